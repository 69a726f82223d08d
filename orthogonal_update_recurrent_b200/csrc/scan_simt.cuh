// scan_simt.cuh -- CUDA-core scan of the Lattice recurrence, exact or chunked.
//
// One CTA per (b, h) sequence, or (SPLIT) a cluster of up to 4 CTAs per sequence
// when the batch has fewer sequences than half the SMs; the slots live in registers
// (octet layout, common.cuh), RQ slot quads per warp. Tokens are processed in order; inputs
// are staged through shared memory TB tokens at a time (loaded into registers
// one block ahead, stored after the current block's compute), and the
// read-out partial sums of the warps are reduced across warps through shared
// memory once per block, in a fixed order (bit-reproducible).
//
// EXACT (CHUNKED = false): §3.1.1 eq. OSR + §3.2 eq. normalized_recurrence +
// §3.3 forget gate, projection by Eq. 14 against the current slot.
// CHUNKED: Eq. 17 (§3.4.1, Appendix B.1): the projection and the normaliser use
// the state at the start of the chunk, kept in a second register set; the
// normaliser n/sqrt(mu^2 n^2 + |Delta|^2) keeps the chunk-start norm n (the
// paper's Appendix D listing scales its rsqrt by the slot norm).
#pragma once
#include "args.h"
#include "common.cuh"

namespace lattice {

constexpr int kScanTB = 8;       // tokens per staged block
constexpr int kScanTBSplit = 16;  // split kernels: longer blocks, half the cluster barriers

// Per-token staged record: x[D] | q[m] | c[m] | mu | eta, padded to a multiple
// of 4 floats so that every record starts 16-byte aligned.
__host__ __device__ inline int scan_record_floats(int D, int m) { return (D + 2 * m + 2 + 3) & ~3; }

// Shared memory: in[2][TB][record] floats, ybuf[2][TB][NW][D] floats and, for the
// reconstruction objective, rbuf[2][NW][D] floats (per-warp partial reconstructions);
// split kernels add ypart[2][TB][D] (the CTA's read-out partials for the cluster sum),
// and with the reconstruction objective rwarp[R][NW][D], rpart[2][R][D] and rsum[R][D]
// (reconstructions per warp, per CTA, over the cluster) for R = TB tokens when chunked
// (a block at a time) and R = 1 when exact (a token at a time).
template <int D>
__host__ __device__ inline size_t scan_smem_bytes(int m, int nw, bool dec, bool split = false,
                                                  bool chunked = true) {
    const size_t tb = split ? kScanTBSplit : kScanTB;
    const size_t rr = chunked ? tb : 1;
    return sizeof(float) * (2ull * tb * scan_record_floats(D, m) + 2ull * tb * nw * D +
                            (dec ? 2ull * nw * D : 0ull) + (split ? 2ull * tb * D : 0ull) +
                            (split && dec ? rr * nw * D + 3ull * rr * D : 0ull));
}

// Cluster barrier and a load from a peer CTA's shared memory (split kernels).
__device__ __forceinline__ void scan_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float scan_ld_peer(const float* local_ptr, uint32_t rank) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local_ptr));
    uint32_t r;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
    return v;
}

// DEC selects the reconstruction objective (§3.1.1 eq. decoding_recurrence): each
// token's write direction is x - sum_i (c_i/|s_i|) s_i, with the slots of the state
// the token's projection uses (the current state; the chunk-start state when
// CHUNKED). On one CTA per sequence it costs one cross-warp reduction and one barrier
// per token; on a cluster (SPLIT, below) the sums also cross the CTAs.
// LIN1 (chunked only) selects the chunk linearisation of eq. recurrence_linear1
// (§3.4.1): the projection part of each token's update scales the chunk-start slot
// instead of the running one.
// SPLIT: each sequence runs on a cluster of a.G CTAs of 8 warps; CTA g owns slots
// [g*spc, (g+1)*spc), spc <= 32. Under the similarity objective the slots evolve
// independently, so the CTAs share only the read-out: each block's per-CTA partial
// y is added over the cluster through distributed shared memory, ranks in a fixed
// order (one cluster barrier per block of tokens). With the reconstruction objective,
// chunked (chunks made of whole blocks), the residual of every token uses the
// chunk-start state, so each block's reconstructions sum_i (c_i/|s0_i|) s0_i are formed
// before its tokens: per CTA over its slots, then over the cluster the same way (a
// second cluster barrier per block). Exact, every token's reconstruction is summed over
// the cluster before the token's update (a cluster barrier per token).
template <int D, int RQ, bool CHUNKED, bool DEC, bool LIN1 = false, bool SPLIT = false>
__global__ void __launch_bounds__(SPLIT ? 256 : 512) scan_simt_kernel(ScanArgs a) {
    static_assert(!(SPLIT && RQ != 1), "split kernels: one slot per octet");
    constexpr int TB = SPLIT ? kScanTBSplit : kScanTB;  // tokens per staged block
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    extern __shared__ __align__(16) float smem[];
    const int NW = blockDim.x >> 5;
    const int NT = blockDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    const int G = SPLIT ? a.G : 1, crank = SPLIT ? (int)(blockIdx.x % G) : 0;
    const int bh = blockIdx.x / G;
    const int b = bh / a.H, h = bh % a.H;
    const int m = a.m, T = a.T, H = a.H;
    const int per_tok = scan_record_floats(D, m);  // x | q | c | mu | eta | pad
    float* in_buf = smem;
    float* ybuf = smem + 2 * TB * per_tok;
    float* rbuf = ybuf + 2 * TB * NW * D;  // DEC only
    float* ypart = rbuf + (DEC ? 2 * NW * D : 0);  // SPLIT only: [2][TB][D]
    constexpr int RR = CHUNKED ? TB : 1;              // reconstructions formed at a time
    float* rwarp = ypart + (SPLIT ? 2 * TB * D : 0);  // SPLIT and DEC: [RR][NW][D]
    float* rpart = rwarp + RR * NW * D;               // [2][RR][D], read by the cluster
    float* rsum = rpart + 2 * RR * D;                 // [RR][D]

    // ---- load the initial state into registers
    float s[RQ][EPL];
    float s0[CHUNKED ? RQ : 1][CHUNKED ? EPL : 1];
    float n0sq[RQ], n0[RQ];
    int slot[RQ];
    const float* S0bh = a.S0 + (size_t)bh * m * D;
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        slot[r] = 4 * (warp + NW * r) + oct;
        if constexpr (SPLIT) slot[r] = slot[r] < a.spc ? crank * a.spc + slot[r] : m;  // m: no slot
        if (slot[r] < m) {
            load_row_f32<D>(S0bh + (size_t)slot[r] * D, j, s[r]);
        } else {
#pragma unroll
            for (int k = 0; k < EPL; ++k) s[r][k] = 0.f;
        }
        n0sq[r] = 0.f;
        n0[r] = 1.f;
    }

    // ---- staging helpers
    const int n_blocks = (T + TB - 1) / TB;
    const int stage_total = TB * per_tok;
    // per-thread staging registers: the host launches NW >= 4 warps when RQ == 1, NW = 16
    // otherwise, and 8 warps for split kernels
    constexpr int kMinThreads = SPLIT ? 256 : (RQ == 1 ? 128 : 512);
    constexpr int kStgM = SPLIT ? 128 : kMaxM;  // split kernels: m <= 4 CTAs x 32 slots
    constexpr int kStg = (TB * (D + 2 * kStgM + 4) + kMinThreads - 1) / kMinThreads;
    float stg[kStg];
    auto stage_load = [&](int blk) {
        const int t0 = blk * TB;
#pragma unroll
        for (int u = 0; u < kStg; ++u) {
            int idx = tid + u * NT;
            float v = 0.f;
            if (idx < stage_total) {
                int tok = idx / per_tok, e = idx - tok * per_tok;
                int t = t0 + tok;
                if (t < T) {
                    size_t bth = ((size_t)b * T + t) * H + h;
                    if (e < D) v = load_elem(a.x, a.x_bf16, bth * D + e);
                    else if (e < D + m) v = load_elem(a.q, a.q_bf16, bth * m + (e - D));
                    else if (e < D + 2 * m) v = a.c[bth * m + (e - D - m)];
                    else if (e == D + 2 * m) v = a.mu[bth];
                    else if (e == D + 2 * m + 1) v = a.eta ? a.eta[bth] : 1.f;
                }
            }
            stg[u] = v;
        }
    };
    auto stage_store = [&](int buf) {
        float* dst = in_buf + buf * stage_total;
#pragma unroll
        for (int u = 0; u < kStg; ++u) {
            int idx = tid + u * NT;
            if (idx < stage_total) dst[idx] = stg[u];
        }
    };

    // Read-out of block fb: fixed-order sum over the warps (and, for split kernels,
    // over the cluster's CTAs, each CTA writing a share of the block's entries).
    auto flush_y = [&](int fb) {
        const int pt0 = fb * TB, ntok = min(TB, T - pt0);
        const float* yb = ybuf + (size_t)(fb & 1) * TB * NW * D;
        if constexpr (!SPLIT) {
            for (int idx = tid; idx < ntok * D; idx += NT) {
                int tok = idx / D, k = idx - tok * D;
                float acc = 0.f;
                for (int w = 0; w < NW; ++w) acc += yb[((size_t)tok * NW + w) * D + k];
                a.y[(((size_t)b * T + pt0 + tok) * H + h) * D + k] = acc;
            }
        } else {
            // the partial buffers alternate by block; the next flush's cluster barrier
            // orders their reuse after every peer has read them
            float* part = ypart + (size_t)(fb & 1) * TB * D;
            for (int idx = tid; idx < ntok * D; idx += NT) {
                int tok = idx / D, k = idx - tok * D;
                float acc = 0.f;
                for (int w = 0; w < NW; ++w) acc += yb[((size_t)tok * NW + w) * D + k];
                part[idx] = acc;
            }
            scan_cluster_sync();
            for (int idx = crank * NT + tid; idx < ntok * D; idx += G * NT) {
                int tok = idx / D, k = idx - tok * D;
                float v[8];  // every peer's load in flight before the fixed-order sum
#pragma unroll
                for (int r = 0; r < 8; ++r) v[r] = r < G ? scan_ld_peer(part + idx, (uint32_t)r) : 0.f;
                float acc = 0.f;
#pragma unroll
                for (int r = 0; r < 8; ++r) if (r < G) acc += v[r];
                a.y[(((size_t)b * T + pt0 + tok) * H + h) * D + k] = acc;
            }
        }
    };

    if (n_blocks > 0) {
        stage_load(0);
        stage_store(0);
    }
    __syncthreads();

    for (int blk = 0; blk < n_blocks; ++blk) {
        const int buf = blk & 1;
        const int t0 = blk * TB;
        // flush the previous block's read-out
        if (blk > 0) flush_y(blk - 1);
        if (blk + 1 < n_blocks) stage_load(blk + 1);

        const float* inb = in_buf + buf * stage_total;
        float* yb = ybuf + (size_t)buf * TB * NW * D;
        const int ntok = min(TB, T - t0);
        if constexpr (SPLIT && DEC && CHUNKED) {
            // chunk-start snapshot (chunks start on block boundaries), then the block's
            // reconstructions: per warp, per CTA, and over the cluster in rank order
            if (t0 % a.chunk == 0) {
                float n2 = 0.f;
#pragma unroll
                for (int k = 0; k < EPL; ++k) { s0[0][k] = s[0][k]; n2 = fmaf(s[0][k], s[0][k], n2); }
                n0sq[0] = octet_sum(n2);
                n0[0] = __fsqrt_rn(n0sq[0]);
            }
            for (int tok = 0; tok < ntok; ++tok) {
                const float* rec = inb + tok * per_tok;
                const float cv = slot[0] < m ? rec[D + m + slot[0]] : 0.f;
                float f[1], rp[EPL];
                f[0] = n0sq[0] > 0.f ? __fdiv_rn(cv, __fsqrt_rn(n0sq[0])) : 0.f;
                recon_warp_partial<D, 1>(s0, f, rp);
                if (oct == 0) {
#pragma unroll
                    for (int k = 0; k < EPL; ++k) rwarp[((size_t)tok * NW + warp) * D + O::pos(j, k)] = rp[k];
                }
            }
            __syncthreads();
            float* part = rpart + (size_t)(blk & 1) * TB * D;  // the next cluster barrier orders its reuse
            for (int idx = tid; idx < ntok * D; idx += NT) {
                const int tok = idx / D, k = idx - tok * D;
                float acc = 0.f;
                for (int w = 0; w < NW; ++w) acc += rwarp[((size_t)tok * NW + w) * D + k];
                part[idx] = acc;
            }
            scan_cluster_sync();
            for (int idx = tid; idx < ntok * D; idx += NT) {
                float v[8];  // every peer's load in flight before the fixed-order sum
#pragma unroll
                for (int r = 0; r < 8; ++r) v[r] = r < G ? scan_ld_peer(part + idx, (uint32_t)r) : 0.f;
                float acc = 0.f;
#pragma unroll
                for (int r = 0; r < 8; ++r) if (r < G) acc += v[r];
                rsum[idx] = acc;
            }
            __syncthreads();
        }
        for (int tok = 0; tok < ntok; ++tok) {
            const int t = t0 + tok;
            const float* rec = inb + tok * per_tok;
            float xv[EPL];
            load_row_f32<D>(rec, j, xv);
            const float mu = rec[D + 2 * m], eta = rec[D + 2 * m + 1];

            if constexpr (CHUNKED && !(SPLIT && DEC)) {  // (split DEC: taken per block above)
                if (t % a.chunk == 0) {  // chunk start: snapshot the state and its norms
#pragma unroll
                    for (int r = 0; r < RQ; ++r) {
                        float n2 = 0.f;
#pragma unroll
                        for (int k = 0; k < EPL; ++k) { s0[r][k] = s[r][k]; n2 = fmaf(s[r][k], s[r][k], n2); }
                        n0sq[r] = octet_sum(n2);
                        n0[r] = __fsqrt_rn(n0sq[r]);
                    }
                }
            }
            if constexpr (SPLIT && DEC && CHUNKED) {  // the block's reconstructions, formed above
#pragma unroll
                for (int k = 0; k < EPL; ++k) xv[k] -= rsum[(size_t)tok * D + O::pos(j, k)];
            } else if constexpr (SPLIT && DEC) {
                // exact: this token's reconstruction from the current slots, per warp, per
                // CTA (part, double-buffered by token), then over the cluster in rank order
                float nn = 0.f;
#pragma unroll
                for (int k = 0; k < EPL; ++k) nn = fmaf(s[0][k], s[0][k], nn);
                const float nsq = octet_sum(nn);
                const float cv = slot[0] < m ? rec[D + m + slot[0]] : 0.f;
                float f[1], rp[EPL];
                f[0] = nsq > 0.f ? __fdiv_rn(cv, __fsqrt_rn(nsq)) : 0.f;
                recon_warp_partial<D, 1>(s, f, rp);
                if (oct == 0) {
#pragma unroll
                    for (int k = 0; k < EPL; ++k) rwarp[warp * D + O::pos(j, k)] = rp[k];
                }
                __syncthreads();
                float* part = rpart + (size_t)(t & 1) * D;  // the next cluster barrier orders its reuse
                for (int idx = tid; idx < D; idx += NT) {
                    float acc = 0.f;
                    for (int w = 0; w < NW; ++w) acc += rwarp[w * D + idx];
                    part[idx] = acc;
                }
                scan_cluster_sync();
                for (int idx = tid; idx < D; idx += NT) {
                    float v[8];
#pragma unroll
                    for (int r = 0; r < 8; ++r) v[r] = r < G ? scan_ld_peer(part + idx, (uint32_t)r) : 0.f;
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r) if (r < G) acc += v[r];
                    rsum[idx] = acc;
                }
                __syncthreads();
#pragma unroll
                for (int k = 0; k < EPL; ++k) xv[k] -= rsum[O::pos(j, k)];
            } else if constexpr (DEC) {  // x <- x - sum_i (c_i/|s_i|) s_i over every slot of the CTA
                float f[RQ], rp[EPL];
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    const float cv = slot[r] < m ? rec[D + m + slot[r]] : 0.f;
                    float nsq;
                    if constexpr (CHUNKED) {
                        nsq = n0sq[r];
                    } else {
                        float nn = 0.f;
#pragma unroll
                        for (int k = 0; k < EPL; ++k) nn = fmaf(s[r][k], s[r][k], nn);
                        nsq = octet_sum(nn);
                    }
                    f[r] = nsq > 0.f ? __fdiv_rn(cv, __fsqrt_rn(nsq)) : 0.f;
                }
                if constexpr (CHUNKED) recon_warp_partial<D, RQ>(s0, f, rp);
                else recon_warp_partial<D, RQ>(s, f, rp);
                float* rb = rbuf + (size_t)(t & 1) * NW * D;
                if (oct == 0) {
#pragma unroll
                    for (int k = 0; k < EPL; ++k) rb[warp * D + O::pos(j, k)] = rp[k];
                }
                __syncthreads();
#pragma unroll
                for (int k = 0; k < EPL; ++k) {
                    float acc = 0.f;
                    for (int w = 0; w < NW; ++w) acc += rb[w * D + O::pos(j, k)];
                    xv[k] -= acc;
                }
            }
            float xx = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; ++k) xx = fmaf(xv[k], xv[k], xx);
            xx = octet_sum(xx);
            float p[RQ], n2[RQ];
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                float pp = 0.f, nn = 0.f;
#pragma unroll
                for (int k = 0; k < EPL; ++k) {
                    if constexpr (CHUNKED) {
                        pp = fmaf(s0[r][k], xv[k], pp);
                    } else {
                        pp = fmaf(s[r][k], xv[k], pp);
                        nn = fmaf(s[r][k], s[r][k], nn);
                    }
                }
                p[r] = pp;
                n2[r] = nn;
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    p[r] += __shfl_xor_sync(0xffffffffu, p[r], o);
                    if constexpr (!CHUNKED) n2[r] += __shfl_xor_sync(0xffffffffu, n2[r], o);
                }
            }
            float yp[EPL];
#pragma unroll
            for (int k = 0; k < EPL; ++k) yp[k] = 0.f;
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                const bool valid = slot[r] < m;
                const float cv = valid ? rec[D + m + slot[r]] : 0.f;
                const float qv = valid ? rec[D + slot[r]] : 0.f;
                if constexpr (CHUNKED && LIN1) {
                    float alpha_s, alpha_0, gamma;
                    if (a.cnorm) {  // no per-token normaliser: the bare write (beta = 1)
                        const bool ok = n0sq[r] > 0.f;
                        const float ac = ok ? __fdiv_rn(eta * cv, n0[r]) : 0.f;   // eta c / n
                        const float rr = ok ? __fdiv_rn(p[r], n0sq[r]) : 0.f;     // p / n^2
                        alpha_s = mu;
                        alpha_0 = -ac * rr;
                        gamma = ac;
                    } else if constexpr (DEC) {  // |x_perp|^2 summed directly (see update_coefs_perp)
                        const float pp2 = octet_sum(perp2_partial<EPL>(xv, s0[r], p[r], n0sq[r]));
                        update_coefs_lin1_perp<true>(n0sq[r], p[r], pp2, cv, mu, eta, n0[r], alpha_s, alpha_0, gamma);
                    } else {
                        update_coefs_lin1<true>(n0sq[r], p[r], xx, cv, mu, eta, n0[r], alpha_s, alpha_0, gamma);
                    }
                    if (!valid) { alpha_s = 0.f; alpha_0 = 0.f; gamma = 0.f; }
#pragma unroll
                    for (int k = 0; k < EPL; ++k) {
                        s[r][k] = fmaf(alpha_s, s[r][k], fmaf(alpha_0, s0[r][k], gamma * xv[k]));
                        yp[k] = fmaf(qv, s[r][k], yp[k]);
                    }
                } else {
                    float alpha, gamma;
                    if (CHUNKED && a.cnorm) {  // no per-token normaliser: the bare write (beta = 1)
                        const bool ok = n0sq[r] > 0.f;
                        const float ac = ok ? __fdiv_rn(eta * cv, n0[r]) : 0.f;   // eta c / n
                        const float rr = ok ? __fdiv_rn(p[r], n0sq[r]) : 0.f;     // p / n^2
                        alpha = ok ? fmaf(-ac, rr, mu) : 1.f;
                        gamma = ac;
                    } else if constexpr (DEC) {  // |x_perp|^2 summed directly (see update_coefs_perp)
                        const float nr2 = CHUNKED ? n0sq[r] : n2[r];
                        const float pp2 = octet_sum(perp2_partial<EPL>(xv, CHUNKED ? s0[r] : s[r], p[r], nr2));
                        update_coefs_perp<true>(nr2, p[r], pp2, cv, mu, eta, CHUNKED ? n0[r] : 1.f, alpha, gamma);
                    } else {
                        update_coefs<CHUNKED>(CHUNKED ? n0sq[r] : n2[r], p[r], xx, cv, mu, eta,
                                              CHUNKED ? n0[r] : 1.f, alpha, gamma);
                    }
                    if (!valid) { alpha = 0.f; gamma = 0.f; }
#pragma unroll
                    for (int k = 0; k < EPL; ++k) {
                        s[r][k] = fmaf(alpha, s[r][k], gamma * xv[k]);
                        yp[k] = fmaf(qv, s[r][k], yp[k]);
                    }
                }
            }
            if constexpr (CHUNKED) {  // normalisation at chunk boundaries: after the chunk's last read-out
                if (a.cnorm && ((t + 1) % a.chunk == 0 || t + 1 == T)) {
#pragma unroll
                    for (int r = 0; r < RQ; ++r) {
                        float nn = 0.f;
#pragma unroll
                        for (int k = 0; k < EPL; ++k) nn = fmaf(s[r][k], s[r][k], nn);
                        nn = octet_sum(nn);
                        if (nn > 0.f) {
                            const float nr = __fsqrt_rn(nn);
#pragma unroll
                            for (int k = 0; k < EPL; ++k) s[r][k] = __fdiv_rn(s[r][k], nr);
                        }
                    }
                }
            }
            // reduce the read-out over the 4 octets of the warp (reduce-scatter)
            float* ydst = yb + ((size_t)tok * NW + warp) * D;
            if constexpr (EPL >= 4) {
                const int hi = (lane >> 4) & 1, mid = (lane >> 3) & 1;
                float v1[EPL / 2];
#pragma unroll
                for (int k = 0; k < EPL / 2; ++k) {
                    float send = hi ? yp[k] : yp[k + EPL / 2];
                    float keep = hi ? yp[k + EPL / 2] : yp[k];
                    v1[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
                float v2[EPL / 4];
#pragma unroll
                for (int k = 0; k < EPL / 4; ++k) {
                    float send = mid ? v1[k] : v1[k + EPL / 4];
                    float keep = mid ? v1[k + EPL / 4] : v1[k];
                    v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                const int kbase = hi * (EPL / 2) + mid * (EPL / 4);
#pragma unroll
                for (int k = 0; k < EPL / 4; ++k) ydst[O::pos(j, kbase + k)] = v2[k];
            } else {  // EPL == 2
                const int hi = (lane >> 4) & 1, mid = (lane >> 3) & 1;
                float send = hi ? yp[0] : yp[1];
                float keep = hi ? yp[1] : yp[0];
                float v = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                if (!mid) ydst[O::pos(j, hi)] = v;
            }
        }
        if (blk + 1 < n_blocks) stage_store(buf ^ 1);
        __syncthreads();
    }
    // flush the last block
    if (n_blocks > 0) flush_y(n_blocks - 1);
    if constexpr (SPLIT) scan_cluster_sync();  // no CTA leaves while a peer may still read its partials
    // final state
    float* Sbh = a.S_out + (size_t)bh * m * D;
#pragma unroll
    for (int r = 0; r < RQ; ++r)
        if (slot[r] < m) store_row_f32<D, false>(Sbh + (size_t)slot[r] * D, j, s[r]);
}

}  // namespace lattice
