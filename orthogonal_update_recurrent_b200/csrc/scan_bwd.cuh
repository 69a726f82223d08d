// scan_bwd.cuh -- CUDA-core backward pass of the Lattice scan (similarity
// objective), exact recurrence or chunked form (Eq. 17).
//
// "Lattice: Learning to Efficiently Compress the Memory" prints no backward
// formulas; this kernel evaluates the reverse-mode derivative of the forward that
// scan_simt.cuh computes, for L = sum_t dy_t . y_t + dS_T . S_T:
//   per slot and token  n2 = |z|^2, p = z.x, xx = |x|^2 (z = the running slot for
//   the exact recurrence, the chunk-start slot for Eq. 17), a = eta c/n,
//   r = p/n2, u = mu - a r, w2 = mu^2 n2 + a^2 (xx - p r), iw = target/sqrt(w2)
//   (target 1, or n for Eq. 17's normaliser), s_t = (u iw) s_{t-1} + (a iw) x,
//   y_t = sum_i q_i s_t,i.
// The adjoint walks the tokens backwards, carrying dL/ds_t in registers.
//
// Each (b, h) sequence runs on a cluster of G <= 4 CTAs (G = 1: a single CTA); CTA g
// owns slots [g*spc, (g+1)*spc) in registers in the octet layout (common.cuh).
// Slots evolve independently under the similarity objective, so the CTAs share
// nothing but the per-token sums over slots (dx, dmu, deta): each CTA reduces its
// own warps, then, once per block of tokens, the cluster adds the G partials
// through distributed shared memory in a fixed order (one cluster barrier per
// block, partial buffers double-buffered). States are rebuilt by recomputation, so
// memory stays O(T/L):
//   1. a forward sweep stores the state at the start of every segment of L
//      tokens (L a multiple of the chunk size) in the workspace;
//   2. for each segment, last to first: recompute its states from the
//      checkpoint into the segment tape (workspace, L2-resident), then run the
//      adjoint over the segment's tokens in reverse, reading the tape.
// Per-token gradients that sum over slots (dx, dmu, deta) are reduced within
// the warp by shuffles and across warps through shared memory in a fixed order,
// so results are bit-reproducible.
#pragma once
#include "args.h"
#include "common.cuh"

namespace lattice {

constexpr int kBwdTB = 8;        // tokens per staged block
constexpr int kBwdTBSplit = 16;  // cluster kernels: longer blocks, half the cluster barriers


// Staged record per token: x[D] | dy[D] | q[spc] | c[spc] | mu | eta (q and c of
// this CTA's slots only), padded so that every record (and its dy) starts 16-byte
// aligned. Records are double-buffered: the next block's are loaded into registers
// while the current block computes.
__host__ __device__ inline int bwd_record_floats(int D, int spc) { return (2 * D + 2 * spc + 2 + 3) & ~3; }

// Threads per CTA: 512 for one CTA per sequence, 256 in a cluster (<= 32 slots per CTA).
__host__ __device__ constexpr int bwd_threads(bool split) { return split ? 256 : 512; }

__host__ __device__ inline size_t bwd_smem_bytes(int D, int spc, int nw, bool split) {
    const size_t tb = split ? kBwdTBSplit : kBwdTB;
    return sizeof(float) * (2ull * tb * bwd_record_floats(D, spc) + tb * nw * D + tb * nw * 2 +
                            2ull * tb * (D + 2));
}

// 1/sqrt(x) for x > 0: the hardware approximation and one Newton step.
__device__ __forceinline__ float bwd_rsqrt(float x) {
    const float y = rsqrtf(x);
    return y * fmaf(-0.5f * x * y, y, 1.5f);
}

// Cluster primitives (distributed shared memory).
__device__ __forceinline__ void bwd_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float bwd_ld_peer(const float* local_ptr, uint32_t rank) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local_ptr));
    uint32_t r;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
    return v;
}


// Forward coefficients of one slot and token, with the intermediates the adjoint needs.
struct SlotFwd {
    bool ok;
    float n2, inv_n, inv_n2, r, a, praw, perp2, w2, iw, u, alpha, gamma;
};

__device__ __forceinline__ SlotFwd slot_fwd(float n2, float p, float xx, float c, float mu, float eta,
                                            bool chunked) {
    SlotFwd f;
    f.ok = n2 > 0.f;
    f.n2 = f.ok ? n2 : 1.f;
    f.inv_n = bwd_rsqrt(f.n2);
    f.inv_n2 = f.inv_n * f.inv_n;
    f.r = p * f.inv_n2;
    f.a = eta * c * f.inv_n;
    f.praw = fmaf(-p, f.r, xx);
    f.perp2 = fmaxf(f.praw, 0.f);
    f.w2 = fmaf(f.a * f.a, f.perp2, mu * mu * f.n2);
    f.ok = f.ok && f.w2 > 0.f;
    const float target = chunked ? f.n2 * f.inv_n : 1.f;
    f.iw = bwd_rsqrt(f.ok ? f.w2 : 1.f) * target;
    f.u = fmaf(-f.a, f.r, mu);
    f.alpha = f.ok ? f.u * f.iw : 1.f;
    f.gamma = f.ok ? f.a * f.iw : 0.f;
    return f;
}

// Adjoint of slot_fwd: from dL/dalpha and dL/dgamma to dL/dp, dL/dn2, dL/dxx,
// dL/dmu, dL/deta, dL/dc. A degenerate slot (ok false) had constant coefficients.
struct SlotBwd {
    float pb, n2b, xxb, mub, etab, cb;
};

__device__ __forceinline__ SlotBwd slot_bwd(const SlotFwd& f, float p, float c, float mu, float eta,
                                            float alphab, float gammab, bool chunked) {
    SlotBwd g{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (!f.ok) return g;
    const float ub = alphab * f.iw;                       // alpha = u iw
    const float iwb = fmaf(alphab, f.u, gammab * f.a);    // gamma = a iw
    float ab = fmaf(gammab, f.iw, -ub * f.r);
    float rb = -ub * f.a;                                 // u = mu - a r
    g.mub = ub;
    // iw = target w2^(-1/2): d iw / d w2 = -iw^3 / (2 target^2), target^2 = n2 or 1
    const float iw3 = f.iw * f.iw * f.iw;
    const float w2b = -0.5f * iwb * (chunked ? iw3 * f.inv_n2 : iw3);
    g.mub = fmaf(w2b, 2.f * mu * f.n2, g.mub);            // w2 = mu^2 n2 + a^2 perp2
    g.n2b = w2b * mu * mu;
    ab = fmaf(w2b, 2.f * f.a * f.perp2, ab);
    const float perp2b = f.praw > 0.f ? w2b * f.a * f.a : 0.f;
    g.xxb = perp2b;                                       // perp2 = xx - p r
    g.pb = -perp2b * f.r;
    rb = fmaf(-perp2b, p, rb);
    g.pb = fmaf(rb, f.inv_n2, g.pb);                      // r = p / n2
    g.n2b = fmaf(-rb * f.r, f.inv_n2, g.n2b);
    g.etab = ab * c * f.inv_n;                            // a = eta c / n
    g.cb = ab * eta * f.inv_n;
    float nb = -ab * f.a * f.inv_n;
    if (chunked) nb = fmaf(iwb * f.iw, f.inv_n, nb);      // target = n
    g.n2b = fmaf(nb, 0.5f * f.inv_n, g.n2b);              // n = sqrt(n2)
    return g;
}

// Sum a per-lane D-vector partial over the 4 octets of the warp and store the
// warp's total to dst[D] (each lane stores EPL/4 of its octet positions).
template <int D>
__device__ __forceinline__ void warp_octets_sum_store(const float* v, float* dst, int lane) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    const int j = lane & 7;
    const int hi = (lane >> 4) & 1, mid = (lane >> 3) & 1;
    if constexpr (EPL >= 4) {
        float v1[EPL / 2];
#pragma unroll
        for (int k = 0; k < EPL / 2; ++k) {
            const float send = hi ? v[k] : v[k + EPL / 2];
            const float keep = hi ? v[k + EPL / 2] : v[k];
            v1[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        float v2[EPL / 4];
#pragma unroll
        for (int k = 0; k < EPL / 4; ++k) {
            const float send = mid ? v1[k] : v1[k + EPL / 4];
            const float keep = mid ? v1[k + EPL / 4] : v1[k];
            v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const int kbase = hi * (EPL / 2) + mid * (EPL / 4);
#pragma unroll
        for (int k = 0; k < EPL / 4; ++k) dst[O::pos(j, kbase + k)] = v2[k];
    } else {  // EPL == 2
        const float send = hi ? v[0] : v[1];
        const float keep = hi ? v[1] : v[0];
        float t = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        t += __shfl_xor_sync(0xffffffffu, t, 8);
        if (!mid) dst[O::pos(j, hi)] = t;
    }
}

// SPLIT: launched in clusters (G > 1) with at most 32 slots per CTA. The CTA has
// bwd_threads(SPLIT) threads whatever its slot count (idle warps only stage inputs).
template <int D, int RQ, bool CHUNKED, bool SPLIT>
__global__ void __launch_bounds__(bwd_threads(SPLIT)) scan_bwd_kernel(BwdArgs a) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    constexpr int NT = bwd_threads(SPLIT), NW = NT / 32;
    constexpr int TB = SPLIT ? kBwdTBSplit : kBwdTB;  // tokens per staged block
    // staging registers per thread: one block of the largest record this instantiation takes
    constexpr int kMaxSpc = SPLIT ? 32 : 64 * RQ;
    constexpr int KS = (TB * ((2 * D + 2 * kMaxSpc + 2 + 3) & ~3) + NT - 1) / NT;
    // a cluster CTA has one warp per scheduler, so the next tape entry is loaded one
    // token ahead; with 16 warps the others hide that latency and the registers are short
    constexpr bool kPrefetchTape = SPLIT;
    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    const int G = a.G, crank = blockIdx.x % G;  // cluster rank (clusters span G consecutive CTAs)
    const int bh = blockIdx.x / G, b = bh / a.H, h = bh % a.H;
    const int m = a.m, T = a.T, H = a.H, L = a.seg, SPC = a.spc;
    const int R = bwd_record_floats(D, SPC);
    float* rec_buf = smem;                                   // [2][TB][R]
    float* dx_buf = smem + 2 * TB * R;                   // [TB][NW][D]
    float* sc_buf = dx_buf + (size_t)TB * NW * D;        // [TB][NW][2]: dmu, deta partials
    float* cta_part = sc_buf + (size_t)TB * NW * 2;      // [2][TB][D + 2]: this CTA's sums (G > 1)
    const int nseg = T > 0 ? (T + L - 1) / L : 1;
    float* ckpt = a.ws + ((size_t)bh * G + crank) * bwd_ws_floats_per_seq(T, SPC, D, L);  // [nseg-1][SPC][D]
    float* tape = ckpt + (size_t)(nseg - 1) * SPC * D;                                     // [L][SPC][D]
    const size_t st_sz = (size_t)SPC * D;  // one checkpoint or tape entry

    int slot[RQ], lslot[RQ];  // global slot (rows of S0, dS_T, dS0, c, q) and row in this CTA's scratch
    bool valid[RQ];
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        lslot[r] = 4 * (warp + NW * r) + oct;
        slot[r] = crank * SPC + lslot[r];
        valid[r] = lslot[r] < SPC && slot[r] < m;
    }
    auto load_rows = [&](const float* base, const int* row, float (*v)[EPL]) {
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            if (valid[r]) load_row_f32<D>(base + (size_t)row[r] * D, j, v[r]);
            else {
#pragma unroll
                for (int k = 0; k < EPL; ++k) v[r][k] = 0.f;
            }
        }
    };
    auto store_rows = [&](float* base, const int* row, const float (*v)[EPL]) {
#pragma unroll
        for (int r = 0; r < RQ; ++r)
            if (valid[r]) store_row_f32<D, false>(base + (size_t)row[r] * D, j, v[r]);
    };
    auto load_state = [&](const float* base, float (*v)[EPL]) { load_rows(base, slot, v); };
    auto store_state = [&](float* base, const float (*v)[EPL]) { store_rows(base, slot, v); };
    auto load_scratch = [&](const float* base, float (*v)[EPL]) { load_rows(base, lslot, v); };
    auto store_scratch = [&](float* base, const float (*v)[EPL]) { store_rows(base, lslot, v); };

    // Staging of tokens [t0, t0 + n): fetch into registers (all loads in flight at
    // once), later put into one of the two record buffers. The forward sweeps need
    // x, c, mu, eta only.
    float stg[KS];
    auto fetch = [&](int t0, int n, bool need_qdy) {
#pragma unroll
        for (int u = 0; u < KS; ++u) {
            const int idx = tid + u * NT;
            float v = 0.f;
            if (idx < n * R) {
                const int tok = idx / R, e = idx - tok * R;
                const size_t bth = ((size_t)b * T + t0 + tok) * H + h;
                if (e < D) v = load_elem(a.x, a.x_bf16, bth * D + e);
                else if (e < 2 * D) { if (need_qdy) v = a.dy[bth * D + (e - D)]; }
                else if (e < 2 * D + 2 * SPC) {
                    const bool is_c = e >= 2 * D + SPC;
                    const int ls = e - 2 * D - (is_c ? SPC : 0), gs = crank * SPC + ls;
                    if (gs < m) {
                        if (is_c) v = a.c[bth * m + gs];
                        else if (need_qdy) v = load_elem(a.q, a.q_bf16, bth * m + gs);
                    }
                } else if (e == 2 * D + 2 * SPC) v = a.mu[bth];
                else if (e == 2 * D + 2 * SPC + 1) v = a.eta ? a.eta[bth] : 1.f;
            }
            stg[u] = v;
        }
    };
    auto put = [&](int buf, int n) {
        float* dst = rec_buf + (size_t)buf * TB * R;
#pragma unroll
        for (int u = 0; u < KS; ++u) {
            const int idx = tid + u * NT;
            if (idx < n * R) dst[idx] = stg[u];
        }
    };

    float s[RQ][EPL], s0[CHUNKED ? RQ : 1][EPL];
    float n0sq[RQ];
    // One forward token from the record rec: s <- alpha s + gamma x.
    auto forward_token = [&](int t, const float* rec) {
        if constexpr (CHUNKED) {
            if (t % a.chunk == 0) {
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    float nn = 0.f;
#pragma unroll
                    for (int k = 0; k < EPL; ++k) { s0[r][k] = s[r][k]; nn = fmaf(s[r][k], s[r][k], nn); }
                    n0sq[r] = octet_sum(nn);
                }
            }
        }
        float xv[EPL];
        load_row_f32<D>(rec, j, xv);
        const float mu = rec[2 * D + 2 * SPC], eta = rec[2 * D + 2 * SPC + 1];
        float xx = 0.f, p[RQ], n2[RQ];
#pragma unroll
        for (int k = 0; k < EPL; ++k) xx = fmaf(xv[k], xv[k], xx);
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            float pp = 0.f, nn = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; ++k) {
                if constexpr (CHUNKED) pp = fmaf(s0[r][k], xv[k], pp);
                else { pp = fmaf(s[r][k], xv[k], pp); nn = fmaf(s[r][k], s[r][k], nn); }
            }
            p[r] = pp;
            n2[r] = nn;
        }
        xx = octet_sum(xx);
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            p[r] = octet_sum(p[r]);
            if constexpr (!CHUNKED) n2[r] = octet_sum(n2[r]);
        }
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            const float cv = valid[r] ? rec[2 * D + SPC + lslot[r]] : 0.f;
            SlotFwd f = slot_fwd(CHUNKED ? n0sq[r] : n2[r], p[r], xx, cv, mu, eta, CHUNKED);
            const float al = valid[r] ? f.alpha : 0.f, ga = valid[r] ? f.gamma : 0.f;
#pragma unroll
            for (int k = 0; k < EPL; ++k) s[r][k] = fmaf(al, s[r][k], ga * xv[k]);
        }
    };
    // Forward over tokens [t_begin, t_end) from the state in s. tape_base != null:
    // store the state before each token at tape_base[t - t_begin]. ckpts: store the
    // state before each segment start t (t % L == 0, 0 < t < t_end) as a checkpoint.
    auto forward = [&](int t_begin, int t_end, float* tape_base, bool ckpts) {
        const int nblk = (t_end - t_begin + TB - 1) / TB;
        if (nblk == 0) return;
        __syncthreads();  // the record buffers are free
        fetch(t_begin, min(TB, t_end - t_begin), false);
        put(0, min(TB, t_end - t_begin));
        __syncthreads();
        for (int k = 0; k < nblk; ++k) {
            const int t0 = t_begin + k * TB, n = min(TB, t_end - t0);
            const int t1 = t0 + TB, n1 = k + 1 < nblk ? min(TB, t_end - t1) : 0;
            if (n1 > 0) fetch(t1, n1, false);
            const float* rb = rec_buf + (size_t)(k & 1) * TB * R;
            for (int tok = 0; tok < n; ++tok) {
                const int t = t0 + tok;
                if (ckpts && t > 0 && t % L == 0) store_scratch(ckpt + (size_t)(t / L - 1) * st_sz, s);
                if (tape_base) store_scratch(tape_base + (size_t)(t - t_begin) * st_sz, s);
                forward_token(t, rb + tok * R);
            }
            if (n1 > 0) put((k + 1) & 1, n1);
            __syncthreads();
        }
    };

    // ---- 1. checkpoints at every segment start (the last segment needs none beyond)
    load_state(a.S0 + (size_t)bh * m * D, s);
    if (nseg > 1) {
        forward(0, (nseg - 1) * L, nullptr, true);
        store_scratch(ckpt + (size_t)(nseg - 2) * st_sz, s);  // the last segment's start
    }

    // ---- 2. segments, last to first
    int pbuf = 0;       // partial buffer of the next block (G > 1)
    float gb[RQ][EPL];  // dL/ds_t
    if (a.dST) load_state(a.dST + (size_t)bh * m * D, gb);
    else {
#pragma unroll
        for (int r = 0; r < RQ; ++r)
#pragma unroll
            for (int k = 0; k < EPL; ++k) gb[r][k] = 0.f;
    }
    float acc[CHUNKED ? RQ : 1][EPL];  // chunked: sum over the chunk's tokens of dL/dp x
    float n2acc[RQ];                   // chunked: sum of dL/dn2
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        n2acc[r] = 0.f;
        if constexpr (CHUNKED) {
#pragma unroll
            for (int k = 0; k < EPL; ++k) acc[r][k] = 0.f;
        }
    }
    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int ts = seg * L, te = min(T, ts + L);
        // 2a. rebuild the segment's states into the tape
        if (seg == 0) load_state(a.S0 + (size_t)bh * m * D, s);
        else load_scratch(ckpt + (size_t)(seg - 1) * st_sz, s);
        forward(ts, te, tape, false);
        float spn[kPrefetchTape ? RQ : 1][EPL];  // s_{t-1} of the next token, loaded one token ahead
        if constexpr (kPrefetchTape) {
            if (te > ts) load_scratch(tape + (size_t)(te - 1 - ts) * st_sz, spn);
        }
        // 2b. adjoint over the segment's tokens, last to first (blocks from the end)
        const int nblk = (te - ts + TB - 1) / TB;
        if (nblk > 0) {
            __syncthreads();  // the record buffers are free
            const int f0 = max(ts, te - TB);
            fetch(f0, te - f0, true);
            put(0, te - f0);
            __syncthreads();
        }
        for (int kb = 0; kb < nblk; ++kb) {
            const int tb_end = te - kb * TB;
            const int t0 = max(ts, tb_end - TB), n = tb_end - t0;
            const int t0n = max(ts, t0 - TB), n1 = kb + 1 < nblk ? t0 - t0n : 0;
            if (n1 > 0) fetch(t0n, n1, true);
            const float* rbuf = rec_buf + (size_t)(kb & 1) * TB * R;
            for (int tok = n - 1; tok >= 0; --tok) {
                const int t = t0 + tok;
                const float* rec = rbuf + tok * R;
                const size_t bth = ((size_t)b * T + t) * H + h;
                float sp[RQ][EPL];  // s_{t-1}
                if constexpr (kPrefetchTape) {
#pragma unroll
                    for (int r = 0; r < RQ; ++r)
#pragma unroll
                        for (int k = 0; k < EPL; ++k) sp[r][k] = spn[r][k];
                    if (t > ts) load_scratch(tape + (size_t)(t - 1 - ts) * st_sz, spn);
                } else {
                    load_scratch(tape + (size_t)(t - ts) * st_sz, sp);
                }
                if constexpr (CHUNKED) {
                    if (t == te - 1 || (t + 1) % a.chunk == 0) {  // entering a chunk from its end
                        const int tc = (t / a.chunk) * a.chunk;
                        load_scratch(tape + (size_t)(tc - ts) * st_sz, s0);
#pragma unroll
                        for (int r = 0; r < RQ; ++r) {
                            float nn = 0.f;
#pragma unroll
                            for (int k = 0; k < EPL; ++k) nn = fmaf(s0[r][k], s0[r][k], nn);
                            n0sq[r] = octet_sum(nn);
                        }
                    }
                }
                float xv[EPL], yb[EPL];
                load_row_f32<D>(rec, j, xv);
                load_row_f32<D>(rec + D, j, yb);
                const float mu = rec[2 * D + 2 * SPC], eta = rec[2 * D + 2 * SPC + 1];
                // lane-local dot products, then one batch of octet reductions
                float xx = 0.f, xy = 0.f;
#pragma unroll
                for (int k = 0; k < EPL; ++k) { xx = fmaf(xv[k], xv[k], xx); xy = fmaf(xv[k], yb[k], xy); }
                float p[RQ], n2[RQ], spy[RQ], spg[RQ], xg[RQ];
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    float pp = 0.f, nn = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int k = 0; k < EPL; ++k) {
                        if constexpr (CHUNKED) pp = fmaf(s0[r][k], xv[k], pp);
                        else { pp = fmaf(sp[r][k], xv[k], pp); nn = fmaf(sp[r][k], sp[r][k], nn); }
                        a1 = fmaf(sp[r][k], yb[k], a1);
                        a2 = fmaf(sp[r][k], gb[r][k], a2);
                        a3 = fmaf(xv[k], gb[r][k], a3);
                    }
                    p[r] = pp; n2[r] = nn; spy[r] = a1; spg[r] = a2; xg[r] = a3;
                }
                xx = octet_sum(xx);
                xy = octet_sum(xy);
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    p[r] = octet_sum(p[r]);
                    if constexpr (!CHUNKED) n2[r] = octet_sum(n2[r]);
                    spy[r] = octet_sum(spy[r]);
                    spg[r] = octet_sum(spg[r]);
                    xg[r] = octet_sum(xg[r]);
                }
                float dxp[EPL];
#pragma unroll
                for (int k = 0; k < EPL; ++k) dxp[k] = 0.f;
                float mub = 0.f, etab = 0.f;
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    const float cv = valid[r] ? rec[2 * D + SPC + lslot[r]] : 0.f;
                    const float qv = valid[r] ? rec[2 * D + lslot[r]] : 0.f;
                    const SlotFwd f = slot_fwd(CHUNKED ? n0sq[r] : n2[r], p[r], xx, cv, mu, eta, CHUNKED);
                    // read-out y_t = sum_i q_i s_t,i, s_t = alpha s_{t-1} + gamma x
                    const float qb = fmaf(f.alpha, spy[r], f.gamma * xy);
                    // dL/ds_t including the read-out: g = gb + q dy
                    const float alphab = fmaf(qv, spy[r], spg[r]);  // s_{t-1} . g
                    const float gammab = fmaf(qv, xy, xg[r]);       // x . g
                    SlotBwd d = slot_bwd(f, p[r], cv, mu, eta, alphab, gammab, CHUNKED);
                    if (!valid[r]) d = SlotBwd{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    const float al = valid[r] ? f.alpha : 0.f, ga = valid[r] ? f.gamma : 0.f;
#pragma unroll
                    for (int k = 0; k < EPL; ++k) {
                        const float g = fmaf(qv, yb[k], gb[r][k]);
                        const float z = CHUNKED ? s0[r][k] : sp[r][k];
                        dxp[k] = fmaf(ga, g, fmaf(d.pb, z, fmaf(2.f * d.xxb, xv[k], dxp[k])));
                        float ng = al * g;
                        if constexpr (!CHUNKED) ng = fmaf(d.pb, xv[k], fmaf(2.f * d.n2b, sp[r][k], ng));
                        else acc[r][k] = fmaf(d.pb, xv[k], acc[r][k]);
                        gb[r][k] = ng;
                    }
                    if constexpr (CHUNKED) n2acc[r] += d.n2b;
                    mub += d.mub;
                    etab += d.etab;
                    if (valid[r] && j == 0) {
                        a.dq[bth * m + slot[r]] = qb;
                        a.dc[bth * m + slot[r]] = d.cb;
                    }
                }
                if constexpr (CHUNKED) {
                    if (t % a.chunk == 0) {  // the chunk-start slot is also s_{t-1}
#pragma unroll
                        for (int r = 0; r < RQ; ++r) {
#pragma unroll
                            for (int k = 0; k < EPL; ++k) {
                                gb[r][k] += fmaf(2.f * n2acc[r], s0[r][k], acc[r][k]);
                                acc[r][k] = 0.f;
                            }
                            n2acc[r] = 0.f;
                        }
                    }
                }
                // per-warp partials of the slot sums
                warp_octets_sum_store<D>(dxp, dx_buf + ((size_t)tok * NW + warp) * D, lane);
                mub += __shfl_xor_sync(0xffffffffu, mub, 8);
                mub += __shfl_xor_sync(0xffffffffu, mub, 16);
                etab += __shfl_xor_sync(0xffffffffu, etab, 8);
                etab += __shfl_xor_sync(0xffffffffu, etab, 16);
                if (lane == 0) {
                    sc_buf[((size_t)tok * NW + warp) * 2] = mub;
                    sc_buf[((size_t)tok * NW + warp) * 2 + 1] = etab;
                }
            }
            __syncthreads();
            if (G == 1) {  // fixed-order sums over the warps, straight to the outputs
                for (int idx = tid; idx < n * D; idx += NT) {
                    const int tok = idx / D, k = idx - tok * D;
                    float v = 0.f;
                    for (int w = 0; w < NW; ++w) v += dx_buf[((size_t)tok * NW + w) * D + k];
                    a.dx[(((size_t)b * T + t0 + tok) * H + h) * D + k] = v;
                }
                for (int idx = tid; idx < n * 2; idx += NT) {
                    const int tok = idx >> 1, which = idx & 1;
                    float v = 0.f;
                    for (int w = 0; w < NW; ++w) v += sc_buf[((size_t)tok * NW + w) * 2 + which];
                    const size_t bth = ((size_t)b * T + t0 + tok) * H + h;
                    if (which == 0) a.dmu[bth] = v;
                    else if (a.deta) a.deta[bth] = v;
                }
            } else {
                // this CTA's sums over its warps (fixed order) ...
                float* part = cta_part + (size_t)(pbuf & 1) * TB * (D + 2);
                for (int idx = tid; idx < n * (D + 2); idx += NT) {
                    const int tok = idx / (D + 2), k = idx - tok * (D + 2);
                    float v = 0.f;
                    if (k < D) for (int w = 0; w < NW; ++w) v += dx_buf[((size_t)tok * NW + w) * D + k];
                    else for (int w = 0; w < NW; ++w) v += sc_buf[((size_t)tok * NW + w) * 2 + (k - D)];
                    part[idx] = v;
                }
                bwd_cluster_sync();  // every CTA's partials of this block are in place
                // ... then the cluster's sum (ranks in order), each CTA a share of the entries.
                // The partial buffers alternate, so the next block writes the other one while
                // peers may still read this one; the next cluster barrier orders the reuse.
                for (int idx = crank * NT + tid; idx < n * (D + 2); idx += G * NT) {
                    const int tok = idx / (D + 2), k = idx - tok * (D + 2);
                    float pv[8];  // every peer's load in flight before the fixed-order sum
#pragma unroll
                    for (int r = 0; r < 8; ++r) pv[r] = r < G ? bwd_ld_peer(part + idx, (uint32_t)r) : 0.f;
                    float v = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r) if (r < G) v += pv[r];
                    const size_t bth = ((size_t)b * T + t0 + tok) * H + h;
                    if (k < D) a.dx[bth * D + k] = v;
                    else if (k == D) a.dmu[bth] = v;
                    else if (a.deta) a.deta[bth] = v;
                }
                ++pbuf;
            }
            if (n1 > 0) put((kb + 1) & 1, n1);
            __syncthreads();  // next block's records in place; dx_buf free
        }
    }
    if (G > 1) bwd_cluster_sync();  // no CTA leaves while a peer may still read its partials
    store_state(a.dS0 + (size_t)bh * m * D, gb);
}

}  // namespace lattice
