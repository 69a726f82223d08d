// step.cuh -- decode step and read-out kernels (CUDA cores, HBM-bound).
//
// Decode step: one new token per (b, h); the state row of every slot is read
// from HBM, updated by the exact recurrence (§3.1.1 eq. OSR, §3.2 unit-sphere
// projection, §3.3 forget gate, §3.4 Eq. 14 projection) and written back in
// place; y = sum_i q_i s_i uses the updated slots. The state (2 * 4 * m * d
// bytes of traffic per head) dominates, so each lane issues all of its
// streaming 16-byte loads before any arithmetic.
#pragma once
#include "args.h"
#include "common.cuh"
#include "tc_ptx.cuh"
#include "waits.cuh"

namespace lattice {


// The step of one head, after its state rows (s), input (xv), mu and eta are in
// registers; cv(r) and qv(r) give the intensity and query of the lane's slot r (from
// registers, or read where they are needed): the update of every slot, written back
// to Sbh, and y. NW warps, RQ slot quads per warp (4*NW*RQ >= m), lane layout as in
// common.cuh. DEC selects the reconstruction objective (§3.1.1 eq.
// decoding_recurrence): the write direction is x - sum_i (c_i/|s_i|) s_i, from the
// state before the step. Uses ysm (and esm) in shared memory; ends after a CTA
// barrier, with ysm read by the final sum.
template <int D, int RQ, bool DEC, class CV, class QV>
__device__ __forceinline__ void step_head(float (&s)[RQ][Octet<D>::EPL], float (&xv)[Octet<D>::EPL],
                                          CV cv, QV qv, float mu, float eta,
                                          float* Sbh, const int (&slot)[RQ], int m, float (*ysm)[D],
                                          float* esm, float* y) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    const int NW = blockDim.x >> 5;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    float p[RQ], n2[RQ];
    if constexpr (DEC) {  // x <- x - sum_i (c_i/|s_i|) s_i over every slot of the CTA
        // |s_i|^2 (kept for the update: the slots do not change before it), two partial
        // sums per lane to halve the dependent chain
        float f[RQ], rp[EPL];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            float n0 = 0.f, n1 = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; k += 2) {
                n0 = fmaf(s[r][k], s[r][k], n0);
                n1 = fmaf(s[r][k + 1], s[r][k + 1], n1);
            }
            n2[r] = n0 + n1;
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1)
#pragma unroll
            for (int r = 0; r < RQ; ++r) n2[r] += __shfl_xor_sync(0xffffffffu, n2[r], o);
        // c_i / |s_i| with a Newton-refined reciprocal square root (within 2 ulp): the slots
        // are renormalised to the unit sphere by this very step, so no bias accumulates
#pragma unroll
        for (int r = 0; r < RQ; ++r) f[r] = n2[r] > 0.f ? cv(r) * ptx::rsqrt_nr(n2[r]) : 0.f;
        recon_warp_partial<D, RQ>(s, f, rp);
        if (oct == 0) {
#pragma unroll
            for (int k = 0; k < EPL; ++k) ysm[warp][O::pos(j, k)] = rp[k];
        }
        __syncthreads();
        // one thread per element sums the warps (fixed order) and forms x - sum ...
        for (int e = tid; e < D; e += blockDim.x) {
            float acc = 0.f;
            for (int w = 0; w < NW; ++w) acc += ysm[w][e];
            esm[e] = acc;
        }
        __syncthreads();  // ... which every lane then reads (ysm is free for the read-out)
#pragma unroll
        for (int k = 0; k < EPL; ++k) xv[k] -= esm[O::pos(j, k)];
    }
    float xx = 0.f;
    if constexpr (DEC) {
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            float p0 = 0.f, p1 = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; k += 2) {
                p0 = fmaf(s[r][k], xv[k], p0);
                p1 = fmaf(s[r][k + 1], xv[k + 1], p1);
            }
            p[r] = p0 + p1;
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1)
#pragma unroll
            for (int r = 0; r < RQ; ++r) p[r] += __shfl_xor_sync(0xffffffffu, p[r], o);
    } else {
#pragma unroll
        for (int k = 0; k < EPL; ++k) xx = fmaf(xv[k], xv[k], xx);
        xx = octet_sum(xx);
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            float pp = 0.f, nn = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; ++k) {
                pp = fmaf(s[r][k], xv[k], pp);
                nn = fmaf(s[r][k], s[r][k], nn);
            }
            p[r] = pp;
            n2[r] = nn;
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                p[r] += __shfl_xor_sync(0xffffffffu, p[r], o);
                n2[r] += __shfl_xor_sync(0xffffffffu, n2[r], o);
            }
        }
    }
    float pp2[RQ];  // DEC: |x - (p/n2) s|^2 per slot, all slots' octet sums interleaved
    if constexpr (DEC) {
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            const float rr = n2[r] > 0.f ? p[r] * ptx::rcp_nr(n2[r]) : 0.f;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; k += 2) {
                const float u0 = fmaf(-rr, s[r][k], xv[k]);
                const float u1 = fmaf(-rr, s[r][k + 1], xv[k + 1]);
                a0 = fmaf(u0, u0, a0);
                a1 = fmaf(u1, u1, a1);
            }
            pp2[r] = a0 + a1;
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1)
#pragma unroll
            for (int r = 0; r < RQ; ++r) pp2[r] += __shfl_xor_sync(0xffffffffu, pp2[r], o);
    }
    float yp[EPL];
#pragma unroll
    for (int k = 0; k < EPL; ++k) yp[k] = 0.f;
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        float alpha, gamma;
        if constexpr (DEC) {  // |x_perp|^2 summed directly: the residual can be near a slot
            update_coefs_perp<false>(n2[r], p[r], pp2[r], cv(r), mu, eta, 1.f, alpha, gamma);
        } else {
            update_coefs<false>(n2[r], p[r], xx, cv(r), mu, eta, 1.f, alpha, gamma);
        }
        const float qr = qv(r);
#pragma unroll
        for (int k = 0; k < EPL; ++k) {
            s[r][k] = fmaf(alpha, s[r][k], gamma * xv[k]);
            yp[k] = fmaf(qr, s[r][k], yp[k]);
        }
        if (slot[r] < m) store_row_f32<D, true>(Sbh + (size_t)slot[r] * D, j, s[r]);
    }
    // read-out: octets of the warp, then warps (fixed order)
#pragma unroll
    for (int k = 0; k < EPL; ++k) {
        yp[k] += __shfl_xor_sync(0xffffffffu, yp[k], 8);
        yp[k] += __shfl_xor_sync(0xffffffffu, yp[k], 16);
    }
    if (oct == 0) {
#pragma unroll
        for (int k = 0; k < EPL; ++k) ysm[warp][O::pos(j, k)] = yp[k];
    }
    __syncthreads();
    for (int k = tid; k < D; k += blockDim.x) {
        float acc = 0.f;
        for (int w = 0; w < NW; ++w) acc += ysm[w][k];
        y[k] = acc;
    }
}

// One CTA per (b, h): every lane issues all of its streaming 16-byte state loads
// first, then runs step_head.
template <int D, int RQ, bool DEC>
__global__ void __launch_bounds__(512) step_kernel(StepArgs a) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    __shared__ __align__(16) float ysm[16][D];
    __shared__ __align__(16) float esm[DEC ? D : 1];  // DEC: the token's write direction
    const int NW = blockDim.x >> 5;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    const size_t bh = blockIdx.x;
    const int m = a.m;
    float* Sbh = a.S + bh * (size_t)m * D;

    float s[RQ][EPL];
    int slot[RQ];
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        slot[r] = 4 * (warp + NW * r) + oct;
        if (slot[r] < m) load_row_f32_stream<D>(Sbh + (size_t)slot[r] * D, j, s[r]);
        else {
#pragma unroll
            for (int k = 0; k < EPL; ++k) s[r][k] = 0.f;
        }
    }
    float xv[EPL];
    if (a.x_bf16) load_row_any<D>(static_cast<const __nv_bfloat16*>(a.x) + bh * D, true, j, xv);
    else load_row_any<D>(static_cast<const float*>(a.x) + bh * D, false, j, xv);
    const float mu = a.mu[bh];
    const float eta = a.eta ? a.eta[bh] : 1.f;
    float cv[RQ], qv[RQ];
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        const bool valid = slot[r] < m;
        cv[r] = valid ? a.c[bh * m + slot[r]] : 0.f;
        qv[r] = valid ? load_elem(a.q, a.q_bf16, bh * m + slot[r]) : 0.f;
    }
    step_head<D, RQ, DEC>(s, xv, [&](int r) { return cv[r]; }, [&](int r) { return qv[r]; }, mu, eta, Sbh,
                          slot, m, ysm, esm, a.y + bh * D);
}

// Persistent form: a grid of G CTAs (as many as fit: two per SM at m = d = 128), CTA g
// taking heads g, g+G, ... While a CTA computes one head from registers, the copy
// engine already brings the next head's state (m*D*4 bytes, one bulk copy per 16 KB)
// into its shared memory, and per-thread asynchronous copies bring that head's x, c,
// q, mu and eta. So every CTA keeps a state load in flight through its arithmetic,
// which the one-CTA-per-head kernel cannot: there the SM's loads stop whenever both
// resident CTAs compute, which bounds the reconstruction objective's longer
// arithmetic. Needs S and x 16-byte aligned (the ABI requires both). The wait on each
// copy is bounded (waits.cuh): on timeout the CTA stops taking heads and still drains
// its copy.
struct StepPfLayout {
    // [state: m*D fp32][small inputs, two sets by head parity: x | c | q | mu, eta]
    uint32_t state_bytes, x_off, c_off, q_off, mu_off, small_bytes, bytes;
    __host__ __device__ StepPfLayout(int m, int D, bool x_bf16) {
        state_bytes = (uint32_t)m * D * 4;
        x_off = 0;
        c_off = (uint32_t)D * (x_bf16 ? 2 : 4);
        q_off = (c_off + (uint32_t)m * 4 + 15) & ~15u;
        mu_off = (q_off + (uint32_t)m * 4 + 15) & ~15u;  // room for fp32 q
        small_bytes = mu_off + 16;
        bytes = state_bytes + 2 * small_bytes;
    }
};

template <int D, int RQ, bool DEC>
__global__ void __launch_bounds__(512) step_pf_kernel(StepArgs a) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    __shared__ __align__(16) float ysm[16][D];
    __shared__ __align__(16) float esm[DEC ? D : 1];
    __shared__ __align__(8) uint64_t bar_mem;
    __shared__ uint32_t abort_mem;
    extern __shared__ __align__(128) uint8_t buf[];
    const int NW = blockDim.x >> 5;
    const int nthr = blockDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    const int m = a.m;
    const int nheads = a.B * a.H;
    const StepPfLayout L(m, D, a.x_bf16);
    const uint32_t bar = ptx::smem_u32(&bar_mem);
    volatile uint32_t* abort = &abort_mem;
    const uint32_t sbuf = ptx::smem_u32(buf);
    const uint32_t xbytes = (uint32_t)D * (a.x_bf16 ? 2 : 4);
    // q rides along in 4-byte pieces when its rows are 4-byte aligned, else it is read
    // from global memory where it is needed
    const uint32_t qrow = (uint32_t)m * (a.q_bf16 ? 2 : 4);
    const bool q_smem = ((reinterpret_cast<uintptr_t>(a.q) & 3u) == 0) && (qrow & 3u) == 0;

    // head bh (the it-th of this CTA): its state by bulk copies (thread 0) into the state
    // buffer, its x (16-byte pieces), c, q, mu and eta (4-byte pieces) by per-thread copies
    // into small-input set it % 2, which stays readable while the next head's copies land
    auto prefetch = [&](int bh, int it) {
        if (tid == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            ptx::mbar_arrive_expect_tx(bar, L.state_bytes);
            const uint8_t* src = reinterpret_cast<const uint8_t*>(a.S + (size_t)bh * m * D);
            for (uint32_t o = 0; o < L.state_bytes; o += 16384u) {
                const uint32_t n = L.state_bytes - o < 16384u ? L.state_bytes - o : 16384u;
                ptx::bulk_load_g2s(sbuf + o, src + o, n, bar, pol);
            }
        }
        const uint32_t sm = sbuf + L.state_bytes + (it & 1) * L.small_bytes;
        const uint8_t* xs = static_cast<const uint8_t*>(a.x) + (size_t)bh * xbytes;
        for (uint32_t o = 16u * tid; o < xbytes; o += 16u * nthr) ptx::cp_async16(sm + L.x_off + o, xs + o);
        for (int i = tid; i < m; i += nthr) ptx::cp_async4(sm + L.c_off + 4 * i, a.c + (size_t)bh * m + i);
        if (q_smem) {
            const uint8_t* qs = static_cast<const uint8_t*>(a.q) + (size_t)bh * qrow;
            for (uint32_t o = 4u * tid; o < qrow; o += 4u * nthr) ptx::cp_async4(sm + L.q_off + o, qs + o);
        }
        if (tid == 0) ptx::cp_async4(sm + L.mu_off, a.mu + bh);
        if (tid == 1 && a.eta) ptx::cp_async4(sm + L.mu_off + 4, a.eta + bh);
        ptx::cp_async_commit();
    };

    int slot[RQ];
#pragma unroll
    for (int r = 0; r < RQ; ++r) slot[r] = 4 * (warp + NW * r) + oct;
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        abort_mem = 0u;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int it = 0;
    bool pending = false;  // a bulk copy issued whose completion no thread has seen yet
    if ((int)blockIdx.x < nheads) {
        prefetch(blockIdx.x, 0);
        pending = true;
    }
    for (int bh = blockIdx.x; bh < nheads; bh += gridDim.x, ++it) {
        tc_wait(bar, it & 1, abort);
        ptx::cp_async_wait_all();
        __syncthreads();  // every thread's small copies landed; abort is settled
        if (*abort) break;
        pending = false;
        const uint8_t* sm = buf + L.state_bytes + (it & 1) * L.small_bytes;
        float s[RQ][EPL], xv[EPL];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            if (slot[r] < m) load_row_f32<D>(reinterpret_cast<const float*>(buf) + (size_t)slot[r] * D, j, s[r]);
            else {
#pragma unroll
                for (int k = 0; k < EPL; ++k) s[r][k] = 0.f;
            }
        }
        load_row_any<D>(sm + L.x_off, a.x_bf16, j, xv);
        const float mu = *reinterpret_cast<const float*>(sm + L.mu_off);
        const float eta = a.eta ? *reinterpret_cast<const float*>(sm + L.mu_off + 4) : 1.f;
        __syncthreads();  // the state buffer is read: the next head's copy may overwrite it
        if (bh + (int)gridDim.x < nheads) {
            prefetch(bh + gridDim.x, it + 1);
            pending = true;
        }
        // c and q are read from this head's small-input set where the arithmetic needs them
        const float* cs = reinterpret_cast<const float*>(sm + L.c_off);
        const size_t qbase = (size_t)bh * m;
        step_head<D, RQ, DEC>(
            s, xv, [&](int r) { return slot[r] < m ? cs[slot[r]] : 0.f; },
            [&](int r) {
                return slot[r] >= m ? 0.f
                                    : (q_smem ? load_elem(sm + L.q_off, a.q_bf16, slot[r])
                                              : load_elem(a.q, a.q_bf16, qbase + slot[r]));
            },
            mu, eta, a.S + (size_t)bh * m * D, slot, m, ysm, esm, a.y + (size_t)bh * D);
    }
    // no copy may still write into shared memory when the CTA retires
    ptx::cp_async_wait_all();
    if (pending && tid == 0) tc_drain(bar, it & 1);
}


// y[b][h][:] = sum_i q_i s_i (§2 eq. LA read-out; Appendix D y = q @ S).
template <int D, int RQ>
__global__ void __launch_bounds__(512) readout_kernel(ReadoutArgs a) {
    using O = Octet<D>;
    constexpr int EPL = O::EPL;
    __shared__ __align__(16) float ysm[16][D];
    const int NW = blockDim.x >> 5;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 7, oct = lane >> 3;
    const size_t bh = blockIdx.x;
    const int m = a.m;
    const float* Sbh = a.S + bh * (size_t)m * D;
    float s[RQ][EPL];
    float qv[RQ];
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        const int slot = 4 * (warp + NW * r) + oct;
        if (slot < m) {
            load_row_f32_stream<D>(Sbh + (size_t)slot * D, j, s[r]);
            qv[r] = load_elem(a.q, a.q_bf16, bh * m + slot);
        } else {
#pragma unroll
            for (int k = 0; k < EPL; ++k) s[r][k] = 0.f;
            qv[r] = 0.f;
        }
    }
    float yp[EPL];
#pragma unroll
    for (int k = 0; k < EPL; ++k) yp[k] = 0.f;
#pragma unroll
    for (int r = 0; r < RQ; ++r)
#pragma unroll
        for (int k = 0; k < EPL; ++k) yp[k] = fmaf(qv[r], s[r][k], yp[k]);
#pragma unroll
    for (int k = 0; k < EPL; ++k) {
        yp[k] += __shfl_xor_sync(0xffffffffu, yp[k], 8);
        yp[k] += __shfl_xor_sync(0xffffffffu, yp[k], 16);
    }
    if (oct == 0) {
#pragma unroll
        for (int k = 0; k < EPL; ++k) ysm[warp][O::pos(j, k)] = yp[k];
    }
    __syncthreads();
    for (int k = tid; k < D; k += blockDim.x) {
        float acc = 0.f;
        for (int w = 0; w < NW; ++w) acc += ysm[w][k];
        a.y[bh * D + k] = acc;
    }
}

}  // namespace lattice
