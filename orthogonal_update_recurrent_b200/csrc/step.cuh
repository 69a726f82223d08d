// step.cuh -- decode step and read-out kernels (CUDA cores, HBM-bound).
//
// Decode step: one new token per (b, h); the state row of every slot is read
// from HBM, updated by the exact recurrence (§3.1.1 eq. OSR, §3.2 unit-sphere
// projection, §3.3 forget gate, §3.4 Eq. 14 projection) and written back in
// place; y = sum_i q_i s_i uses the updated slots. The state (2 * 4 * m * d
// bytes of traffic per head) dominates, so each lane issues all of its
// streaming 16-byte loads before any arithmetic.
#pragma once
#include "common.cuh"

namespace lattice {

struct StepArgs {
    float* S;
    const void* x; bool x_bf16;
    const float* c;
    const void* q; bool q_bf16;
    const float* mu;
    const float* eta;  // may be null
    float* y;
    int B, H, m;
};

// One CTA per (b, h); NW warps, RQ slot quads per warp (4*NW*RQ >= m). DEC selects
// the reconstruction objective (§3.1.1 eq. decoding_recurrence): the write direction
// is x - sum_i (c_i/|s_i|) s_i, from the state before the step.
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
    if constexpr (DEC) {  // x <- x - sum_i (c_i/|s_i|) s_i over every slot of the CTA
        float f[RQ], rp[EPL];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            float nn = 0.f;
#pragma unroll
            for (int k = 0; k < EPL; ++k) nn = fmaf(s[r][k], s[r][k], nn);
            nn = octet_sum(nn);
            f[r] = nn > 0.f ? __fdiv_rn(cv[r], __fsqrt_rn(nn)) : 0.f;
        }
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
#pragma unroll
    for (int k = 0; k < EPL; ++k) xx = fmaf(xv[k], xv[k], xx);
    xx = octet_sum(xx);

    float p[RQ], n2[RQ];
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
    float yp[EPL];
#pragma unroll
    for (int k = 0; k < EPL; ++k) yp[k] = 0.f;
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
        float alpha, gamma;
        if constexpr (DEC) {  // |x_perp|^2 summed directly: the residual can be near a slot
            const float pp2 = octet_sum(perp2_partial<EPL>(xv, s[r], p[r], n2[r]));
            update_coefs_perp<true>(n2[r], p[r], pp2, cv[r], mu, eta, 1.f, alpha, gamma);
        } else {
            update_coefs<false>(n2[r], p[r], xx, cv[r], mu, eta, 1.f, alpha, gamma);
        }
#pragma unroll
        for (int k = 0; k < EPL; ++k) {
            s[r][k] = fmaf(alpha, s[r][k], gamma * xv[k]);
            yp[k] = fmaf(qv[r], s[r][k], yp[k]);
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
        a.y[bh * D + k] = acc;
    }
}

struct ReadoutArgs {
    const float* S;
    const void* q; bool q_bf16;
    float* y;
    int B, H, m;
};

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
