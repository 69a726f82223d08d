// common.cuh -- device helpers shared by the Lattice kernels (sm_100a).
//
// Slot layout on CUDA cores ("octet" layout): a slot s_i in R^D is held by 8
// consecutive lanes of a warp; a warp therefore holds 4 slots at once (one per
// octet). Lane j (0..7) of an octet owns EPL = D/8 elements, in VW-wide
// vectors: element k of the lane lives at position VW*(j + 8*(k/VW)) + k%VW.
// With this interleave, vector r of the 8 lanes covers one contiguous span of
// 8*VW elements, so a row load or store is fully coalesced, and a dot product
// over the slot is a lane-local sum followed by a 3-level octet shuffle.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lattice {

// Device status word: set by kernels that gave up a bounded wait.
__device__ unsigned int g_device_status = 0;
constexpr unsigned int kStatusTimeout = 1u;

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_device_status, kStatusTimeout); }

// Reads, and zeroes when set, this translation unit's copy of the status word: every
// translation unit of the library is a module of its own with its own copy, so the C
// ABI asks each unit in turn.
static inline cudaError_t read_clear_module_status(unsigned int* v) {
    unsigned int zero = 0;
    *v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_device_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
    return e;
}

template <int D>
struct Octet {
    static_assert(D == 16 || D == 32 || D == 64 || D == 128, "D must be 16, 32, 64 or 128");
    static constexpr int EPL = D / 8;                 // elements per lane
    static constexpr int VW = EPL >= 4 ? 4 : EPL;     // vector width
    static constexpr int NV = EPL / VW;               // vectors per lane
    __device__ __forceinline__ static int pos(int j, int k) {
        return VW * (j + 8 * (k / VW)) + (k % VW);
    }
};

// Load the lane's EPL elements of a D-vector of fp32.
template <int D>
__device__ __forceinline__ void load_row_f32(const float* __restrict__ row, int j, float* v) {
    using O = Octet<D>;
#pragma unroll
    for (int r = 0; r < O::NV; ++r) {
        const float* p = row + O::VW * (j + 8 * r);
        if constexpr (O::VW == 4) {
            float4 t = *reinterpret_cast<const float4*>(p);
            v[4 * r] = t.x; v[4 * r + 1] = t.y; v[4 * r + 2] = t.z; v[4 * r + 3] = t.w;
        } else {
            float2 t = *reinterpret_cast<const float2*>(p);
            v[2 * r] = t.x; v[2 * r + 1] = t.y;
        }
    }
}

// Streaming (evict-first) variant for state rows read once per call.
template <int D>
__device__ __forceinline__ void load_row_f32_stream(const float* row, int j, float* v) {
    using O = Octet<D>;
#pragma unroll
    for (int r = 0; r < O::NV; ++r) {
        const float* p = row + O::VW * (j + 8 * r);
        if constexpr (O::VW == 4) {
            float4 t = __ldcs(reinterpret_cast<const float4*>(p));
            v[4 * r] = t.x; v[4 * r + 1] = t.y; v[4 * r + 2] = t.z; v[4 * r + 3] = t.w;
        } else {
            float2 t = __ldcs(reinterpret_cast<const float2*>(p));
            v[2 * r] = t.x; v[2 * r + 1] = t.y;
        }
    }
}

template <int D, bool STREAM>
__device__ __forceinline__ void store_row_f32(float* row, int j, const float* v) {
    using O = Octet<D>;
#pragma unroll
    for (int r = 0; r < O::NV; ++r) {
        float* p = row + O::VW * (j + 8 * r);
        if constexpr (O::VW == 4) {
            float4 t = make_float4(v[4 * r], v[4 * r + 1], v[4 * r + 2], v[4 * r + 3]);
            if constexpr (STREAM) __stcs(reinterpret_cast<float4*>(p), t);
            else *reinterpret_cast<float4*>(p) = t;
        } else {
            float2 t = make_float2(v[2 * r], v[2 * r + 1]);
            if constexpr (STREAM) __stcs(reinterpret_cast<float2*>(p), t);
            else *reinterpret_cast<float2*>(p) = t;
        }
    }
}

// Load the lane's elements of a D-vector stored as bf16 or fp32 (global or shared).
template <int D>
__device__ __forceinline__ void load_row_any(const void* row, bool bf16, int j, float* v) {
    using O = Octet<D>;
    if (!bf16) {
        load_row_f32<D>(static_cast<const float*>(row), j, v);
        return;
    }
    const __nv_bfloat16* b = static_cast<const __nv_bfloat16*>(row);
#pragma unroll
    for (int r = 0; r < O::NV; ++r) {
        const __nv_bfloat16* p = b + O::VW * (j + 8 * r);
        if constexpr (O::VW == 4) {
            uint2 t = *reinterpret_cast<const uint2*>(p);
            v[4 * r + 0] = __uint_as_float(t.x << 16);
            v[4 * r + 1] = __uint_as_float(t.x & 0xffff0000u);
            v[4 * r + 2] = __uint_as_float(t.y << 16);
            v[4 * r + 3] = __uint_as_float(t.y & 0xffff0000u);
        } else {
            uint32_t t = *reinterpret_cast<const uint32_t*>(p);
            v[2 * r + 0] = __uint_as_float(t << 16);
            v[2 * r + 1] = __uint_as_float(t & 0xffff0000u);
        }
    }
}

__device__ __forceinline__ float load_elem(const void* base, bool bf16, size_t i) {
    if (bf16) {
        uint16_t u = static_cast<const uint16_t*>(base)[i];
        return __uint_as_float(static_cast<uint32_t>(u) << 16);
    }
    return static_cast<const float*>(base)[i];
}

__device__ __forceinline__ float octet_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

// Reconstruction objective ("Lattice: Learning to Efficiently Compress the
// Memory", §3.1.1 eq. decoding_recurrence): the write direction is -e with
// e = sum_i c_i s_i/|s_i| - x. This is the warp's share of sum_i f_i s_i
// (f_i = c_i/|s_i|) over the slots it holds, summed over its four octets, so
// every octet ends with the warp's partial for its lane's element positions.
template <int D, int RQ>
__device__ __forceinline__ void recon_warp_partial(const float (*s)[Octet<D>::EPL], const float* f,
                                                   float* rp) {
    constexpr int EPL = Octet<D>::EPL;
#pragma unroll
    for (int k = 0; k < EPL; ++k) rp[k] = 0.f;
#pragma unroll
    for (int r = 0; r < RQ; ++r)
#pragma unroll
        for (int k = 0; k < EPL; ++k) rp[k] = fmaf(f[r], s[r][k], rp[k]);
#pragma unroll
    for (int k = 0; k < EPL; ++k) {
        rp[k] += __shfl_xor_sync(0xffffffffu, rp[k], 8);
        rp[k] += __shfl_xor_sync(0xffffffffu, rp[k], 16);
    }
}

// Per-slot update coefficients. The new slot is alpha*s + gamma*x.
//   n2 = |s_ref|^2, p = s_ref . x, xx = |x|^2 (s_ref = current slot for the exact
//   recurrence, chunk-start slot for the chunked form).
//   w = (mu - a p/n2) s + a x with a = eta c / n; |w|^2 = mu^2 n2 + a^2 (xx - p^2/n2)
//   (Pythagoras: the write is orthogonal to s_ref). The result is scaled to norm
//   `target` (1 for the exact recurrence's unit sphere, |s0| for the chunked
//   form's normaliser). Zero-norm updates keep the slot.
// PRECISE selects correctly rounded reciprocal square root and division. The
// chunked form carries each slot's norm from chunk to chunk without restoring
// it, so a systematic one-ulp bias in the normaliser accumulates linearly over
// the sequence (about 6e-3 after 65536 tokens); the exact recurrence projects
// onto the unit sphere every token and can use the fast approximations.
template <bool PRECISE>
__device__ __forceinline__ void update_coefs(float n2, float p, float xx, float c, float mu,
                                             float eta, float target, float& alpha,
                                             float& gamma) {
    bool ok = n2 > 0.f;
    float n2s = ok ? n2 : 1.f;
    float inv_n = PRECISE ? __frsqrt_rn(n2s) : rsqrtf(n2s);
    float r = PRECISE ? __fdiv_rn(p, n2s) : __fdividef(p, n2s);  // p / n^2
    float a = eta * c * inv_n;              // eta c / n
    float perp2 = fmaxf(fmaf(-p, r, xx), 0.f);  // |x_perp|^2
    float w2 = fmaf(a * a, perp2, mu * mu * n2s);
    ok = ok && (w2 > 0.f);
    float iw = (PRECISE ? __frsqrt_rn(ok ? w2 : 1.f) : rsqrtf(ok ? w2 : 1.f)) * target;
    alpha = ok ? fmaf(-a, r, mu) * iw : 1.f;
    gamma = ok ? a * iw : 0.f;
}

// As update_coefs, with |x_perp|^2 = |x - (p/n2) s_ref|^2 given, summed directly over
// the elements instead of as xx - p^2/n2. The reconstruction objective's write
// direction can be long and nearly parallel to a slot (|x|^2 ~ 1e4 against
// |x_perp|^2 ~ 4), where that difference cancels away most of fp32's digits.
template <bool PRECISE>
__device__ __forceinline__ void update_coefs_perp(float n2, float p, float perp2, float c, float mu,
                                                  float eta, float target, float& alpha,
                                                  float& gamma) {
    bool ok = n2 > 0.f;
    float n2s = ok ? n2 : 1.f;
    float inv_n = PRECISE ? __frsqrt_rn(n2s) : rsqrtf(n2s);
    float r = PRECISE ? __fdiv_rn(p, n2s) : __fdividef(p, n2s);
    float a = eta * c * inv_n;
    float w2 = fmaf(a * a, perp2, mu * mu * n2s);
    ok = ok && (w2 > 0.f);
    float iw = (PRECISE ? __frsqrt_rn(ok ? w2 : 1.f) : rsqrtf(ok ? w2 : 1.f)) * target;
    alpha = ok ? fmaf(-a, r, mu) * iw : 1.f;
    gamma = ok ? a * iw : 0.f;
}

// The lane's share of |x - (p/n2) s|^2 (octet-summed by the caller).
template <int EPL>
__device__ __forceinline__ float perp2_partial(const float* x, const float* s, float p, float n2) {
    const float r = n2 > 0.f ? __fdiv_rn(p, n2) : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < EPL; ++k) {
        const float u = fmaf(-r, s[k], x[k]);
        acc = fmaf(u, u, acc);
    }
    return acc;
}

// As update_coefs_lin1, with |x_perp|^2 given (see update_coefs_perp).
template <bool PRECISE>
__device__ __forceinline__ void update_coefs_lin1_perp(float n2, float p, float perp2, float c, float mu,
                                                       float eta, float target, float& alpha_s,
                                                       float& alpha_0, float& gamma) {
    bool ok = n2 > 0.f;
    float n2s = ok ? n2 : 1.f;
    float inv_n = PRECISE ? __frsqrt_rn(n2s) : rsqrtf(n2s);
    float r = PRECISE ? __fdiv_rn(p, n2s) : __fdividef(p, n2s);
    float a = eta * c * inv_n;
    float w2 = fmaf(a * a, perp2, mu * mu * n2s);
    ok = ok && (w2 > 0.f);
    float iw = (PRECISE ? __frsqrt_rn(ok ? w2 : 1.f) : rsqrtf(ok ? w2 : 1.f)) * target;
    alpha_s = ok ? mu * iw : 1.f;
    alpha_0 = ok ? -a * r * iw : 0.f;
    gamma = ok ? a * iw : 0.f;
}

// As update_coefs, split for the chunk linearisation of eq. recurrence_linear1
// (§3.4.1): the new slot is alpha_s*s + alpha_0*s0 + gamma*x, where the forget part
// mu scales the running slot s and the projection part (-a p/n^2) the chunk-start
// slot s0 (alpha_s + alpha_0 is update_coefs' alpha).
template <bool PRECISE>
__device__ __forceinline__ void update_coefs_lin1(float n2, float p, float xx, float c, float mu,
                                                  float eta, float target, float& alpha_s,
                                                  float& alpha_0, float& gamma) {
    bool ok = n2 > 0.f;
    float n2s = ok ? n2 : 1.f;
    float inv_n = PRECISE ? __frsqrt_rn(n2s) : rsqrtf(n2s);
    float r = PRECISE ? __fdiv_rn(p, n2s) : __fdividef(p, n2s);
    float a = eta * c * inv_n;
    float perp2 = fmaxf(fmaf(-p, r, xx), 0.f);
    float w2 = fmaf(a * a, perp2, mu * mu * n2s);
    ok = ok && (w2 > 0.f);
    float iw = (PRECISE ? __frsqrt_rn(ok ? w2 : 1.f) : rsqrtf(ok ? w2 : 1.f)) * target;
    alpha_s = ok ? mu * iw : 1.f;
    alpha_0 = ok ? -a * r * iw : 0.f;
    gamma = ok ? a * iw : 0.f;
}

}  // namespace lattice
