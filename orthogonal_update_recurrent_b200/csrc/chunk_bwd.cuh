// chunk_bwd.cuh -- backward pass of the chunked recurrence (Eq. 17) in chunk-parallel
// form, one cluster of CTAs per sequence: the matrix products on the tensor cores
// (tf32 with a hi/lo split of each operand), the rest in fp32 on CUDA cores.
//
// Reverse-mode derivative of the forward of "Lattice: Learning to Efficiently
// Compress the Memory" §3.4.1 Eq. 17 with the chunk normaliser of eq. beta_chunk
// (Appendix B.1), for the loss L = sum_t dy_t.y_t + dS_T.S_T. The pages print no
// backward; this is the derivative of their forward, arranged so that only the state
// adjoint crosses chunk boundaries. Inside a chunk of L tokens with chunk-start state
// S0, each (token t, slot i) has gates g, kappa that depend on S0 and the token alone:
//   s_t,i = g_t,i s_t-1,i + kappa_t,i h_t,   h_t = -x_t,   y_t = sum_i q_t,i s_t,i.
// With D_i[k][t] = prod_{l=t+1..k} g_l,i, the prefix A_t,i = prod_{l<=t} g_l,i, the
// suffix U_t,i = prod_{l>t} g_l,i and dS, the adjoint of the chunk-end state s_L:
//   dq_t,i     = A_t,i (dy_t.s0_i) + sum_{j<=t} D_i[t][j] kappa_j,i (dy_t.h_j)
//   dkappa_t,i = U_t,i (h_t.dS_i) + sum_{k>=t} D_i[k][t] q_k,i (h_t.dy_k)
//   g_t,i dg_t,i = s_L,i.dS_i + sum_{k>=t} (q_k,i dq_k,i - kappa_k,i dkappa_k,i)
// The last line is the log-derivative identity of a gated linear recurrence (dg is
// the running state before the token dotted with the adjoint after it). The gates'
// own derivative, through hdot = h.s0_i, |h|^2, |s0_i|^2, c, mu and eta, follows per
// (token, slot), and then
//   dx_t = -sum_{k>=t} P[k][t] dy_k - sum_i kappa_t,i U_t,i dS_i
//          - sum_i dhdot_t,i s0_i + 2 (sum_i d|h|^2_t,i) x_t,
//   P[k][t] = sum_i q_k,i kappa_t,i D_i[k][t]       (the chunk's causal scores),
//   dS_prev,i = A_L,i dS_i + sum_t A_t,i q_t,i dy_t - sum_t dhdot_t,i x_t
//               + 2 (sum_t d|s0|^2_t,i) s0_i,
// the adjoint carried into the previous chunk. Every product of gates is formed
// directly, never as a quotient of products; the one division is dg = (g dg) / g.
//
// Layout: a sequence's slots are split over a cluster of G = ceil(m/16) CTAs of 512
// threads, 16 slots each. Under the similarity objective the slots evolve
// independently, so the chain from chunk to chunk stays inside each CTA; only the
// token-indexed sums over slots (dx, dmu, deta) cross CTAs, added through distributed
// shared memory in rank order (bit-reproducible). A forward sweep first stores each
// chunk's start state in the workspace; the backward sweep then walks the chunks in
// reverse, loading each chunk's inputs and start state into registers while the chunk
// after it finishes. Thread roles inside a phase:
//   pairs      thread -> (token tid/16 and tid/16 + 32, slot tid%16)
//   slot warps warp w -> slot w; lane -> tokens 2l, 2l+1 (scans) or D/32 state columns
//   MMA tiles  warp w -> 16x16 / 16xD/4 / 16x8 output tiles of the matrix products, on
//              the tensor cores (mma.sync, tf32 with a hi/lo split: about fp32 accuracy)
#pragma once
#include "args.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace lattice {

template <int D>
struct CbLayout {
    static constexpr int XS = D + 4;              // row stride, [token][D] and [slot][D]
    static constexpr int PS = kCbMaxL + 8;        // row stride, [token][token] and [slot][token]
    static constexpr int TS = kCbSlots + 1;       // row stride, [token][slot]
    static constexpr int TSA = kCbMaxL * TS;
    static constexpr int X = 0;                   // x of the chunk (fp32)
    static constexpr int DY = X + kCbMaxL * XS;   // dy
    static constexpr int DX = DY + kCbMaxL * XS;  // this CTA's share of dx
    static constexpr int SA = DX + kCbMaxL * XS;  // two state buffers (start / end of chunk)
    static constexpr int SB = SA + kCbSlots * XS;
    static constexpr int DS = SB + kCbSlots * XS; // adjoint of the chunk-end state
    static constexpr int M2 = DS + kCbSlots * XS; // [t][j] dy_t.h_j (lower triangle); later [i][D] scratch
    static constexpr int P = M2 + kCbMaxL * PS;   // [k][t] causal scores
    static constexpr int KST = P + kCbMaxL * PS;  // [i][t] kappa U
    static constexpr int AQT = KST + kCbSlots * PS;  // [i][t] A q
    static constexpr int HBT = AQT + kCbSlots * PS;  // [i][t] d hdot
    static constexpr int CC = HBT + kCbSlots * PS;   // [t][i] arrays from here
    static constexpr int QQ = CC + TSA, GG = QQ + TSA, KT = GG + TSA, M1 = KT + TSA,
                         M3 = M1 + TSA, AA = M3 + TSA, SUF = AA + TSA, DQ = SUF + TSA,
                         DKT = DQ + TSA;
    static constexpr int MU = DKT + TSA, ETA = MU + kCbMaxL, HH = ETA + kCbMaxL,
                         HHB = HH + kCbMaxL, MUB = HHB + kCbMaxL, ETAB = MUB + kCbMaxL;
    static constexpr int N2 = ETAB + kCbMaxL, E0 = N2 + kCbSlots, AL = E0 + kCbSlots;
    // 16-token blocks: q times the in-block prefix of g, kappa times the in-block suffix,
    // and the products of the whole blocks between two blocks (pairs b1 < b2)
    static constexpr int QA = AL + kCbSlots, KU = QA + TSA, W = KU + TSA;
    static constexpr int FLOATS = W + 6 * kCbSlots;
    static constexpr size_t BYTES = (size_t)FLOATS * 4;
    static_assert(BYTES <= 232448, "shared memory per CTA");
    static_assert(X % 4 == 0 && DY % 4 == 0 && DX % 4 == 0 && SA % 4 == 0 && SB % 4 == 0 &&
                      DS % 4 == 0 && P % 4 == 0 && KST % 4 == 0 && AQT % 4 == 0 && HBT % 4 == 0,
                  "16-byte rows");
};

// CPT = D/32 consecutive floats per lane.
template <int N>
__device__ __forceinline__ void cb_ld(const float* p, float* v) {
    if constexpr (N == 4) {
        const float4 t = *reinterpret_cast<const float4*>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (N == 2) {
        const float2 t = *reinterpret_cast<const float2*>(p);
        v[0] = t.x; v[1] = t.y;
    } else {
        v[0] = *p;
    }
}
template <int N>
__device__ __forceinline__ void cb_st(float* p, const float* v) {
    if constexpr (N == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
        *p = v[0];
    }
}

__device__ __forceinline__ float cb_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float cb_half_sum(float v) {  // over the 16 lanes of a half-warp
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Gates of Eq. 17 / eq. beta_chunk for one (token, slot):
//   hhat = hdot/n2, khat = c/sqrt(n2), tt = khat^2 |h|^2 - n2 hhat^2 khat^2,
//   den = mu^2 n2 + eta^2 max(tt, 0), beta = sqrt(n2)/sqrt(den),
//   g = beta (mu + eta hhat khat), kappa = -beta eta khat;
// den == 0 (a zero-norm update) keeps the slot: g = 1, kappa = 0. Reciprocal square
// roots are the hardware approximation with one Newton step (ptx::rsqrt_nr).
__device__ __forceinline__ void cb_gates(float hd, float hh, float n2, float c, float mu, float eta,
                                         float& g, float& kt) {
    const float rn = ptx::rsqrt_nr(n2), r2 = rn * rn;
    const float hhat = hd * r2, khat = c * rn;
    const float tt = khat * khat * hh - n2 * hhat * hhat * khat * khat;
    const float den = mu * mu * n2 + eta * eta * fmaxf(tt, 0.f);
    if (den == 0.f) {
        g = 1.f;
        kt = 0.f;
        return;
    }
    const float beta = n2 * rn * ptx::rsqrt_nr(den);
    g = beta * (mu + eta * hhat * khat);
    kt = -beta * eta * khat;
}

struct CbGateGrad {
    float cb, mub, etab, hdb, hhb, n2b;
};

// Derivative of cb_gates: gb = dL/dg, ktb = dL/dkappa in; the derivatives with respect
// to c, mu, eta, hdot, |h|^2 and n2 out (zero for a kept slot).
__device__ __forceinline__ CbGateGrad cb_gates_bwd(float hd, float hh, float n2, float c, float mu,
                                                   float eta, float gb, float ktb) {
    CbGateGrad r{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float rn = ptx::rsqrt_nr(n2), r2 = rn * rn;   // 1/sqrt(n2), 1/n2
    const float hhat = hd * r2, khat = c * rn;
    const float tt = khat * khat * hh - n2 * hhat * hhat * khat * khat;
    const float ttp = fmaxf(tt, 0.f);
    const float den = mu * mu * n2 + eta * eta * ttp;
    if (den == 0.f) return r;
    const float rd = ptx::rsqrt_nr(den);
    const float beta = n2 * rn * rd;
    // g = beta (mu + eta hhat khat), kappa = -beta eta khat
    const float betab = gb * (mu + eta * hhat * khat) - ktb * eta * khat;
    float mub = gb * beta;
    float etab = gb * beta * hhat * khat - ktb * beta * khat;
    float hhatb = gb * beta * eta * khat;
    float khatb = gb * beta * eta * hhat - ktb * beta * eta;
    // beta = sqrt(n2) den^(-1/2)
    float n2b = 0.5f * betab * beta * r2;
    const float denb = -0.5f * betab * beta * rd * rd;
    // den = mu^2 n2 + eta^2 max(tt, 0)
    mub += denb * 2.f * mu * n2;
    n2b += denb * mu * mu;
    etab += denb * 2.f * eta * ttp;
    const float ttb = tt > 0.f ? denb * eta * eta : 0.f;
    // tt = khat^2 hh - n2 hhat^2 khat^2
    khatb += ttb * (2.f * khat * hh - 2.f * n2 * hhat * hhat * khat);
    r.hhb = ttb * khat * khat;
    n2b -= ttb * hhat * hhat * khat * khat;
    hhatb -= ttb * 2.f * n2 * hhat * khat * khat;
    // khat = c n2^(-1/2), hhat = hdot / n2
    r.cb = khatb * rn;
    n2b -= 0.5f * khatb * c * r2 * rn;
    r.hdb = hhatb * r2;
    n2b -= hhatb * hd * r2 * r2;
    r.mub = mub;
    r.etab = etab;
    r.n2b = n2b;
    return r;
}

// acc[NT][4] += A (16 x K) . B (K x 8NT) on the tensor cores (mma.sync m16n8k8, tf32).
// Each operand is split into its tf32 part and the tf32 remainder, and three MMAs per
// step add lo.hi + hi.lo + hi.hi: products keep about fp32 accuracy. Element (r, k) of A
// is A[r*am + k*ak] and element (k, n) of B is B[k*bk + n*bn], both pointers already at
// the tile's origin; k runs over [k0, k1), a multiple of 8 long. acc[nt] holds rows
// lane/4 and lane/4 + 8, columns 8nt + 2(lane%4) and the next.
template <int NT>
__device__ __forceinline__ void cb_mma(float (&acc)[NT][4], const float* A, int am, int ak,
                                       const float* B, int bk, int bn, int k0, int k1, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll 2
    for (int k = k0; k < k1; k += 8) {
        const float av[4] = {A[g * am + (k + c) * ak], A[(g + 8) * am + (k + c) * ak],
                             A[g * am + (k + c + 4) * ak], A[(g + 8) * am + (k + c + 4) * ak]};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            ah[r] = ptx::cvt_tf32(av[r]);
            al[r] = ptx::cvt_tf32(av[r] - __uint_as_float(ah[r]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float b0 = B[(k + c) * bk + (8 * nt + g) * bn];
            const float b1 = B[(k + c + 4) * bk + (8 * nt + g) * bn];
            const uint32_t bh[2] = {ptx::cvt_tf32(b0), ptx::cvt_tf32(b1)};
            const uint32_t bl[2] = {ptx::cvt_tf32(b0 - __uint_as_float(bh[0])),
                                    ptx::cvt_tf32(b1 - __uint_as_float(bh[1]))};
            ptx::mma_tf32(acc[nt], al, bh);
            ptx::mma_tf32(acc[nt], ah, bl);
            ptx::mma_tf32(acc[nt], ah, bh);
        }
    }
}
// cb_mma with a per-slot scale: SIDE 1 scales A's element (r, k) by scale[k], SIDE 2
// scales B's element (k, n) by scale[8nt + n].
template <int NT, int SIDE>
__device__ __forceinline__ void cb_mma_s(float (&acc)[NT][4], const float* A, int am, int ak,
                                         const float* B, int bk, int bn, int k0, int k1, int lane,
                                         const float* scale) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll 2
    for (int k = k0; k < k1; k += 8) {
        float av[4] = {A[g * am + (k + c) * ak], A[(g + 8) * am + (k + c) * ak],
                       A[g * am + (k + c + 4) * ak], A[(g + 8) * am + (k + c + 4) * ak]};
        if (SIDE == 1) {
            const float s0 = scale[k + c], s1 = scale[k + c + 4];
            av[0] *= s0; av[1] *= s0; av[2] *= s1; av[3] *= s1;
        }
        uint32_t ah[4], al[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            ah[r] = ptx::cvt_tf32(av[r]);
            al[r] = ptx::cvt_tf32(av[r] - __uint_as_float(ah[r]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float b0 = B[(k + c) * bk + (8 * nt + g) * bn];
            float b1 = B[(k + c + 4) * bk + (8 * nt + g) * bn];
            if (SIDE == 2) {
                const float sn = scale[8 * nt + g];
                b0 *= sn; b1 *= sn;
            }
            const uint32_t bh[2] = {ptx::cvt_tf32(b0), ptx::cvt_tf32(b1)};
            const uint32_t bl[2] = {ptx::cvt_tf32(b0 - __uint_as_float(bh[0])),
                                    ptx::cvt_tf32(b1 - __uint_as_float(bh[1]))};
            ptx::mma_tf32(acc[nt], al, bh);
            ptx::mma_tf32(acc[nt], ah, bl);
            ptx::mma_tf32(acc[nt], ah, bh);
        }
    }
}

template <int NT>
__device__ __forceinline__ void cb_zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
}

template <int D>
__global__ void __launch_bounds__(kCbThreads, 1) chunk_bwd_kernel(const BwdArgs a) {
    using Lo = CbLayout<D>;
    constexpr int XS = Lo::XS, PS = Lo::PS, TS = Lo::TS;
    constexpr int CPT = D / 32;   // state columns per lane
    constexpr int DV = D / 4;     // float4s per row
    extern __shared__ __align__(16) float sm[];
    float* sX = sm + Lo::X;
    float* sDY = sm + Lo::DY;
    float* sDX = sm + Lo::DX;
    float* sDS = sm + Lo::DS;
    float* sM2 = sm + Lo::M2;
    float* sP = sm + Lo::P;
    float* sKST = sm + Lo::KST;
    float* sAQT = sm + Lo::AQT;
    float* sHBT = sm + Lo::HBT;
    float* sC = sm + Lo::CC;
    float* sQ = sm + Lo::QQ;
    float* sG = sm + Lo::GG;
    float* sKT = sm + Lo::KT;
    float* sM1 = sm + Lo::M1;   // dy.s0, then dg
    float* sM3 = sm + Lo::M3;   // h.dS
    float* sA = sm + Lo::AA;
    float* sU = sm + Lo::SUF;
    float* sDQ = sm + Lo::DQ;
    float* sDKT = sm + Lo::DKT; // dkappa, then d|s0|^2 per (token, slot)
    float* sMU = sm + Lo::MU;
    float* sETA = sm + Lo::ETA;
    float* sHH = sm + Lo::HH;
    float* sHHB = sm + Lo::HHB;
    float* sMUB = sm + Lo::MUB;
    float* sETAB = sm + Lo::ETAB;
    float* sN2 = sm + Lo::N2;
    float* sE0 = sm + Lo::E0;
    float* sAL = sm + Lo::AL;
    float* sQA = sm + Lo::QA;
    float* sKU = sm + Lo::KU;
    float* sW = sm + Lo::W;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G, crank = G > 1 ? (int)ptx::cluster_ctarank() : 0;
    const int bh = blockIdx.x / G, bidx = bh / a.H, hidx = bh % a.H;
    const int T = a.T, H = a.H, m = a.m, C = a.chunk;
    const int slot0 = crank * kCbSlots;
    const int nvalid = min(kCbSlots, m - slot0);  // >= 1
    const int nc = T > 0 ? (T + C - 1) / C : 0;
    const bool has_eta = a.eta != nullptr;
    float* ws = a.ws + (size_t)(bh * G + crank) * nc * kCbSlots * D;
    const size_t sbase = ((size_t)bidx * H + hidx) * m * D;  // this (b,h)'s state
    auto tok = [&](int t) { return ((size_t)bidx * T + t) * H + hidx; };
    auto cta_sync = [&]() {
        if (G > 1) ptx::cluster_sync(); else __syncthreads();
    };

    // pairs
    const int pi = tid & 15, pt0 = tid >> 4;  // tokens pt0 and pt0 + 32
    const bool pvalid = pi < nvalid;
    // slot warps: slot `warp`, columns lane*CPT .. +CPT
    const int wi = warp;
    const bool wvalid = wi < nvalid;
    const int wc = lane * CPT;

    // ---- stage one chunk's token inputs (x, and with dy: dy, q); |x_t|^2 per token. The
    // loads go to registers first (stage_load, issued a phase ahead where possible) and
    // are converted and stored to shared memory by stage_store.
    constexpr int NI = kCbMaxL * DV / kCbThreads;   // row pieces per thread (D >= 32: >= 1)
    struct Pre {
        float4 x[NI], dy[NI];   // x raw: fp32, or bf16 pairs in the .x/.y bit patterns
        uint32_t c[2], q[2];    // q raw (fp32 bits, or the bf16 bits)
        float mu, eta;
    };
    auto stage_load = [&](Pre& pr, int t0, int L, bool bwd) {
#pragma unroll
        for (int it = 0; it < NI; ++it) {
            const int e = tid + it * kCbThreads, t = e / DV, c4 = e % DV;
            pr.x[it] = make_float4(0.f, 0.f, 0.f, 0.f);
            pr.dy[it] = pr.x[it];
            if (t < L) {
                const size_t ro = tok(t0 + t) * D + 4 * c4;
                if (a.x_bf16) {
                    const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.x) + ro);
                    pr.x[it].x = __uint_as_float(u.x);
                    pr.x[it].y = __uint_as_float(u.y);
                } else {
                    pr.x[it] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + ro);
                }
                if (bwd) pr.dy[it] = *reinterpret_cast<const float4*>(a.dy + ro);
            }
        }
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int e = tid + it * kCbThreads, t = e >> 4, i = e & 15;
            pr.c[it] = 0u;
            pr.q[it] = 0u;
            if (t < L && i < nvalid) {
                const size_t ro = tok(t0 + t) * m + slot0 + i;
                pr.c[it] = __float_as_uint(a.c[ro]);
                if (bwd)
                    pr.q[it] = a.q_bf16 ? (uint32_t)(static_cast<const unsigned short*>(a.q)[ro])
                                        : __float_as_uint(static_cast<const float*>(a.q)[ro]);
            }
        }
        pr.mu = 0.f;
        pr.eta = 1.f;
        if (tid < L) {
            pr.mu = a.mu[tok(t0 + tid)];
            if (has_eta) pr.eta = a.eta[tok(t0 + tid)];
        }
    };
    auto stage_store = [&](const Pre& pr, bool bwd) {
#pragma unroll
        for (int it = 0; it < NI; ++it) {
            const int e = tid + it * kCbThreads, t = e / DV, c4 = e % DV;
            float4 v = pr.x[it];
            if (a.x_bf16) {
                const uint32_t u0 = __float_as_uint(v.x), u1 = __float_as_uint(v.y);
                v = make_float4(__uint_as_float(u0 << 16), __uint_as_float(u0 & 0xffff0000u),
                                __uint_as_float(u1 << 16), __uint_as_float(u1 & 0xffff0000u));
            }
            *reinterpret_cast<float4*>(sX + t * XS + 4 * c4) = v;
            if (bwd) *reinterpret_cast<float4*>(sDY + t * XS + 4 * c4) = pr.dy[it];
            // |x_t|^2: the DV threads of a row are consecutive lanes (DV divides 32 or is 32)
            float s = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
            for (int o = DV / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (c4 == 0) sHH[t] = s;
        }
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int e = tid + it * kCbThreads, t = e >> 4, i = e & 15;
            sC[t * TS + i] = __uint_as_float(pr.c[it]);
            sQ[t * TS + i] = a.q_bf16 ? __uint_as_float(pr.q[it] << 16) : __uint_as_float(pr.q[it]);
        }
        if (tid < kCbMaxL) {
            sMU[tid] = pr.mu;
            sETA[tid] = pr.eta;
        }
    };

    // ---- projection MMAs in 16x16 tiles: hdot = -X S^T into sDQ (a temporary); with
    // bwd also dy.s0 = DY S0^T into sM1, h.dS = -X dS^T into sM3, and the lower
    // triangle of dy_t.h_j = -DY X^T into sM2.
    auto projections = [&](const float* S, bool bwd) {
        const int ntask = bwd ? 22 : 4;
        const int g = lane >> 2, c = lane & 3;
        for (int task = warp; task < ntask; task += kCbThreads / 32) {
            float acc[2][4];
            cb_zero(acc);
            float* out;
            int ostr, r0, c0;
            float sgn;
            if (task < 12) {
                const int gm = task >> 2;
                r0 = 16 * (task & 3);
                c0 = 0;
                cb_mma<2>(acc, (gm == 1 ? sDY : sX) + r0 * XS, XS, 1, gm == 2 ? sDS : S, 1, XS, 0, D, lane);
                out = gm == 0 ? sDQ : (gm == 1 ? sM1 : sM3);
                ostr = TS;
                sgn = gm == 1 ? 1.f : -1.f;
            } else {
                const int u = task - 12;
                const int rb = u < 1 ? 0 : (u < 3 ? 1 : (u < 6 ? 2 : 3));
                r0 = 16 * rb;
                c0 = 16 * (u - rb * (rb + 1) / 2);
                cb_mma<2>(acc, sDY + r0 * XS, XS, 1, sX + c0 * XS, 1, XS, 0, D, lane);
                out = sM2;
                ostr = PS;
                sgn = -1.f;
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float* o = out + (r0 + g) * ostr + c0 + 8 * nt + 2 * c;
                o[0] = sgn * acc[nt][0];
                o[1] = sgn * acc[nt][1];
                o[8 * ostr] = sgn * acc[nt][2];
                o[8 * ostr + 1] = sgn * acc[nt][3];
            }
        }
    };

    // ---- gates of the pairs' (token, slot) entries from hdot (sDQ); hdot also out
    // for the gate derivative.
    auto pair_gates = [&](int L, float* hd_out) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int t = pt0 + 32 * h2;
            float g = 1.f, kt = 0.f;
            const float hd = sDQ[t * TS + pi];
            if (t < L && pvalid) cb_gates(hd, sHH[t], sN2[pi], sC[t * TS + pi], sMU[t], sETA[t], g, kt);
            sG[t * TS + pi] = g;
            sKT[t * TS + pi] = kt;
            if (hd_out) hd_out[h2] = hd;
        }
    };

    // ---- per-slot products of the gates over the chunk (slot warps; lane: tokens 2l, 2l+1):
    // A (inclusive prefix), U (exclusive suffix), A_L; kappa U and (bwd) A q by slot.
    auto slot_scans = [&](bool bwd) {
        const int t0 = 2 * lane, t1 = t0 + 1;
        const float g0 = sG[t0 * TS + wi], g1 = sG[t1 * TS + wi];
        const float a1 = g0 * g1;
        float p = a1, s = a1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float up = __shfl_up_sync(0xffffffffu, p, o);
            const float dn = __shfl_down_sync(0xffffffffu, s, o);
            if (lane >= o) p *= up;
            if (lane + o < 32) s *= dn;
        }
        float ex = __shfl_up_sync(0xffffffffu, p, 1);  // product of lanes below
        float rt = __shfl_down_sync(0xffffffffu, s, 1); // product of lanes above
        if (lane == 0) ex = 1.f;
        if (lane == 31) rt = 1.f;
        const float A0 = ex * g0, A1 = p, U1 = rt, U0 = g1 * rt;
        const float AL = __shfl_sync(0xffffffffu, p, 31);
        if (lane == 0) sAL[wi] = AL;
        const float k0 = sKT[t0 * TS + wi], k1 = sKT[t1 * TS + wi];
        *reinterpret_cast<float2*>(sKST + wi * PS + t0) = make_float2(k0 * U0, k1 * U1);
        if (bwd) {
            sA[t0 * TS + wi] = A0;
            sA[t1 * TS + wi] = A1;
            sU[t0 * TS + wi] = U0;
            sU[t1 * TS + wi] = U1;
            const float q0 = sQ[t0 * TS + wi], q1 = sQ[t1 * TS + wi];
            *reinterpret_cast<float2*>(sAQT + wi * PS + t0) = make_float2(A0 * q0, A1 * q1);
            // the same products inside 16-token blocks (8 lanes each), and the block totals
            float pb = a1, sb = a1;
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, pb, o);
                const float dn = __shfl_down_sync(0xffffffffu, sb, o);
                if ((lane & 7) >= o) pb *= up;
                if ((lane & 7) + o < 8) sb *= dn;
            }
            float exb = __shfl_up_sync(0xffffffffu, pb, 1);
            float rtb = __shfl_down_sync(0xffffffffu, sb, 1);
            if ((lane & 7) == 0) exb = 1.f;
            if ((lane & 7) == 7) rtb = 1.f;
            sQA[t0 * TS + wi] = q0 * exb * g0;
            sQA[t1 * TS + wi] = q1 * pb;
            sKU[t0 * TS + wi] = k0 * g1 * rtb;
            sKU[t1 * TS + wi] = k1 * rtb;
            const float G1 = __shfl_sync(0xffffffffu, pb, 15), G2 = __shfl_sync(0xffffffffu, pb, 23);
            if (lane == 0) {   // pairs (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
                sW[0 * kCbSlots + wi] = 1.f;
                sW[1 * kCbSlots + wi] = G1;
                sW[2 * kCbSlots + wi] = G1 * G2;
                sW[3 * kCbSlots + wi] = 1.f;
                sW[4 * kCbSlots + wi] = G2;
                sW[5 * kCbSlots + wi] = 1.f;
            }
        }
    };

    // Slot warps: load a state (global, 16 slots of this CTA) into S, with |s_i|^2.
    auto load_state = [&](float* S, const float* src, size_t stride_slot, bool valid) {
        float v[CPT];
        if (valid) {
            cb_ld<CPT>(src + (size_t)wi * stride_slot + wc, v);
        } else {
#pragma unroll
            for (int c = 0; c < CPT; ++c) v[c] = 0.f;
        }
        cb_st<CPT>(S + wi * XS + wc, v);
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) s += v[c] * v[c];
        s = cb_warp_sum(s);
        if (lane == 0) sN2[wi] = s;
    };

    float* Scur = sm + Lo::SA;
    float* Soth = sm + Lo::SB;

    // ================= forward sweep: the start state of every chunk into the workspace
    const int g4 = lane >> 2, c4 = lane & 3;   // MMA fragment coordinates
    load_state(Scur, a.S0 + sbase + (size_t)slot0 * D, D, wvalid);
    Pre pre;
    if (nc > 0) stage_load(pre, 0, min(C, T), false);
    for (int k = 0; k < nc; ++k) {
        const int t0 = k * C, L = min(C, T - t0), kend = (L + 7) & ~7;
        {   // checkpoint, and |s_i|^2 of this chunk's start state
            float v[CPT];
            cb_ld<CPT>(Scur + wi * XS + wc, v);
            cb_st<CPT>(ws + ((size_t)k * kCbSlots + wi) * D + wc, v);
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) s += v[c] * v[c];
            s = cb_warp_sum(s);
            if (lane == 0) sN2[wi] = s;
        }
        stage_store(pre, false);
        __syncthreads();
        projections(Scur, false);
        __syncthreads();
        pair_gates(L, nullptr);
        __syncthreads();
        slot_scans(false);
        __syncthreads();
        if (k + 1 < nc) stage_load(pre, t0 + C, min(C, T - t0 - C), false);   // next chunk's inputs
        // S_next,i = A_L,i S_i - sum_t kappa_t,i U_t,i x_t   (h = -x): [16 slots] x [8 columns] per warp
        for (int task = warp; task < D / 8; task += kCbThreads / 32) {
            float acc[1][4];
            cb_zero(acc);
            cb_mma<1>(acc, sKST, PS, 1, sX + 8 * task, XS, 1, 0, kend, lane);
            const int col = 8 * task + 2 * c4;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = g4 + 8 * r;
                const float al = sAL[i];
                Soth[i * XS + col] = al * Scur[i * XS + col] - acc[0][2 * r];
                Soth[i * XS + col + 1] = al * Scur[i * XS + col + 1] - acc[0][2 * r + 1];
            }
        }
        __syncthreads();
        float* t = Scur; Scur = Soth; Soth = t;
    }
    // Scur = S_T, the end state of the last chunk.

    // ================= backward sweep
    {   // dS = dS_T; e0 = s_T.dS
        float v[CPT], s[CPT];
        if (a.dST && wvalid) {
            cb_ld<CPT>(a.dST + sbase + (size_t)(slot0 + wi) * D + wc, v);
        } else {
#pragma unroll
            for (int c = 0; c < CPT; ++c) v[c] = 0.f;
        }
        cb_st<CPT>(sDS + wi * XS + wc, v);
        cb_ld<CPT>(Scur + wi * XS + wc, s);
        float e = 0.f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) e += s[c] * v[c];
        e = cb_warp_sum(e);
        if (lane == 0) sE0[wi] = e;
    }
    float* SL = Scur;   // end state of the chunk being differentiated
    float* S0 = Soth;   // its start state (from the workspace)
    float pck[CPT];     // the start state's row piece of this lane, loaded a phase ahead
    if (nc > 0) {
        stage_load(pre, (nc - 1) * C, T - (nc - 1) * C, true);
        cb_ld<CPT>(ws + ((size_t)(nc - 1) * kCbSlots + wi) * D + wc, pck);
    }
    for (int k = nc - 1; k >= 0; --k) {
        const int t0 = k * C, L = min(C, T - t0), kend = (L + 7) & ~7;
        {   // start state (and |s_i|^2) and token inputs into shared memory
            cb_st<CPT>(S0 + wi * XS + wc, pck);
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) s += pck[c] * pck[c];
            s = cb_warp_sum(s);
            if (lane == 0) sN2[wi] = s;
        }
        stage_store(pre, true);
        __syncthreads();
        projections(S0, true);
        __syncthreads();
        float hd[2] = {0.f, 0.f};
        pair_gates(L, hd);
        __syncthreads();

        slot_scans(true);
        __syncthreads();

        // The decayed sums over token pairs, split by 16-token blocks. For k in block bk
        // and t in an earlier block bt, D_i[k][t] = KU-suffix(t) * W_i(bt, bk) * QA-prefix(k)
        // (the in-block suffix after t, the whole blocks between, the in-block prefix up to
        // k), so each pair of blocks is a 16x16 matrix product with a per-slot scale:
        //   P[k][t]   += sum_i QA_k,i W_i KU_t,i                  (bt < bk)
        //   dq_t,i    += Ahat_t,i sum_{bj<bt} W_i (M2[t][bj] . KU_bj)_i
        //   dkappa_t,i += Uhat_t,i sum_{bk>bt} W_i (M2[bk][t]^T . QA_bk)_i
        // (Ahat, Uhat: the in-block prefix and suffix; the in-block loops that follow form
        // them as they walk the block, and apply them to the block sums stored here).
        {
            const int g = lane >> 2, c = lane & 3;
            auto pidx = [](int b1, int b2) { return b1 == 0 ? b2 - 1 : (b1 == 1 ? b2 + 1 : 5); };
            for (int task = warp; task < 14; task += kCbThreads / 32) {
                float acc[2][4];
                cb_zero(acc);
                if (task < 6) {   // scores of block pair (bt, bk), bt < bk
                    const int bt = task < 3 ? 0 : (task < 5 ? 1 : 2);
                    const int bk = task < 3 ? task + 1 : (task < 5 ? task - 1 : 3);
                    cb_mma_s<2, 1>(acc, sQA + 16 * bk * TS, TS, 1, sKU + 16 * bt * TS, 1, TS, 0, kCbSlots, lane,
                                   sW + pidx(bt, bk) * kCbSlots);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        float* o = sP + (16 * bk + g) * PS + 16 * bt + 8 * nt + 2 * c;
                        o[0] = acc[nt][0];
                        o[1] = acc[nt][1];
                        o[8 * PS] = acc[nt][2];
                        o[8 * PS + 1] = acc[nt][3];
                    }
                } else if (task < 10) {   // dq of block bt from the earlier blocks
                    const int bt = task - 6;
                    for (int bj = 0; bj < bt; ++bj)
                        cb_mma_s<2, 2>(acc, sM2 + 16 * bt * PS + 16 * bj, PS, 1, sKU + 16 * bj * TS, TS, 1, 0, 16,
                                       lane, sW + pidx(bj, bt) * kCbSlots);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int t = 16 * bt + g + 8 * (r >> 1), i = 8 * nt + 2 * c + (r & 1);
                            sDQ[t * TS + i] = bt > 0 ? acc[nt][r] : 0.f;
                        }
                } else {   // dkappa of block bt from the later blocks
                    const int bt = task - 10;
                    for (int bk = bt + 1; bk < 4; ++bk)
                        cb_mma_s<2, 2>(acc, sM2 + 16 * bk * PS + 16 * bt, 1, PS, sQA + 16 * bk * TS, TS, 1, 0, 16,
                                       lane, sW + pidx(bt, bk) * kCbSlots);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int t = 16 * bt + g + 8 * (r >> 1), i = 8 * nt + 2 * c + (r & 1);
                            sDKT[t * TS + i] = bt < 3 ? acc[nt][r] : 0.f;
                        }
                }
            }
        }
        __syncthreads();

        // in-block parts: dq over j <= t in t's block (pairs), the scores and dkappa over
        // k >= t in t's block (half-warps: lanes = slots; tokens hw and 63 - hw)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int t = pt0 + 32 * h2;
            float dq = 0.f;
            if (t < L) {
                dq = sA[t * TS + pi] * sM1[t * TS + pi];
                float Dp = 1.f;
                for (int j = t; j >= (t & ~15); --j) {
                    dq += Dp * sKT[j * TS + pi] * sM2[t * PS + j];
                    Dp *= sG[j * TS + pi];
                }
                dq += Dp * sDQ[t * TS + pi];   // Dp is now Ahat_t
            }
            sDQ[t * TS + pi] = dq;
        }
        {
            const int hw = tid >> 4;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                const int t = h2 == 0 ? hw : kCbMaxL - 1 - hw;
                const int bb = (h2 == 0 ? (hw & ~1) : kCbMaxL - 2 - (hw & ~1)) & ~15;  // warp-uniform block
                const float ktv = sKT[t * TS + pi];
                float Dp = 1.f, dk = 0.f;
                float v[16];
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    const int kk = bb + n;
                    v[n] = 0.f;
                    if (kk >= t) {
                        const float w = sQ[kk * TS + pi] * Dp;
                        v[n] = ktv * w;
                        dk += w * sM2[kk * PS + t];
                        if (n < 15) Dp *= sG[(kk + 1) * TS + pi];   // stays inside the block
                    }
                }
                // reduce the 16 values over the half-warp's 16 lanes: lane n keeps entry n
#pragma unroll
                for (int s = 8; s >= 1; s >>= 1) {
                    const bool up = (pi & s) != 0;
#pragma unroll
                    for (int n = 0; n < s; ++n) {
                        const float send = up ? v[n] : v[n + s];
                        const float keep = up ? v[n + s] : v[n];
                        v[n] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                    }
                }
                sP[(bb + pi) * PS + t] = v[0];
                // Dp is now Uhat_t, the product of g over the block after t
                sDKT[t * TS + pi] = t < L ? Dp * sDKT[t * TS + pi] + sU[t * TS + pi] * sM3[t * TS + pi] + dk : 0.f;
            }
        }
        __syncthreads();

        // g dg = s_L.dS + reverse cumulative sum of q dq - kappa dkappa (slot warps)
        {
            const int ta = 2 * lane, tb = ta + 1;
            const float r0 = sQ[ta * TS + wi] * sDQ[ta * TS + wi] - sKT[ta * TS + wi] * sDKT[ta * TS + wi];
            const float r1 = sQ[tb * TS + wi] * sDQ[tb * TS + wi] - sKT[tb * TS + wi] * sDKT[tb * TS + wi];
            float s = r0 + r1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float dn = __shfl_down_sync(0xffffffffu, s, o);
                if (lane + o < 32) s += dn;
            }
            float rt = __shfl_down_sync(0xffffffffu, s, 1);
            if (lane == 31) rt = 0.f;
            const float e0 = sE0[wi];
            const float ea = e0 + s, eb = e0 + r1 + rt;
            sM1[ta * TS + wi] = ea / sG[ta * TS + wi];
            sM1[tb * TS + wi] = eb / sG[tb * TS + wi];
        }
        __syncthreads();

        // derivative of the gates (pairs); dq and dc out; sums over the slots per token
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int t = pt0 + 32 * h2;
            CbGateGrad gg{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (t < L && pvalid) {
                gg = cb_gates_bwd(hd[h2], sHH[t], sN2[pi], sC[t * TS + pi], sMU[t], sETA[t],
                                  sM1[t * TS + pi], sDKT[t * TS + pi]);
                const size_t ro = tok(t0 + t) * m + slot0 + pi;
                a.dc[ro] = gg.cb;
                a.dq[ro] = sDQ[t * TS + pi];
            }
            sHBT[pi * PS + t] = gg.hdb;
            sDKT[t * TS + pi] = gg.n2b;
            const float hs = cb_half_sum(gg.hhb), ms = cb_half_sum(gg.mub), es = cb_half_sum(gg.etab);
            if (pi == 0) {
                sHHB[t] = hs;
                sMUB[t] = ms;
                sETAB[t] = es;
            }
        }
        __syncthreads();

        // this CTA's share of dx (16 tokens x D/4 columns per warp) and the MMA part of the
        // carried adjoint, sum_t A_t,i q_t,i dy_t - sum_t dhdot_t,i x_t (16 slots x 8 columns
        // per warp, into the scratch that sM2 no longer needs)
        float* sTMP = sM2;
        {
            constexpr int NT = D / 32;
            const int rb = warp >> 2, col0 = (warp & 3) * (D / 4);
            if (16 * rb < L) {
                float acc[NT][4];
                cb_zero(acc);
                cb_mma<NT>(acc, sP + 16 * rb, 1, PS, sDY + col0, XS, 1, 16 * rb, kend, lane);
                cb_mma<NT>(acc, sKST + 16 * rb, 1, PS, sDS + col0, XS, 1, 0, kCbSlots, lane);
                cb_mma<NT>(acc, sHBT + 16 * rb, 1, PS, S0 + col0, XS, 1, 0, kCbSlots, lane);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int t = 16 * rb + g4 + 8 * r, col = col0 + 8 * nt + 2 * c4;
                        const float h2 = 2.f * sHHB[t];
                        sDX[t * XS + col] = h2 * sX[t * XS + col] - acc[nt][2 * r];
                        sDX[t * XS + col + 1] = h2 * sX[t * XS + col + 1] - acc[nt][2 * r + 1];
                    }
            }
            if (warp < D / 8) {
                float a1[1][4], a2[1][4];
                cb_zero(a1);
                cb_zero(a2);
                cb_mma<1>(a1, sAQT, PS, 1, sDY + 8 * warp, XS, 1, 0, kend, lane);
                cb_mma<1>(a2, sHBT, PS, 1, sX + 8 * warp, XS, 1, 0, kend, lane);
                const int col = 8 * warp + 2 * c4;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int i = g4 + 8 * r;
                    sTMP[i * XS + col] = a1[0][2 * r] - a2[0][2 * r];
                    sTMP[i * XS + col + 1] = a1[0][2 * r + 1] - a2[0][2 * r + 1];
                }
            }
        }
        cta_sync();   // every CTA's dx share, dmu and deta sums are in place
        if (k > 0) {   // the previous chunk's inputs and start state, while this one finishes
            stage_load(pre, t0 - C, C, true);
            cb_ld<CPT>(ws + ((size_t)(k - 1) * kCbSlots + wi) * D + wc, pck);
        }

        // the adjoint carried into the previous chunk (slot warps), in place; e0 for it
        {
            const float nb = cb_warp_sum(sDKT[(2 * lane) * TS + wi] + sDKT[(2 * lane + 1) * TS + wi]);
            float acc[CPT], dv[CPT], sv[CPT];
            cb_ld<CPT>(sTMP + wi * XS + wc, acc);
            cb_ld<CPT>(sDS + wi * XS + wc, dv);
            cb_ld<CPT>(S0 + wi * XS + wc, sv);
            const float al = sAL[wi];
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[c] += al * dv[c] + 2.f * nb * sv[c];
            cb_st<CPT>(sDS + wi * XS + wc, acc);
            float e = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) e += sv[c] * acc[c];
            e = cb_warp_sum(e);
            if (lane == 0) sE0[wi] = e;
        }
        // dx, dmu, deta of the tokens t = crank (mod G): the cluster's shares in rank order
        {
            const uint32_t dxa = ptx::smem_u32(sDX), mua = ptx::smem_u32(sMUB), eta_a = ptx::smem_u32(sETAB);
            const int nrow = L > crank ? (L - crank + G - 1) / G : 0;
            for (int e = tid; e < nrow * DV; e += kCbThreads) {
                const int t = crank + G * (e / DV), c4 = e % DV;
                const uint32_t off = (uint32_t)(t * XS + 4 * c4) * 4u;
                float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int g = 0; g < G; ++g) {
                    const float4 v = G > 1 ? ptx::ld_cluster_v4(ptx::mapa(dxa + off, (uint32_t)g))
                                           : *reinterpret_cast<const float4*>(sDX + t * XS + 4 * c4);
                    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
                }
                *reinterpret_cast<float4*>(a.dx + tok(t0 + t) * D + 4 * c4) = s;
            }
            if (tid < nrow) {
                const int t = crank + G * tid;
                float sm_ = 0.f, se = 0.f;
                for (int g = 0; g < G; ++g) {
                    if (G > 1) {
                        sm_ += ptx::ld_cluster_f32(ptx::mapa(mua + 4u * t, (uint32_t)g));
                        if (has_eta) se += ptx::ld_cluster_f32(ptx::mapa(eta_a + 4u * t, (uint32_t)g));
                    } else {
                        sm_ += sMUB[t];
                        se += sETAB[t];
                    }
                }
                a.dmu[tok(t0 + t)] = sm_;
                if (has_eta && a.deta) a.deta[tok(t0 + t)] = se;
            }
        }
        cta_sync();   // no CTA rewrites its shares while a peer may still read them
        float* tmp = SL; SL = S0; S0 = tmp;
    }
    if (wvalid) {
        float v[CPT];
        cb_ld<CPT>(sDS + wi * XS + wc, v);
        cb_st<CPT>(a.dS0 + sbase + (size_t)(slot0 + wi) * D + wc, v);
    }
}

}  // namespace lattice
