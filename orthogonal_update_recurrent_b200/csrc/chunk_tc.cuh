// chunk_tc.cuh -- tensor-core (tcgen05) chunked scan of the Lattice recurrence.
//
// Computes the chunked form, Eq. 17 of "Lattice: Learning to Efficiently
// Compress the Memory" (§3.4.1 and Appendix B.1), chunk size C = 64: inside a
// chunk every token's per-slot gate g and write coefficient kappa come from the
// chunk-start state S0 (projection p = x . s0, normaliser of eq. beta_chunk with
// the chunk-start norm as in the Appendix D listing), and the state follows the
// diagonal-gated linear recurrence  s_i <- g_i s_i + kappa_i x.
//
// Chunk-parallel evaluation. Products of gates over a whole chunk reach 1e-58
// on the paper-shaped workloads (small-norm slots get small or negative gates),
// so nothing is ever divided by a product longer than one 16-token sub-chunk:
//   y_t   = sum_i q_ti A_ti s0_i + sum_{j<=t} P_tj x_j,  A_t = prod_{l<=t} g_l
//   P_tj  = sum_i QR_b(t)_i KD(j)_i           for j in sub-chunk b (16b..16b+15)
//   QR_b(t) = q_t prod_{l=16b..t} g_l          (t >= 16b; plain products)
//   KD(j)   = kappa_j / prod_{l=16b..j} g_l    (division inside one sub-chunk)
//   S_C   = diag(A_C) S0 + sum_j (kappa_j prod_{l=j+1..C-1} g_l) x_j^T
// with kappa_j prod_{l=j+1..C-1} g_l = KD(j) F_b, F_b = prod_{l>=16b} g_l.
//
// One CTA per (b, h) sequence. The fp32 state lives in tensor memory as
// S = diag(sigma) T: the chunk decay diag(A_C) is folded into the per-slot scale
// sigma, so the state-update GEMM accumulates straight onto T; rows whose
// sigma*A_C drops below 2^-100 (the old state is then below fp32 resolution)
// are rescaled in TMEM first, and T is renormalised when sigma leaves
// [2^-32, 2^32]. The GEMMs that carry the state use hi+lo bf16 operand pairs
// (kept in tensor memory), so the carried state keeps close to fp32 accuracy
// over thousands of chunks. Per chunk (fp32 TMEM accumulators):
//   G1: D1  [m x C]  = (S0hi + S0lo) . X^T       projections x_t . s0_i (A in TMEM)
//   G7: T   [m x d] += (KShi + KSlo)^T . X       state update (A in TMEM)
//   G4: Y^T [d x C]  = S0hi^T . QR_0^T           inter-chunk read-out (smem operands)
//   G6: Y^T [d x C] += X^T . P_causal^T          intra-chunk read-out
// and the causal scores P = QR_b . KD_b^T (16 x 16 blocks, keys of sub-chunk b) with
// warp-synchronous MMAs (mma.sync) on two warps of their own.
//
// Warp roles (640 threads, 5 warpgroups). Warps 0-15 are workers: warp 4*sb + q
// owns TMEM lane quadrant q (slots 32q..32q+31) and sub-chunk sb. It computes
// the gates of tokens 16sb..16sb+15 for its 32 slots (the 64-token gate
// recurrence runs as four independent 16-token pieces, tied together by four
// sub-chunk products per slot exchanged through shared memory), converts state
// columns sb*d/4..(sb+1)*d/4, stores y for
// tokens 16sb..16sb+15 and prepares |x|^2, mu, eta of four tokens of the next
// chunk. Warp 16 issues every MMA, warp 17 every TMA copy (an MMA issue blocks
// its warp while the MMA runs, so neither sits on a worker), warps 18 and 19 form
// the masked scores. The state chain (G1 -> gates -> G7 -> state conversion -> next
// G1) is signalled separately from the read-out path (scores, G6), which overlaps
// the next chunk.
// Every mbarrier wait is bounded by %globaltimer: on timeout the kernel sets the
// device status word, skips the remaining work and still meets every named barrier.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "scan_simt.cuh"
#include "tc_ptx.cuh"
#include "waits.cuh"

namespace lattice {

constexpr int kTcC = 64;            // chunk size of the tensor-core path
constexpr int kTcSub = 16;          // sub-chunk: the longest product ever divided by
constexpr int kTcWorkers = 512;     // 16 worker warps: 4 lane quadrants x 4 sub-chunks
constexpr int kTcThreads = kTcWorkers + 128;  // + control warpgroup (MMA warp, TMA warp, 2 idle)

inline bool chunk_tc_supported(int m, int d, int chunk, bool x_bf16, bool q_bf16) {
    return chunk == kTcC && x_bf16 && q_bf16 && (m == 64 || m == 128) && (d == 64 || d == 128);
}

template <int MS, int DS>
struct TcLayout {
    static constexpr int NST = 2;                         // X stages
    static constexpr uint32_t X_STAGE = DS * 128;         // DS/64 blocks x 64 rows x 128 B
    static constexpr uint32_t S0_TILE = MS * DS * 2;      // DS/64 blocks x m rows x 128 B
    static constexpr uint32_t ROW_TILE = MS * 128;        // [m][64] bf16, one 128 B row per slot
    static constexpr uint32_t Q_TILE = kTcC * MS * 2;     // [C][m] bf16, row-major (TMA)
    static constexpr uint32_t C_TILE = kTcC * MS * 4;     // [C][m] fp32, row-major (TMA)
    static constexpr uint32_t X_OFF = 0;
    static constexpr uint32_t Q_OFF = X_OFF + NST * X_STAGE;
    static constexpr uint32_t CC_OFF = Q_OFF + Q_TILE;
    static constexpr uint32_t S0HI_OFF = CC_OFF + C_TILE;          // A of the read-out GEMM
    static constexpr uint32_t QR_OFF = S0HI_OFF + S0_TILE;         // QR_0..QR_3
    static constexpr uint32_t KD_OFF = QR_OFF + 4 * ROW_TILE;
    static constexpr uint32_t P_OFF = KD_OFF + ROW_TILE;           // [C][128 B]
    static constexpr uint32_t AUX_OFF = P_OFF + kTcC * 128;        // [NST][C/2][2] float4
    static constexpr uint32_t MUETA_OFF = AUX_OFF + NST * kTcC * 16;  // [C] {mu, eta}, with the q/c stage
    static constexpr uint32_t GSUB_OFF = MUETA_OFF + kTcC * 8;        // [4][m] float
    static constexpr uint32_t TSQ_OFF = GSUB_OFF + 4 * MS * 4;        // [4][m] float
    static constexpr uint32_t BAR_OFF = TSQ_OFF + 4 * MS * 4;         // 8 mbarriers
    static constexpr uint32_t MISC_OFF = BAR_OFF + 8 * 8;
    static constexpr uint32_t BYTES = MISC_OFF + 64;
    static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;          // room to align the base
    // TMEM columns: fp32 state T | D1 (projections; its columns also hold the bf16
    // hi/lo pairs of the state-update operand KS, whose lifetime never overlaps
    // D1's) | (unused) | Y^T, double-buffered | S0 hi/lo bf16 pairs (two per column, d/2 each)
    static constexpr uint32_t T_COL = 0;
    static constexpr uint32_t D1_COL = DS;
    static constexpr uint32_t KSHI_TCOL = D1_COL;
    static constexpr uint32_t KSLO_TCOL = D1_COL + kTcC / 2;
    static constexpr uint32_t Y_COL = DS + 2 * kTcC;               // + (chunk & 1) * C
    static constexpr uint32_t S0HI_TCOL = DS + 4 * kTcC;
    static constexpr uint32_t S0LO_TCOL = S0HI_TCOL + DS / 2;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(S0LO_TCOL + DS / 2 <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
    static constexpr uint32_t TX_BYTES = X_STAGE;
    static constexpr uint32_t QC_BYTES = Q_TILE + C_TILE;
};

struct TcMaps {
    CUtensorMap x, q, c;
};

__device__ __forceinline__ uint4 pack8(const float* v) {
    uint4 u;
    u.x = ptx::pack_bf16x2(v[0], v[1]);
    u.y = ptx::pack_bf16x2(v[2], v[3]);
    u.z = ptx::pack_bf16x2(v[4], v[5]);
    u.w = ptx::pack_bf16x2(v[6], v[7]);
    return u;
}

// hi = v truncated to bf16 (the top 16 bits: one byte permute per pair, no
// conversion unit), lo = bf16_rn(v - hi) (v - hi is exact in fp32). hi + lo
// carries ~16 mantissa bits and, since lo is rounded to nearest, no bias.
__device__ __forceinline__ void split2(float2 v, uint32_t& hi, uint32_t& lo) {
    const uint32_t bx = __float_as_uint(v.x), by = __float_as_uint(v.y);
    hi = __byte_perm(bx, by, 0x7632);
    const float2 h = make_float2(__uint_as_float(bx & 0xffff0000u), __uint_as_float(by & 0xffff0000u));
    const float2 l = ptx::f2add(v, ptx::f2neg(h));
    lo = ptx::pack_bf16x2(l.x, l.y);
}

template <int MS, int DS>
__global__ void __launch_bounds__(kTcThreads, 1)
    chunk_tc_kernel(const __grid_constant__ TcMaps maps, ScanArgs a) {
    using Lay = TcLayout<MS, DS>;
    constexpr int NSUB = kTcC / kTcSub;   // 4 sub-chunks, one per worker group
    constexpr int DCOL = DS / NSUB;       // state columns converted by each group
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H;
    const int nch = (T + kTcC - 1) / kTcC;
    constexpr int MMA_WARP = 16, TMA_WARP = 17;

    // mbarriers: X stage landed [2], q/c landed, D1 ready, T updated (G7), (unused),
    // read-out complete (G6), S0 operand read (G4)
    const uint32_t bar_full0 = sbase + Lay::BAR_OFF;
    const uint32_t bar_qc = sbase + Lay::BAR_OFF + 16;
    const uint32_t bar_d1 = sbase + Lay::BAR_OFF + 24;
    const uint32_t bar_t = sbase + Lay::BAR_OFF + 32;
    const uint32_t bar_y = sbase + Lay::BAR_OFF + 48;
    const uint32_t bar_g4 = sbase + Lay::BAR_OFF + 56;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
    volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 4);
    // per X stage: set when a token of that chunk has mu^2 below 2^-60, where the normaliser's
    // argument may be denormal or zero (a zero-norm update keeps the slot)
    volatile uint32_t* zmu = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 8);
    float* aux = reinterpret_cast<float*>(smem + Lay::AUX_OFF);
    float* gsub = reinterpret_cast<float*>(smem + Lay::GSUB_OFF);   // [NSUB][MS] sub-chunk products
    float* tsqp = reinterpret_cast<float*>(smem + Lay::TSQ_OFF);    // [NSUB][MS] partial |s|^2

    // named barriers (ids, participants): workers + MMA warp, or workers + TMA warp
    constexpr uint32_t BAR_INIT = 1, BAR_G = 2, BAR_A = 3, BAR_S0 = 4, BAR_P = 5;
    constexpr uint32_t N_WM = kTcWorkers + 32;
    constexpr uint32_t N_WMS = kTcWorkers + 32 + 64;  // + the two score warps (BAR_A, BAR_P)
    constexpr int SCORE_WARP0 = 18;                    // warps 18, 19: the causal scores

    if (warp == MMA_WARP) {
        if (lane == 0) {
            for (int j = 0; j < 8; ++j) ptx::mbar_init(sbase + Lay::BAR_OFF + 8 * j, 1);
            ptx::mbar_init(bar_qc, 1 + 32);  // TMA bytes + the TMA warp's 32 copy arrivals (mu, eta)
            *abort = 0u;
            zmu[0] = 0u;
            zmu[1] = 0u;
            ptx::fence_mbar_init();
        }
        __syncwarp();
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), Lay::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= kTcWorkers / 32) {
        // ================================================================ control
        if (warp == MMA_WARP) {
            // -------------------------------------------------- MMA issue (warp-converged,
            // one elected lane issues; descriptors get per-MMA start-address offsets)
            constexpr uint32_t idesc_g1 = ptx::idesc_bf16(MS, kTcC, 0, 0);
            constexpr uint32_t idesc_g7 = ptx::idesc_bf16(MS, DS, 0, 1);
            constexpr uint32_t idesc_g4 = ptx::idesc_bf16(DS, kTcC, 1, 1);
            constexpr uint32_t idesc_g6 = ptx::idesc_bf16(DS, kTcC, 1, 0);
            auto off = [](uint32_t bytes) { return uint64_t(bytes >> 4); };
            auto g1 = [&](int k) {  // D1 = (S0hi + S0lo) . X_k^T  (M = m, N = C, K = d)
                const uint64_t dK_x = ptx::sdesc_sw128(sbase + Lay::X_OFF, 16, 1024);
                const uint32_t xo = (k & 1) * Lay::X_STAGE;
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < DS / 16; ++kk) {
                        const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
                        ptx::mma_bf16_tmem_a_elect(tmem + Lay::D1_COL,
                                                   tmem + (part ? Lay::S0LO_TCOL : Lay::S0HI_TCOL) + kk * 8,
                                                   dK_x + off(xo + kb * 64 * 128 + ko), idesc_g1,
                                                   (part | kk) != 0);
                    }
            };
            if (nch > 0) {
                ptx::named_bar(BAR_INIT, N_WM);  // S0 operand written
                ptx::tc_fence_after();
                if (tc_wait_warp(bar_full0, 0, abort)) g1(0);
                ptx::mma_commit_elect(bar_d1);
            }
            const uint64_t dM_x = ptx::sdesc_sw128(sbase + Lay::X_OFF, 64 * 128, 1024);
            const uint64_t dM_qr = ptx::sdesc_sw128(sbase + Lay::QR_OFF, MS * 128, 1024);
            const uint64_t dM_s0hi = ptx::sdesc_sw128(sbase + Lay::S0HI_OFF, MS * 128, 1024);
            const uint64_t dK_p = ptx::sdesc_sw128(sbase + Lay::P_OFF, 16, 1024);
            for (int k = 0; k < nch; ++k) {
                const uint32_t xo = (k & 1) * Lay::X_STAGE;
                const uint32_t ycol = Lay::Y_COL + (k & 1) * kTcC;
                ptx::named_bar(BAR_A, N_WMS);  // KS in TMEM, QR/KD written, T prescaled
                ptx::tc_fence_after();
                if (tc_live(abort)) {
                    // G7: T += (KShi + KSlo)^T . X  (M = m, N = d, K = C); A in TMEM, B MN-major
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < kTcC / 16; ++kk)
                            ptx::mma_bf16_tmem_a_elect(tmem + Lay::T_COL,
                                                       tmem + (part ? Lay::KSLO_TCOL : Lay::KSHI_TCOL) + kk * 8,
                                                       dM_x + off(xo + kk * 2048), idesc_g7, 1);
                }
                ptx::mma_commit_elect(bar_t);
                if (tc_live(abort)) {
                    // G4: Y^T = S0hi^T . QR_0^T  (M = d, N = C, K = m); both MN-major
#pragma unroll
                    for (int kk = 0; kk < MS / 16; ++kk)
                        ptx::mma_bf16_elect(tmem + ycol, dM_s0hi + off(kk * 2048), dM_qr + off(kk * 2048),
                                            idesc_g4, kk > 0);
                }
                ptx::mma_commit_elect(bar_g4);
                ptx::named_bar(BAR_S0, N_WM);  // S0 operand of chunk k+1 written
                ptx::tc_fence_after();
                if (k + 1 < nch) {
                    if (tc_wait_warp(bar_full0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1, abort)) g1(k + 1);
                    ptx::mma_commit_elect(bar_d1);
                }
                ptx::named_bar(BAR_P, N_WMS);  // masked scores written
                ptx::tc_fence_after();
                if (tc_live(abort)) {
                    // G6: Y^T += X^T . P^T  (M = d, N = C, K = C); A MN-major, B K-major
#pragma unroll
                    for (int kk = 0; kk < kTcC / 16; ++kk)
                        ptx::mma_bf16_elect(tmem + ycol, dM_x + off(xo + kk * 2048), dK_p + off(kk * 32),
                                            idesc_g6, 1);
                }
                ptx::mma_commit_elect(bar_y);
            }
            if (nch > 0) tc_drain(bar_y, (nch - 1) & 1);  // every MMA done before TMEM goes away
        } else if (warp == TMA_WARP) {
            // -------------------------------------------------- TMA issue (lane 0)
            int last_x[2] = {-1, -1}, last_qc = -1;
            auto issue_x = [&](int k) {  // X of chunk k -> stage k % 2
                const int s = k & 1;
                last_x[s] = k;
                const uint32_t bar = bar_full0 + 8 * s;
                ptx::mbar_arrive_expect_tx(bar, Lay::TX_BYTES);
#pragma unroll
                for (int kb = 0; kb < DS / 64; ++kb)
                    ptx::tma_load_4d(sbase + Lay::X_OFF + s * Lay::X_STAGE + kb * (64 * 128), &maps.x, bar,
                                     kb * 64, h, k * kTcC, b);
            };
            // q and c of chunk k -> the single q/c stage (lane 0, tensor copies), with mu and
            // eta of its 64 tokens (every lane two tokens, cp.async: a token's mu is one float
            // at a stride of H floats, too narrow for a tensor copy); each lane arrives on the
            // stage's barrier once its copies have landed. Called by every lane.
            auto issue_qc = [&](int k) {
                last_qc = k;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(bar_qc, Lay::QC_BYTES);
                    ptx::tma_load_4d(sbase + Lay::Q_OFF, &maps.q, bar_qc, 0, h, k * kTcC, b);
                    ptx::tma_load_4d(sbase + Lay::CC_OFF, &maps.c, bar_qc, 0, h, k * kTcC, b);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int tau = lane + 32 * j, t = k * kTcC + tau;
                    if (t < T) {
                        const size_t bth = ((size_t)b * T + t) * H + h;
                        ptx::cp_async4(sbase + Lay::MUETA_OFF + tau * 8, a.mu + bth);
                        if (a.eta) ptx::cp_async4(sbase + Lay::MUETA_OFF + tau * 8 + 4, a.eta + bth);
                    }
                }
                ptx::cp_async_mbar_arrive_noinc(bar_qc);
            };
            auto prefetch_l2 = [&](int k) {  // X, q and c of chunk k into L2
#pragma unroll
                for (int kb = 0; kb < DS / 64; ++kb) ptx::tma_prefetch_l2_4d(&maps.x, kb * 64, h, k * kTcC, b);
                ptx::tma_prefetch_l2_4d(&maps.q, 0, h, k * kTcC, b);
                ptx::tma_prefetch_l2_4d(&maps.c, 0, h, k * kTcC, b);
            };
            if (lane == 0 && nch > 0) {
                ptx::prefetch_tensormap(&maps.x);
                ptx::prefetch_tensormap(&maps.q);
                ptx::prefetch_tensormap(&maps.c);
                issue_x(0);
            }
            if (nch > 0) issue_qc(0);
            if (lane == 0 && nch > 0) {
                if (nch > 1) issue_x(1);
                for (int j = 1; j < 4 && j < nch; ++j) prefetch_l2(j);
            }
            for (int k = 0; k < nch; ++k) {
                ptx::named_bar(BAR_G, N_WM);  // every worker is done reading q, c and mu, eta of chunk k
                if (k + 1 < nch) issue_qc(k + 1);
                if (lane == 0) {
                    // X of chunk k is read last by G6_k; then its stage takes chunk k+2
                    if (k + 2 < nch && tc_wait(bar_y, k & 1, abort)) {
                        issue_x(k + 2);
                        if (k + 4 < nch) prefetch_l2(k + 4);
                    }
                }
                __syncwarp();
            }
            ptx::cp_async_wait_all();
            if (lane == 0) {  // no TMA write may be in flight when the CTA retires
#pragma unroll
                for (int s = 0; s < 2; ++s)
                    if (last_x[s] >= 0) tc_drain(bar_full0 + 8 * s, (last_x[s] >> 1) & 1);
                if (last_qc >= 0) tc_drain(bar_qc, last_qc & 1);
            }
            __syncwarp();
        } else if (warp == SCORE_WARP0 || warp == SCORE_WARP0 + 1) {
            // -------------------------------------------------- score warps
            // The causal scores P_tj = sum_i QR_b(t)_i KD(j)_i (K = m), one 16 x 16 block
            // (tokens 16wt.., keys 16b.., b <= wt) at a time, with warp-synchronous MMAs
            // (m16n8k16, bf16 operands by ldmatrix.trans from the slot-major QR and KD tiles,
            // fp32 in registers), masked to j <= t in the diagonal block and written in bf16
            // to the score tile for G6. Warp 18 takes token blocks 0 and 3, warp 19 blocks 1
            // and 2 (five blocks each). On tcgen05 these 16-column blocks cost the tensor
            // pipe about a hundred cycles per K = 16 step, 32 steps a chunk, queued ahead of
            // the next chunk's projection.
            const int lj = lane >> 3, lr = lane & 7, gq = lane >> 2, cq = lane & 3;
            uint8_t* ps = smem + Lay::P_OFF;
            const uint32_t kd_a = sbase + Lay::KD_OFF;
            auto block = [&](int wt, int bk) {
                const uint32_t qr_a = sbase + Lay::QR_OFF + bk * Lay::ROW_TILE;
                float acc[2][4];
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < MS / 16; ++ks) {
                    uint32_t af[4], bf[4];
                    {   // A = QR^T block: stored rows are slots (K), columns tokens (M)
                        const int row = 16 * ks + 8 * (lj >> 1) + lr;
                        const int col = 16 * wt + 8 * (lj & 1);
                        ptx::ldsm_x4_t(qr_a + row * 128 + (((col >> 3) ^ (row & 7)) << 4), af);
                    }
                    {   // B = KD^T block: stored rows are slots (K), columns keys (N)
                        const int row = 16 * ks + 8 * (lj & 1) + lr;
                        const int col = 16 * bk + 8 * (lj >> 1);
                        ptx::ldsm_x4_t(kd_a + row * 128 + (((col >> 3) ^ (row & 7)) << 4), bf);
                    }
                    ptx::mma16816(acc[0], af, bf);      // keys 16bk .. 16bk+7
                    ptx::mma16816(acc[1], af, bf + 2);  // keys 16bk+8 .. 16bk+15
                }
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int t = 16 * wt + gq + 8 * hf, j = 16 * bk + 8 * n + 2 * cq;
                        const float v0 = (j > t) ? 0.f : acc[n][2 * hf];
                        const float v1 = (j + 1 > t) ? 0.f : acc[n][2 * hf + 1];
                        *reinterpret_cast<uint32_t*>(ps + ptx::sw128_off(t, j)) = ptx::pack_bf16x2(v0, v1);
                    }
            };
            const int wa = warp == SCORE_WARP0 ? 0 : 1, wb = warp == SCORE_WARP0 ? 3 : 2;
            for (int k = 0; k < nch; ++k) {
                ptx::named_bar(BAR_A, N_WMS);  // QR and KD of chunk k written
                // G6 of the previous chunk has read the old scores
                if (k > 0) tc_wait(bar_y, (k - 1) & 1, abort);
                __syncwarp();
                ptx::tc_fence_after();
                if (!*abort) {
                    for (int bk = 0; bk <= wa; ++bk) block(wa, bk);
                    for (int bk = 0; bk <= wb; ++bk) block(wb, bk);
                }
                ptx::fence_proxy_async_smem();  // G6 reads the scores through the async proxy
                ptx::named_bar(BAR_P, N_WMS);
            }
        }
    } else {
        // ================================================================ workers
        // warp 4*sb + q4 owns TMEM lane quadrant q4 and sub-chunk sb
        const int q4 = warp & 3, sb = warp >> 2;
        const bool active = (MS == 128) || (lane < 16);
        const int i = (MS == 128) ? (32 * q4 + lane) : (16 * q4 + (lane & 15));  // slot
        const uint32_t lane_base = uint32_t(32 * q4) << 16;
        // y column in the Y^T accumulator (M = d) and P row (M = 64: lanes 0-15 per quadrant)
        const bool ycol_ok = (DS == 128) || (lane < 16);
        const int kcol = (DS == 128) ? (32 * q4 + lane) : (16 * q4 + lane);
        uint8_t* s0hi = smem + Lay::S0HI_OFF;
        uint8_t* qr = smem + Lay::QR_OFF;
        uint8_t* kd = smem + Lay::KD_OFF;
        uint8_t* ps = smem + Lay::P_OFF;
        const uint16_t* qsm = reinterpret_cast<const uint16_t*>(smem + Lay::Q_OFF);
        const float* csm = reinterpret_cast<const float*>(smem + Lay::CC_OFF);

        // a block of DCOL state columns starting at col0 -> hi/lo bf16 operand rows: both
        // into tensor memory (A of the projection GEMM; warp-collective), hi into shared
        // memory too (A of the read-out GEMM). Lanes without a slot store zeros.
        auto store_s0 = [&](int col0, const float* v) {
            const int kb = col0 >> 6;
            uint32_t hw[DCOL / 2], lw[DCOL / 2];
#pragma unroll
            for (int e = 0; e < DCOL / 2; ++e) split2(make_float2(v[2 * e], v[2 * e + 1]), hw[e], lw[e]);
            if (active) {
#pragma unroll
                for (int ch = 0; ch < DCOL / 8; ++ch)
                    *reinterpret_cast<uint4*>(s0hi + kb * Lay::ROW_TILE +
                                              ptx::sw128_chunk(i, ((col0 & 63) >> 3) + ch)) =
                        make_uint4(hw[4 * ch], hw[4 * ch + 1], hw[4 * ch + 2], hw[4 * ch + 3]);
            }
            ptx::tmem_st<DCOL / 2>(tmem + lane_base + Lay::S0HI_TCOL + col0 / 2, hw);
            ptx::tmem_st<DCOL / 2>(tmem + lane_base + Lay::S0LO_TCOL + col0 / 2, lw);
        };
        // mu and eta of chunk k, copied by the TMA warp's lanes with the chunk's q and c
        // (loaded by the workers themselves, their latency landed on the chunk)
        const float* mueta = reinterpret_cast<const float*>(smem + Lay::MUETA_OFF);
        // per-token mu, eta, |x|^2, mu^2 of 4 tokens of chunk k (this warp's share) into
        // aux[k % 2], laid out per token pair {mu0 mu1 eta0 eta1 | xx0 xx1 mu2_0 mu2_1}
        auto aux_part = [&](int k) {
            const int s = k & 1;
            const int u = lane >> 3, part = lane & 7;
            const int tau = 4 * warp + u;
            tc_wait(bar_qc, k & 1, abort);  // the q/c stage of chunk k, with its mu and eta
            float mu = 0.f, eta = 1.f;
            if (part == 0 && k * kTcC + tau < T) {
                mu = mueta[tau * 2];
                if (a.eta) eta = mueta[tau * 2 + 1];
            }
            const bool ok = tc_wait(bar_full0 + 8 * s, (k >> 1) & 1, abort);
            const uint8_t* xs = smem + Lay::X_OFF + s * Lay::X_STAGE;
            float2 acc = ptx::f2(0.f);
            if (ok) {
#pragma unroll
                for (int kb = 0; kb < DS / 64; ++kb) {
                    // the 8 lanes of a token read its 8 chunks of 16 B (any order sums the row)
                    uint4 v = *reinterpret_cast<const uint4*>(xs + kb * (64 * 128) + tau * 128 + part * 16);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xv = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
                        acc = ptx::f2fma(xv, xv, acc);
                    }
                }
            }
            const float xx = octet_sum(acc.x + acc.y);
            if (part == 0) {
                float* A = aux + (s * (kTcC / 2) + (tau >> 1)) * 8 + (tau & 1);
                const float mu2 = mu * mu;
                A[0] = mu;
                A[2] = eta;
                A[4] = xx;
                A[6] = mu2;
                if (!(mu2 >= 8.6736174e-19f)) zmu[s] = 1u;  // mu^2 < 2^-60 (or zero)
            }
        };
        // 8 tokens (half hf of this group's 16) of chunk kc from the Y^T accumulator
        auto store_y = [&](int kc, int hf) {
            uint32_t yv[8];
            ptx::tmem_ld8(tmem + lane_base + Lay::Y_COL + (kc & 1) * kTcC + sb * kTcSub + 8 * hf, yv);
            ptx::tmem_wait_ld();
            if (!ycol_ok || *abort) return;
            const int t0 = kc * kTcC + sb * kTcSub + 8 * hf;
            float* yb = a.y + (((size_t)b * T + t0) * H + h) * DS + kcol;
            const size_t stride = (size_t)H * DS;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (t0 + u < T) yb[u * stride] = __uint_as_float(yv[u]);
        };

        // ---- prologue: initial state T = S0 (sigma = 1), operands, norms, aux of chunk 0
        float sigma = 1.f;
        {
            const float* S0g = a.S0 + ((size_t)bh * MS + i) * DS + sb * DCOL;
            float v[DCOL];
            uint32_t r[DCOL];
            float ns = 0.f;
#pragma unroll
            for (int e = 0; e < DCOL; e += 4) {
                float4 t4 = active ? *reinterpret_cast<const float4*>(S0g + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[e] = t4.x; v[e + 1] = t4.y; v[e + 2] = t4.z; v[e + 3] = t4.w;
            }
#pragma unroll
            for (int e = 0; e < DCOL; ++e) {
                ns = fmaf(v[e], v[e], ns);
                r[e] = __float_as_uint(v[e]);
            }
            ptx::tmem_st<DCOL>(tmem + lane_base + Lay::T_COL + sb * DCOL, r);
            store_s0(sb * DCOL, v);
            ptx::tmem_wait_st();
            if (active) tsqp[sb * MS + i] = ns;
        }
        for (int o = tid; o < int(kTcC * 128 / 16); o += kTcWorkers)  // score blocks above the diagonal
            reinterpret_cast<uint4*>(ps)[o] = make_uint4(0u, 0u, 0u, 0u);
        if (nch > 0) {
            aux_part(0);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        if (nch > 0) ptx::named_bar(BAR_INIT, N_WM);
        // n = |s0|, 1/n and 1/n^2 of this lane's slot for the next chunk's gates
        float n, inv_n, inv_n2;
        auto load_norm = [&]() {
            float nsq = 0.f;
            if (active)
#pragma unroll
                for (int g = 0; g < NSUB; ++g) nsq += tsqp[g * MS + i];
            if (!active) nsq = 1.f;
            inv_n = ptx::rsqrt_nr(nsq);
            n = nsq * inv_n;
            inv_n2 = inv_n * inv_n;
        };
        load_norm();

        for (int k = 0; k < nch; ++k) {
            const int s = k & 1;
            // ---- phase A: gates of this group's 16 tokens (needs D1 = S0 . X_k^T)
            tc_wait(bar_d1, k & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
            uint32_t pr[kTcSub];
            ptx::tmem_ld16(tmem + lane_base + Lay::D1_COL + sb * kTcSub, pr);
            ptx::tmem_wait_ld();
            tc_wait(bar_qc, k & 1, abort);  // q and c of chunk k in shared memory
            __syncwarp();
            const bool zero_mu = zmu[s] != 0u;
            // per slot: n = |s0|; the gate of token t is g = mu - (eta c/n^2)(p/n) scaled by
            // n / sqrt(den), den = mu^2 n^2 + (eta c/n)^2 |x_perp|^2, i.e. by
            // 1/sqrt(mu^2 + (eta c/n^2)^2 |x_perp|^2); kappa/n = (eta c/n^2) by the same factor
            const float4* ax = reinterpret_cast<const float4*>(aux) + (s * (kTcC / 2) + sb * (kTcSub / 2)) * 2;
            float gv[kTcSub], kdv[kTcSub], base[kTcSub];
            float R = 1.f;
#pragma unroll
            for (int u = 0; u < kTcSub; u += 2) {
                const float4 z0 = ax[u], z1 = ax[u + 1];  // {mu eta} x2, {|x|^2 mu^2} x2
                const int tau = sb * kTcSub + u;
                const float2 cc = make_float2(csm[tau * MS + i], csm[(tau + 1) * MS + i]);
                const float2 qq = make_float2(__uint_as_float(uint32_t(qsm[tau * MS + i]) << 16),
                                              __uint_as_float(uint32_t(qsm[(tau + 1) * MS + i]) << 16));
                const float2 pp = make_float2(__uint_as_float(pr[u]), __uint_as_float(pr[u + 1]));
                const float2 mu = make_float2(z0.x, z0.y), eta = make_float2(z0.z, z0.w);
                const float2 xx = make_float2(z1.x, z1.y), mu2 = make_float2(z1.z, z1.w);
                const float2 e2 = ptx::f2mul(cc, ptx::f2mul(eta, ptx::f2(inv_n2)));  // eta c / n^2
                const float2 pn = ptx::f2mul(pp, ptx::f2(inv_n));                    // p / n
                float2 perp = ptx::f2fma(ptx::f2neg(pn), pn, xx);                     // |x_perp|^2
                perp.x = fmaxf(perp.x, 0.f);
                perp.y = fmaxf(perp.y, 0.f);
                const float2 den = ptx::f2fma(ptx::f2mul(e2, e2), perp, mu2);
                const float2 bn = ptx::rsqrt2_nr(den);
                float2 g = ptx::f2mul(bn, ptx::f2fma(ptx::f2neg(e2), pn, mu));
                float2 kn = ptx::f2mul(bn, e2);                                       // kappa / n
                if (zero_mu) {  // denormal-safe normaliser; a zero-norm update keeps the slot
                    const float2 bs = make_float2(den.x > 0.f ? ptx::rsqrt_nr(den.x) : 0.f,
                                                  den.y > 0.f ? ptx::rsqrt_nr(den.y) : 0.f);
                    g = ptx::f2mul(bs, ptx::f2fma(ptx::f2neg(e2), pn, mu));
                    kn = ptx::f2mul(bs, e2);
                    if (!(den.x > 0.f)) { g.x = 1.f; kn.x = 0.f; }
                    if (!(den.y > 0.f)) { g.y = 1.f; kn.y = 0.f; }
                }
                gv[u] = g.x;
                gv[u + 1] = g.y;
                kdv[u] = kn.x;
                kdv[u + 1] = kn.y;
                R *= g.x;
                const float R0 = R;
                R *= g.y;
                const float2 qb = ptx::f2mul(qq, make_float2(R0, R));              // q_t prod_{16sb..t} g
                base[u] = qb.x;
                base[u + 1] = qb.y;
            }
            if (active) gsub[sb * MS + i] = R;
            {   // KD(t) = kappa_t / prod_{16sb..t} g: one reciprocal, then a backward product
                float inv = n * ptx::rcp_nr(copysignf(fmaxf(fabsf(R), 1e-37f), R));
#pragma unroll
                for (int u = kTcSub - 1; u >= 0; --u) {
                    kdv[u] *= inv;
                    inv *= gv[u];
                }
            }
            if (active) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int g8 = 2 * sb + hh;
                    *reinterpret_cast<uint4*>(qr + sb * Lay::ROW_TILE + ptx::sw128_chunk(i, g8)) = pack8(base + 8 * hh);
                    *reinterpret_cast<uint4*>(kd + ptx::sw128_chunk(i, g8)) = pack8(kdv + 8 * hh);
                }
            }
            ptx::tc_fence_before();
            ptx::named_bar(BAR_G, N_WM);  // sub-chunk products known; q, c and D1 read
            ptx::tc_fence_after();
            if (tid == 0) zmu[s] = 0u;  // every worker read it before the barrier
            float G[NSUB];
#pragma unroll
            for (int g = 0; g < NSUB; ++g) G[g] = active ? gsub[g * MS + i] : 1.f;
            float F = 1.f, AC = 1.f;  // prod_{c >= sb} G_c, prod_c G_c
#pragma unroll
            for (int g = NSUB - 1; g >= 0; --g) {
                AC *= G[g];
                if (g >= sb) F *= G[g];
            }
            const float sig_c = sigma * AC;                     // sigma * A_C
            const bool pre = !(fabsf(sig_c) >= 7.8886091e-31f);  // 2^-100, or not finite
            const float inv_sig = pre ? 1.f : ptx::rcp_nr(sig_c);  // |sig_c| >= 2^-100: a normal float
            if (active) {
                // query operands of the other sub-chunks' key blocks for this group's tokens:
                // plain products for the earlier blocks, zeros for the later ones
#pragma unroll
                for (int bb = 0; bb < NSUB; ++bb) {
                    if (bb == sb) continue;
                    float cgb = 1.f;  // prod_{c=bb..sb-1} G_c
#pragma unroll
                    for (int g = 0; g < NSUB; ++g)
                        if (g >= bb && g < sb) cgb *= G[g];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint4 u4 = make_uint4(0u, 0u, 0u, 0u);
                        if (bb < sb) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 v = ptx::f2mul(make_float2(base[8 * hh + 2 * e], base[8 * hh + 2 * e + 1]),
                                                            ptx::f2(cgb));
                                w[e] = ptx::pack_bf16x2(v.x, v.y);
                            }
                            u4 = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        *reinterpret_cast<uint4*>(qr + bb * Lay::ROW_TILE + ptx::sw128_chunk(i, 2 * sb + hh)) = u4;
                    }
                }
            }
            {   // state-update coefficients KS(t) = KD(t) F_sb / (sigma A_C) -> tensor memory
                const float ksc = active ? F * inv_sig : 0.f;
                uint32_t hw[8], lw[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    split2(ptx::f2mul(make_float2(kdv[2 * e], kdv[2 * e + 1]), ptx::f2(ksc)), hw[e], lw[e]);
                ptx::tmem_st8(tmem + lane_base + Lay::KSHI_TCOL + 8 * sb, hw);
                ptx::tmem_st8(tmem + lane_base + Lay::KSLO_TCOL + 8 * sb, lw);
            }
            // rows whose old state fell below fp32 resolution: T <- sigma A_C T, sigma = 1
            if (__any_sync(0xffffffffu, pre && active)) {
                const float sc = (pre && active) ? (isfinite(sig_c) ? sig_c : 0.f) : 1.f;
                uint32_t r[DCOL];
                ptx::tmem_ld<DCOL>(tmem + lane_base + Lay::T_COL + sb * DCOL, r);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < DCOL; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * sc);
                ptx::tmem_st<DCOL>(tmem + lane_base + Lay::T_COL + sb * DCOL, r);
            }
            ptx::tmem_wait_st();
            sigma = pre ? 1.f : sig_c;
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar(BAR_A, N_WMS);

            // ---- phase B: y of the previous chunk (first half), while G7 and G4 run
            if (k > 0) {
                tc_wait(bar_y, (k - 1) & 1, abort);
                __syncwarp();
                ptx::tc_fence_after();
                store_y(k - 1, 0);
            }
            // state after the chunk (S = sigma T') and the next chunk's S0 operands
            tc_wait(bar_t, k & 1, abort);  // G7 complete
            __syncwarp();
            ptx::tc_fence_after();
            const bool renorm = !(fabsf(sigma) >= 2.3283064e-10f && fabsf(sigma) <= 4.2949673e9f);
            const bool any_renorm = __any_sync(0xffffffffu, renorm && active);  // tcgen05.st is warp-collective
            {
                uint32_t r[DCOL];
                float v[DCOL];
                ptx::tmem_ld<DCOL>(tmem + lane_base + Lay::T_COL + sb * DCOL, r);
                ptx::tmem_wait_ld();
                float2 ts = ptx::f2(0.f);
#pragma unroll
                for (int e = 0; e < DCOL; e += 2) {
                    const float2 vv = ptx::f2mul(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])),
                                                 ptx::f2(sigma));  // true state
                    ts = ptx::f2fma(vv, vv, ts);
                    v[e] = vv.x;
                    v[e + 1] = vv.y;
                }
                if (any_renorm) {
#pragma unroll
                    for (int e = 0; e < DCOL; ++e)
                        if (renorm) r[e] = __float_as_uint(v[e]);
                    ptx::tmem_st<DCOL>(tmem + lane_base + Lay::T_COL + sb * DCOL, r);
                }
                if (active) tsqp[sb * MS + i] = ts.x + ts.y;
                if (k + 1 == nch) {
                    if (active) {
                        float* So = a.S_out + ((size_t)bh * MS + i) * DS + sb * DCOL;
#pragma unroll
                        for (int e = 0; e < DCOL; e += 4)
                            *reinterpret_cast<float4*>(So + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    }
                } else {
                    tc_wait(bar_g4, k & 1, abort);  // the read-out GEMM is done with S0hi
                    __syncwarp();
                    store_s0(sb * DCOL, v);
                }
                ptx::tmem_wait_st();
            }
            if (renorm) sigma = 1.f;
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar(BAR_S0, N_WM);
            load_norm();
            if (k > 0) store_y(k - 1, 1);  // second half of the previous chunk's y

            // ---- masked scores, next chunk's per-token inputs

            if (k + 1 < nch) aux_part(k + 1);
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar(BAR_P, N_WMS);
        }
        if (nch > 0) {  // read-out of the last chunk
            tc_wait(bar_y, (nch - 1) & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
            store_y(nch - 1, 0);
            store_y(nch - 1, 1);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == MMA_WARP) ptx::tmem_dealloc(tmem, Lay::TMEM_COLS);
}

// ---------------------------------------------------------------- host side

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D map over [B][T][H][inner] (innermost first: inner, H, T, B), box {box0, 1, C, 1}.
inline bool make_map_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize,
                        int inner, int H, int T, int B, int box0, bool swizzle) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * H,
                             (cuuint64_t)inner * esize * H * T};
    cuuint32_t box[4] = {(cuuint32_t)box0, 1, (cuuint32_t)kTcC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MS, int DS>
cudaError_t launch_chunk_tc_t(const ScanArgs& a, cudaStream_t st) {
    using Lay = TcLayout<MS, DS>;
    TcMaps maps;
    if (!make_map_4d(&maps.x, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DS, a.H, a.T, a.B, 64, true) ||
        !make_map_4d(&maps.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, MS, a.H, a.T, a.B, MS, false) ||
        !make_map_4d(&maps.c, a.c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, MS, a.H, a.T, a.B, MS, false))
        return cudaErrorInvalidValue;
    auto k = chunk_tc_kernel<MS, DS>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lay::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kTcThreads, Lay::SMEM_ALLOC, st>>>(maps, a);
    return cudaGetLastError();
}

inline cudaError_t launch_chunk_tc(const ScanArgs& a, int d, cudaStream_t st) {
    if (a.m == 128 && d == 128) return launch_chunk_tc_t<128, 128>(a, st);
    if (a.m == 128 && d == 64) return launch_chunk_tc_t<128, 64>(a, st);
    if (a.m == 64 && d == 128) return launch_chunk_tc_t<64, 128>(a, st);
    if (a.m == 64 && d == 64) return launch_chunk_tc_t<64, 64>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace lattice
