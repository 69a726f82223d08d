// chunk_split.cuh -- tensor-core chunked scan with each sequence's slots split over a
// 4-CTA cluster (64 slots: 16 per CTA).
//
// Computes the same chunked form as chunk_tc.cuh (Eq. 17 of "Lattice: Learning to
// Efficiently Compress the Memory", §3.4.1 and Appendix B.1, chunk size 64), for
// workloads with fewer sequences than SMs. The recurrence never couples two slots:
// a slot's gates, write coefficients and state depend on that slot and on the
// token alone. Only the read-out y_t = sum_i q_ti s_i sums over slots. So CTA r of
// the cluster owns slots 16r..16r+15 and runs their whole state chain alone. Each
// CTA forms its partial read-out Y_r [C x d] in tensor memory, and the cluster
// reduce-scatters the partials through distributed shared memory: asynchronous
// remote stores count their bytes on the receiver's mbarrier, and CTA r adds the
// four partials of y columns r*d/4..(r+1)*d/4 (in a fixed order) and stores them.
//
// With 16 slots per CTA, every GEMM puts tokens or state columns on the MMA's M
// side (M = 64 or d) and the 16 slots on N or K:
//   G1: D1^T [C x 16] = X . (S0hi + S0lo)^T     projections (K = d)
//   G7: T^T  [d x 16] += X^T . (KShi + KSlo)    state update (K = C)
//   G4: Y_r  [C x d]  = QR_0 . S0hi             inter-chunk read-out (K = 16)
//   G5: P_r  [C x 16] = QR_b . KD_b^T, b = 0..3 scores per key sub-chunk (K = 16)
//   G6: Y_r  [C x d] += P_r . X                 intra-chunk read-out (K = C)
// The fp32 state lives in tensor memory transposed, T^T (lanes = state columns,
// 16 slot columns), as S = diag(sigma) T with the same chunk-decay folding,
// rescaling and renormalisation as the one-CTA-per-sequence kernel. The
// state-carrying operands are hi+lo bf16 pairs. Products of gates are only ever
// divided within a 16-token sub-chunk.
//
// Warp roles (448 threads). Warps 0-7 run the state chain. Warp w = 4j + q owns
// TMEM lane quadrant q. For the gates, lane l handles token 16q + (l % 16) (one
// sub-chunk per quadrant) and slots 8j + 4(l / 16) .. +3; the sub-chunk's running
// gate products are a segmented scan over 16 lanes. For the state, it handles
// state columns of quadrant q and slots 8j..8j+7. Warps 8-11 (quadrant w % 4) do
// the read-out work off the state chain: per-token inputs of the next chunk, the
// causal mask of the scores, and the cluster reduction and store of y. Warp 12
// issues every MMA, warp 13 every TMA copy. Every wait is bounded; a CTA that gives
// up a wait skips the rest of its work, so its peers time out on their next
// reduction wait and do the same.
#pragma once
#include "chunk_tc.cuh"

namespace lattice {

constexpr int kSpSlots = 16;                    // slots per CTA
constexpr int kSpNC = 4;                        // CTAs per sequence (64 slots)
constexpr int kSpWorkers = 256;                 // 8 state-chain warps
constexpr int kSpReadout = 128;                 // 4 read-out warps
constexpr int kSpThreads = kSpWorkers + kSpReadout + 64;  // + MMA warp + TMA warp

inline bool chunk_split_supported(int m, int d, int chunk, bool x_bf16, bool q_bf16) {
    return chunk == kTcC && x_bf16 && q_bf16 && m == kSpSlots * kSpNC && (d == 64 || d == 128);
}

template <int DS>
struct SpLayout {
    static constexpr int DSL = DS / kSpNC;                // y columns reduced by each CTA
    static constexpr uint32_t X_STAGE = DS * 128;         // [C][d] bf16 in d/64 SW128 blocks
    static constexpr uint32_t ROWT = kTcC * 128;          // [C rows][128 B] SW128 tile
    static constexpr uint32_t DROWT = DS * 128;           // [d rows][128 B] SW128 tile
    static constexpr uint32_t X_OFF = 0;
    static constexpr uint32_t S0HI_OFF = X_OFF + 2 * X_STAGE;   // [d][16 slots] bf16 (row = column e)
    static constexpr uint32_t S0LO_OFF = S0HI_OFF + DROWT;
    static constexpr uint32_t QR_OFF = S0LO_OFF + DROWT;        // 4 x [C][16 slots]
    static constexpr uint32_t KD_OFF = QR_OFF + 4 * ROWT;       // [C][16 slots]
    static constexpr uint32_t KSHI_OFF = KD_OFF + ROWT;         // [C][16 slots]
    static constexpr uint32_t KSLO_OFF = KSHI_OFF + ROWT;
    static constexpr uint32_t P_OFF = KSLO_OFF + ROWT;          // [C][C]
    static constexpr uint32_t RECV_OFF = P_OFF + ROWT;          // [2][NC][C][d/NC] fp32
    static constexpr uint32_t RECV_BYTES = 2 * kSpNC * kTcC * DSL * 4;
    static constexpr uint32_t Q_OFF = RECV_OFF + RECV_BYTES;    // [C][16] bf16
    static constexpr uint32_t C_OFF = Q_OFF + kTcC * kSpSlots * 2;   // [C][16] fp32
    static constexpr uint32_t AUX_OFF = C_OFF + kTcC * kSpSlots * 4;  // [2][C] float4
    static constexpr uint32_t GSUB_OFF = AUX_OFF + 2 * kTcC * 16;    // [4][16] float
    static constexpr uint32_t TSQ_OFF = GSUB_OFF + 4 * kSpSlots * 4;  // [4][16] float
    static constexpr uint32_t SIG_OFF = TSQ_OFF + 4 * kSpSlots * 4;   // [2][16] float
    static constexpr uint32_t PSC_OFF = SIG_OFF + 2 * kSpSlots * 4;   // [16] float: rescale factors
    static constexpr uint32_t BAR_OFF = PSC_OFF + kSpSlots * 4;       // 14 mbarriers
    static constexpr uint32_t MISC_OFF = BAR_OFF + 14 * 8;
    static constexpr uint32_t BYTES = MISC_OFF + 64;
    static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;
    // TMEM columns: T^T | D1^T | P | Y double-buffered
    static constexpr uint32_t T_COL = 0;
    static constexpr uint32_t D1_COL = kSpSlots;
    static constexpr uint32_t P_COL = 2 * kSpSlots;
    static constexpr uint32_t Y_COL = 2 * kSpSlots + kTcC;     // + (chunk & 1) * d
    static constexpr uint32_t TMEM_COLS = (Y_COL + 2 * DS <= 256) ? 256 : 512;
    static constexpr uint32_t TX_BYTES = X_STAGE;
    static constexpr uint32_t QC_BYTES = kTcC * kSpSlots * 6;
    static_assert(Q_OFF % 1024 == 0 && P_OFF % 1024 == 0, "tile alignment");
};

// Per-slot chunk decay and rescaling decision, evaluated identically by every thread
// that needs it (the gate side for KS, the state side for the rescale).
__device__ __forceinline__ void sp_decay(const float* G4, int q, float sigma, float& F, float& AC,
                                         float& sig_c, bool& pre) {
    F = 1.f;
    AC = 1.f;
#pragma unroll
    for (int c = 3; c >= 0; --c) {
        AC *= G4[c];
        if (c >= q) F *= G4[c];
    }
    sig_c = sigma * AC;
    pre = !(fabsf(sig_c) >= 7.8886091e-31f);  // 2^-100, or not finite
}

__device__ __forceinline__ bool tc_wait_cluster(uint32_t bar, uint32_t parity, volatile uint32_t* abort) {
    if (*abort) return false;
    const uint64_t t0 = ptx::globaltimer();
    for (;;) {
        if (ptx::mbar_try_wait_cluster(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (ptx::globaltimer() - t0 > kTcWaitNs) {
            *abort = 1u;
            flag_timeout();
            return false;
        }
    }
}

template <int DS>
__global__ void __launch_bounds__(kSpThreads, 1)
    chunk_split_kernel(const __grid_constant__ TcMaps maps, ScanArgs a) {
    using Lay = SpLayout<DS>;
    constexpr int DSL = Lay::DSL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = (int)ptx::cluster_ctarank();
    const int bh = blockIdx.x / kSpNC, b = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H;
    const int nch = (T + kTcC - 1) / kTcC;
    constexpr int RO_WARP0 = kSpWorkers / 32, MMA_WARP = RO_WARP0 + 4, TMA_WARP = MMA_WARP + 1;

    // mbarriers: X stage landed [2], q/c landed, D1 ready, T updated (G7), S0 operand
    // read (G4), scores ready (G5), read-out GEMMs done (G6), peers' partial y in [2],
    // per-token inputs ready [2] (per chunk parity), read-out buffer drained [2]
    const uint32_t bar_full0 = sbase + Lay::BAR_OFF;
    const uint32_t bar_qc = sbase + Lay::BAR_OFF + 16;
    const uint32_t bar_d1 = sbase + Lay::BAR_OFF + 24;
    const uint32_t bar_t = sbase + Lay::BAR_OFF + 32;
    const uint32_t bar_g4 = sbase + Lay::BAR_OFF + 40;
    const uint32_t bar_p5 = sbase + Lay::BAR_OFF + 48;
    const uint32_t bar_y = sbase + Lay::BAR_OFF + 56;
    const uint32_t bar_recv0 = sbase + Lay::BAR_OFF + 64;   // armed with the bytes of 4 CTAs' partials
    const uint32_t bar_aux0 = sbase + Lay::BAR_OFF + 80;    // 128 arrivals: the read-out threads
    const uint32_t bar_yfree0 = sbase + Lay::BAR_OFF + 96;  // 128 arrivals
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
    volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 4);
    volatile uint32_t* zmu = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 8);
    // per chunk parity: set when some slot's old state must be rescaled before the state-update GEMM
    volatile uint32_t* pflag = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 16);
    float* psc = reinterpret_cast<float*>(smem + Lay::PSC_OFF);
    float4* aux = reinterpret_cast<float4*>(smem + Lay::AUX_OFF);
    float* gsub = reinterpret_cast<float*>(smem + Lay::GSUB_OFF);
    float* tsqp = reinterpret_cast<float*>(smem + Lay::TSQ_OFF);
    float* sig = reinterpret_cast<float*>(smem + Lay::SIG_OFF);

    // named barriers: workers + MMA warp (INIT, A, S0), workers + TMA warp (G),
    // read-out warps (arrive) + MMA warp (P), workers alone (N), workers + MMA warp
    // only in chunks with a rescale (T)
    constexpr uint32_t BAR_INIT = 1, BAR_G = 2, BAR_A = 3, BAR_S0 = 4, BAR_P = 5, BAR_N = 6, BAR_T = 7;
    constexpr uint32_t N_WM = kSpWorkers + 32, N_RM = kSpReadout + 32;

    if (warp == MMA_WARP) {
        if (lane == 0) {
            for (int j = 0; j < 8; ++j) ptx::mbar_init(sbase + Lay::BAR_OFF + 8 * j, 1);
            ptx::mbar_init(bar_recv0, 1);
            ptx::mbar_init(bar_recv0 + 8, 1);
            ptx::mbar_init(bar_aux0, kSpReadout);
            ptx::mbar_init(bar_aux0 + 8, kSpReadout);
            ptx::mbar_init(bar_yfree0, kSpReadout);
            ptx::mbar_init(bar_yfree0 + 8, kSpReadout);
            *abort = 0u;
            zmu[0] = 0u;
            zmu[1] = 0u;
            pflag[0] = 0u;
            pflag[1] = 0u;
            ptx::fence_mbar_init();
        }
        __syncwarp();
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), Lay::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // every CTA's barriers exist before any peer arrives on them
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issue
        constexpr uint32_t idesc_g1 = ptx::idesc_bf16(kTcC, kSpSlots, 0, 1);
        constexpr uint32_t idesc_g7 = ptx::idesc_bf16(DS, kSpSlots, 1, 1);
        constexpr uint32_t idesc_g4 = ptx::idesc_bf16(kTcC, DS, 0, 0);
        constexpr uint32_t idesc_g5 = ptx::idesc_bf16(kTcC, kSpSlots, 0, 0);
        constexpr uint32_t idesc_g6 = ptx::idesc_bf16(kTcC, DS, 0, 1);
        auto off = [](uint32_t bytes) { return uint64_t(bytes >> 4); };
        auto g1 = [&](int k) {  // D1^T = X_k . (S0hi + S0lo)^T  (M = C, N = 16, K = d)
            const uint64_t dK_x = ptx::sdesc_sw128(sbase + Lay::X_OFF, 16, 1024);
            const uint64_t dM_hi = ptx::sdesc_sw128(sbase + Lay::S0HI_OFF, 8192, 1024);
            const uint64_t dM_lo = ptx::sdesc_sw128(sbase + Lay::S0LO_OFF, 8192, 1024);
            const uint32_t xo = (k & 1) * Lay::X_STAGE;
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk) {
                    const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
                    ptx::mma_bf16_elect(tmem + Lay::D1_COL, dK_x + off(xo + kb * 64 * 128 + ko),
                                        (part ? dM_lo : dM_hi) + off(kk * 2048), idesc_g1, (part | kk) != 0);
                }
        };
        if (nch > 0) {
            ptx::named_bar(BAR_INIT, N_WM);
            ptx::tc_fence_after();
            if (tc_wait_warp(bar_full0, 0, abort)) g1(0);
            ptx::mma_commit_elect(bar_d1);
        }
        const uint64_t dM_x = ptx::sdesc_sw128(sbase + Lay::X_OFF, 64 * 128, 1024);
        const uint64_t dM_kshi = ptx::sdesc_sw128(sbase + Lay::KSHI_OFF, 8192, 1024);
        const uint64_t dM_kslo = ptx::sdesc_sw128(sbase + Lay::KSLO_OFF, 8192, 1024);
        const uint64_t dK_qr = ptx::sdesc_sw128(sbase + Lay::QR_OFF, 16, 1024);
        const uint64_t dK_kd = ptx::sdesc_sw128(sbase + Lay::KD_OFF, 16, 1024);
        const uint64_t dK_s0hi = ptx::sdesc_sw128(sbase + Lay::S0HI_OFF, 16, 1024);
        const uint64_t dK_p = ptx::sdesc_sw128(sbase + Lay::P_OFF, 16, 1024);
        for (int k = 0; k < nch; ++k) {
            const uint32_t xo = (k & 1) * Lay::X_STAGE;
            const uint32_t ycol = Lay::Y_COL + (k & 1) * DS;
            ptx::named_bar(BAR_A, N_WM);  // KS, QR, KD written
            if (pflag[k & 1]) ptx::named_bar(BAR_T, N_WM);  // T^T rescaled (rare)
            ptx::tc_fence_after();
            if (tc_live(abort)) {
                // G7: T^T += X^T . KS  (M = d, N = 16, K = C); both MN-major
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < kTcC / 16; ++kk)
                        ptx::mma_bf16_elect(tmem + Lay::T_COL, dM_x + off(xo + kk * 2048),
                                            (part ? dM_kslo : dM_kshi) + off(kk * 2048), idesc_g7, 1);
            }
            ptx::mma_commit_elect(bar_t);
            // the read-out of chunk k-2 (same accumulator buffer) has been drained
            const bool yfree = k < 2 || tc_wait_warp(bar_yfree0 + 8 * (k & 1), ((k - 2) >> 1) & 1, abort);
            ptx::tc_fence_after();
            if (yfree && tc_live(abort)) {
                // G4: Y_r = QR_0 . S0hi  (M = C, N = d, K = 16); both K-major
                ptx::mma_bf16_elect(tmem + ycol, dK_qr, dK_s0hi, idesc_g4, 0);
            }
            ptx::mma_commit_elect(bar_g4);
            if (tc_live(abort)) {
                // G5: P[:, 16b..16b+15] = QR_b . KD_b^T  (M = C, N = 16, K = 16)
#pragma unroll
                for (int sb = 0; sb < 4; ++sb)
                    ptx::mma_bf16_elect(tmem + Lay::P_COL + sb * 16, dK_qr + off(sb * Lay::ROWT),
                                        dK_kd + off(sb * 16 * 128), idesc_g5, 0);
            }
            ptx::mma_commit_elect(bar_p5);
            ptx::named_bar(BAR_S0, N_WM);  // S0 operands of chunk k+1 written
            ptx::tc_fence_after();
            if (k + 1 < nch) {
                if (tc_wait_warp(bar_full0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1, abort)) g1(k + 1);
                ptx::mma_commit_elect(bar_d1);
            }
            ptx::named_bar(BAR_P, N_RM);  // masked scores written by the read-out warps
            ptx::tc_fence_after();
            if (tc_live(abort)) {
                // G6: Y_r += P . X  (M = C, N = d, K = C); A K-major, B MN-major
#pragma unroll
                for (int kk = 0; kk < kTcC / 16; ++kk)
                    ptx::mma_bf16_elect(tmem + ycol, dK_p + off(kk * 32), dM_x + off(xo + kk * 2048), idesc_g6, 1);
            }
            ptx::mma_commit_elect(bar_y);
        }
        if (nch > 0) tc_drain(bar_y, (nch - 1) & 1);
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------------ TMA issue (lane 0)
        int last_x[2] = {-1, -1}, last_qc = -1;
        const int s_lo = rank * kSpSlots;  // this CTA's slots in the q and c rows
        auto issue_x = [&](int k) {
            const int s = k & 1;
            last_x[s] = k;
            const uint32_t bar = bar_full0 + 8 * s;
            ptx::mbar_arrive_expect_tx(bar, Lay::TX_BYTES);
#pragma unroll
            for (int kb = 0; kb < DS / 64; ++kb)
                ptx::tma_load_4d(sbase + Lay::X_OFF + s * Lay::X_STAGE + kb * (64 * 128), &maps.x, bar, kb * 64,
                                 h, k * kTcC, b);
        };
        auto issue_qc = [&](int k) {
            last_qc = k;
            ptx::mbar_arrive_expect_tx(bar_qc, Lay::QC_BYTES);
            ptx::tma_load_4d(sbase + Lay::Q_OFF, &maps.q, bar_qc, s_lo, h, k * kTcC, b);
            ptx::tma_load_4d(sbase + Lay::C_OFF, &maps.c, bar_qc, s_lo, h, k * kTcC, b);
        };
        auto prefetch_l2 = [&](int k) {
#pragma unroll
            for (int kb = 0; kb < DS / 64; ++kb) ptx::tma_prefetch_l2_4d(&maps.x, kb * 64, h, k * kTcC, b);
            ptx::tma_prefetch_l2_4d(&maps.q, s_lo, h, k * kTcC, b);
            ptx::tma_prefetch_l2_4d(&maps.c, s_lo, h, k * kTcC, b);
        };
        if (lane == 0 && nch > 0) {
            ptx::prefetch_tensormap(&maps.x);
            ptx::prefetch_tensormap(&maps.q);
            ptx::prefetch_tensormap(&maps.c);
            issue_x(0);
            issue_qc(0);
            if (nch > 1) issue_x(1);
            for (int j = 1; j < 4 && j < nch; ++j) prefetch_l2(j);
        }
        for (int k = 0; k < nch; ++k) {
            ptx::named_bar(BAR_G, N_WM);  // q and c of chunk k consumed
            if (lane == 0) {
                if (k + 1 < nch) issue_qc(k + 1);
                if (k + 2 < nch && tc_wait(bar_y, k & 1, abort)) {  // G6_k was X_k's last reader
                    issue_x(k + 2);
                    if (k + 4 < nch) prefetch_l2(k + 4);
                }
            }
            __syncwarp();
        }
        if (lane == 0) {
#pragma unroll
            for (int s = 0; s < 2; ++s)
                if (last_x[s] >= 0) tc_drain(bar_full0 + 8 * s, (last_x[s] >> 1) & 1);
            if (last_qc >= 0) tc_drain(bar_qc, last_qc & 1);
        }
        __syncwarp();
    } else if (warp >= RO_WARP0) {
        // ------------------------------------------------------------ read-out warps
        const int q = warp & 3;
        const int rt = tid - kSpWorkers;  // 0..127
        const uint32_t lane_base = uint32_t(32 * q) << 16;
        const bool row_ok = lane < 16;     // M = 64 accumulators: lanes 0-15 of each quadrant
        const int trow = 16 * q + lane;    // accumulator row (token) of this lane
        // per-token mu, eta, |x|^2, mu^2 of chunk k: 2 threads per token, each half of x
        auto aux_chunk = [&](int k) {
            const int s = k & 1;
            const int tk = rt >> 1, half = rt & 1;
            const int t = k * kTcC + tk;
            float mu = 0.f, eta = 1.f;
            if (half == 0 && t < T) {
                const size_t bth = ((size_t)b * T + t) * H + h;
                mu = __ldg(a.mu + bth);
                if (a.eta) eta = __ldg(a.eta + bth);
            }
            const bool ok = tc_wait(bar_full0 + 8 * s, (k >> 1) & 1, abort);
            const uint8_t* xs = smem + Lay::X_OFF + s * Lay::X_STAGE;
            float2 acc = ptx::f2(0.f);
            if (ok) {
#pragma unroll
                for (int u = 0; u < DS / 16; ++u) {  // DS/16 chunks of 16 B per thread
                    const int ch = half * (DS / 16) + u;  // block ch/8, chunk ch%8 (any order sums the row)
                    uint4 v = *reinterpret_cast<const uint4*>(xs + (ch >> 3) * (64 * 128) + tk * 128 + (ch & 7) * 16);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 xv = make_float2(__uint_as_float(w[c] << 16), __uint_as_float(w[c] & 0xffff0000u));
                        acc = ptx::f2fma(xv, xv, acc);
                    }
                }
            }
            float xx = acc.x + acc.y;
            xx += __shfl_xor_sync(0xffffffffu, xx, 1);
            if (half == 0) {
                const float mu2 = mu * mu;
                aux[s * kTcC + tk] = make_float4(mu, eta, xx, mu2);
                if (!(mu2 >= 8.6736174e-19f)) zmu[s] = 1u;  // mu^2 < 2^-60 (or zero)
            }
            ptx::mbar_arrive(bar_aux0 + 8 * s);
        };
        // the four partials of this CTA's columns of chunk kc -> y. Summing chunk k-1
        // before sending chunk k keeps two receive buffers enough: a peer's chunk k+1
        // follows its sum of chunk k, which needs this CTA's chunk k, sent after this sum.
        constexpr uint32_t RECV_TX = kSpNC * kTcC * DSL * 4;  // bytes of one chunk's partials
        auto recv_y = [&](int kc) {
            const int par = kc & 1;
            tc_wait_cluster(bar_recv0 + 8 * par, (kc >> 1) & 1, abort);
            if (rt == 0 && kc + 2 < nch) ptx::mbar_arrive_expect_tx(bar_recv0 + 8 * par, RECV_TX);  // chunk kc+2
            if (*abort) return;
            const int tk = rt >> 1;
            const int t = kc * kTcC + tk;
            constexpr int PER = DSL / 2;  // floats per thread: 8 (d = 64) or 16 (d = 128)
            const int c0 = (rt & 1) * PER;
            float acc[PER];
#pragma unroll
            for (int c = 0; c < PER; ++c) acc[c] = 0.f;
#pragma unroll
            for (int src = 0; src < kSpNC; ++src) {
                const float* rb = reinterpret_cast<const float*>(
                                      smem + Lay::RECV_OFF + ((par * kSpNC + src) * kTcC + tk) * (DSL * 4)) + c0;
#pragma unroll
                for (int c = 0; c < PER; c += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(rb + c);
                    acc[c] += v.x; acc[c + 1] += v.y; acc[c + 2] += v.z; acc[c + 3] += v.w;
                }
            }
            if (t < T) {
                float* yp = a.y + (((size_t)b * T + t) * H + h) * DS + rank * DSL + c0;
#pragma unroll
                for (int c = 0; c < PER; c += 4)
                    *reinterpret_cast<float4*>(yp + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
            }
        };
        if (rt == 0) {  // arm the receive barriers of chunks 0 and 1
            if (nch > 0) ptx::mbar_arrive_expect_tx(bar_recv0, RECV_TX);
            if (nch > 1) ptx::mbar_arrive_expect_tx(bar_recv0 + 8, RECV_TX);
        }
        if (nch > 0) aux_chunk(0);
        for (int k = 0; k < nch; ++k) {
            const int par = k & 1;
            if (k + 1 < nch) aux_chunk(k + 1);
            // causal mask of this chunk's scores: row trow, all 64 keys
            tc_wait(bar_p5, k & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + lane_base + Lay::P_COL + 32 * half, r);
                ptx::tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        float v[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int key = 32 * half + 8 * c8 + c;
                            v[c] = (key <= trow) ? __uint_as_float(r[8 * c8 + c]) : 0.f;
                        }
                        *reinterpret_cast<uint4*>(smem + Lay::P_OFF + ptx::sw128_chunk(trow, 4 * half + c8)) = pack8(v);
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar_arrive(BAR_P, N_RM);
            if (k > 0) recv_y(k - 1);
            // partial read-out of this chunk: every peer's quarter of the columns
            tc_wait(bar_y, k & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
#pragma unroll
            for (int p = 0; p < kSpNC; ++p) {
                __syncwarp();  // tcgen05.ld is warp-collective
                uint32_t yv[DSL];
                ptx::tmem_ld<DSL>(tmem + lane_base + Lay::Y_COL + par * DS + p * DSL, yv);
                ptx::tmem_wait_ld();
                if (row_ok && !*abort) {
                    const uint32_t dst = Lay::RECV_OFF + ((par * kSpNC + rank) * kTcC + trow) * (DSL * 4);
                    const uint32_t cdst = ptx::mapa(sbase + dst, (uint32_t)p);
                    const uint32_t cbar = ptx::mapa(bar_recv0 + 8 * par, (uint32_t)p);
#pragma unroll
                    for (int c = 0; c < DSL; c += 4)
                        ptx::st_async_v4(cdst + c * 4, make_float4(__uint_as_float(yv[c]), __uint_as_float(yv[c + 1]),
                                                                   __uint_as_float(yv[c + 2]), __uint_as_float(yv[c + 3])),
                                         cbar);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_yfree0 + 8 * par);  // this buffer may take chunk k+2
        }
        if (nch > 0) recv_y(nch - 1);
    } else {
        // ================================================================ state-chain workers
        const int q = warp & 3, j = warp >> 2;
        const uint32_t lane_base = uint32_t(32 * q) << 16;
        // gate role: token tau (sub-chunk q), slots s0..s0+3
        const int tau = 16 * q + (lane & 15);
        const int s0 = 8 * j + 4 * (lane >> 4);
        const bool seg_last = (lane & 15) == 15;
        // state role: state column e of quadrant q (d = 64: lanes 0-15 of the quadrant), slots 8j..8j+7
        const bool e_ok = (DS == 128) || (lane < 16);
        const int e = (DS == 128) ? (32 * q + lane) : (16 * q + (lane & 15));
        uint8_t* qr = smem + Lay::QR_OFF;
        uint8_t* kd = smem + Lay::KD_OFF;
        const uint16_t* qsm = reinterpret_cast<const uint16_t*>(smem + Lay::Q_OFF);
        const float* csm = reinterpret_cast<const float*>(smem + Lay::C_OFF);

        // state columns e, slots 8j..8j+7 -> |.|^2 partial per slot (butterfly over the
        // quadrant's 32 lanes: lane l ends with slot 4b16 + 2b8 + b4 of its bits)
        auto col_norms = [&](const float* v) {
            float w[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) w[c] = e_ok ? v[c] * v[c] : 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const bool up = lane & 16;
                const float send = up ? w[c] : w[c + 4];
                const float keep = up ? w[c + 4] : w[c];
                w[c] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const bool up = lane & 8;
                const float send = up ? w[c] : w[c + 2];
                const float keep = up ? w[c + 2] : w[c];
                w[c] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            {
                const bool up = lane & 4;
                const float send = up ? w[0] : w[1];
                const float keep = up ? w[1] : w[0];
                w[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            w[0] += __shfl_xor_sync(0xffffffffu, w[0], 2);
            w[0] += __shfl_xor_sync(0xffffffffu, w[0], 1);
            if ((lane & 3) == 0) {
                const int slot = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
                tsqp[q * kSpSlots + 8 * j + slot] = w[0];
            }
        };
        // state columns e, slots 8j..8j+7 -> hi/lo bf16 operand rows (row e, bytes 16j..16j+15)
        auto store_s0 = [&](const float* v) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) split2(make_float2(v[2 * c], v[2 * c + 1]), hw[c], lw[c]);
            if (e_ok) {
                const uint32_t o = ptx::sw128_chunk(e, j);
                *reinterpret_cast<uint4*>(smem + Lay::S0HI_OFF + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(smem + Lay::S0LO_OFF + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        };
        // n = |s0|, 1/n and 1/n^2 of slots s0..s0+3 for the next chunk's gates
        auto load_norms = [&](float* n, float* inv_n, float* inv_n2) {
            const float4 t0 = *reinterpret_cast<const float4*>(tsqp + 0 * kSpSlots + s0);
            const float4 t1 = *reinterpret_cast<const float4*>(tsqp + 1 * kSpSlots + s0);
            const float4 t2 = *reinterpret_cast<const float4*>(tsqp + 2 * kSpSlots + s0);
            const float4 t3 = *reinterpret_cast<const float4*>(tsqp + 3 * kSpSlots + s0);
            const float nsq[4] = {((t0.x + t1.x) + t2.x) + t3.x, ((t0.y + t1.y) + t2.y) + t3.y,
                                  ((t0.z + t1.z) + t2.z) + t3.z, ((t0.w + t1.w) + t2.w) + t3.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                inv_n[c] = ptx::rsqrt_nr(nsq[c]);
                n[c] = nsq[c] * inv_n[c];
                inv_n2[c] = inv_n[c] * inv_n[c];
            }
        };

        // ---- prologue: T^T = S0^T (sigma = 1), S0 operands, norms
        {
            // tiles of the earlier-sub-chunk query operands stay zero where a later
            // sub-chunk's tokens would be (never written below)
            uint4* z = reinterpret_cast<uint4*>(qr);
            for (int o = tid; o < int(4 * Lay::ROWT / 16); o += kSpWorkers) z[o] = make_uint4(0u, 0u, 0u, 0u);
            if (tid < 2 * kSpSlots) sig[tid] = 1.f;
            float v[8];
            uint32_t r[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int slot = rank * kSpSlots + 8 * j + c;
                v[c] = e_ok ? a.S0[((size_t)bh * (kSpSlots * kSpNC) + slot) * DS + e] : 0.f;
                r[c] = __float_as_uint(v[c]);
            }
            ptx::tmem_st8(tmem + lane_base + Lay::T_COL + 8 * j, r);
            col_norms(v);
            store_s0(v);
            ptx::tmem_wait_st();
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        if (nch > 0) ptx::named_bar(BAR_INIT, N_WM);
        float n[4], inv_n[4], inv_n2[4];
        load_norms(n, inv_n, inv_n2);

        for (int k = 0; k < nch; ++k) {
            const int s = k & 1;
            // ---- phase A: gates of token tau for slots s0..s0+3
            tc_wait(bar_d1, k & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
            float p4[4];
            {
                uint32_t pr[8];
                ptx::tmem_ld8(tmem + lane_base + Lay::D1_COL + 8 * j, pr);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // lanes 16-31 take slots 4..7 of lane l-16's token
                    const float up = __shfl_sync(0xffffffffu, __uint_as_float(pr[4 + c]), lane & 15);
                    p4[c] = (lane < 16) ? __uint_as_float(pr[c]) : up;
                }
            }
            tc_wait(bar_aux0 + 8 * s, (k >> 1) & 1, abort);  // per-token inputs of chunk k
            tc_wait(bar_qc, k & 1, abort);
            __syncwarp();
            const bool zero_mu = zmu[s] != 0u;
            const float4 z = aux[s * kTcC + tau];  // mu, eta, |x|^2, mu^2
            const float4 cv = *reinterpret_cast<const float4*>(csm + tau * kSpSlots + s0);
            const uint2 qv = *reinterpret_cast<const uint2*>(qsm + tau * kSpSlots + s0);
            const float qf[4] = {__uint_as_float(qv.x << 16), __uint_as_float(qv.x & 0xffff0000u),
                                 __uint_as_float(qv.y << 16), __uint_as_float(qv.y & 0xffff0000u)};
            const float cf[4] = {cv.x, cv.y, cv.z, cv.w};
            float g[4], kn[4];
#pragma unroll
            for (int c = 0; c < 4; c += 2) {
                const float2 cc = make_float2(cf[c], cf[c + 1]);
                const float2 pp = make_float2(p4[c], p4[c + 1]);
                const float2 e2 = ptx::f2mul(cc, ptx::f2mul(ptx::f2(z.y), make_float2(inv_n2[c], inv_n2[c + 1])));
                const float2 pn = ptx::f2mul(pp, make_float2(inv_n[c], inv_n[c + 1]));
                float2 perp = ptx::f2fma(ptx::f2neg(pn), pn, ptx::f2(z.z));
                perp.x = fmaxf(perp.x, 0.f);
                perp.y = fmaxf(perp.y, 0.f);
                const float2 den = ptx::f2fma(ptx::f2mul(e2, e2), perp, ptx::f2(z.w));
                float2 bn = ptx::rsqrt2_nr(den);
                if (zero_mu) {
                    bn = make_float2(den.x > 0.f ? ptx::rsqrt_nr(den.x) : 0.f, den.y > 0.f ? ptx::rsqrt_nr(den.y) : 0.f);
                }
                float2 gg = ptx::f2mul(bn, ptx::f2fma(ptx::f2neg(e2), pn, ptx::f2(z.x)));
                float2 kk = ptx::f2mul(bn, e2);  // kappa / n
                if (zero_mu) {
                    if (!(den.x > 0.f)) { gg.x = 1.f; kk.x = 0.f; }
                    if (!(den.y > 0.f)) { gg.y = 1.f; kk.y = 0.f; }
                }
                g[c] = gg.x; g[c + 1] = gg.y;
                kn[c] = kk.x; kn[c + 1] = kk.y;
            }
            // running products over the sub-chunk's 16 tokens (segmented inclusive scan)
            float R[4] = {g[0], g[1], g[2], g[3]};
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float t = __shfl_up_sync(0xffffffffu, R[c], o, 16);
                    if ((lane & 15) >= o) R[c] *= t;
                }
            }
            float base[4], kdv[4], Gq[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                base[c] = qf[c] * R[c];                               // q_t prod_{16q..t} g
                kdv[c] = kn[c] * n[c] * ptx::rcp_nr(copysignf(fmaxf(fabsf(R[c]), 1e-37f), R[c]));  // kappa / prod
                Gq[c] = __shfl_sync(0xffffffffu, R[c], 15, 16);       // the sub-chunk's product
            }
            if (seg_last)
                *reinterpret_cast<float4*>(gsub + q * kSpSlots + s0) = make_float4(Gq[0], Gq[1], Gq[2], Gq[3]);
            {
                const uint32_t o = ptx::sw128_off(tau, s0);
                *reinterpret_cast<uint2*>(qr + q * Lay::ROWT + o) =
                    make_uint2(ptx::pack_bf16x2(base[0], base[1]), ptx::pack_bf16x2(base[2], base[3]));
                *reinterpret_cast<uint2*>(kd + o) =
                    make_uint2(ptx::pack_bf16x2(kdv[0], kdv[1]), ptx::pack_bf16x2(kdv[2], kdv[3]));
            }
            ptx::tc_fence_before();
            ptx::named_bar(BAR_G, N_WM);
            ptx::tc_fence_after();
            if (tid == 0) zmu[s] = 0u;
            {   // gate side: cross-sub-chunk query operands, state-update coefficients
                float G[4][4];  // [sub-chunk][slot]
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 t4 = *reinterpret_cast<const float4*>(gsub + c * kSpSlots + s0);
                    G[c][0] = t4.x; G[c][1] = t4.y; G[c][2] = t4.z; G[c][3] = t4.w;
                }
                const float4 sg = *reinterpret_cast<const float4*>(sig + s * kSpSlots + s0);
                const float sgv[4] = {sg.x, sg.y, sg.z, sg.w};
                float ksc[4], sig_new[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float G4[4] = {G[0][c], G[1][c], G[2][c], G[3][c]};
                    float F, AC, sig_c;
                    bool pre;
                    sp_decay(G4, q, sgv[c], F, AC, sig_c, pre);
                    ksc[c] = F * (pre ? 1.f : ptx::rcp_nr(sig_c));  // |sig_c| >= 2^-100: a normal float
                    sig_new[c] = pre ? 1.f : sig_c;
                }
#pragma unroll
                for (int bb = 0; bb < 3; ++bb) {
                    if (bb >= q) break;
                    float v[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float cgb = 1.f;  // prod_{sub-chunks bb..q-1}
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc)
                            if (cc >= bb && cc < q) cgb *= G[cc][c];
                        v[c] = base[c] * cgb;
                    }
                    *reinterpret_cast<uint2*>(qr + bb * Lay::ROWT + ptx::sw128_off(tau, s0)) =
                        make_uint2(ptx::pack_bf16x2(v[0], v[1]), ptx::pack_bf16x2(v[2], v[3]));
                }
                uint32_t hw[2], lw[2];
                split2(ptx::f2mul(make_float2(kdv[0], kdv[1]), make_float2(ksc[0], ksc[1])), hw[0], lw[0]);
                split2(ptx::f2mul(make_float2(kdv[2], kdv[3]), make_float2(ksc[2], ksc[3])), hw[1], lw[1]);
                const uint32_t o = ptx::sw128_off(tau, s0);
                *reinterpret_cast<uint2*>(smem + Lay::KSHI_OFF + o) = make_uint2(hw[0], hw[1]);
                *reinterpret_cast<uint2*>(smem + Lay::KSLO_OFF + o) = make_uint2(lw[0], lw[1]);
                if (tau == 0) {
                    *reinterpret_cast<float4*>(sig + (s ^ 1) * kSpSlots + s0) =
                        make_float4(sig_new[0], sig_new[1], sig_new[2], sig_new[3]);
                    float sc[4];
                    bool any = false;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float G4[4] = {G[0][c], G[1][c], G[2][c], G[3][c]};
                        float F, AC, sig_c;
                        bool pre;
                        sp_decay(G4, q, sgv[c], F, AC, sig_c, pre);
                        sc[c] = pre ? (isfinite(sig_c) ? sig_c : 0.f) : 1.f;
                        any = any || pre;
                    }
                    *reinterpret_cast<float4*>(psc + s0) = make_float4(sc[0], sc[1], sc[2], sc[3]);
                    if (any) pflag[s] = 1u;
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar(BAR_A, N_WM);
            if (pflag[s]) {  // the same decision as the MMA warp's
                // columns whose decayed old state fell below fp32 resolution: T <- sigma A_C T
                const float4 sa = *reinterpret_cast<const float4*>(psc + 8 * j);
                const float4 sb4 = *reinterpret_cast<const float4*>(psc + 8 * j + 4);
                const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb4.x, sb4.y, sb4.z, sb4.w};
                ptx::tc_fence_after();
                uint32_t r[8];
                ptx::tmem_ld8(tmem + lane_base + Lay::T_COL + 8 * j, r);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * sc[c]);
                ptx::tmem_st8(tmem + lane_base + Lay::T_COL + 8 * j, r);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::named_bar(BAR_T, N_WM);
            }

            // ---- phase B: state after the chunk, next S0 operands
            tc_wait(bar_t, k & 1, abort);
            __syncwarp();
            ptx::tc_fence_after();
            {
                const float4 sa = *reinterpret_cast<const float4*>(sig + (s ^ 1) * kSpSlots + 8 * j);
                const float4 sb4 = *reinterpret_cast<const float4*>(sig + (s ^ 1) * kSpSlots + 8 * j + 4);
                const float sg[8] = {sa.x, sa.y, sa.z, sa.w, sb4.x, sb4.y, sb4.z, sb4.w};
                uint32_t r[8];
                float v[8];
                ptx::tmem_ld8(tmem + lane_base + Lay::T_COL + 8 * j, r);
                ptx::tmem_wait_ld();
                bool any_renorm = false;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    v[c] = __uint_as_float(r[c]) * sg[c];
                    const bool rn = !(fabsf(sg[c]) >= 2.3283064e-10f && fabsf(sg[c]) <= 4.2949673e9f);
                    if (rn) r[c] = __float_as_uint(v[c]);
                    any_renorm = any_renorm || rn;
                }
                if (any_renorm) ptx::tmem_st8(tmem + lane_base + Lay::T_COL + 8 * j, r);  // warp-uniform
                if (k + 1 == nch) {
                    if (e_ok) {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            a.S_out[((size_t)bh * (kSpSlots * kSpNC) + rank * kSpSlots + 8 * j + c) * DS + e] = v[c];
                    }
                } else {
                    tc_wait(bar_g4, k & 1, abort);  // G4 is done with S0hi
                    __syncwarp();
                    store_s0(v);
                }
                ptx::tmem_wait_st();
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::named_bar(BAR_S0, N_WM);
                // the next chunk's slot norms, while the projection GEMM runs
                if (k + 1 < nch) col_norms(v);
            }
            if (tid == 0) pflag[s] = 0u;  // read by every worker and the MMA warp before BAR_S0
            if (tau == 0) {  // renormalised slots restart at sigma = 1
                float* sp = sig + (s ^ 1) * kSpSlots + s0;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (!(fabsf(sp[c]) >= 2.3283064e-10f && fabsf(sp[c]) <= 4.2949673e9f)) sp[c] = 1.f;
            }
            if (k + 1 < nch) {
                ptx::named_bar(BAR_N, kSpWorkers);  // every slot's partial norms written
                load_norms(n, inv_n, inv_n2);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // no peer still writes into this CTA's shared memory
    ptx::tc_fence_after();
    if (warp == MMA_WARP) ptx::tmem_dealloc(tmem, Lay::TMEM_COLS);
}

template <int DS>
cudaError_t launch_chunk_split_t(const ScanArgs& a, cudaStream_t st) {
    using Lay = SpLayout<DS>;
    TcMaps maps;
    const int m = kSpSlots * kSpNC;
    if (!make_map_4d(&maps.x, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DS, a.H, a.T, a.B, 64, true) ||
        !make_map_4d(&maps.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, m, a.H, a.T, a.B, kSpSlots, false) ||
        !make_map_4d(&maps.c, a.c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, m, a.H, a.T, a.B, kSpSlots, false))
        return cudaErrorInvalidValue;
    auto k = chunk_split_kernel<DS>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.H * kSpNC);
    cfg.blockDim = dim3(kSpThreads);
    cfg.dynamicSmemBytes = Lay::SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSpNC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k, maps, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

inline cudaError_t launch_chunk_split(const ScanArgs& a, int d, cudaStream_t st) {
    if (a.m != kSpSlots * kSpNC) return cudaErrorNotSupported;
    if (d == 128) return launch_chunk_split_t<128>(a, st);
    if (d == 64) return launch_chunk_split_t<64>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace lattice
