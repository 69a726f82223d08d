// chunk_reg.cuh -- chunked scan with each sequence's 64 slots split over a 4-CTA
// cluster, the state chain held in registers and advanced with warp-synchronous
// tensor-core MMAs, the read-out on tcgen05 tensor cores.
//
// Computes the chunked form, Eq. 17 of "Lattice: Learning to Efficiently Compress the
// Memory" (§3.4.1 and Appendix B.1), chunk size 64, as chunk_tc.cuh and
// chunk_split.cuh do. Each chunk of a sequence depends on the state the previous
// chunk left, through the projections p = x . s0 and the normaliser of
// eq. beta_chunk, so a sequence is a chain of T/64 dependent steps and its time is
// the chain's latency times the number of chunks. This kernel keeps that chain off
// every asynchronous round trip. Per CTA (16 slots) four chain warps, one per SM
// sub-partition, hold the fp32 state in registers and, per chunk:
//   projection  D[t][i] = x_t . s0_i            warp w: tokens 16w..16w+15, all slots
//   gates       g, kappa of Eq. 17 per (token, slot), in the MMA's output registers
//   scans       running products R (prefix) and Suf (suffix) of the gates over the
//               warp's 16-token sub-chunk: shuffles over the fragment's rows
//   update      S <- diag(A_C) S + sum_b f_b . (X_b^T KS_b)   warp w: state columns
//               w*d/4..(w+1)*d/4; KS_j = kappa_j Suf(j) per sub-chunk b, scaled after
//               the MMA by f_b = prod_{c>b} G_c (G_c: sub-chunk products), so no
//               product of gates is ever divided in the state chain
// with mma.sync m16n8k16 (bf16 operands, fp32 accumulation in registers; the state
// operand is a hi+lo bf16 pair, so the carried state keeps close to fp32 accuracy)
// and two 128-thread named barriers per chunk: one after the gates (sub-chunk
// products and KS exchanged through shared memory), one after the update (the next
// chunk's state operand and slot norms). An asynchronous tcgen05 MMA would put a
// commit, an mbarrier wake-up and a tensor-memory load on the chain twice per chunk.
//
// The read-out y_t = sum_i q_ti s_i(t) is off the chain and uses the chunk-parallel
// form of chunk_split.cuh: the chain warps write QR_b(t) = q_t prod_{l=16b..t} g_l
// (times the sub-chunk products in between) and KD(j) = kappa_j / prod_{l=16b..j} g_l
// (a division inside one 16-token sub-chunk only) and the chunk-start state hi part;
// one MMA warp issues, on tcgen05 with fp32 accumulators in tensor memory,
//   G4: Y_r  [C x d]  = QR_0 . S0hi                 inter-chunk read-out (K = 16)
//   G5: P_r  [C x 16] = QR_b . KD_b^T, b = 0..3     scores per key sub-chunk
//   G6: Y_r  [C x d] += P_r . X                     intra-chunk read-out (K = C)
// and four read-out warps mask the scores, reduce-scatter the four CTAs' partial
// Y_r through distributed shared memory (asynchronous remote stores that count
// their bytes on the receiver's mbarrier; each CTA sums its quarter of the columns
// in a fixed order) and store y. One TMA warp streams x, q and c through a ring of
// 64-token stages (no multicast); its lanes add each stage's mu and eta (cp.async),
// counted on the same stage barrier. Every mbarrier wait is bounded (waits.cuh).
#pragma once
#include "chunk_split.cuh"

namespace lattice {

constexpr int kRgM = 64;                        // slots per sequence
constexpr int kRgReadout = 128;                 // 4 read-out warps

inline bool chunk_reg_supported(int m, int d, int chunk, bool x_bf16, bool q_bf16) {
    return (chunk == kTcC || chunk == 16) && x_bf16 && q_bf16 && m == kRgM && (d == 64 || d == 128);
}

// SPC slots per CTA (16: clusters of 4 CTAs; 8: clusters of 8), state width DS, chunk
// size CH (64, or 16: four chunks per 64-token ring stage and read-out round).
template <int DS, int SPC, int CH>
struct RgLayout {
    static_assert(SPC == 8 || SPC == 16, "8 or 16 slots per CTA");
    static_assert(CH == 64 || CH == 16, "chunk size 64 or 16");
    static constexpr int HALVES = SPC / 8;                 // 8-slot halves, each with its own 4 chain warps
    static constexpr int CHAIN = 128 * HALVES;             // chain threads
    static constexpr int THREADS = CHAIN + kRgReadout + 64;  // + 4 read-out warps, MMA warp, TMA warp
    static constexpr int NST = DS == 128 ? (CH == 16 ? 2 : 3) : 4;  // x/q/c ring depth (stages of 64 tokens)
    static constexpr int NC = kRgM / SPC;                  // CTAs per sequence (cluster size)
    static constexpr int DSL = DS / NC;                    // y columns reduced by each CTA
    static constexpr uint32_t X_STAGE = DS * 128;          // [C][d] bf16 in d/64 SW128 blocks
    static constexpr uint32_t Q_STAGE = kTcC * SPC * 2;    // [C][SPC] bf16
    static constexpr uint32_t C_STAGE = kTcC * SPC * 4;    // [C][SPC] fp32
    static constexpr uint32_t X_OFF = 0;
    static constexpr uint32_t Q_OFF = X_OFF + NST * X_STAGE;
    static constexpr uint32_t C_OFF = Q_OFF + NST * Q_STAGE;
    // chunk-start state, double-buffered by chunk parity: [d rows = state column e][128 B],
    // the slots' hi parts at columns 0..SPC-1, lo parts at 16..16+SPC-1 (SW128); the
    // columns up to 16 stay zero (the read-out GEMM takes K = 16)
    static constexpr uint32_t S0_BUF = DS * 128;
    static constexpr uint32_t S0_OFF = C_OFF + NST * C_STAGE;
    // C = 16: the read-out's stacked chunk-start states of a stage, double-buffered by
    // stage parity: [d rows][128 B], chunk c's hi part at columns 16c..16c+SPC-1
    static constexpr uint32_t S0ST_OFF = S0_OFF + 2 * S0_BUF;
    static constexpr int S0_TILES = CH == 16 ? 4 : 2;
    static constexpr uint32_t QR_OFF = S0_OFF + S0_TILES * S0_BUF;  // [C][128 B]: QR_b at columns 16b..
    static constexpr uint32_t KT_OFF = QR_OFF + kTcC * 128;     // [C][128 B]: KD at 0.., KS hi at 16.., lo at 32..
    static constexpr uint32_t P_OFF = KT_OFF + kTcC * 128;      // [C][C] bf16 masked scores
    static constexpr uint32_t RECV_OFF = P_OFF + kTcC * 128;    // [2][NC][C][d/NC] fp32
    static constexpr uint32_t RECV_BYTES = 2 * NC * kTcC * DSL * 4;
    // outgoing partials, one [C][d/NC] fp32 block per peer (this CTA's own block goes
    // straight into its receive buffer), moved by one bulk copy per peer
    static constexpr uint32_t PEER_BLOCK = kTcC * DSL * 4;
    static constexpr uint32_t STG_OFF = RECV_OFF + RECV_BYTES;
    // mu, eta of each ring stage's 64 tokens, [NST][C][2] fp32, copied by the TMA warp's lanes
    static constexpr uint32_t MUE_OFF = STG_OFF + (NC - 1) * PEER_BLOCK;
    static constexpr uint32_t GSUB_OFF = MUE_OFF + 4 * kTcC * 2 * 4;  // [4 sub-chunks][16] (SPC used)
    static constexpr uint32_t TSQ_OFF = GSUB_OFF + 4 * 16 * 4;        // [2][4 warps][16] (SPC used)
    static constexpr uint32_t BAR_OFF = TSQ_OFF + 2 * 4 * 16 * 4;
    static constexpr int NBAR = 2 * NST + 8;
    static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr uint32_t BYTES = MISC_OFF + 64;
    static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;
    // TMEM columns: P | Y double-buffered
    static constexpr uint32_t P_COL = 0;
    static constexpr uint32_t Y_COL = kTcC;
    static constexpr uint32_t TMEM_COLS = (Y_COL + 2 * DS <= 256) ? 256 : 512;
    static constexpr uint32_t STAGE_TX = X_STAGE + Q_STAGE + C_STAGE;
    static_assert(S0_OFF % 1024 == 0 && QR_OFF % 1024 == 0 && KT_OFF % 1024 == 0 && P_OFF % 1024 == 0,
                  "SW128 tiles are 1024-byte aligned");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

template <int DS, int SPC, int CH>
__global__ void __launch_bounds__(RgLayout<DS, SPC, CH>::THREADS, 1)
    chunk_reg_kernel(const __grid_constant__ TcMaps maps, ScanArgs a) {
    using Lay = RgLayout<DS, SPC, CH>;
    constexpr int DSL = Lay::DSL;
    constexpr int NC = Lay::NC;
    constexpr int CHAIN = Lay::CHAIN;
    constexpr int NT = 1;  // 8-slot n-tiles per chain warp
    constexpr int NST = Lay::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = (int)ptx::cluster_ctarank();
    const int bh = blockIdx.x / NC, b = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H;
    const int nch = (T + kTcC - 1) / kTcC;  // ring stages of 64 tokens (chunks when C = 64)
    constexpr int RO_WARP0 = CHAIN / 32, MMA_WARP = RO_WARP0 + 4, TMA_WARP = MMA_WARP + 1;

    // mbarriers: ring stage full [NST] (TMA bytes) and empty [NST] (the chain warps + the
    // MMA warp's commit after G6), scores ready (G4, G5), read-out done (G6), peers'
    // partial y in [2], per-token inputs ready [2], read-out buffer drained [2]
    const uint32_t bar_full0 = sbase + Lay::BAR_OFF;
    const uint32_t bar_empty0 = bar_full0 + 8 * NST;
    const uint32_t bar_p5 = bar_empty0 + 8 * NST;
    const uint32_t bar_y = bar_p5 + 8;
    const uint32_t bar_recv0 = bar_y + 8;
    const uint32_t bar_yfree0 = bar_recv0 + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
    volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::MISC_OFF + 4);
    float* gsub = reinterpret_cast<float*>(smem + Lay::GSUB_OFF);
    float* tsq = reinterpret_cast<float*>(smem + Lay::TSQ_OFF);

    // named barriers: each half's 4 chain warps alone (C1 after the gates, C2 after the
    // update: ids 1, 2 for half 0 and 5, 6 for half 1), every chain warp (INIT, at the
    // start), chain warps (arrive) + MMA warp (A: read-out operands written), read-out
    // warps (arrive) + MMA warp (P: masked scores written)
    constexpr uint32_t BAR_A = 3, BAR_P = 4, BAR_INIT = 7, BAR_RO = 8;
    constexpr uint32_t N_CM = CHAIN + 32, N_RM = kRgReadout + 32;

    if (warp == MMA_WARP) {
        if (lane == 0) {
            for (int s = 0; s < NST; ++s) {
                ptx::mbar_init(bar_full0 + 8 * s, 1 + 32);  // TMA bytes + the TMA warp's 32 copy arrivals
                ptx::mbar_init(bar_empty0 + 8 * s, CHAIN / 32 + 1);
            }
            ptx::mbar_init(bar_p5, 1);
            ptx::mbar_init(bar_y, 1);
            ptx::mbar_init(bar_recv0, 1);
            ptx::mbar_init(bar_recv0 + 8, 1);
            ptx::mbar_init(bar_yfree0, kRgReadout);
            ptx::mbar_init(bar_yfree0 + 8, kRgReadout);
            *abort = 0u;
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
        // ------------------------------------------------------------ MMA issue (tcgen05)
        constexpr uint32_t idesc_g4 = ptx::idesc_bf16(kTcC, DS, 0, 0);
        constexpr uint32_t idesc_g5 = ptx::idesc_bf16(kTcC, kTcSub, 0, 0);
        constexpr uint32_t idesc_g6 = ptx::idesc_bf16(kTcC, DS, 0, 1);
        auto off = [](uint32_t bytes) { return uint64_t(bytes >> 4); };
        const uint64_t dK_qr = ptx::sdesc_sw128(sbase + Lay::QR_OFF, 16, 1024);
        const uint64_t dK_kd = ptx::sdesc_sw128(sbase + Lay::KT_OFF, 16, 1024);
        const uint64_t dK_s0 = ptx::sdesc_sw128(sbase + (CH == 64 ? Lay::S0_OFF : Lay::S0ST_OFF), 16, 1024);
        const uint64_t dK_p = ptx::sdesc_sw128(sbase + Lay::P_OFF, 16, 1024);
        const uint64_t dM_x = ptx::sdesc_sw128(sbase + Lay::X_OFF, 64 * 128, 1024);
        for (int k = 0; k < nch; ++k) {
            const int s = k % NST, p = k & 1;
            const uint32_t ycol = Lay::Y_COL + p * DS;
            ptx::named_bar(BAR_A, N_CM);  // QR, KD of chunk k and its start state written
            ptx::tc_fence_after();
            // the read-out of chunk k-2 (same accumulator buffer) has been drained
            const bool yfree = k < 2 || tc_wait_warp(bar_yfree0 + 8 * p, ((k - 2) >> 1) & 1, abort);
            ptx::tc_fence_after();
            if (yfree && tc_live(abort)) {
                if constexpr (CH == 64) {
                    // G4: Y_r = QR_0 . S0hi  (M = C, N = d, K = 16); both K-major
                    ptx::mma_bf16_elect(tmem + ycol, dK_qr, dK_s0 + off(p * Lay::S0_BUF), idesc_g4, 0);
                } else {
                    // G4: Y_r = QR_bd . S0stack  (K = 64: chunk c's rows of QR meet chunk c's start state)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::mma_bf16_elect(tmem + ycol, dK_qr + off(32 * kk), dK_s0 + off(p * Lay::S0_BUF + 32 * kk),
                                            idesc_g4, kk > 0);
                }
                // G5: P[:, 16b..16b+15] = QR_b . KD_b^T  (M = C, N = 16, K = 16)
#pragma unroll
                for (int sb = 0; sb < 4; ++sb)
                    ptx::mma_bf16_elect(tmem + Lay::P_COL + sb * 16, dK_qr + off(32 * sb),
                                        dK_kd + off(sb * 16 * 128), idesc_g5, 0);
            }
            ptx::mma_commit_elect(bar_p5);
            ptx::named_bar(BAR_P, N_RM);  // masked scores written by the read-out warps
            ptx::tc_fence_after();
            const bool xok = tc_wait_warp(bar_full0 + 8 * s, (k / NST) & 1, abort);
            if (xok && tc_live(abort)) {
                // G6: Y_r += P . X  (M = C, N = d, K = C); A K-major, B MN-major
#pragma unroll
                for (int kk = 0; kk < kTcC / 16; ++kk)
                    ptx::mma_bf16_elect(tmem + ycol, dK_p + off(kk * 32),
                                        dM_x + off(s * Lay::X_STAGE + kk * 2048), idesc_g6, 1);
            }
            ptx::mma_commit_elect(bar_y);
            ptx::mma_commit_elect(bar_empty0 + 8 * s);  // the MMAs are done with stage s
        }
        if (nch > 0) tc_drain(bar_y, (nch - 1) & 1);
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------------ TMA issue
        // Lane 0 issues the tensor copies of x, q and c of each 64-token stage; every lane
        // copies mu and eta of two of its tokens (cp.async, 4 bytes: a token's mu is one
        // float at a stride of H floats, too narrow for a tensor copy) and arrives on the
        // stage's full barrier once they have landed, so the chain warps find the
        // per-token inputs in shared memory with the rest of the stage.
        if (nch > 0) {
            const int s_lo = rank * SPC;  // this CTA's slots in the q and c rows
            int last[NST];
#pragma unroll
            for (int s = 0; s < NST; ++s) last[s] = -1;
            auto prefetch_l2 = [&](int k) {
#pragma unroll
                for (int kb = 0; kb < DS / 64; ++kb) ptx::tma_prefetch_l2_4d(&maps.x, kb * 64, h, k * kTcC, b);
                ptx::tma_prefetch_l2_4d(&maps.q, s_lo, h, k * kTcC, b);
                ptx::tma_prefetch_l2_4d(&maps.c, s_lo, h, k * kTcC, b);
            };
            if (lane == 0) {
                ptx::prefetch_tensormap(&maps.x);
                ptx::prefetch_tensormap(&maps.q);
                ptx::prefetch_tensormap(&maps.c);
                for (int k = NST; k < NST + 4 && k < nch; ++k) prefetch_l2(k);
            }
            for (int k = 0; k < nch; ++k) {
                const int s = k % NST;
                if (k >= NST && !tc_wait_warp(bar_empty0 + 8 * s, ((k / NST) - 1) & 1, abort)) break;
                const uint32_t full = bar_full0 + 8 * s;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(full, Lay::STAGE_TX);
#pragma unroll
                    for (int kb = 0; kb < DS / 64; ++kb)
                        ptx::tma_load_4d(sbase + Lay::X_OFF + s * Lay::X_STAGE + kb * (64 * 128), &maps.x, full,
                                         kb * 64, h, k * kTcC, b);
                    ptx::tma_load_4d(sbase + Lay::Q_OFF + s * Lay::Q_STAGE, &maps.q, full, s_lo, h, k * kTcC, b);
                    ptx::tma_load_4d(sbase + Lay::C_OFF + s * Lay::C_STAGE, &maps.c, full, s_lo, h, k * kTcC, b);
                }
                const uint32_t me = sbase + Lay::MUE_OFF + s * (kTcC * 8);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int tau = lane + 32 * j, t = k * kTcC + tau;
                    if (t < T) {
                        const size_t bth = ((size_t)b * T + t) * H + h;
                        ptx::cp_async4(me + tau * 8, a.mu + bth);
                        if (a.eta) ptx::cp_async4(me + tau * 8 + 4, a.eta + bth);
                    }
                }
                ptx::cp_async_mbar_arrive_noinc(full);
                last[s] = k;
                if (lane == 0 && k + NST + 4 < nch) prefetch_l2(k + NST + 4);
            }
            ptx::cp_async_wait_all();
            if (lane == 0) {
#pragma unroll
                for (int s = 0; s < NST; ++s)  // no TMA write may be in flight when the CTA retires
                    if (last[s] >= 0) tc_drain(bar_full0 + 8 * s, (last[s] / NST) & 1);
            }
        }
        __syncwarp();
    } else if (warp >= RO_WARP0) {
        // ------------------------------------------------------------ read-out warps
        const int q = warp & 3;
        const int rt = tid - CHAIN;        // 0..127
        const uint32_t lane_base = uint32_t(32 * q) << 16;
        const bool row_ok = lane < 16;     // M = 64 accumulators: lanes 0-15 of each quadrant
        const int trow = 16 * q + lane;    // accumulator row (token) of this lane
        // the NC partials of this CTA's columns of chunk kc -> y. Summing chunk k-1 before
        // sending chunk k keeps two receive buffers enough: a peer's chunk k+1 follows its
        // sum of chunk k, which needs this CTA's chunk k, sent after this sum. A partial
        // block is [C rows][d/NC fp32 columns] with the 16-byte chunk j of row r stored at
        // position j ^ (r mod G) (G chunks per row), so that neither the writers (one row
        // per lane) nor the readers (one chunk per lane) meet bank conflicts.
        constexpr int G = DSL / 4;          // 16-byte chunks per row of a partial block
        constexpr uint32_t RECV_TX = (NC - 1) * Lay::PEER_BLOCK;  // bytes of one chunk's partials from the peers
        auto recv_y = [&](int kc) {
            const int par = kc & 1;
            tc_wait_cluster(bar_recv0 + 8 * par, (kc >> 1) & 1, abort);
            if (rt == 0 && kc + 2 < nch) ptx::mbar_arrive_expect_tx(bar_recv0 + 8 * par, RECV_TX);  // chunk kc+2
            if (*abort) return;
            constexpr int TPR = kRgReadout / G;  // tokens per round
            const int gg = rt % G;
#pragma unroll
            for (int r = 0; r < kTcC / TPR; ++r) {
                const int tk = r * TPR + rt / G;
                const uint32_t o = tk * (DSL * 4) + ((gg ^ (tk & (G - 1))) << 4);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int src = 0; src < NC; ++src) {
                    const float4 v = *reinterpret_cast<const float4*>(smem + Lay::RECV_OFF + (par * NC + src) * Lay::PEER_BLOCK + o);
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                const int t = kc * kTcC + tk;
                if (t < T)
                    *reinterpret_cast<float4*>(a.y + (((size_t)b * T + t) * H + h) * DS + rank * DSL + 4 * gg) = acc;
            }
        };
        if (rt == 0) {  // arm the receive barriers of chunks 0 and 1
            if (nch > 0) ptx::mbar_arrive_expect_tx(bar_recv0, RECV_TX);
            if (nch > 1) ptx::mbar_arrive_expect_tx(bar_recv0 + 8, RECV_TX);
        }
        for (int k = 0; k < nch; ++k) {
            const int par = k & 1;
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
            // partial read-out of this chunk: every peer's block of columns, staged in shared
            // memory and sent with one bulk copy per peer (this CTA's own block goes straight
            // into its receive buffer)
            tc_wait(bar_y, k & 1, abort);
            if (rt == 0) ptx::bulk_wait_read_all();  // the previous chunk's copies have read the staging
            ptx::named_bar(BAR_RO, kRgReadout);
            ptx::tc_fence_after();
#pragma unroll
            for (int pp = 0; pp < NC; ++pp) {
                __syncwarp();  // tcgen05.ld is warp-collective
                uint32_t yv[DSL];
                ptx::tmem_ld<DSL>(tmem + lane_base + Lay::Y_COL + par * DS + pp * DSL, yv);
                ptx::tmem_wait_ld();
                if (row_ok) {
                    const uint32_t off = pp == rank ? Lay::RECV_OFF + (par * NC + rank) * Lay::PEER_BLOCK
                                                    : Lay::STG_OFF + (pp - (pp > rank)) * Lay::PEER_BLOCK;
                    uint8_t* dst = smem + off + trow * (DSL * 4);
#pragma unroll
                    for (int c = 0; c < DSL; c += 4)
                        *reinterpret_cast<float4*>(dst + (((c / 4) ^ (trow & (G - 1))) << 4)) =
                            make_float4(__uint_as_float(yv[c]), __uint_as_float(yv[c + 1]),
                                        __uint_as_float(yv[c + 2]), __uint_as_float(yv[c + 3]));
                }
            }
            ptx::fence_proxy_async_smem();  // the staged blocks are read by the copy engine
            ptx::named_bar(BAR_RO, kRgReadout);
            if (rt == 0 && !*abort) {
#pragma unroll
                for (int pp = 0; pp < NC; ++pp) {
                    if (pp == rank) continue;
                    const uint32_t dst = sbase + Lay::RECV_OFF + (par * NC + rank) * Lay::PEER_BLOCK;
                    ptx::bulk_copy_s2cluster(ptx::mapa(dst, (uint32_t)pp),
                                             sbase + Lay::STG_OFF + (pp - (pp > rank)) * Lay::PEER_BLOCK,
                                             Lay::PEER_BLOCK, ptx::mapa(bar_recv0 + 8 * par, (uint32_t)pp));
                }
                ptx::bulk_commit();
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_yfree0 + 8 * par);  // this buffer may take chunk k+2
        }
        if (nch > 0) recv_y(nch - 1);
        if (rt == 0) ptx::bulk_wait_all();  // no copy still reads this CTA's shared memory
    } else {
        // ================================================================ chain warps
        // Chain warp w + 4hv runs half hv of the CTA's slots (8 slots, sh = 8hv..8hv+7); the
        // two halves never exchange anything, so each runs its own chain with its own named
        // barriers and the warp scheduler overlaps one half's gate arithmetic with the other
        // half's MMAs. Fragment coordinates: g = lane/4 (a row: a token, or a state column),
        // cq = lane%4 (a pair of slots sh + 2cq, sh + 2cq + 1); index i of a 4-register
        // fragment is (row g + 8(i/2), slot sh + 2cq + i%2). Warp w owns the state columns
        // w*d/4..(w+1)*d/4 of its half in the update; with C = 64 it also owns the
        // projections and gates of sub-chunk w (tokens 16w..16w+15).
        const int w = warp & 3, hv = warp >> 2, sh = 8 * hv;
        const uint32_t BAR_C1 = hv ? 5 : 1, BAR_C2 = hv ? 6 : 2;
        const int g = lane >> 2, cq = lane & 3;
        constexpr int MT = DS / 64;                   // 16-column m-tiles of the update per warp
        const int e_base = w * (DS / 4);
        const int lj = lane >> 3, lr = lane & 7;      // ldmatrix: matrix lj, row lr
        uint8_t* qr = smem + Lay::QR_OFF;
        uint8_t* kt = smem + Lay::KT_OFF;
        const uint32_t kt_a = sbase + Lay::KT_OFF;

        // fp32 state: st[mt][nt][i] = s_{slot}[e], e = e_base + 16mt + g + 8(i/2)
        float st[MT][NT][4];
        {
            const float* S0g = a.S0 + ((size_t)bh * kRgM + rank * SPC) * DS;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e = e_base + 16 * mt + g + 8 * (i >> 1);
                        const int sl = sh + 8 * nt + 2 * cq + (i & 1);
                        st[mt][nt][i] = S0g[(size_t)sl * DS + e];
                    }
        }
        // the state as the next chunk's operand: hi/lo bf16 into S0 buffer pb (and, with
        // C = 16, its hi part into the read-out's stacked-state tile sto at column scol),
        // and each slot's partial |s|^2 over this warp's columns into tsq[pb][w] (double
        // buffered: a warp may start the next chunk before the others have read them)
        auto write_state = [&](int pb, uint8_t* sto, int scol) {
            uint8_t* dst = smem + Lay::S0_OFF + pb * Lay::S0_BUF;
            float ns[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) ns[nt][0] = ns[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int e = e_base + 16 * mt + g + 8 * hf;
                        const float2 v = make_float2(st[mt][nt][2 * hf], st[mt][nt][2 * hf + 1]);
                        uint32_t hi, lo;
                        split2(v, hi, lo);
                        const int col = sh + 8 * nt + 2 * cq;
                        *reinterpret_cast<uint32_t*>(dst + ptx::sw128_off(e, col)) = hi;
                        *reinterpret_cast<uint32_t*>(dst + ptx::sw128_off(e, 16 + col)) = lo;
                        if (CH == 16) *reinterpret_cast<uint32_t*>(sto + ptx::sw128_off(e, scol + col)) = hi;
                        ns[nt][0] = fmaf(v.x, v.x, ns[nt][0]);
                        ns[nt][1] = fmaf(v.y, v.y, ns[nt][1]);
                    }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float v = ns[nt][j];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (g == 0) tsq[pb * 64 + w * 16 + sh + 8 * nt + 2 * cq + j] = v;
                }
        };
        // n = |s0|, 1/n, 1/n^2 of this thread's slots (index 2nt + j: slot 8nt + 2cq + j)
        float nrm[2 * NT], inv_n[2 * NT], inv_n2[2 * NT];
        auto load_norms = [&](int pb) {
#pragma unroll
            for (int u = 0; u < 2 * NT; ++u) {
                const float* t4 = tsq + pb * 64 + sh + 8 * (u >> 1) + 2 * cq + (u & 1);
                const float nsq = ((t4[0] + t4[16]) + t4[32]) + t4[48];
                inv_n[u] = ptx::rsqrt_nr(nsq);
                nrm[u] = nsq * inv_n[u];
                inv_n2[u] = inv_n[u] * inv_n[u];
            }
        };
        // B fragments (k = 16 rows from row0, n = 8 slots per n-tile) of a hi/lo operand pair
        // stored row-major in an SW128 tile: hi slots at columns col0 + 8nt, lo at col0 + 16 + 8nt.
        // ldmatrix.trans turns the stored [k][n] rows into the fragment layout.
        auto load_b_pairs = [&](uint32_t tile, int row0, int col0, uint32_t (&bfr)[2][NT][2]) {
            const int row = row0 + 8 * (lj & 1) + lr;
            const uint32_t ra = tile + row * 128;
            uint32_t r4[4];
            if constexpr (NT == 2) {
                ptx::ldsm_x4_t(ra + ((((col0 >> 3) + (lj >> 1)) ^ (row & 7)) << 4), r4);
                bfr[0][0][0] = r4[0]; bfr[0][0][1] = r4[1]; bfr[0][1][0] = r4[2]; bfr[0][1][1] = r4[3];
                ptx::ldsm_x4_t(ra + ((((col0 >> 3) + 2 + (lj >> 1)) ^ (row & 7)) << 4), r4);
                bfr[1][0][0] = r4[0]; bfr[1][0][1] = r4[1]; bfr[1][1][0] = r4[2]; bfr[1][1][1] = r4[3];
            } else {
                ptx::ldsm_x4_t(ra + ((((col0 >> 3) + 2 * (lj >> 1)) ^ (row & 7)) << 4), r4);
                bfr[0][0][0] = r4[0]; bfr[0][0][1] = r4[1]; bfr[1][0][0] = r4[2]; bfr[1][0][1] = r4[3];
            }
        };
        // projections D[t][i] = x_t . (s0hi_i + s0lo_i) of the 16 tokens at stage rows
        // row0..row0+15, all the CTA's slots; pr[nt][i] in the fragment layout
        auto project = [&](uint32_t xs_a, uint32_t s0_a, int row0, float (&pr)[NT][4], float (&xx)[2]) {
            float2 xa = ptx::f2(0.f), xb = ptx::f2(0.f);  // |x|^2 partials of rows g and g+8
            float acc[2][2][NT][4];  // [k-step parity][hi, lo][nt][i]
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int v = 0; v < 2; ++v)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[u][v][nt][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < DS / 16; ++ks) {
                uint32_t af[4], bf[2][NT][2];
                {   // A: x rows row0 + 8(lj&1) + lr, columns 16ks + 8(lj>>1)
                    const int row = row0 + 8 * (lj & 1) + lr;
                    const int col = 16 * ks + 8 * (lj >> 1);
                    ptx::ldsm_x4(xs_a + (col >> 6) * (64 * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4), af);
                }
#pragma unroll
                for (int j = 0; j < 4; j += 2) {  // af[0], af[2]: row g; af[1], af[3]: row g+8
                    const float2 u = make_float2(__uint_as_float(af[j] << 16), __uint_as_float(af[j] & 0xffff0000u));
                    const float2 v = make_float2(__uint_as_float(af[j + 1] << 16), __uint_as_float(af[j + 1] & 0xffff0000u));
                    xa = ptx::f2fma(u, u, xa);
                    xb = ptx::f2fma(v, v, xb);
                }
                load_b_pairs(s0_a, 16 * ks, sh, bf);  // the state rows e = 16ks..16ks+15
#pragma unroll
                for (int v = 0; v < 2; ++v)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) ptx::mma16816(acc[ks & 1][v][nt], af, bf[v][nt]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    pr[nt][i] = (acc[0][0][nt][i] + acc[1][0][nt][i]) + (acc[0][1][nt][i] + acc[1][1][nt][i]);
            xx[0] = xa.x + xa.y;
            xx[1] = xb.x + xb.y;
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // the quad's four lanes hold the rest of each row
                xx[j] += __shfl_xor_sync(0xffffffffu, xx[j], 1);
                xx[j] += __shfl_xor_sync(0xffffffffu, xx[j], 2);
            }
        };
        // mu and eta of the tokens at rows row0 + g and row0 + g + 8 of chunk (or stage) k
        // mu and eta of the tokens at rows row0 + g and row0 + g + 8 of ring stage s (stage
        // k), from the shared memory the TMA warp's lanes copied them into. Loaded by the
        // chain warps themselves, their latency landed on the chain.
        auto stage_mueta = [&](int s, int k, int row0, float (&mu)[2], float (&eta)[2]) {
            const float* me = reinterpret_cast<const float*>(smem + Lay::MUE_OFF) + s * (kTcC * 2);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int tau = row0 + g + 8 * j;
                mu[j] = 0.f;
                eta[j] = 1.f;
                if (k * kTcC + tau < T) {
                    mu[j] = me[2 * tau];
                    if (a.eta) eta[j] = me[2 * tau + 1];
                }
            }
        };
        // gates of Eq. 17 (eq. beta_chunk with the chunk-start norm n) of the 16 tokens at
        // rows row0.. of ring stage s; z[hf] = (mu, eta, |x|^2, mu^2) of row g + 8hf:
        //   e2 = eta c / n^2, pn = p / n, den = mu^2 + e2^2 max(|x|^2 - pn^2, 0),
        //   g = (mu - e2 pn) / sqrt(den), kappa = n e2 / sqrt(den); den = 0 keeps the slot
        auto gates = [&](const float (&pr)[NT][4], int s, const float4 (&zr)[2], int row0, bool zero_mu,
                         float (&gt)[NT][4], float (&kap)[NT][4], float (&qv)[NT][4]) {
            const float* cs = reinterpret_cast<const float*>(smem + Lay::C_OFF + s * Lay::C_STAGE);
            const uint16_t* qs = reinterpret_cast<const uint16_t*>(smem + Lay::Q_OFF + s * Lay::Q_STAGE);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int tk = row0 + g + 8 * hf;
                const float4 z = zr[hf];  // mu, eta, |x|^2, mu^2
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int u0 = 2 * nt;  // norm index of slot 8nt + 2cq
                    const float2 cc = *reinterpret_cast<const float2*>(cs + tk * SPC + sh + 8 * nt + 2 * cq);
                    const uint32_t q2 = *reinterpret_cast<const uint32_t*>(qs + tk * SPC + sh + 8 * nt + 2 * cq);
                    const float2 pp = make_float2(pr[nt][2 * hf], pr[nt][2 * hf + 1]);
                    const float2 e2 = ptx::f2mul(cc, ptx::f2mul(ptx::f2(z.y), make_float2(inv_n2[u0], inv_n2[u0 + 1])));
                    const float2 pn = ptx::f2mul(pp, make_float2(inv_n[u0], inv_n[u0 + 1]));
                    float2 perp = ptx::f2fma(ptx::f2neg(pn), pn, ptx::f2(z.z));
                    perp.x = fmaxf(perp.x, 0.f);
                    perp.y = fmaxf(perp.y, 0.f);
                    const float2 den = ptx::f2fma(ptx::f2mul(e2, e2), perp, ptx::f2(z.w));
                    float2 bn = ptx::rsqrt2_nr(den);
                    if (zero_mu)
                        bn = make_float2(den.x > 0.f ? ptx::rsqrt_nr(den.x) : 0.f, den.y > 0.f ? ptx::rsqrt_nr(den.y) : 0.f);
                    float2 gg = ptx::f2mul(bn, ptx::f2fma(ptx::f2neg(e2), pn, ptx::f2(z.x)));
                    float2 kk = ptx::f2mul(ptx::f2mul(bn, e2), make_float2(nrm[u0], nrm[u0 + 1]));  // kappa
                    if (zero_mu) {
                        if (!(den.x > 0.f)) { gg.x = 1.f; kk.x = 0.f; }
                        if (!(den.y > 0.f)) { gg.y = 1.f; kk.y = 0.f; }
                    }
                    gt[nt][2 * hf] = gg.x;
                    gt[nt][2 * hf + 1] = gg.y;
                    kap[nt][2 * hf] = kk.x;
                    kap[nt][2 * hf + 1] = kk.y;
                    qv[nt][2 * hf] = __uint_as_float(q2 << 16);
                    qv[nt][2 * hf + 1] = __uint_as_float(q2 & 0xffff0000u);
                }
            }
        };
        // running products over 16 tokens (rows g and g+8 of each column): R = inclusive
        // prefix, suf = exclusive suffix, Gs = the total
        auto scans = [&](const float (&gt)[NT][4], float (&R)[NT][4], float (&suf)[NT][4], float (&Gs)[NT][2]) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float rl = gt[nt][j], rh = gt[nt][2 + j];
                    float ul = rl, uh = rh;
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) {
                        const float tl = __shfl_up_sync(0xffffffffu, rl, 4 * o);
                        const float th = __shfl_up_sync(0xffffffffu, rh, 4 * o);
                        const float dl = __shfl_down_sync(0xffffffffu, ul, 4 * o);
                        const float dh = __shfl_down_sync(0xffffffffu, uh, 4 * o);
                        if (g >= o) { rl *= tl; rh *= th; }
                        if (g + o <= 7) { ul *= dl; uh *= dh; }
                    }
                    rh *= __shfl_sync(0xffffffffu, rl, 28 + cq);        // times prod of rows 0..7
                    const float U = __shfl_sync(0xffffffffu, uh, cq);   // prod of rows 8..15
                    ul *= U;                                            // prod of rows g..15
                    const float nl = __shfl_down_sync(0xffffffffu, ul, 4);
                    const float nh = __shfl_down_sync(0xffffffffu, uh, 4);
                    R[nt][j] = rl;
                    R[nt][2 + j] = rh;
                    suf[nt][j] = g < 7 ? nl : U;       // prod of rows g+1..15
                    suf[nt][2 + j] = g < 7 ? nh : 1.f;  // prod of rows g+9..15
                    Gs[nt][j] = __shfl_sync(0xffffffffu, rh, 28 + cq);
                }
        };
        // KD = kappa / R (R clamped away from zero, sign kept) and KS = kappa suf (hi + lo)
        // of the fragment's rows into the KT tile, rows kd_row0.. and ks_row0..; the
        // query operand q R into the QR tile at rows qr_row0.., columns qcol.. (unless null)
        auto write_operands = [&](const float (&kap)[NT][4], const float (&R)[NT][4], const float (&suf)[NT][4],
                                  const float (&qv)[NT][4], int kd_row0, int ks_row0, int qcol, float (&qrw)[NT][4],
                                  bool write_kd_qr) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int col = sh + 8 * nt + 2 * cq;
                    float kd[2], ks[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int i = 2 * hf + j;
                        const float r = R[nt][i];
                        kd[j] = kap[nt][i] * ptx::rcp_nr(copysignf(fmaxf(fabsf(r), 1e-37f), r));
                        ks[j] = kap[nt][i] * suf[nt][i];
                        qrw[nt][i] = qv[nt][i] * r;
                    }
                    uint32_t khi, klo;
                    split2(make_float2(ks[0], ks[1]), khi, klo);
                    const int rs = ks_row0 + g + 8 * hf;
                    *reinterpret_cast<uint32_t*>(kt + ptx::sw128_off(rs, 16 + col)) = khi;
                    *reinterpret_cast<uint32_t*>(kt + ptx::sw128_off(rs, 32 + col)) = klo;
                    if (write_kd_qr) {
                        const int rk = kd_row0 + g + 8 * hf;
                        *reinterpret_cast<uint32_t*>(kt + ptx::sw128_off(rk, col)) = ptx::pack_bf16x2(kd[0], kd[1]);
                        *reinterpret_cast<uint32_t*>(qr + ptx::sw128_off(rk, qcol + col)) =
                            ptx::pack_bf16x2(qrw[nt][2 * hf], qrw[nt][2 * hf + 1]);
                    }
                }
        };
        // U[e][i] += sum_{tokens j of stage rows row0..row0+15} x_j[e] KS_j[i] for this warp's
        // columns, KS from the KT tile rows ks_row0.. (B), x^T from the stage (A)
        auto update_mma = [&](uint32_t xs_a, int row0, int ks_row0, float (&u)[MT][NT][4]) {
            uint32_t kf[2][NT][2];
            load_b_pairs(kt_a, ks_row0, 16 + sh, kf);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t af[4];
                {   // A = X^T: x rows row0 + 8(lj>>1) + lr, columns e = e_base + 16mt + 8(lj&1)
                    const int row = row0 + 8 * (lj >> 1) + lr;
                    const int e = e_base + 16 * mt + 8 * (lj & 1);
                    ptx::ldsm_x4_t(xs_a + (e >> 6) * (64 * 128) + row * 128 + ((((e & 63) >> 3) ^ (row & 7)) << 4), af);
                }
#pragma unroll
                for (int v = 0; v < 2; ++v)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) ptx::mma16816(u[mt][nt], af, kf[v][nt]);
            }
        };

        // ---- prologue: operand tiles zeroed (blocks of the query tile that are never
        // written, and with 8 slots per CTA the K padding up to 16)
        for (int o = tid; o < int(kTcC * 128 / 16); o += CHAIN) {
            reinterpret_cast<uint4*>(qr)[o] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4*>(kt)[o] = make_uint4(0u, 0u, 0u, 0u);
        }
        for (int o = tid; o < int(Lay::S0_TILES * Lay::S0_BUF / 16); o += CHAIN)
            reinterpret_cast<uint4*>(smem + Lay::S0_OFF)[o] = make_uint4(0u, 0u, 0u, 0u);
        ptx::named_bar(BAR_INIT, CHAIN);  // every chain thread's zeros before any state is written
        write_state(0, smem + Lay::S0ST_OFF, 0);
        ptx::named_bar(BAR_C2, 128);
        if (CH == 16) load_norms(0);

        if constexpr (CH == 64) {
            const int tok0 = 16 * w;  // this warp's sub-chunk
            for (int k = 0; k < nch; ++k) {
                const int s = k % NST, p = k & 1;
                tc_wait(bar_full0 + 8 * s, (k / NST) & 1, abort);
                const uint32_t xs_a = sbase + Lay::X_OFF + s * Lay::X_STAGE;
                float pr[NT][4], xx[2];
                project(xs_a, sbase + Lay::S0_OFF + p * Lay::S0_BUF, tok0, pr, xx);
                load_norms(p);  // this chunk's slot norms (written with its start state), while the MMAs run
                float mu_n[2], eta_n[2];
                stage_mueta(s, k, tok0, mu_n, eta_n);
                float4 zr[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) zr[j] = make_float4(mu_n[j], eta_n[j], xx[j], mu_n[j] * mu_n[j]);
                // mu^2 < 2^-60 (or zero): the normaliser's argument may be denormal or zero
                const bool zero_mu = __any_sync(0xffffffffu, !(zr[0].w >= 8.6736174e-19f) || !(zr[1].w >= 8.6736174e-19f));
                float gt[NT][4], kap[NT][4], qv[NT][4], R[NT][4], suf[NT][4], Gs[NT][2], qrw[NT][4];
                gates(pr, s, zr, tok0, zero_mu, gt, kap, qv);
                scans(gt, R, suf, Gs);
                if (k > 0) tc_wait(bar_p5, (k - 1) & 1, abort);  // G4/G5 of chunk k-1 are done with QR, KD
                write_operands(kap, R, suf, qv, tok0, tok0, 16 * w, qrw, true);
                if (g == 0) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        *reinterpret_cast<float2*>(gsub + w * 16 + sh + 8 * nt + 2 * cq) = make_float2(Gs[nt][0], Gs[nt][1]);
                }
                ptx::named_bar(BAR_C1, 128);  // every sub-chunk's products and KS of this half written
                // per slot: the chunk decay A_C and f_b = prod_{c>b} G_c of each sub-chunk b
                float AC[2 * NT], fb[3][2 * NT];
#pragma unroll
                for (int u = 0; u < 2 * NT; ++u) {
                    const int sl = sh + 8 * (u >> 1) + 2 * cq + (u & 1);
                    const float G0 = gsub[sl], G1 = gsub[16 + sl], G2 = gsub[32 + sl], G3 = gsub[48 + sl];
                    fb[2][u] = G3;
                    fb[1][u] = G2 * G3;
                    fb[0][u] = G1 * fb[1][u];
                    AC[u] = G0 * fb[0][u];
                }
                // query operands of the earlier key blocks bb < w for this warp's tokens:
                // QR_bb(t) = QR_w(t) prod_{c=bb..w-1} G_c
#pragma unroll
                for (int bb = 0; bb < 3; ++bb) {
                    if (bb >= w) break;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            float v[2];
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const int sl = sh + 8 * nt + 2 * cq + j;
                                float cgb = 1.f;
#pragma unroll
                                for (int c = 0; c < 4; ++c)
                                    if (c >= bb && c < w) cgb *= gsub[c * 16 + sl];
                                v[j] = qrw[nt][2 * hf + j] * cgb;
                            }
                            const int tk = tok0 + g + 8 * hf, col = sh + 8 * nt + 2 * cq;
                            *reinterpret_cast<uint32_t*>(qr + ptx::sw128_off(tk, 16 * bb + col)) =
                                ptx::pack_bf16x2(v[0], v[1]);
                        }
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_arrive(BAR_A, N_CM);  // QR, KD and the chunk-start state are ready for G4/G5

                // ---- state update: per key sub-chunk bb, U_bb[e][i] = sum_{j in bb} x_j[e] KS_j[i]
                float ua[4][MT][NT][4];
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) ua[bb][mt][nt][i] = 0.f;
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) update_mma(xs_a, 16 * bb, 16 * bb, ua[bb]);
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar_empty0 + 8 * s);  // done with x, q, c of stage s
                // S <- A_C S + f_0 U_0 + f_1 U_1 + f_2 U_2 + U_3
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int u = 2 * nt + (i & 1);
                            float v = ua[3][mt][nt][i];
                            v = fmaf(fb[2][u], ua[2][mt][nt][i], v);
                            v = fmaf(fb[1][u], ua[1][mt][nt][i], v);
                            v = fmaf(fb[0][u], ua[0][mt][nt][i], v);
                            st[mt][nt][i] = fmaf(AC[u], st[mt][nt][i], v);
                        }
                if (k + 1 < nch) {
                    write_state((k + 1) & 1, nullptr, 0);  // G4 of chunk k-1 (the buffer's last reader) is done
                    ptx::named_bar(BAR_C2, 128);
                }
            }
        } else {
            // C = 16: each ring stage (64 tokens) holds four consecutive chunks, run one after
            // the other by all four chain warps together. Every warp forms the projections,
            // gates and products of the whole chunk (16 tokens x the CTA's slots); warp 0 writes
            // the chunk's read-out operands (QR in the block-diagonal position of chunk c, KD,
            // the chunk-start state in column block c of the stacked-state tile), and each warp
            // writes KS into its own rows of the KT tile for its update, so one barrier per
            // chunk (the new state) remains on the chain.
            int step = 0;
            for (int k = 0; k < nch; ++k) {
                const int s = k % NST, p = k & 1;
                tc_wait(bar_full0 + 8 * s, (k / NST) & 1, abort);
                float mu_c[4][2], eta_c[4][2];  // this stage's four chunks
#pragma unroll
                for (int c = 0; c < 4; ++c) stage_mueta(s, k, 16 * c, mu_c[c], eta_c[c]);
                bool zero_mu = false;
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 2; ++j) zero_mu = zero_mu || !(mu_c[c][j] * mu_c[c][j] >= 8.6736174e-19f);
                zero_mu = __any_sync(0xffffffffu, zero_mu);  // mu^2 < 2^-60 somewhere in the stage
                if (k > 0) tc_wait(bar_p5, (k - 1) & 1, abort);  // G4/G5 of stage k-1 are done with QR, KD
                const uint32_t xs_a = sbase + Lay::X_OFF + s * Lay::X_STAGE;
                for (int c = 0; c < 4; ++c, ++step) {
                    float pr[NT][4], xx[2];
                    project(xs_a, sbase + Lay::S0_OFF + (step & 1) * Lay::S0_BUF, 16 * c, pr, xx);
                    float4 zr[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        zr[j] = make_float4(mu_c[c][j], eta_c[c][j], xx[j], mu_c[c][j] * mu_c[c][j]);
                    float gt[NT][4], kap[NT][4], qv[NT][4], R[NT][4], suf[NT][4], Gs[NT][2], qrw[NT][4];
                    gates(pr, s, zr, 16 * c, zero_mu, gt, kap, qv);
                    scans(gt, R, suf, Gs);
                    write_operands(kap, R, suf, qv, 16 * c, 16 * w, 16 * c, qrw, w == 0);
                    __syncwarp();
                    float ua[MT][NT][4];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) ua[mt][nt][i] = 0.f;
                    update_mma(xs_a, 16 * c, 16 * w, ua);
                    // S <- G S + U, G the chunk's product of gates
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                st[mt][nt][i] = fmaf(Gs[nt][i & 1], st[mt][nt][i], ua[mt][nt][i]);
                    if (k + 1 < nch || c < 3) {
                        // the next chunk's state operand; its hi part also goes to the read-out's
                        // stacked-state tile of this stage (block c+1) or of the next one (block 0)
                        uint8_t* sto = smem + Lay::S0ST_OFF + (c < 3 ? p : p ^ 1) * Lay::S0_BUF;
                        write_state((step + 1) & 1, sto, c < 3 ? 16 * (c + 1) : 0);
                        ptx::named_bar(BAR_C2, 128);
                        load_norms((step + 1) & 1);
                    }
                    __syncwarp();
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_arrive(BAR_A, N_CM);  // QR, KD and the stage's chunk-start states are ready
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar_empty0 + 8 * s);  // done with x, q, c of stage s
            }
        }
        // final state
        float* So = a.S_out + ((size_t)bh * kRgM + rank * SPC) * DS;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = e_base + 16 * mt + g + 8 * (i >> 1);
                    const int sl = sh + 8 * nt + 2 * cq + (i & 1);
                    So[(size_t)sl * DS + e] = st[mt][nt][i];
                }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // no peer still writes into this CTA's shared memory
    ptx::tc_fence_after();
    if (warp == MMA_WARP) ptx::tmem_dealloc(tmem, Lay::TMEM_COLS);
}

template <int DS, int SPC, int CH>
cudaError_t launch_chunk_reg_t(const ScanArgs& a, cudaStream_t st) {
    using Lay = RgLayout<DS, SPC, CH>;
    TcMaps maps;
    if (!make_map_4d(&maps.x, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DS, a.H, a.T, a.B, 64, true) ||
        !make_map_4d(&maps.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kRgM, a.H, a.T, a.B, SPC, false) ||
        !make_map_4d(&maps.c, a.c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kRgM, a.H, a.T, a.B, SPC, false))
        return cudaErrorInvalidValue;
    auto k = chunk_reg_kernel<DS, SPC, CH>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.H * Lay::NC);
    cfg.blockDim = dim3(Lay::THREADS);
    cfg.dynamicSmemBytes = Lay::SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Lay::NC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k, maps, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Clusters of the kernel with `spc` slots per CTA (8 or 16) that the current device can
// hold at once (each cluster takes 64/spc SMs of one GPC); 0 if the query fails.
template <int DS, int SPC>
int chunk_reg_max_clusters_t() {
    using Lay = RgLayout<DS, SPC, 64>;
    auto k = chunk_reg_kernel<DS, SPC, 64>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM_ALLOC) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Lay::NC * 64);
    cfg.blockDim = dim3(Lay::THREADS);
    cfg.dynamicSmemBytes = Lay::SMEM_ALLOC;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Lay::NC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

inline int chunk_reg_max_clusters(int d, int spc) {
    if (d == 128) return spc == 8 ? chunk_reg_max_clusters_t<128, 8>() : chunk_reg_max_clusters_t<128, 16>();
    if (d == 64) return spc == 8 ? chunk_reg_max_clusters_t<64, 8>() : chunk_reg_max_clusters_t<64, 16>();
    return 0;
}

template <int CH>
cudaError_t launch_chunk_reg_c(const ScanArgs& a, int d, int spc, cudaStream_t st) {
    if (d == 128) return spc == 8 ? launch_chunk_reg_t<128, 8, CH>(a, st) : launch_chunk_reg_t<128, 16, CH>(a, st);
    if (d == 64) return spc == 8 ? launch_chunk_reg_t<64, 8, CH>(a, st) : launch_chunk_reg_t<64, 16, CH>(a, st);
    return cudaErrorNotSupported;
}

inline cudaError_t launch_chunk_reg(const ScanArgs& a, int d, int spc, cudaStream_t st) {
    if (a.m != kRgM || (spc != 8 && spc != 16)) return cudaErrorNotSupported;
    if (a.chunk == 64) return launch_chunk_reg_c<64>(a, d, spc, st);
    if (a.chunk == 16) return launch_chunk_reg_c<16>(a, d, spc, st);
    return cudaErrorNotSupported;
}

}  // namespace lattice
