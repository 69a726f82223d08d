/*
 * lattice.h -- C ABI of the B200 (sm_100a) Lattice compression-layer library.
 *
 * The library computes the state recurrence of "Lattice: Learning to
 * Efficiently Compress the Memory" (Karami, Pascanu, Mirrokni; arXiv
 * 2504.05646) for the similarity objective (h_t = -x_t):
 *
 *   per (batch b, head h), a state of m slots s_i in R^d (rows of S, the
 *   layout of the paper's Appendix D listing), for every token t:
 *     n_i = |s_i|,  p_i = s_i . x_t
 *     w_i = mu_t s_i + eta_t (c_{t,i}/n_i) (x_t - (p_i/n_i^2) s_i)
 *           [§3.1.1 eq. OSR: write only the part of x orthogonal to the slot,
 *            scaled by the writing intensity c; §3.3 eq. dacay_recurrence:
 *            forget gate mu; §3.4 Eq. 14: projection by one dot + one axpy]
 *     s_i <- w_i / |w_i|        [§3.2 eq. normalized_recurrence: unit sphere]
 *     y_t = sum_i q_{t,i} s_i   [read-out with the updated state, §3 General
 *                                Form; Appendix D, y = q @ S_t]
 *   If w_i = 0 (mu = 0 and no orthogonal write) the slot is left unchanged.
 *
 * The chunked form (chunk_size C > 1) is the paper's Eq. 17
 * (recurrence_linear2, §3.4.1 and Appendix B.1): inside a chunk the projection
 * uses the chunk-start state S0 (n_i = |s0_i|, p_i = s0_i . x_t) and the token
 * update is the gated linear recurrence s_i <- g_{t,i} s_i + kappa_{t,i} x_t with
 *   den = mu_t^2 n_i^2 + (eta_t c_{t,i}/n_i)^2 max(0, |x_t|^2 - p_i^2/n_i^2)
 *   g   = n_i (mu_t - eta_t c_{t,i} p_i / n_i^3) / sqrt(den)
 *   kappa = n_i (eta_t c_{t,i} / n_i) / sqrt(den)      [eq. beta_chunk]
 * (g = 1, kappa = 0 where den = 0). The factor n_i = |s0_i| follows the paper's
 * Appendix D listing, whose chunk normaliser keeps each slot's chunk-start
 * norm. Chunks are consecutive blocks of C tokens; the last one may be
 * partial. For unit-norm states, C = 1 is exactly the recurrence above.
 *
 * Layouts (row-major, element strides, no padding):
 *   x    [B][T][H][d]   fp32 or bf16          input written into the slots
 *   c    [B][T][H][m]   fp32                  writing intensities (codes)
 *   q    [B][T][H][m]   fp32 or bf16          read-out queries
 *   mu   [B][T][H]      fp32                  forget gate
 *   eta  [B][T][H]      fp32, or NULL for 1   step size
 *   S    [B][H][m][d]   fp32                  state, one slot per row
 *   y    [B][T][H][d]   fp32                  read-out
 * Decode calls drop the T axis.
 *
 * Ownership and execution: every pointer is caller-owned DEVICE memory. The
 * library allocates nothing and keeps no state besides one device status
 * word (and the static scratch array of lattice_scan_bwd_noalloc, described
 * there). Every call is asynchronous on `stream` (a cudaStream_t passed as
 * void*, NULL = the legacy default stream) and returns after the launch.
 *
 * Errors: arguments are checked on the host before anything is launched; a
 * failed check launches nothing and returns the code. LATTICE_ERR_CUDA means a
 * launch or attribute call failed (call cudaGetLastError for the detail).
 * Device-side waits are bounded: a kernel that gives up sets the status word
 * and returns; lattice_get_device_status() reports it as LATTICE_ERR_TIMEOUT.
 *
 * Supported sizes: d in {16, 32, 64, 128}; 1 <= m <= 256 (m <= 128 for the
 * backward pass); B, H >= 1; T >= 0.
 * The tensor-core chunked kernel serves C = 64, m in {64, 128},
 * d in {64, 128} with bf16 x and q; other chunked shapes run a CUDA-core
 * kernel of the same definition.
 */
#ifndef LATTICE_H_
#define LATTICE_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LATTICE_OK = 0,
    LATTICE_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, partial aliasing  */
    LATTICE_ERR_UNSUPPORTED = 2, /* valid but outside the supported sizes     */
    LATTICE_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed      */
    LATTICE_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up        */
} lattice_status;

typedef enum { LATTICE_F32 = 0, LATTICE_BF16 = 1 } lattice_dtype;

/* Objective (§3.1.1, eq. OSR): what each token writes into the slots.
 *   LATTICE_SIM  dot-product similarity objective, h_t = -x_t: slot i takes
 *                the part of x_t orthogonal to it (eq. similarity_recurrence).
 *   LATTICE_DEC  l2 reconstruction objective, h_t = e_t = phi(S) c_t - x_t with
 *                phi(s_i) = s_i/|s_i| (eq. decoding_stateNorm_loss and
 *                eq. decoding_recurrence): slot i takes the part of the
 *                reconstruction residual x_t - sum_j c_tj s_j/|s_j| orthogonal
 *                to it. e is formed from the state the token's projection uses:
 *                the current state (exact recurrence, decode step) or the
 *                chunk-start state (chunked form, as in the Appendix D listing).
 * DEC runs on the CUDA-core kernels only. The tensor-core choices return
 * LATTICE_ERR_UNSUPPORTED for it, and LATTICE_IMPL_AUTO takes the CUDA-core
 * kernel. */
typedef enum { LATTICE_SIM = 0, LATTICE_DEC = 1 } lattice_mode;

/* Kernel choice for chunked scans.
 *   AUTO            picks the fastest kernel that can run the shape (see
 *                   lattice_chunk_impl).
 *   SIMT            the CUDA-core kernel (any chunk size, fp32 or bf16 x/q).
 *   TCGEN05         the tensor-core kernel with one CTA per sequence
 *                   (chunk 64, bf16 x and q, m and d in {64, 128}).
 *   TCGEN05_SPLIT   the tensor-core kernel with each sequence's 64 slots split
 *                   over a cluster of 4 CTAs (chunk 64, bf16 x and q, m = 64,
 *                   d in {64, 128}); for batches with fewer sequences than SMs.
 *   SPLIT_REG       the same split and read-out, with each CTA's share of the
 *                   state held in registers and advanced chunk to chunk by
 *                   warp-synchronous tensor-core MMAs (mma.sync), which keeps the
 *                   per-chunk dependency chain off every asynchronous round trip
 *                   (chunk 64 or 16, bf16 x and q, m = 64, d in {64, 128}).
 *   SPLIT_REG8      as SPLIT_REG with 8 slots per CTA over a cluster of 8 CTAs:
 *                   half the tensor work on each CTA's chain; needs B*H clusters
 *                   of 8 SMs within one GPC each.
 * An explicit choice that cannot run the shape returns LATTICE_ERR_UNSUPPORTED.
 * All tensor-core choices compute the same chunked form; they differ only in
 * fp32 summation order. */
typedef enum {
    LATTICE_IMPL_AUTO = 0,
    LATTICE_IMPL_SIMT = 1,
    LATTICE_IMPL_TCGEN05 = 2,
    LATTICE_IMPL_TCGEN05_SPLIT = 3,
    LATTICE_IMPL_SPLIT_REG = 4,
    LATTICE_IMPL_SPLIT_REG8 = 5
} lattice_impl;

/* Which kernel LATTICE_IMPL_AUTO runs for a chunked scan of B x H sequences of
 * this shape: SPLIT_REG when it applies (chunk 64 or 16, m = 64) and the current
 * device holds B*H of its 4-CTA clusters at once, else TCGEN05 when it applies,
 * else SIMT (chunk_size 1 is always SIMT). Host function; launches nothing
 * (without a device it assumes the 37 clusters of a 148-SM part). */
lattice_impl lattice_chunk_impl(int B, int H, int m, int d, int chunk_size, lattice_dtype x_dtype,
                                lattice_dtype q_dtype);

/* Whole-sequence forward (the paper's lattice_compress, Appendix D).
 * Reads S0, writes the final state to S_out (S_out == S0 is allowed: the
 * update is then in place; any other overlap between outputs and inputs is
 * LATTICE_ERR_INVALID_ARG) and the read-out of every token to y.
 * chunk_size = 1: exact recurrence; chunk_size > 1: Eq. 17 chunked form.
 * T = 0 copies S0 to S_out and writes nothing else. */
lattice_status lattice_scan_fwd(const void *x, lattice_dtype x_dtype, const float *c,
                                const void *q, lattice_dtype q_dtype, const float *mu,
                                const float *eta, const float *S0, float *S_out, float *y,
                                int B, int T, int H, int m, int d, int chunk_size,
                                lattice_mode mode, void *stream);

/* Chunk form for chunk_size > 1: a linearisation (§3.4.1), optionally OR'ed with
 * LATTICE_CHUNK_NORM_AT_BOUNDARY.
 *   LATTICE_CHUNK_LIN2  Eq. 17 (recurrence_linear2), the default: within a chunk
 *                       each token's gate g = beta (mu + eta hhat khat) scales the
 *                       running slot.
 *   LATTICE_CHUNK_LIN1  eq. recurrence_linear1: the forget part beta mu scales
 *                       the running slot and the projection part beta eta hhat khat
 *                       the chunk-start slot (its chunk form is eq. chunkwise_OSR).
 *   LATTICE_CHUNK_NORM_AT_BOUNDARY  the normalisation ablation of Appendix C
 *                       ("Per-token vs. Per-chunk Normalization"): no per-token
 *                       normaliser inside a chunk (beta = 1); every slot is
 *                       projected onto the unit sphere after each chunk, once the
 *                       chunk's read-outs are done. With chunk_size 1 this is the
 *                       exact recurrence.
 * LIN1 and NORM_AT_BOUNDARY run on the CUDA-core kernel only: tensor-core choices
 * return LATTICE_ERR_UNSUPPORTED, and AUTO takes the CUDA-core kernel. */
typedef enum {
    LATTICE_CHUNK_LIN2 = 0,
    LATTICE_CHUNK_LIN1 = 1,
    LATTICE_CHUNK_NORM_AT_BOUNDARY = 2
} lattice_chunk_form;

/* As lattice_scan_fwd, with an explicit kernel choice (see lattice_impl). */
lattice_status lattice_scan_fwd_impl(const void *x, lattice_dtype x_dtype, const float *c,
                                     const void *q, lattice_dtype q_dtype, const float *mu,
                                     const float *eta, const float *S0, float *S_out, float *y,
                                     int B, int T, int H, int m, int d, int chunk_size,
                                     lattice_mode mode, lattice_impl impl, void *stream);

/* As lattice_scan_fwd_impl, with the chunk form (see lattice_chunk_form; values 0-3;
 * the linearisation is ignored for chunk_size 1). Any other form is
 * LATTICE_ERR_INVALID_ARG. */
lattice_status lattice_scan_fwd_ex(const void *x, lattice_dtype x_dtype, const float *c,
                                   const void *q, lattice_dtype q_dtype, const float *mu,
                                   const float *eta, const float *S0, float *S_out, float *y,
                                   int B, int T, int H, int m, int d, int chunk_size,
                                   lattice_mode mode, lattice_chunk_form form, lattice_impl impl,
                                   void *stream);

/* Backward pass of the similarity-objective scan (exact recurrence for
 * chunk_size 1, Eq. 17 otherwise). The paper prints no backward formulas; this is
 * the reverse-mode derivative of the forward of lattice_scan_fwd with
 * LATTICE_SIM and LATTICE_CHUNK_LIN2, for the scalar loss
 *     L = sum_t dy_t . y_t + dS_T . S_T.
 * Inputs as for lattice_scan_fwd (same layouts and dtypes), plus
 *   dy [B][T][H][d] fp32 (required when T > 0) and dS_T [B][H][m][d] fp32 or NULL (0).
 * Outputs (fp32, device, the inputs' layouts, written in full): dx, dc, dq, dmu,
 *   deta (may be NULL; not written when eta is NULL, i.e. eta = 1) and dS0.
 * States are rebuilt by recomputation from checkpoints every seg_tokens tokens
 * (0 selects the default: the smallest multiple of chunk_size that is >= 64; any
 * other value must be a positive multiple of chunk_size, else
 * LATTICE_ERR_INVALID_ARG). workspace is caller-owned device memory of at least
 * lattice_scan_bwd_workspace_bytes(...) bytes, 16-byte aligned; the call
 * overwrites it and keeps no pointer after it returns (the kernel runs on
 * `stream`). Outputs must not overlap inputs, each other or the workspace
 * (LATTICE_ERR_INVALID_ARG). m <= 128 (larger m: LATTICE_ERR_UNSUPPORTED).
 * Kernels: chunk sizes 2..64 with d in {32, 64, 128}, and x, dy, dx on 16-byte
 * boundaries, run a chunk-parallel kernel: a forward sweep stores every chunk-start
 * state in the workspace, then each chunk, last to first, is differentiated as a whole
 * (matrix products on the tensor cores in tf32 with a hi/lo split of each operand,
 * about fp32 accuracy), and only the state adjoint passes from chunk to chunk;
 * seg_tokens is checked but not used. Other shapes (the exact recurrence included)
 * run token by token on CUDA cores with the segment checkpoints described above.
 * Both are deterministic: sums across CTAs are taken in a fixed order. */
lattice_status lattice_scan_bwd(const void *x, lattice_dtype x_dtype, const float *c,
                                const void *q, lattice_dtype q_dtype, const float *mu,
                                const float *eta, const float *S0, const float *dy,
                                const float *dS_T, float *dx, float *dc, float *dq, float *dmu,
                                float *deta, float *dS0, void *workspace, size_t workspace_bytes,
                                int B, int T, int H, int m, int d, int chunk_size, int seg_tokens,
                                void *stream);

/* Workspace bytes lattice_scan_bwd needs for this shape on the current device: the
 * token kernel's B*H*G*(n_seg - 1 + seg_tokens)*ceil(m/G)*d*4 with
 * n_seg = ceil(T/seg_tokens) (seg_tokens as resolved by lattice_scan_bwd) and G the
 * CTAs per sequence it uses (G = 1 when the batch fills the device's SMs; up to 4
 * otherwise), and, where the chunk-parallel kernel serves the shape, the larger of
 * that and its B*H*ceil(m/16)*ceil(T/chunk)*16*d*4 (every chunk-start state), so that
 * either kernel can run. Returns 0 for arguments lattice_scan_bwd would reject. Host
 * function; launches nothing. */
size_t lattice_scan_bwd_workspace_bytes(int B, int T, int H, int m, int d, int chunk_size,
                                        int seg_tokens);

/* Backward pass that allocates nothing, for callers that cannot call cudaMalloc:
 * for example a plug-in running inside a host application that hands out every
 * byte of device memory through its own pool, or a process that reserved the
 * device's memory up front and may not ask the driver for more. The paper has no
 * counterpart; this is a packaging of lattice_scan_bwd.
 *
 * Arguments, layouts, results and errors are those of lattice_scan_bwd without the
 * workspace: the scratch it needs lives in one static device array of
 * LATTICE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. A shape whose workspace
 * (lattice_scan_bwd_workspace_bytes) exceeds that size returns
 * LATTICE_ERR_UNSUPPORTED before any device work. The caller still allocates the
 * inputs and outputs; the call itself makes no allocation.
 *
 * The first call in each CUDA context (the device's primary context, or a context
 * the caller created and made current) looks up the array's device address in that
 * context with cudaGetSymbolAddress and caches it under the context's unique id; make
 * that first call before any stream capture. Every call shares the one array:
 * calls that overlap on the GPU (on different streams, or from different host
 * threads without ordering) race and corrupt each other's results, so order them. Nothing needs clearing between calls: the kernel
 * writes every scratch word before it reads it. */
#define LATTICE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

lattice_status lattice_scan_bwd_noalloc(const void *x, lattice_dtype x_dtype, const float *c,
                                        const void *q, lattice_dtype q_dtype, const float *mu,
                                        const float *eta, const float *S0, const float *dy,
                                        const float *dS_T, float *dx, float *dc, float *dq,
                                        float *dmu, float *deta, float *dS0, int B, int T, int H,
                                        int m, int d, int chunk_size, int seg_tokens, void *stream);

/* One decode step: the exact recurrence for one new token per (b,h), state
 * updated in place (constant work per token, §1-§2 of the paper).
 *   S [B][H][m][d] in/out, x [B][H][d], c [B][H][m], q [B][H][m],
 *   mu [B][H], eta [B][H] or NULL, y [B][H][d] out. */
lattice_status lattice_step(float *S, const void *x, lattice_dtype x_dtype, const float *c,
                            const void *q, lattice_dtype q_dtype, const float *mu,
                            const float *eta, float *y, int B, int H, int m, int d,
                            lattice_mode mode, void *stream);

/* Read-out without an update: y[b][h][:] = sum_i q[b][h][i] S[b][h][i][:]
 * (§2 eq. LA memory read-out; Appendix D y = q @ S). S [B][H][m][d],
 * q [B][H][m], y [B][H][d]. */
lattice_status lattice_readout(const float *S, const void *q, lattice_dtype q_dtype, float *y,
                               int B, int H, int m, int d, void *stream);

/* Synchronises `stream`, returns LATTICE_ERR_TIMEOUT if any kernel since the
 * last call gave up a bounded wait (and clears the flag), LATTICE_ERR_CUDA if
 * the stream reports an error, else LATTICE_OK. */
lattice_status lattice_get_device_status(void *stream);

/* Failure-detection self-test (the paper has no counterpart): launches one warp
 * that waits, with the same bounded device-side wait the tensor-core kernels use,
 * on an mbarrier that nothing ever completes. After limit_ns nanoseconds (1 ns to
 * 1 s; else LATTICE_ERR_INVALID_ARG, nothing launched) the wait gives up, sets the
 * device status word and the kernel returns, so the next
 * lattice_get_device_status(stream) returns LATTICE_ERR_TIMEOUT (and clears the
 * word) while the CUDA context stays usable. Asynchronous on `stream`. */
lattice_status lattice_selftest_bounded_wait(unsigned long long limit_ns, void *stream);

/* Name and description of the last CUDA error the library saw on this host
 * thread when a call returned LATTICE_ERR_CUDA ("" if none). The text is
 * owned by the library and stays valid until the next call on this thread. */
const char *lattice_last_cuda_error(void);

/* Static English text for a status code. */
const char *lattice_status_string(lattice_status s);

/* Library version, major*10000 + minor*100 + patch. */
int lattice_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LATTICE_H_ */
