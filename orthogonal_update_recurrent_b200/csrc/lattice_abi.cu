// lattice_abi.cu -- extern "C" entry points of liblattice (declared in
// include/lattice.h): argument checks and kernel choice. The launches live in one
// translation unit per kernel family (tu_*.cu, through launch.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "launch.h"
#include "waits.cuh"

using namespace lattice;

namespace {

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
};

Span span(const void* p, size_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Span{a, a + bytes};
}
bool overlap(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }
bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }
bool dtype_ok(lattice_dtype t) { return t == LATTICE_F32 || t == LATTICE_BF16; }
size_t dsize(lattice_dtype t) { return t == LATTICE_BF16 ? 2 : 4; }
bool d_supported(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

thread_local char g_last_error[256] = "";

}  // namespace

namespace lattice {

// SMs of the current device (148 on B200; also the answer without a device).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        return n;
    cudaGetLastError();  // clear the error of a host without a device
    return 148;
}

lattice_status cuda_fail(cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return LATTICE_ERR_CUDA;
}

lattice_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LATTICE_OK : cuda_fail(e);
}

// CTAs per sequence for the CUDA-core scans: when the batch has fewer sequences than
// SMs, a cluster of G CTAs per sequence covers more of the device (G at most 4, at
// least 4 and at most 32 slots per CTA); otherwise 1. Measured on B200: 8-CTA clusters
// (8 slots per CTA) ran the long-context backward at half the speed of 4-CTA ones.
int cluster_split(int B, int H, int m) {
    const long long seqs = (long long)B * H;
    long long G = sm_count() / seqs;
    if (G > 4) G = 4;
    if (G > (m + 3) / 4) G = (m + 3) / 4;
    if (G < 2 || (m + G - 1) / G > 32) return 1;
    return (int)G;
}

}  // namespace lattice

namespace {

// ---- backward
constexpr int kBwdMaxM = 128;  // slots per head of the backward kernels

int bwd_seg(int chunk, int seg) {
    if (seg == 0) return chunk >= 64 ? chunk : chunk * ((64 + chunk - 1) / chunk);
    return (seg > 0 && seg % chunk == 0) ? seg : -1;
}

// CTAs per sequence of the backward kernel (see cluster_split).
int bwd_split(int B, int H, int m) { return cluster_split(B, H, m); }

// One warp waits, with the library's bounded wait, on an mbarrier that nothing ever
// arrives on: after limit_ns the wait gives up, sets the device status word and the
// kernel returns. Used to check, on a live GPU, that a wait that runs out is reported
// on the host and leaves the context usable.
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    const uint32_t b = ptx::smem_u32(&bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(b, 1);
        abort_flag = 0u;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    tc_wait(b, 0, &abort_flag, limit_ns);
}

lattice_status check_dims(int B, int H, int m, int d) {
    if (B < 1 || H < 1 || m < 1 || d < 1) return LATTICE_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return LATTICE_ERR_UNSUPPORTED;
    if (!d_supported(d) || m > kMaxM) return LATTICE_ERR_UNSUPPORTED;
    return LATTICE_OK;
}

}  // namespace

extern "C" {

int lattice_version(void) { return 100; }

const char* lattice_status_string(lattice_status s) {
    switch (s) {
        case LATTICE_OK: return "ok";
        case LATTICE_ERR_INVALID_ARG: return "invalid argument";
        case LATTICE_ERR_UNSUPPORTED: return "unsupported size or dtype";
        case LATTICE_ERR_CUDA: return "CUDA error";
        case LATTICE_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

lattice_impl lattice_chunk_impl(int B, int H, int m, int d, int chunk_size, lattice_dtype x_dtype,
                                lattice_dtype q_dtype) {
    if (chunk_size <= 1) return LATTICE_IMPL_SIMT;
    const bool xb = x_dtype == LATTICE_BF16, qb = q_dtype == LATTICE_BF16;
    if (tc_supported(LATTICE_IMPL_SPLIT_REG, m, d, chunk_size, xb, qb) && B >= 1 && H >= 1 &&
        (long long)B * H <= reg_cluster_capacity(d))
        return LATTICE_IMPL_SPLIT_REG;
    if (tc_supported(LATTICE_IMPL_TCGEN05, m, d, chunk_size, xb, qb)) return LATTICE_IMPL_TCGEN05;
    return LATTICE_IMPL_SIMT;
}

lattice_status lattice_scan_fwd_ex(const void* x, lattice_dtype x_dtype, const float* c,
                                   const void* q, lattice_dtype q_dtype, const float* mu,
                                   const float* eta, const float* S0, float* S_out, float* y,
                                   int B, int T, int H, int m, int d, int chunk_size,
                                   lattice_mode mode, lattice_chunk_form form, lattice_impl impl,
                                   void* stream) {
    if ((int)form < 0 || (int)form > 3) return LATTICE_ERR_INVALID_ARG;
    const bool lin1 = ((int)form & LATTICE_CHUNK_LIN1) != 0;
    const bool cnorm = ((int)form & LATTICE_CHUNK_NORM_AT_BOUNDARY) != 0;
    if (B < 1 || H < 1 || m < 1 || d < 1 || T < 0 || chunk_size < 1) return LATTICE_ERR_INVALID_ARG;
    if (!dtype_ok(x_dtype) || !dtype_ok(q_dtype)) return LATTICE_ERR_INVALID_ARG;
    if (impl != LATTICE_IMPL_AUTO && impl != LATTICE_IMPL_SIMT && impl != LATTICE_IMPL_TCGEN05 &&
        impl != LATTICE_IMPL_TCGEN05_SPLIT && impl != LATTICE_IMPL_SPLIT_REG &&
        impl != LATTICE_IMPL_SPLIT_REG8)
        return LATTICE_ERR_INVALID_ARG;
    if (mode != LATTICE_SIM && mode != LATTICE_DEC) return LATTICE_ERR_INVALID_ARG;
    const bool dec = mode == LATTICE_DEC;
    lattice_status ds = check_dims(B, H, m, d);
    if (ds != LATTICE_OK) return ds;
    if (!S0 || !S_out) return LATTICE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !c || !q || !mu || !y)) return LATTICE_ERR_INVALID_ARG;
    if (!aligned(S0, 16) || !aligned(S_out, 16)) return LATTICE_ERR_INVALID_ARG;
    const size_t nS = (size_t)B * H * m * d * 4;
    const Span sS0 = span(S0, nS), sSo = span(S_out, nS);
    if (S0 != S_out && overlap(sS0, sSo)) return LATTICE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S0 != S_out) {
            cudaError_t e = cudaMemcpyAsync(S_out, S0, nS, cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return LATTICE_OK;
    }
    const size_t ntok = (size_t)B * T * H;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(c, 4) || !aligned(mu, 4) ||
        !aligned(q, dsize(q_dtype)) || (eta && !aligned(eta, 4)))
        return LATTICE_ERR_INVALID_ARG;
    const Span sx = span(x, ntok * d * dsize(x_dtype)), sc = span(c, ntok * m * 4),
               sq = span(q, ntok * m * dsize(q_dtype)), smu = span(mu, ntok * 4),
               seta = span(eta, eta ? ntok * 4 : 0), sy = span(y, ntok * d * 4);
    const Span ins[] = {sx, sc, sq, smu, seta, sS0};
    for (const Span& s : ins)
        if (overlap(s, sy) || (s.lo != sS0.lo && overlap(s, sSo))) return LATTICE_ERR_INVALID_ARG;
    if (overlap(sy, sSo)) return LATTICE_ERR_INVALID_ARG;

    ScanArgs a{x, x_dtype == LATTICE_BF16, c, q, q_dtype == LATTICE_BF16, mu, eta, S0, S_out, y,
               B, T, H, m, chunk_size};
    const bool tc_choice = impl == LATTICE_IMPL_TCGEN05 || impl == LATTICE_IMPL_TCGEN05_SPLIT ||
                           impl == LATTICE_IMPL_SPLIT_REG || impl == LATTICE_IMPL_SPLIT_REG8;
    a.cnorm = cnorm && chunk_size > 1 ? 1 : 0;
    if (chunk_size == 1 && cnorm) {  // normalising after every token is the exact recurrence
        if (tc_choice) return LATTICE_ERR_UNSUPPORTED;
        return launch_scan_simt(a, d, false, dec, false, st);
    }
    if (chunk_size == 1 || dec || lin1 || cnorm) {  // the tensor-core kernels: Eq. 17, per-token normaliser, similarity objective
        if (tc_choice) return LATTICE_ERR_UNSUPPORTED;
        return launch_scan_simt(a, d, chunk_size > 1, dec, lin1, st);
    }
    if (impl == LATTICE_IMPL_AUTO) impl = lattice_chunk_impl(B, H, m, d, chunk_size, x_dtype, q_dtype);
    if (impl != LATTICE_IMPL_SIMT) {
        if (!tc_supported(impl, m, d, chunk_size, a.x_bf16, a.q_bf16)) return LATTICE_ERR_UNSUPPORTED;
        return launch_tc(impl, a, d, st);
    }
    return launch_scan_simt(a, d, true, false, false, st);
}

lattice_status lattice_scan_fwd_impl(const void* x, lattice_dtype x_dtype, const float* c,
                                     const void* q, lattice_dtype q_dtype, const float* mu,
                                     const float* eta, const float* S0, float* S_out, float* y,
                                     int B, int T, int H, int m, int d, int chunk_size,
                                     lattice_mode mode, lattice_impl impl, void* stream) {
    return lattice_scan_fwd_ex(x, x_dtype, c, q, q_dtype, mu, eta, S0, S_out, y, B, T, H, m, d,
                               chunk_size, mode, LATTICE_CHUNK_LIN2, impl, stream);
}

lattice_status lattice_scan_fwd(const void* x, lattice_dtype x_dtype, const float* c,
                                const void* q, lattice_dtype q_dtype, const float* mu,
                                const float* eta, const float* S0, float* S_out, float* y, int B,
                                int T, int H, int m, int d, int chunk_size, lattice_mode mode,
                                void* stream) {
    return lattice_scan_fwd_impl(x, x_dtype, c, q, q_dtype, mu, eta, S0, S_out, y, B, T, H, m, d,
                                 chunk_size, mode, LATTICE_IMPL_AUTO, stream);
}

lattice_status lattice_step(float* S, const void* x, lattice_dtype x_dtype, const float* c,
                            const void* q, lattice_dtype q_dtype, const float* mu,
                            const float* eta, float* y, int B, int H, int m, int d,
                            lattice_mode mode, void* stream) {
    if (!dtype_ok(x_dtype) || !dtype_ok(q_dtype)) return LATTICE_ERR_INVALID_ARG;
    if (mode != LATTICE_SIM && mode != LATTICE_DEC) return LATTICE_ERR_INVALID_ARG;
    const bool dec = mode == LATTICE_DEC;
    lattice_status ds = check_dims(B, H, m, d);
    if (ds != LATTICE_OK) return ds;
    if (!S || !x || !c || !q || !mu || !y) return LATTICE_ERR_INVALID_ARG;
    if (!aligned(S, 16) || !aligned(x, 16) || !aligned(y, 16) || !aligned(c, 4) ||
        !aligned(mu, 4) || !aligned(q, dsize(q_dtype)) || (eta && !aligned(eta, 4)))
        return LATTICE_ERR_INVALID_ARG;
    const size_t nbh = (size_t)B * H;
    const Span sS = span(S, nbh * m * d * 4), sy = span(y, nbh * d * 4);
    const Span ins[] = {span(x, nbh * d * dsize(x_dtype)), span(c, nbh * m * 4),
                        span(q, nbh * m * dsize(q_dtype)), span(mu, nbh * 4),
                        span(eta, eta ? nbh * 4 : 0)};
    for (const Span& s : ins)
        if (overlap(s, sS) || overlap(s, sy)) return LATTICE_ERR_INVALID_ARG;
    if (overlap(sS, sy)) return LATTICE_ERR_INVALID_ARG;
    StepArgs a{S, x, x_dtype == LATTICE_BF16, c, q, q_dtype == LATTICE_BF16, mu, eta, y, B, H, m};
    return launch_step(a, d, dec, static_cast<cudaStream_t>(stream));
}

lattice_status lattice_readout(const float* S, const void* q, lattice_dtype q_dtype, float* y,
                               int B, int H, int m, int d, void* stream) {
    if (!dtype_ok(q_dtype)) return LATTICE_ERR_INVALID_ARG;
    lattice_status ds = check_dims(B, H, m, d);
    if (ds != LATTICE_OK) return ds;
    if (!S || !q || !y) return LATTICE_ERR_INVALID_ARG;
    if (!aligned(S, 16) || !aligned(y, 16) || !aligned(q, dsize(q_dtype))) return LATTICE_ERR_INVALID_ARG;
    const size_t nbh = (size_t)B * H;
    const Span sy = span(y, nbh * d * 4);
    if (overlap(sy, span(S, nbh * m * d * 4)) || overlap(sy, span(q, nbh * m * dsize(q_dtype))))
        return LATTICE_ERR_INVALID_ARG;
    ReadoutArgs a{S, q, q_dtype == LATTICE_BF16, y, B, H, m};
    return launch_readout(a, d, static_cast<cudaStream_t>(stream));
}

size_t lattice_scan_bwd_workspace_bytes(int B, int T, int H, int m, int d, int chunk_size,
                                        int seg_tokens) {
    if (B < 1 || H < 1 || m < 1 || d < 1 || T < 0 || chunk_size < 1) return 0;
    if (check_dims(B, H, m, d) != LATTICE_OK || m > kBwdMaxM) return 0;
    const int seg = bwd_seg(chunk_size, seg_tokens);
    if (seg < 1) return 0;
    const int G = bwd_split(B, H, m), spc = (m + G - 1) / G;
    const size_t tok = (size_t)B * H * G * bwd_ws_floats_per_seq(T, spc, d, seg) * sizeof(float);
    if (!chunk_bwd_supported(m, d, chunk_size)) return tok;
    // the chunk-parallel kernel serves the shape; the token kernel stays the fallback
    // for buffers it cannot read with vector loads, so the workspace covers both
    const size_t cb = chunk_bwd_ws_floats(B, T, H, m, d, chunk_size) * sizeof(float);
    return cb > tok ? cb : tok;
}

lattice_status lattice_scan_bwd(const void* x, lattice_dtype x_dtype, const float* c,
                                const void* q, lattice_dtype q_dtype, const float* mu,
                                const float* eta, const float* S0, const float* dy,
                                const float* dS_T, float* dx, float* dc, float* dq, float* dmu,
                                float* deta, float* dS0, void* workspace, size_t workspace_bytes,
                                int B, int T, int H, int m, int d, int chunk_size, int seg_tokens,
                                void* stream) {
    if (B < 1 || H < 1 || m < 1 || d < 1 || T < 0 || chunk_size < 1) return LATTICE_ERR_INVALID_ARG;
    if (!dtype_ok(x_dtype) || !dtype_ok(q_dtype)) return LATTICE_ERR_INVALID_ARG;
    lattice_status ds = check_dims(B, H, m, d);
    if (ds != LATTICE_OK) return ds;
    if (m > kBwdMaxM) return LATTICE_ERR_UNSUPPORTED;
    const int seg = bwd_seg(chunk_size, seg_tokens);
    if (seg < 1) return LATTICE_ERR_INVALID_ARG;
    const size_t need = lattice_scan_bwd_workspace_bytes(B, T, H, m, d, chunk_size, seg_tokens);
    if (!S0 || !dS0 || !workspace || workspace_bytes < need) return LATTICE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !c || !q || !mu || !dy || !dx || !dc || !dq || !dmu))
        return LATTICE_ERR_INVALID_ARG;
    if (!aligned(S0, 16) || !aligned(dS0, 16) || !aligned(workspace, 16) || (dS_T && !aligned(dS_T, 16)))
        return LATTICE_ERR_INVALID_ARG;
    const size_t ntok = (size_t)B * T * H, nS = (size_t)B * H * m * d * 4;
    if (T > 0 && (!aligned(x, dsize(x_dtype)) || !aligned(c, 4) || !aligned(mu, 4) || !aligned(q, dsize(q_dtype)) ||
                  !aligned(dy, 4) || !aligned(dx, 4) || !aligned(dc, 4) || !aligned(dq, 4) ||
                  !aligned(dmu, 4) || (eta && !aligned(eta, 4)) || (deta && !aligned(deta, 4))))
        return LATTICE_ERR_INVALID_ARG;
    float* deta_w = eta ? deta : nullptr;
    const size_t tb = T > 0 ? 1 : 0;  // token-indexed buffers are empty when T == 0
    const Span ins[] = {span(x, tb * ntok * d * dsize(x_dtype)), span(c, tb * ntok * m * 4),
                        span(q, tb * ntok * m * dsize(q_dtype)), span(mu, tb * ntok * 4),
                        span(eta, eta ? tb * ntok * 4 : 0), span(S0, nS),
                        span(dy, tb * ntok * d * 4), span(dS_T, dS_T ? nS : 0)};
    const Span outs[] = {span(dx, tb * ntok * d * 4), span(dc, tb * ntok * m * 4),
                         span(dq, tb * ntok * m * 4), span(dmu, tb * ntok * 4),
                         span(deta_w, deta_w ? tb * ntok * 4 : 0), span(dS0, nS),
                         span(workspace, need)};
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
        for (const Span& s : ins)
            if (overlap(outs[i], s)) return LATTICE_ERR_INVALID_ARG;
        for (size_t k = i + 1; k < sizeof(outs) / sizeof(outs[0]); ++k)
            if (overlap(outs[i], outs[k])) return LATTICE_ERR_INVALID_ARG;
    }
    // Chunks of 2..64 tokens: the chunk-parallel kernel, when x, dy and dx take 16-byte
    // vector accesses; otherwise (and for the exact recurrence) the token kernel.
    if (chunk_bwd_supported(m, d, chunk_size) &&
        (T == 0 || (aligned(x, 16) && aligned(dy, 16) && aligned(dx, 16)))) {
        const int G = chunk_bwd_ctas(m);
        BwdArgs a{x, x_dtype == LATTICE_BF16, c, q, q_dtype == LATTICE_BF16, mu, eta, S0, dy, dS_T,
                  dx, dc, dq, dmu, deta_w, dS0, static_cast<float*>(workspace), B, T, H, m, chunk_size,
                  seg, G, kCbSlots};
        return launch_chunk_bwd(a, d, static_cast<cudaStream_t>(stream));
    }
    const int G = bwd_split(B, H, m);
    BwdArgs a{x, x_dtype == LATTICE_BF16, c, q, q_dtype == LATTICE_BF16, mu, eta, S0, dy, dS_T,
              dx, dc, dq, dmu, deta_w, dS0, static_cast<float*>(workspace), B, T, H, m, chunk_size, seg,
              G, (m + G - 1) / G};
    return launch_bwd(a, d, static_cast<cudaStream_t>(stream));
}

lattice_status lattice_selftest_bounded_wait(unsigned long long limit_ns, void* stream) {
    if (limit_ns < 1 || limit_ns > 1000000000ull) return LATTICE_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return launch_status();
}

lattice_status lattice_get_device_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    // every translation unit's copy of the status word (each unit is a module of its own)
    cudaError_t (*const units[])(unsigned int*) = {read_clear_module_status, status_simt_exact,
                                                   status_simt_chunked, status_step, status_bwd, status_tc};
    unsigned int any = 0;
    for (auto unit : units) {
        unsigned int v = 0;
        e = unit(&v);
        if (e != cudaSuccess) return cuda_fail(e);
        any |= v;
    }
    return any ? LATTICE_ERR_TIMEOUT : LATTICE_OK;
}

const char* lattice_last_cuda_error(void) { return g_last_error; }

}  // extern "C"

// ---- backward pass without allocation: scratch in a static device array
namespace {

constexpr size_t kNoAllocScratchBytes = LATTICE_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocCacheEntries = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// The array's device address differs from context to context (each context loads its
// own copy of the module), so the looked-up address is cached per context, keyed by
// the driver's unique context id. A caller running inside its own driver-API context,
// or a process that reset the device and so got a new primary context, gets a fresh
// lookup instead of an address that belongs to another context.
struct NoAllocEntry {
    unsigned long long ctx_id;
    void* addr;
};
std::mutex g_noalloc_mutex;
NoAllocEntry g_noalloc_cache[kNoAllocCacheEntries] = {};
int g_noalloc_next = 0;

typedef CUresult (*PfnCtxGetCurrent)(CUcontext*);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long*);

// Unique id of the context current on this thread (false if none is current).
bool current_ctx_id(unsigned long long* id) {
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PfnCtxGetId>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_scratch in the current context, looked up once per
// context with cudaGetSymbolAddress (a host-side query, no stream work). In host
// code the array's name is only a host-side stand-in, never a device address.
lattice_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    unsigned long long id = 0;
    bool have_id = current_ctx_id(&id);
    if (have_id) {
        for (const NoAllocEntry& en : g_noalloc_cache)
            if (en.addr && en.ctx_id == id) {
                *out = en.addr;
                return LATTICE_OK;
            }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's primary context current if none is
    if (e != cudaSuccess) return cuda_fail(e);
    if (!have_id) have_id = current_ctx_id(&id);
    if (have_id) {
        g_noalloc_cache[g_noalloc_next] = NoAllocEntry{id, p};
        g_noalloc_next = (g_noalloc_next + 1) % kNoAllocCacheEntries;
    }
    *out = p;
    return LATTICE_OK;
}

}  // namespace

extern "C" lattice_status lattice_scan_bwd_noalloc(
    const void* x, lattice_dtype x_dtype, const float* c, const void* q, lattice_dtype q_dtype,
    const float* mu, const float* eta, const float* S0, const float* dy, const float* dS_T,
    float* dx, float* dc, float* dq, float* dmu, float* deta, float* dS0, int B, int T, int H,
    int m, int d, int chunk_size, int seg_tokens, void* stream) {
    const size_t need = lattice_scan_bwd_workspace_bytes(B, T, H, m, d, chunk_size, seg_tokens);
    if (need == 0)  // a rejected shape: lattice_scan_bwd names the error before using the workspace
        return lattice_scan_bwd(x, x_dtype, c, q, q_dtype, mu, eta, S0, dy, dS_T, dx, dc, dq, dmu,
                                deta, dS0, nullptr, 0, B, T, H, m, d, chunk_size, seg_tokens, stream);
    if (need > kNoAllocScratchBytes) return LATTICE_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    lattice_status s = noalloc_scratch(&scratch);
    if (s != LATTICE_OK) return s;
    return lattice_scan_bwd(x, x_dtype, c, q, q_dtype, mu, eta, S0, dy, dS_T, dx, dc, dq, dmu, deta,
                            dS0, scratch, kNoAllocScratchBytes, B, T, H, m, d, chunk_size, seg_tokens,
                            stream);
}
