// lattice_abi.cu -- extern "C" entry points of liblattice (declared in
// include/lattice.h): argument checks, kernel choice and launches.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/lattice.h"
#include "common.cuh"
#include "scan_simt.cuh"
#include "step.cuh"
#include "chunk_tc.cuh"
#include "chunk_split.cuh"
#include "chunk_reg.cuh"
#include "scan_bwd.cuh"

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

lattice_status launch_clusters(const void* kernel, int grid, int block, size_t smem, int G,
                               cudaStream_t st, void** args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, args);
    if (e != cudaSuccess) return cuda_fail(e);
    return launch_status();
}

// ---- exact / chunked CUDA-core scan
template <int D, int RQ, bool CH, bool DEC, bool LIN1>
lattice_status launch_scan_simt_t(const ScanArgs& a, int nw, cudaStream_t st) {
    size_t smem = scan_smem_bytes<D>(a.m, nw, DEC);
    auto k = scan_simt_kernel<D, RQ, CH, DEC, LIN1>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
    k<<<a.B * a.H, nw * 32, smem, st>>>(a);
    return launch_status();
}

// one cluster of a.G CTAs (8 warps each) per sequence; similarity objective
template <int D, bool CH, bool LIN1>
lattice_status launch_scan_simt_split(const ScanArgs& a, cudaStream_t st) {
    const size_t smem = scan_smem_bytes<D>(a.m, 8, false, true);
    auto k = scan_simt_kernel<D, 1, CH, false, LIN1, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
    ScanArgs arg = a;
    void* args[] = {&arg};
    return launch_clusters(reinterpret_cast<const void*>(k), a.B * a.H * a.G, 256, smem, a.G, st, args);
}

template <int D, bool CH, bool DEC, bool LIN1>
lattice_status launch_scan_simt_d(const ScanArgs& a, cudaStream_t st) {
    if constexpr (!DEC) {  // the reconstruction objective couples every slot on every token
        const int G = cluster_split(a.B, a.H, a.m);
        if (G > 1) {
            ScanArgs s = a;
            s.G = G;
            s.spc = (a.m + G - 1) / G;
            return launch_scan_simt_split<D, CH, LIN1>(s, st);
        }
    }
    const int quads = (a.m + 3) / 4;
    if (quads <= 16) return launch_scan_simt_t<D, 1, CH, DEC, LIN1>(a, quads < 4 ? 4 : quads, st);
    if (quads <= 32) return launch_scan_simt_t<D, 2, CH, DEC, LIN1>(a, 16, st);
    return launch_scan_simt_t<D, 4, CH, DEC, LIN1>(a, 16, st);
}

template <bool CH, bool DEC, bool LIN1>
lattice_status launch_scan_simt_m(const ScanArgs& a, int d, cudaStream_t st) {
    switch (d) {
        case 16: return launch_scan_simt_d<16, CH, DEC, LIN1>(a, st);
        case 32: return launch_scan_simt_d<32, CH, DEC, LIN1>(a, st);
        case 64: return launch_scan_simt_d<64, CH, DEC, LIN1>(a, st);
        case 128: return launch_scan_simt_d<128, CH, DEC, LIN1>(a, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

// exact: CH = false (LIN1 does not apply); chunked: either linearisation
template <bool CH>
lattice_status launch_scan_simt(const ScanArgs& a, int d, bool dec, bool lin1, cudaStream_t st) {
    if constexpr (!CH) {
        return dec ? launch_scan_simt_m<false, true, false>(a, d, st) : launch_scan_simt_m<false, false, false>(a, d, st);
    } else {
        if (lin1)
            return dec ? launch_scan_simt_m<true, true, true>(a, d, st) : launch_scan_simt_m<true, false, true>(a, d, st);
        return dec ? launch_scan_simt_m<true, true, false>(a, d, st) : launch_scan_simt_m<true, false, false>(a, d, st);
    }
}

// ---- decode step / read-out: NW warps x RQ quads per warp
void step_shape(int m, int& nw, int& rq) {
    const int quads = (m + 3) / 4;
    if (quads <= 8) { nw = quads; rq = 1; }
    else if (quads <= 16) { nw = 8; rq = 2; }
    else if (quads <= 32) { nw = 8; rq = 4; }
    else { nw = 16; rq = 4; }
}

// The persistent decode step (step_pf_kernel): as many CTAs as fit on the device at
// once (cached per device, m and x dtype), each taking every G-th head.
constexpr int kStepMaxDevices = 16;

template <int D, int RQ, bool DEC>
lattice_status launch_step_pf(const StepArgs& a, int nw, int nheads, cudaStream_t st) {
    const StepPfLayout L(a.m, D, a.x_bf16);
    auto k = step_pf_kernel<D, RQ, DEC>;
    static int cache[kStepMaxDevices][2][kMaxM + 1];  // CTAs resident on the device; 0 = unknown
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    int* slot = dev < kStepMaxDevices ? &cache[dev][a.x_bf16 ? 1 : 0][a.m] : nullptr;
    int resident = slot ? *slot : 0;
    if (resident == 0) {
        // the largest buffer this instantiation can take (every m it serves, fp32 x), so
        // that a later launch with a larger m never meets a smaller limit
        const int m_max = 64 * RQ < kMaxM ? 64 * RQ : kMaxM;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)StepPfLayout(m_max, D, false).bytes);
        if (e != cudaSuccess) return cuda_fail(e);
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, nw * 32, L.bytes);
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        if (per_sm < 1) return LATTICE_ERR_UNSUPPORTED;
        resident = per_sm * sms;
        if (slot) *slot = resident;
    }
    k<<<dim3(nheads < resident ? nheads : resident), dim3(nw * 32), L.bytes, st>>>(a);
    return launch_status();
}

// Decode step. Under the reconstruction objective, with at least as many heads as SMs,
// the persistent kernel streams the next head's state in while computing the current
// one (measured at the decode shape, m = d = 128, 8192 heads: 234 us per step against
// 277 us). Otherwise every head has its own CTA, which loads its state straight into
// registers: the similarity objective's short arithmetic hides behind the other
// resident CTA's loads (186 us per step there, 193 us persistent).
template <int D, bool DEC>
lattice_status launch_step_dm(const StepArgs& a, cudaStream_t st) {
    int nw, rq;
    step_shape(a.m, nw, rq);
    const int nheads = a.B * a.H;
    int sms = 0, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nheads >= sms) {
        switch (rq) {
            case 1: return launch_step_pf<D, 1, DEC>(a, nw, nheads, st);
            case 2: return launch_step_pf<D, 2, DEC>(a, nw, nheads, st);
            default: return launch_step_pf<D, 4, DEC>(a, nw, nheads, st);
        }
    }
    dim3 grid(nheads), block(nw * 32);
    switch (rq) {
        case 1: step_kernel<D, 1, DEC><<<grid, block, 0, st>>>(a); break;
        case 2: step_kernel<D, 2, DEC><<<grid, block, 0, st>>>(a); break;
        default: step_kernel<D, 4, DEC><<<grid, block, 0, st>>>(a); break;
    }
    return launch_status();
}

template <int D>
lattice_status launch_step_d(const StepArgs& a, bool dec, cudaStream_t st) {
    return dec ? launch_step_dm<D, true>(a, st) : launch_step_dm<D, false>(a, st);
}

template <int D>
lattice_status launch_readout_d(const ReadoutArgs& a, cudaStream_t st) {
    int nw, rq;
    step_shape(a.m, nw, rq);
    dim3 grid(a.B * a.H), block(nw * 32);
    switch (rq) {
        case 1: readout_kernel<D, 1><<<grid, block, 0, st>>>(a); break;
        case 2: readout_kernel<D, 2><<<grid, block, 0, st>>>(a); break;
        default: readout_kernel<D, 4><<<grid, block, 0, st>>>(a); break;
    }
    return launch_status();
}

// ---- backward
constexpr int kBwdMaxM = 128;

int bwd_seg(int chunk, int seg) {
    if (seg == 0) return chunk >= 64 ? chunk : chunk * ((64 + chunk - 1) / chunk);
    return (seg > 0 && seg % chunk == 0) ? seg : -1;
}

// CTAs per sequence of the backward kernel (see cluster_split).
int bwd_split(int B, int H, int m) { return cluster_split(B, H, m); }

template <int D, int RQ, bool CH, bool SPLIT>
lattice_status launch_bwd_t(const BwdArgs& a, cudaStream_t st) {
    constexpr int nt = bwd_threads(SPLIT);
    const size_t smem = bwd_smem_bytes(D, a.spc, nt / 32, SPLIT);
    auto k = scan_bwd_kernel<D, RQ, CH, SPLIT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
    if (a.G == 1) {
        k<<<a.B * a.H, nt, smem, st>>>(a);
        return launch_status();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.H * a.G));
    cfg.blockDim = dim3((unsigned)nt);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k, a);
    if (e != cudaSuccess) return cuda_fail(e);
    return launch_status();
}

// One CTA per sequence: 16 warps, one slot (m <= 64) or two (m <= 128) per octet.
// Clusters: 8 warps per CTA, one slot per octet (bwd_split keeps <= 32 slots per CTA).
template <int D, bool CH>
lattice_status launch_bwd_d(const BwdArgs& a, cudaStream_t st) {
    if (a.G == 1) return a.m <= 64 ? launch_bwd_t<D, 1, CH, false>(a, st) : launch_bwd_t<D, 2, CH, false>(a, st);
    return launch_bwd_t<D, 1, CH, true>(a, st);
}

template <bool CH>
lattice_status launch_bwd(const BwdArgs& a, int d, cudaStream_t st) {
    switch (d) {
        case 16: return launch_bwd_d<16, CH>(a, st);
        case 32: return launch_bwd_d<32, CH>(a, st);
        case 64: return launch_bwd_d<64, CH>(a, st);
        case 128: return launch_bwd_d<128, CH>(a, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

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

// Clusters of 4 CTAs of the register-chain kernel the current device holds at once
// (queried once per device; without a device, the SMs / 4 of a 148-SM B200).
int reg_cluster_capacity(int d) {
    static int cache[64][2] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return sm_count() / 4;
    }
    int& c = cache[dev][d == 128 ? 1 : 0];
    if (c == 0) {
        c = chunk_reg_max_clusters(d, 16);
        if (c <= 0) c = -1;
    }
    return c > 0 ? c : sm_count() / 4;
}

lattice_impl lattice_chunk_impl(int B, int H, int m, int d, int chunk_size, lattice_dtype x_dtype,
                                lattice_dtype q_dtype) {
    if (chunk_size <= 1) return LATTICE_IMPL_SIMT;
    const bool xb = x_dtype == LATTICE_BF16, qb = q_dtype == LATTICE_BF16;
    if (chunk_reg_supported(m, d, chunk_size, xb, qb) && B >= 1 && H >= 1 &&
        (long long)B * H <= reg_cluster_capacity(d))
        return LATTICE_IMPL_SPLIT_REG;
    if (chunk_tc_supported(m, d, chunk_size, xb, qb)) return LATTICE_IMPL_TCGEN05;
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
        return launch_scan_simt<false>(a, d, dec, false, st);
    }
    if (chunk_size == 1 || dec || lin1 || cnorm) {  // the tensor-core kernels: Eq. 17, per-token normaliser, similarity objective
        if (tc_choice) return LATTICE_ERR_UNSUPPORTED;
        return chunk_size == 1 ? launch_scan_simt<false>(a, d, dec, false, st)
                               : launch_scan_simt<true>(a, d, dec, lin1, st);
    }
    if (impl == LATTICE_IMPL_AUTO) impl = lattice_chunk_impl(B, H, m, d, chunk_size, x_dtype, q_dtype);
    if (impl == LATTICE_IMPL_SPLIT_REG || impl == LATTICE_IMPL_SPLIT_REG8) {
        if (!chunk_reg_supported(m, d, chunk_size, a.x_bf16, a.q_bf16)) return LATTICE_ERR_UNSUPPORTED;
        cudaError_t e = launch_chunk_reg(a, d, impl == LATTICE_IMPL_SPLIT_REG8 ? 8 : 16, st);
        return e == cudaSuccess ? LATTICE_OK : cuda_fail(e);
    }
    if (impl == LATTICE_IMPL_TCGEN05_SPLIT) {
        if (!chunk_split_supported(m, d, chunk_size, a.x_bf16, a.q_bf16)) return LATTICE_ERR_UNSUPPORTED;
        cudaError_t e = launch_chunk_split(a, d, st);
        return e == cudaSuccess ? LATTICE_OK : cuda_fail(e);
    }
    if (impl == LATTICE_IMPL_TCGEN05) {
        if (!chunk_tc_supported(m, d, chunk_size, a.x_bf16, a.q_bf16)) return LATTICE_ERR_UNSUPPORTED;
        cudaError_t e = launch_chunk_tc(a, d, st);
        return e == cudaSuccess ? LATTICE_OK : cuda_fail(e);
    }
    return launch_scan_simt<true>(a, d, false, false, st);
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (d) {
        case 16: return launch_step_d<16>(a, dec, st);
        case 32: return launch_step_d<32>(a, dec, st);
        case 64: return launch_step_d<64>(a, dec, st);
        default: return launch_step_d<128>(a, dec, st);
    }
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (d) {
        case 16: return launch_readout_d<16>(a, st);
        case 32: return launch_readout_d<32>(a, st);
        case 64: return launch_readout_d<64>(a, st);
        default: return launch_readout_d<128>(a, st);
    }
}

size_t lattice_scan_bwd_workspace_bytes(int B, int T, int H, int m, int d, int chunk_size,
                                        int seg_tokens) {
    if (B < 1 || H < 1 || m < 1 || d < 1 || T < 0 || chunk_size < 1) return 0;
    if (check_dims(B, H, m, d) != LATTICE_OK || m > kBwdMaxM) return 0;
    const int seg = bwd_seg(chunk_size, seg_tokens);
    if (seg < 1) return 0;
    const int G = bwd_split(B, H, m), spc = (m + G - 1) / G;
    return (size_t)B * H * G * bwd_ws_floats_per_seq(T, spc, d, seg) * sizeof(float);
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
    const int G = bwd_split(B, H, m);
    BwdArgs a{x, x_dtype == LATTICE_BF16, c, q, q_dtype == LATTICE_BF16, mu, eta, S0, dy, dS_T,
              dx, dc, dq, dmu, deta_w, dS0, static_cast<float*>(workspace), B, T, H, m, chunk_size, seg,
              G, (m + G - 1) / G};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return chunk_size == 1 ? launch_bwd<false>(a, d, st) : launch_bwd<true>(a, d, st);
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
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e);
    if (v && (e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero))) != cudaSuccess)
        return cuda_fail(e);
    return v ? LATTICE_ERR_TIMEOUT : LATTICE_OK;
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
