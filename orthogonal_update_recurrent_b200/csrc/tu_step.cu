// tu_step.cu -- launches of the decode step and read-out kernels (step.cuh).
#include "common.cuh"
#include "launch.h"
#include "step.cuh"

namespace lattice {
namespace {

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

}  // namespace

lattice_status launch_step(const StepArgs& a, int d, bool dec, cudaStream_t st) {
    switch (d) {
        case 16: return launch_step_d<16>(a, dec, st);
        case 32: return launch_step_d<32>(a, dec, st);
        case 64: return launch_step_d<64>(a, dec, st);
        case 128: return launch_step_d<128>(a, dec, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

lattice_status launch_readout(const ReadoutArgs& a, int d, cudaStream_t st) {
    switch (d) {
        case 16: return launch_readout_d<16>(a, st);
        case 32: return launch_readout_d<32>(a, st);
        case 64: return launch_readout_d<64>(a, st);
        case 128: return launch_readout_d<128>(a, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

cudaError_t status_step(unsigned int* v) { return read_clear_module_status(v); }

}  // namespace lattice
