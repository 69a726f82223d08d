// tu_bwd.cu -- launches of the backward-pass kernels (scan_bwd.cuh, chunk_bwd.cuh).
#include "chunk_bwd.cuh"
#include "common.cuh"
#include "launch.h"
#include "scan_bwd.cuh"

namespace lattice {
namespace {

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
lattice_status launch_bwd_c(const BwdArgs& a, int d, cudaStream_t st) {
    switch (d) {
        case 16: return launch_bwd_d<16, CH>(a, st);
        case 32: return launch_bwd_d<32, CH>(a, st);
        case 64: return launch_bwd_d<64, CH>(a, st);
        case 128: return launch_bwd_d<128, CH>(a, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

template <int D>
lattice_status launch_chunk_bwd_t(const BwdArgs& a, cudaStream_t st) {
    const size_t smem = CbLayout<D>::BYTES;
    auto k = chunk_bwd_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.H * a.G));
    cfg.blockDim = dim3((unsigned)kCbThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.G > 1 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, k, a);
    if (e != cudaSuccess) return cuda_fail(e);
    return launch_status();
}

}  // namespace

// The chunk-parallel backward (chunk_bwd.cuh); a.G must be chunk_bwd_ctas(m).
lattice_status launch_chunk_bwd(const BwdArgs& a, int d, cudaStream_t st) {
    switch (d) {
        case 32: return launch_chunk_bwd_t<32>(a, st);
        case 64: return launch_chunk_bwd_t<64>(a, st);
        case 128: return launch_chunk_bwd_t<128>(a, st);
    }
    return LATTICE_ERR_UNSUPPORTED;
}

lattice_status launch_bwd(const BwdArgs& a, int d, cudaStream_t st) {
    return a.chunk == 1 ? launch_bwd_c<false>(a, d, st) : launch_bwd_c<true>(a, d, st);
}

cudaError_t status_bwd(unsigned int* v) { return read_clear_module_status(v); }

}  // namespace lattice
