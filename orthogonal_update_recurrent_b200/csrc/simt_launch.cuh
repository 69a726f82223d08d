// simt_launch.cuh -- launch templates of the CUDA-core scans, shared by the exact
// and chunked translation units (tu_simt_exact.cu, tu_simt_chunked.cu). Included by
// those two units only.
#pragma once
#include "common.cuh"
#include "launch.h"
#include "scan_simt.cuh"

namespace lattice {
namespace {

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

// one cluster of a.G CTAs (8 warps each) per sequence
template <int D, bool CH, bool DEC, bool LIN1>
lattice_status launch_scan_simt_split(const ScanArgs& a, cudaStream_t st) {
    const size_t smem = scan_smem_bytes<D>(a.m, 8, DEC, true, CH);
    auto k = scan_simt_kernel<D, 1, CH, DEC, LIN1, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
    ScanArgs arg = a;
    void* args[] = {&arg};
    return launch_clusters(reinterpret_cast<const void*>(k), a.B * a.H * a.G, 256, smem, a.G, st, args);
}

template <int D, bool CH, bool DEC, bool LIN1>
lattice_status launch_scan_simt_d(const ScanArgs& a, cudaStream_t st) {
    // The reconstruction objective couples every slot on every token: split, its
    // reconstructions are summed over the cluster once per token (exact) or once per
    // 16-token block (chunked, chunks made of whole blocks, d <= 64, where a block's
    // reconstruction buffers fit in shared memory).
    if constexpr (!DEC || !CH || D <= 64) {
        const int G = cluster_split(a.B, a.H, a.m);
        if (G > 1 && (!DEC || !CH || a.chunk % kScanTBSplit == 0)) {
            ScanArgs s = a;
            s.G = G;
            s.spc = (a.m + G - 1) / G;
            return launch_scan_simt_split<D, CH, DEC, LIN1>(s, st);
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

}  // namespace
}  // namespace lattice
