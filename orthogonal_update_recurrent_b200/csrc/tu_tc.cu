// tu_tc.cu -- launches of the tensor-core chunked scans: one CTA per sequence
// (chunk_tc.cuh), the cluster kernel (chunk_split.cuh) and the register-chain cluster
// kernel (chunk_reg.cuh).
#include "chunk_reg.cuh"
#include "launch.h"

namespace lattice {

bool tc_supported(lattice_impl impl, int m, int d, int chunk, bool x_bf16, bool q_bf16) {
    switch (impl) {
        case LATTICE_IMPL_TCGEN05: return chunk_tc_supported(m, d, chunk, x_bf16, q_bf16);
        case LATTICE_IMPL_TCGEN05_SPLIT: return chunk_split_supported(m, d, chunk, x_bf16, q_bf16);
        case LATTICE_IMPL_SPLIT_REG:
        case LATTICE_IMPL_SPLIT_REG8: return chunk_reg_supported(m, d, chunk, x_bf16, q_bf16);
        default: return false;
    }
}

lattice_status launch_tc(lattice_impl impl, const ScanArgs& a, int d, cudaStream_t st) {
    cudaError_t e = cudaErrorNotSupported;
    switch (impl) {
        case LATTICE_IMPL_TCGEN05: e = launch_chunk_tc(a, d, st); break;
        case LATTICE_IMPL_TCGEN05_SPLIT: e = launch_chunk_split(a, d, st); break;
        case LATTICE_IMPL_SPLIT_REG: e = launch_chunk_reg(a, d, 16, st); break;
        case LATTICE_IMPL_SPLIT_REG8: e = launch_chunk_reg(a, d, 8, st); break;
        default: return LATTICE_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? LATTICE_OK : cuda_fail(e);
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

cudaError_t status_tc(unsigned int* v) { return read_clear_module_status(v); }

}  // namespace lattice
