// chunk_tc.cuh -- tensor-core (tcgen05) chunked scan. Not built yet: every
// chunked call runs the CUDA-core kernel.
#pragma once
#include "common.cuh"
#include "scan_simt.cuh"

namespace lattice {

inline bool chunk_tc_supported(int, int, int, bool, bool) { return false; }
inline cudaError_t launch_chunk_tc(const ScanArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace lattice
