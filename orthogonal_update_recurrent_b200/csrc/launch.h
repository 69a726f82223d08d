// launch.h -- host interface between the C ABI (lattice_abi.cu) and the kernel
// families. Each family is compiled in a translation unit of its own (tu_*.cu), so
// that the units build in parallel and each is optimised as a whole; this header
// carries no device code.
#pragma once
#include <cuda_runtime.h>

#include "../../include/lattice.h"
#include "args.h"

namespace lattice {

// lattice_abi.cu: error recording and device queries shared by every unit
lattice_status cuda_fail(cudaError_t e);
lattice_status launch_status();
int sm_count();
// CTAs per sequence for the CUDA-core kernels (a cluster when > 1)
int cluster_split(int B, int H, int m);

// tu_simt_exact.cu, tu_simt_chunked.cu: CUDA-core scans, exact or chunked (either linearisation)
lattice_status launch_scan_simt_exact(const ScanArgs& a, int d, bool dec, cudaStream_t st);
lattice_status launch_scan_simt_chunked(const ScanArgs& a, int d, bool dec, bool lin1, cudaStream_t st);
inline lattice_status launch_scan_simt(const ScanArgs& a, int d, bool chunked, bool dec, bool lin1, cudaStream_t st) {
    return chunked ? launch_scan_simt_chunked(a, d, dec, lin1, st) : launch_scan_simt_exact(a, d, dec, st);
}

// tu_step.cu: decode step and read-out
lattice_status launch_step(const StepArgs& a, int d, bool dec, cudaStream_t st);
lattice_status launch_readout(const ReadoutArgs& a, int d, cudaStream_t st);

// tu_bwd.cu: backward pass (a.G, a.spc set by the caller)
lattice_status launch_bwd(const BwdArgs& a, int d, cudaStream_t st);
lattice_status launch_chunk_bwd(const BwdArgs& a, int d, cudaStream_t st);

// tu_tc.cu: tensor-core chunked scans
bool tc_supported(lattice_impl impl, int m, int d, int chunk, bool x_bf16, bool q_bf16);
lattice_status launch_tc(lattice_impl impl, const ScanArgs& a, int d, cudaStream_t st);
// clusters of 4 CTAs of the register-chain kernel the current device holds at once
int reg_cluster_capacity(int d);

// each unit's device status word (read, and zeroed when set)
cudaError_t status_simt_exact(unsigned int* v);
cudaError_t status_simt_chunked(unsigned int* v);
cudaError_t status_step(unsigned int* v);
cudaError_t status_bwd(unsigned int* v);
cudaError_t status_tc(unsigned int* v);

}  // namespace lattice
