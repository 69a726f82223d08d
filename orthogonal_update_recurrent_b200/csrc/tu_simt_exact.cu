// tu_simt_exact.cu -- launches of the exact recurrence on CUDA cores (scan_simt.cuh).
#include "simt_launch.cuh"

namespace lattice {

lattice_status launch_scan_simt_exact(const ScanArgs& a, int d, bool dec, cudaStream_t st) {
    return dec ? launch_scan_simt_m<false, true, false>(a, d, st) : launch_scan_simt_m<false, false, false>(a, d, st);
}

cudaError_t status_simt_exact(unsigned int* v) { return read_clear_module_status(v); }

}  // namespace lattice
