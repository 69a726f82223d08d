// tu_simt_chunked.cu -- launches of the chunked form on CUDA cores (scan_simt.cuh),
// either linearisation, either objective.
#include "simt_launch.cuh"

namespace lattice {

lattice_status launch_scan_simt_chunked(const ScanArgs& a, int d, bool dec, bool lin1, cudaStream_t st) {
    if (lin1)
        return dec ? launch_scan_simt_m<true, true, true>(a, d, st) : launch_scan_simt_m<true, false, true>(a, d, st);
    return dec ? launch_scan_simt_m<true, true, false>(a, d, st) : launch_scan_simt_m<true, false, false>(a, d, st);
}

cudaError_t status_simt_chunked(unsigned int* v) { return read_clear_module_status(v); }

}  // namespace lattice
