// args.h -- kernel argument blocks and the size rules the host needs, with no device
// code, so that the C ABI's translation unit can build them without compiling any
// kernel. Each kernel family's header includes this file.
#pragma once
#include <stddef.h>

#if defined(__CUDACC__)
#define LATTICE_HD __host__ __device__
#else
#define LATTICE_HD
#endif

namespace lattice {

constexpr int kMaxM = 256;  // most slots per head on every path

// scan_simt.cuh, chunk_tc.cuh, chunk_split.cuh, chunk_reg.cuh
struct ScanArgs {
    const void* x; bool x_bf16;
    const float* c;
    const void* q; bool q_bf16;
    const float* mu;
    const float* eta;            // may be null (=> 1)
    const float* S0;
    float* S_out;
    float* y;
    int B, T, H, m, chunk;
    int cnorm;  // chunked CUDA-core path: no per-token normaliser, unit slots after each chunk
    int G;      // SPLIT kernels: CTAs per sequence (a cluster), each owning spc slots
    int spc;
};

// step.cuh: decode step
struct StepArgs {
    float* S;
    const void* x; bool x_bf16;
    const float* c;
    const void* q; bool q_bf16;
    const float* mu;
    const float* eta;  // may be null
    float* y;
    int B, H, m;
};

// step.cuh: read-out of a given state
struct ReadoutArgs {
    const float* S;
    const void* q; bool q_bf16;
    float* y;
    int B, H, m;
};

// scan_bwd.cuh: backward pass
struct BwdArgs {
    const void* x; bool x_bf16;
    const float* c;
    const void* q; bool q_bf16;
    const float* mu;
    const float* eta;  // may be null (=> 1)
    const float* S0;
    const float* dy;
    const float* dST;  // may be null (=> 0)
    float* dx; float* dc; float* dq; float* dmu;
    float* deta;       // may be null
    float* dS0;
    float* ws;         // workspace: per (b,h) and CTA, (nseg - 1) checkpoints then the L-token tape
    int B, T, H, m, chunk, seg;
    int G;             // CTAs per sequence (a cluster when > 1)
    int spc;           // slots per CTA
};

// Floats of backward workspace per (b,h) sequence and CTA (m: the CTA's slots).
LATTICE_HD inline size_t bwd_ws_floats_per_seq(int T, int m, int D, int seg) {
    const int nseg = T > 0 ? (T + seg - 1) / seg : 1;
    return (size_t)(nseg - 1 + seg) * m * D;
}

// Chunk-parallel backward (chunk_bwd.cuh): 16 slots per CTA, 512 threads, chunks of
// 2..64 tokens, a sequence's slots on a cluster of ceil(m/16) <= 8 CTAs.
constexpr int kCbSlots = 16;
constexpr int kCbThreads = 512;
constexpr int kCbMaxL = 64;
constexpr int kCbMaxG = 8;

inline bool chunk_bwd_supported(int m, int d, int chunk) {
    return chunk >= 2 && chunk <= kCbMaxL && (d == 32 || d == 64 || d == 128) && m >= 1 &&
           m <= kCbMaxG * kCbSlots;
}
inline int chunk_bwd_ctas(int m) { return (m + kCbSlots - 1) / kCbSlots; }
// Workspace floats of the chunk-parallel backward: each CTA's slots of every chunk-start state.
inline size_t chunk_bwd_ws_floats(int B, int T, int H, int m, int D, int chunk) {
    const size_t nc = T > 0 ? (size_t)((T + chunk - 1) / chunk) : 0;
    return (size_t)B * H * chunk_bwd_ctas(m) * nc * kCbSlots * D;
}

}  // namespace lattice
