// kg_profile.cuh -- launch counters and optional CUDA-event timing per kernel kind.
//
// Every launch the library makes is counted by kind.  When profiling is enabled, each
// counted launch is bracketed by a pair of CUDA events recorded on the launch's own stream;
// kron_gptq_profile_read() waits for them and accumulates the elapsed time per kind.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kg {

enum ProfKind : int {
    PK_INIT = 0,     // workspace initialisation, padding, validation
    PK_LEAF = 1,     // in-tile anti-diagonal sweeps
    PK_PUSH = 2,     // trailing band updates (row and column chains)
    PK_PREPARE = 3,  // factor preparation kernels
    PK_LOSS = 4,     // loss and scale kernels
    PK_SOLVE = 5,    // reserved: no launch of this kind
    PK_COUNT = 8
};

// Host-side profiler state (defined in kg_profile.cu).
void prof_before(int kind, cudaStream_t st);
void prof_after(int kind, cudaStream_t st);
bool prof_timing();                          // event timing on (kron_gptq_profile_enable)
void prof_counts(int64_t out[PK_COUNT]);     // launches counted so far, per kind
void prof_add(const int64_t add[PK_COUNT]);  // count launches made by a graph replay

struct ProfScope {
    int kind;
    cudaStream_t st;
    ProfScope(int k, cudaStream_t s) : kind(k), st(s) { prof_before(k, s); }
    ~ProfScope() { prof_after(kind, st); }
};

// Launch statement wrapped in a profiling scope of the given kind.
#define KG_PROF(kind, st, ...)                      \
    do {                                           \
        ::kg::ProfScope _kg_ps((kind), (st));      \
        __VA_ARGS__;                               \
    } while (0)

}  // namespace kg
