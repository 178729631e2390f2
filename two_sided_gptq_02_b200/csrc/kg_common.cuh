// kg_common.cuh -- internal helpers shared by the CUDA sources of the kron_gptq library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kron_gptq.h"

namespace kg {

// Tile edge of the anti-diagonal sweep and of the trailing-update GEMMs.  W is cut into
// KG_T x KG_T tiles; tiles on one tile anti-diagonal (I + J = D) are mutually independent
// because none lies to the top-left of another ("FastKron", Section 2.3).
constexpr int KG_T = 64;

// The device status word lives at the start of every workspace.
struct DevStatus {
    int code;        // KG_OK or a negative kg_status
    int detail;      // first offending index (row*cols+col or pivot), for diagnostics
    int pad[62];
};
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void set_status(DevStatus* st, int code, int detail) {
    // the first error wins; later ones keep the earlier diagnostics
    if (atomicCAS(&st->code, 0, code) == 0) st->detail = detail;
}

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

#define KG_CUDA_TRY(expr)                                   \
    do {                                                    \
        cudaError_t _e = (expr);                            \
        if (_e != cudaSuccess) return KG_ERR_CUDA;          \
    } while (0)

#define KG_LAUNCH_CHECK()                                   \
    do {                                                    \
        cudaError_t _e = cudaGetLastError();                \
        if (_e != cudaSuccess) return KG_ERR_CUDA;          \
    } while (0)

template <typename T>
struct Vec2;
template <>
struct Vec2<float> { using type = float2; };
template <>
struct Vec2<double> { using type = double2; };

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization may
// start while the previous kernel of its stream is still running: it must call grid_dep_wait()
// before touching anything that kernel writes (the wait returns once it has completed and its
// memory is visible; without the launch attribute it returns at once).  grid_dep_launch() lets the
// next kernel of the stream start launching early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace kg
