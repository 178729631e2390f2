// kg_blas.cuh -- the library's cuBLAS handle: one per host thread and device, created on the
// first call that needs a plain dense GEMM and kept for the life of the process.  Callers set the
// stream and hand cuBLAS a workspace slice before every use.  Handles are never destroyed: a
// destructor at thread or process exit could run after the CUDA runtime has shut down, so the
// handle of a thread that exits stays allocated.  Callers that spawn many short-lived threads
// should make these calls from a long-lived one.
#pragma once

#include <cublas_v2.h>

#include <vector>

#include "kg_common.cuh"

namespace kg {

inline int blas_handle(cublasHandle_t* out) {
    struct Entry {
        int dev;
        cublasHandle_t h;
    };
    static thread_local std::vector<Entry> handles;
    int dev = 0;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    for (auto& e : handles)
        if (e.dev == dev) {
            *out = e.h;
            return KG_OK;
        }
    cublasHandle_t h = nullptr;
    if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return KG_ERR_CUDA;
    handles.push_back({dev, h});
    *out = h;
    return KG_OK;
}

// stream and workspace for the next calls on handle h
inline int blas_bind(cublasHandle_t h, cudaStream_t st, void* ws, size_t bytes) {
    if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return KG_ERR_CUDA;
    if (cublasSetWorkspace(h, ws, bytes) != CUBLAS_STATUS_SUCCESS) return KG_ERR_CUDA;
    return KG_OK;
}

}  // namespace kg
