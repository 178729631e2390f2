// kg_entropy.cu -- empirical entropy of integer codes: the memory cost of Z under a good entropy
// coder ("WaterKron and FlipFlop Hessian", Section 2.1: the integers are unbounded and entropy
// coded, so their cost is the entropy of their distribution).  Plug-in estimate in bits per entry:
//     H = -sum_z (c_z / N) log2(c_z / N) = log2 N - (1/N) sum_z c_z log2 c_z,
// with c_z the number of entries equal to z.
//
// Four launches on the caller's stream: the range [zmin, zmax] of the codes; zero that many bins;
// the histogram (per-block in shared memory when the range is small, else atomics on the global
// bins); one block sums c log2 c in fp64.  A range wider than the workspace's bins is reported as
// KG_ERR_RANGE and the result is NaN.
#include <limits.h>
#include <math.h>

#include "kg_common.cuh"

namespace kg {

struct EntHdr {
    int zmin, zmax;
};
constexpr size_t kEntHdrBytes = 256;
constexpr int kEntSmemBins = 8192;
constexpr int kEntThreads = 256;

__global__ void k_ent_init(EntHdr* h) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        h->zmin = INT_MAX;
        h->zmax = INT_MIN;
    }
}

__global__ void k_ent_range(const int32_t* __restrict__ Z, int64_t N, EntHdr* h) {
    int lo = INT_MAX, hi = INT_MIN;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < N; p += stride) {
        const int z = Z[p];
        lo = min(lo, z);
        hi = max(hi, z);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMin(&h->zmin, lo);
        atomicMax(&h->zmax, hi);
    }
}

__device__ __forceinline__ int64_t ent_bins(const EntHdr* h) { return (int64_t)h->zmax - (int64_t)h->zmin + 1; }

__global__ void k_ent_zero(const EntHdr* h, uint32_t* __restrict__ bins, int64_t cap) {
    const int64_t nb = min(ent_bins(h), cap);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) bins[b] = 0u;
}

__global__ void __launch_bounds__(kEntThreads) k_ent_hist(const int32_t* __restrict__ Z, int64_t N, const EntHdr* h,
                                                          uint32_t* __restrict__ bins, int64_t cap, DevStatus* status) {
    __shared__ uint32_t sh[kEntSmemBins];
    const int64_t nb = ent_bins(h);
    if (nb > cap) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, KG_ERR_RANGE, 0);
        return;
    }
    const int zmin = h->zmin;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t p0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (nb <= kEntSmemBins) {
        for (int b = threadIdx.x; b < nb; b += blockDim.x) sh[b] = 0u;
        __syncthreads();
        for (int64_t p = p0; p < N; p += stride) atomicAdd(&sh[Z[p] - zmin], 1u);
        __syncthreads();
        for (int b = threadIdx.x; b < nb; b += blockDim.x)
            if (sh[b]) atomicAdd(&bins[b], sh[b]);
    } else {
        for (int64_t p = p0; p < N; p += stride) atomicAdd(&bins[(int64_t)Z[p] - zmin], 1u);
    }
}

__global__ void __launch_bounds__(1024) k_ent_sum(const EntHdr* h, const uint32_t* __restrict__ bins, int64_t cap,
                                                  int64_t N, double* out) {
    __shared__ double part[32];
    const int64_t nb = ent_bins(h);
    if (nb > cap) {
        if (threadIdx.x == 0) *out = NAN;
        return;
    }
    double acc = 0.0;
    for (int64_t b = threadIdx.x; b < nb; b += blockDim.x) {
        const double c = (double)bins[b];
        if (c > 0.0) acc += c * log2(c);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) *out = log2((double)N) - v / (double)N;
    }
}

}  // namespace kg

using namespace kg;

extern "C" size_t kron_gptq_code_entropy_workspace_size(int64_t max_bins) {
    if (max_bins < 1) max_bins = 1;
    return kStatusBytes + kEntHdrBytes + align_up((size_t)max_bins * sizeof(uint32_t), 256);
}

extern "C" int kron_gptq_code_entropy(const int32_t* Z, int64_t count, double* out_bits, void* ws, size_t ws_bytes,
                                      void* stream) {
    if (count < 0 || !out_bits) return KG_ERR_ARG;
    if (count >= ((int64_t)1 << 32)) return KG_ERR_UNSUPPORTED;   // 32-bit bin counters
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (ws_bytes < kron_gptq_code_entropy_workspace_size(1)) return KG_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* base = static_cast<unsigned char*>(ws);
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    KG_CUDA_TRY(cudaMemsetAsync(status, 0, kStatusBytes, st));
    if (count == 0) {
        KG_CUDA_TRY(cudaMemsetAsync(out_bits, 0, sizeof(double), st));
        return KG_OK;
    }
    if (!Z) return KG_ERR_ARG;
    EntHdr* h = reinterpret_cast<EntHdr*>(base + kStatusBytes);
    uint32_t* bins = reinterpret_cast<uint32_t*>(base + kStatusBytes + kEntHdrBytes);
    const int64_t cap = (int64_t)((ws_bytes - kStatusBytes - kEntHdrBytes) / sizeof(uint32_t));
    const int nb = 148 * 8;
    k_ent_init<<<1, 32, 0, st>>>(h);
    KG_LAUNCH_CHECK();
    k_ent_range<<<nb, kEntThreads, 0, st>>>(Z, count, h);
    KG_LAUNCH_CHECK();
    k_ent_zero<<<nb, kEntThreads, 0, st>>>(h, bins, cap);
    KG_LAUNCH_CHECK();
    k_ent_hist<<<nb, kEntThreads, 0, st>>>(Z, count, h, bins, cap, status);
    KG_LAUNCH_CHECK();
    k_ent_sum<<<1, 1024, 0, st>>>(h, bins, cap, count, out_bits);
    KG_LAUNCH_CHECK();
    return KG_OK;
}
