// kg_loss.cu -- proxy loss, per-row scales and the small C-ABI utilities.
//
// Loss ("FastKron: Efficient Quantization with Kronecker-Factored Hessians", Section 2.2):
//     D_{A,B} = || B^{1/2} (V - W) A^{1/2} ||_F^2 = tr(D A_d D^T B_d),   D = V - W,
//             = sum_{i,j} (D A_d)_{ij} (B_d D)_{ij}.
// One 64x64 tile of P = D A_d and of Q = B_d D per block (fp64 tensor path), the elementwise
// product summed per block, then a fixed-order sum of the block partials.
#include <algorithm>

#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_profile.cuh"

namespace kg {

template <typename In>
__global__ void k_mean_diag2(const In* __restrict__ A, int64_t n, const In* __restrict__ B, int64_t m,
                             double* out) {
    __shared__ double red[2][256];
    double sa = 0.0, sb = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += 256) sa += (double)A[i * n + i];
    for (int64_t i = threadIdx.x; i < m; i += 256) sb += (double)B[i * m + i];
    red[0][threadIdx.x] = sa;
    red[1][threadIdx.x] = sb;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) {
            red[0][threadIdx.x] += red[0][threadIdx.x + w];
            red[1][threadIdx.x] += red[1][threadIdx.x + w];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[0] = red[0][0] / (double)n;
        out[1] = red[1][0] / (double)m;
    }
}

template <typename Real, typename Fac>
__global__ void __launch_bounds__(Dmma64::kThreads)
k_loss_tiles(const Real* __restrict__ W, const Real* __restrict__ V, int64_t m, int64_t n,
             const Fac* __restrict__ A, const Fac* __restrict__ B, const double* __restrict__ meanAB, double damp,
             double* __restrict__ partial) {
    __shared__ Dmma64::Smem sm;
    __shared__ double red[Dmma64::kThreads];
    const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
    const int tid = threadIdx.x;
    auto Dv = [&](int64_t i, int64_t j) -> double {
        return (i < m && j < n) ? (double)V[i * n + j] - (double)W[i * n + j] : 0.0;
    };
    // P tile = D[r0:, :] A[:, c0:]
    Dmma64::Acc accP, acc;
    Dmma64::zero(accP);
    const int Kn = (int)ceil_div(n, Dmma64::BK) * Dmma64::BK;
    auto la1 = [&](int k0, double (*As)[Dmma64::SA]) {
        for (int idx = tid; idx < 64 * Dmma64::BK; idx += Dmma64::kThreads) {
            const int r = idx / Dmma64::BK, k = idx % Dmma64::BK;
            As[r][k] = Dv(r0 + r, k0 + k);
        }
    };
    auto lb1 = [&](int k0, double (*Bs)[Dmma64::SB]) {
        for (int idx = tid; idx < Dmma64::BK * 64; idx += Dmma64::kThreads) {
            const int k = idx / 64, c = idx % 64;
            const int64_t kk = k0 + k, cc = c0 + c;
            Bs[k][c] = (kk < n && cc < n) ? (double)A[kk * n + cc] : 0.0;
        }
    };
    Dmma64::run(accP, sm, Kn, la1, lb1);
    // Q tile = B[r0:, :] D[:, c0:]
    Dmma64::zero(acc);
    const int Km = (int)ceil_div(m, Dmma64::BK) * Dmma64::BK;
    auto la2 = [&](int k0, double (*As)[Dmma64::SA]) {
        for (int idx = tid; idx < 64 * Dmma64::BK; idx += Dmma64::kThreads) {
            const int r = idx / Dmma64::BK, k = idx % Dmma64::BK;
            const int64_t rr = r0 + r, kk = k0 + k;
            As[r][k] = (rr < m && kk < m) ? (double)B[rr * m + kk] : 0.0;
        }
    };
    auto lb2 = [&](int k0, double (*Bs)[Dmma64::SB]) {
        for (int idx = tid; idx < Dmma64::BK * 64; idx += Dmma64::kThreads) {
            const int k = idx / 64, c = idx % 64;
            Bs[k][c] = Dv(k0 + k, c0 + c);
        }
    };
    Dmma64::run(acc, sm, Km, la2, lb2);
    __syncthreads();
    const double dA = damp * meanAB[0], dB = damp * meanAB[1];
    double s = 0.0;
    dmma_for_each2(accP, acc, [&](int r, int c, double p, double q) {
        const double d = Dv(r0 + r, c0 + c);
        s += (p + dA * d) * (q + dB * d);
    });
    red[tid] = s;
    __syncthreads();
    for (int w = Dmma64::kThreads / 2; w > 0; w >>= 1) {
        if (tid < w) red[tid] += red[tid + w];
        __syncthreads();
    }
    if (tid == 0) partial[blockIdx.y * gridDim.x + blockIdx.x] = red[0];
}

__global__ void k_sum_partials(const double* __restrict__ partial, int64_t count, double* out) {
    __shared__ double red[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < count; i += 256) s += partial[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0];
}

template <typename Real>
__global__ void k_row_scales(const Real* __restrict__ W, int64_t m, int64_t n, int qmax, Real* __restrict__ s) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int64_t i = warp; i < m; i += nwarps) {
        Real mx = Real(0);
        for (int64_t j = lane; j < n; j += 32) mx = fmax(mx, fabs(W[i * n + j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s[i] = (mx > Real(0)) ? mx / Real(qmax) : Real(1);
    }
}

template <typename Real, typename Fac>
static int loss_impl(const Real* W, const Real* V, int64_t m, int64_t n, const Fac* A, const Fac* B, double damp,
                     double* out, unsigned char* base, cudaStream_t st) {
    double* meanAB = reinterpret_cast<double*>(base + kStatusBytes);
    double* partial = reinterpret_cast<double*>(base + kStatusBytes + 256);
    const int64_t gx = ceil_div(n, 64), gy = ceil_div(m, 64);
    KG_PROF(PK_LOSS, st, k_mean_diag2<Fac><<<1, 256, 0, st>>>(A, n, B, m, meanAB));
    KG_LAUNCH_CHECK();
    KG_PROF(PK_LOSS, st, k_loss_tiles<Real, Fac><<<dim3((unsigned)gx, (unsigned)gy), Dmma64::kThreads, 0, st>>>(W, V, m, n, A, B, meanAB, damp, partial));
    KG_LAUNCH_CHECK();
    KG_PROF(PK_LOSS, st, k_sum_partials<<<1, 256, 0, st>>>(partial, gx * gy, out));
    KG_LAUNCH_CHECK();
    return KG_OK;
}

}  // namespace kg

using namespace kg;

extern "C" int kron_gptq_version(void) { return 10000; }

extern "C" const char* kron_gptq_status_string(int status) {
    switch (status) {
        case KG_OK: return "ok";
        case KG_ERR_ARG: return "invalid argument";
        case KG_ERR_UNSUPPORTED: return "unsupported dtype or grid";
        case KG_ERR_CUDA: return "CUDA runtime error";
        case KG_ERR_WORKSPACE: return "workspace too small";
        case KG_ERR_NOT_PD: return "factor is not positive definite";
        case KG_ERR_NONFINITE: return "non-finite or non-positive input";
        case KG_ERR_TIMEOUT: return "device wait timed out";
        case KG_ERR_RANGE: return "code out of the representable range";
        default: return "unknown status";
    }
}

extern "C" int kron_gptq_sync_status(const void* ws, void* stream) {
    if (!ws) return KG_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int code = 0;
    if (cudaMemcpyAsync(&code, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return KG_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KG_ERR_CUDA;
    return code;
}

extern "C" size_t kron_gptq_loss_workspace_size(int64_t m, int64_t n) {
    if (m <= 0 || n <= 0) return kStatusBytes + 512;
    return kStatusBytes + 256 + align_up((size_t)(ceil_div(m, 64) * ceil_div(n, 64)) * 8, 256);
}

extern "C" int kron_gptq_loss(const void* W, const void* V, int64_t m, int64_t n, int dtype, const void* A,
                              const void* B, int fac_dtype, double damp, double* out_loss, void* ws, size_t ws_bytes,
                              void* stream) {
    if ((dtype != KG_F32 && dtype != KG_F64) || (fac_dtype != KG_F32 && fac_dtype != KG_F64)) return KG_ERR_UNSUPPORTED;
    if (m < 1 || n < 1 || !W || !V || !A || !B || !out_loss || !(damp >= 0.0)) return KG_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (ws_bytes < kron_gptq_loss_workspace_size(m, n)) return KG_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* base = static_cast<unsigned char*>(ws);
    KG_CUDA_TRY(cudaMemsetAsync(base, 0, kStatusBytes, st));
    if (dtype == KG_F64) {
        if (fac_dtype == KG_F64)
            return loss_impl<double, double>((const double*)W, (const double*)V, m, n, (const double*)A,
                                             (const double*)B, damp, out_loss, base, st);
        return loss_impl<double, float>((const double*)W, (const double*)V, m, n, (const float*)A, (const float*)B,
                                        damp, out_loss, base, st);
    }
    if (fac_dtype == KG_F64)
        return loss_impl<float, double>((const float*)W, (const float*)V, m, n, (const double*)A, (const double*)B,
                                        damp, out_loss, base, st);
    return loss_impl<float, float>((const float*)W, (const float*)V, m, n, (const float*)A, (const float*)B, damp,
                                   out_loss, base, st);
}

extern "C" int kron_gptq_row_scales(const void* W, int64_t m, int64_t n, int dtype, int qmax, void* out_scale,
                                    void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (m < 0 || n < 0 || qmax <= 0) return KG_ERR_ARG;
    if (m == 0) return KG_OK;
    if (!W || !out_scale) return KG_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int blocks = (int)std::min<int64_t>(148 * 8, ceil_div(m, 8));
    if (dtype == KG_F64)
        KG_PROF(PK_LOSS, st, k_row_scales<double><<<blocks, 256, 0, st>>>((const double*)W, m, n, qmax, (double*)out_scale));
    else
        KG_PROF(PK_LOSS, st, k_row_scales<float><<<blocks, 256, 0, st>>>((const float*)W, m, n, qmax, (float*)out_scale));
    KG_LAUNCH_CHECK();
    return KG_OK;
}
