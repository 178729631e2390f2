// kg_factors.cu -- Kronecker factors of H = E[a a^T (x) b b^T] from samples, on the device.
//
// "FastKron", Section 3.2 and Appendix E.2: with a the input of the linear unit and b the gradient
// at its output, the Hessian is an expectation of Kronecker products, not itself one, and is
// approximated by A (x) B.  "WaterKron and FlipFlop Hessian", Table 1 and Section 5: three ways.
//   Marginal:   A = E[a a^T],  B = E[b b^T]                       (independence)
//   Frobenius:  alternating least squares on ||H - A (x) B||_F, from B = I:
//               A = E[(b^T B b) a a^T] / ||B||_F^2,  B = E[(a^T A a) b b^T] / ||A||_F^2
//   FlipFlop:   the same alternation with the reciprocal weighting, from B = I:
//               A = E[(b^T B^-1 b) a a^T] / m,       B = E[(a^T A^-1 a) b b^T] / n
// E is the mean over the N samples.  One iteration updates A, then B.
//
// Everything is fp64 and GEMM-shaped: a weighted Gram X^T diag(w) X is one GEMM of X with its
// row-scaled copy; the weights x_k^T M x_k are one GEMM (Y = X M) and a row-wise dot; for
// FlipFlop M^-1 = U^T U with U from kron_gptq_prepare (damping 0), so x_k^T M^-1 x_k = ||U x_k||^2.
// The GEMMs are the library's own DGEMM on the FP64 tensor path (kg_dgemm.cuh); the samples and
// every operand are kept zero-padded to multiples of 64 in the workspace, so the padding adds
// nothing to any product.
#include <algorithm>

#include "kg_common.cuh"
#include "kg_dgemm.cuh"
#include "kg_profile.cuh"

namespace kg {

static inline int64_t pad64(int64_t x) { return ceil_div(x, 64) * 64; }

// dst (rp x cp, zero padded) = src (rows x cols, row-major, any dtype promoted to fp64); with a
// status word, non-finite input is reported
template <typename T>
__global__ void k_fac_pad(const T* __restrict__ src, int64_t rows, int64_t cols, double* __restrict__ dst,
                          int64_t rp, int64_t cp, DevStatus* status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < rp * cp; p += stride) {
        const int64_t r = p / cp, c = p - r * cp;
        double v = 0.0;
        if (r < rows && c < cols) {
            v = (double)src[r * cols + c];
            if (status && !isfinite(v)) set_status(status, KG_ERR_NONFINITE, (int)std::min<int64_t>(r * cols + c, INT32_MAX));
        }
        dst[p] = v;
    }
}

// w_r = f * sum_j Y[r][j] X[r][j]  (squares == 0)  or  f * sum_j Y[r][j]^2  (squares == 1), with
// f = fh / *fd when fd is given, else fh.  One warp per row.
__global__ void k_fac_rowform(const double* __restrict__ Y, const double* __restrict__ X, int64_t N, int64_t k,
                              int squares, double fh, const double* __restrict__ fd, double* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < N; r += warps) {
        double acc = 0.0;
        for (int64_t j = lane; j < k; j += 32) {
            const double y = Y[r * k + j];
            acc += squares ? y * y : y * X[r * k + j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) w[r] = acc * (fd ? fh / *fd : fh);
    }
}

// Xw[r][j] = X[r][j] w_r
__global__ void k_fac_scale_rows(const double* __restrict__ X, const double* __restrict__ w, int64_t N, int64_t k,
                                 double* __restrict__ Xw) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < N * k; p += stride) Xw[p] = X[p] * w[p / k];
}

// out (k x k) = (G + G^T) / 2 on the leading block of the padded G (ld gp)
__global__ void k_fac_sym_out(const double* __restrict__ G, int64_t gp, double* __restrict__ out, int64_t k) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < k * k; p += stride) {
        const int64_t i = p / k, j = p - i * k;
        out[p] = 0.5 * (G[i * gp + j] + G[j * gp + i]);
    }
}

__global__ void k_fac_eye(double* __restrict__ M, int64_t k) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < k * k; p += stride)
        M[p] = (p / k == p % k) ? 1.0 : 0.0;
}

// *out = sum of squares of cnt entries (one block)
__global__ void __launch_bounds__(1024) k_fac_sumsq(const double* __restrict__ M, int64_t cnt, double* out) {
    __shared__ double part[32];
    double acc = 0.0;
    for (int64_t p = threadIdx.x; p < cnt; p += blockDim.x) acc += M[p] * M[p];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) *out = v;
    }
}

// the first error wins
__global__ void k_fac_merge_status(DevStatus* dst, const DevStatus* src) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && src->code != 0) set_status(dst, src->code, src->detail);
}

struct FacLayout {
    int64_t Np, np, mp, kp;
    size_t off_a, off_b, off_y, off_xw, off_w, off_u, off_upad, off_g, off_scal, off_prep, total;
};

static FacLayout fac_layout(int64_t N, int64_t n, int64_t m) {
    const int64_t k = std::max(n, m);
    FacLayout L{};
    L.Np = pad64(N); L.np = pad64(n); L.mp = pad64(m); L.kp = pad64(k);
    size_t off = kStatusBytes;
    auto take = [&](size_t& o, size_t bytes) { o = off; off = align_up(off + bytes, 256); };
    take(L.off_a, (size_t)(L.Np * L.np) * 8);
    take(L.off_b, (size_t)(L.Np * L.mp) * 8);
    take(L.off_y, (size_t)(L.Np * L.kp) * 8);
    take(L.off_xw, (size_t)(L.Np * L.kp) * 8);
    take(L.off_w, (size_t)L.Np * 8);
    take(L.off_u, (size_t)(k * k) * 8);
    take(L.off_upad, (size_t)(L.kp * L.kp) * 8);
    take(L.off_g, (size_t)(L.kp * L.kp) * 8);
    take(L.off_scal, 256);
    take(L.off_prep, kron_gptq_prepare_workspace_size(k));
    L.total = off;
    return L;
}

struct Fac {
    cudaStream_t st;
    DevStatus* status;
    double *y, *xw, *w, *u, *upad, *g, *scal;
    void* prep;
    size_t prep_bytes;
    int64_t N, Np;
};

static int grid_for(int64_t cnt) { return (int)std::max<int64_t>(1, std::min<int64_t>(148 * 4, ceil_div(cnt, 256))); }

// G (k x k) = X^T diag(w) X (the weights carry every constant), symmetrised; X is Np x px, zero padded.
static int fac_gram(const Fac& f, const double* X, int64_t px, int64_t k, double* G) {
    k_fac_scale_rows<<<grid_for(f.Np * px), 256, 0, f.st>>>(X, f.w, f.Np, px, f.xw);
    KG_LAUNCH_CHECK();
    if (!dgemm(f.st, DG_TRANS_A, (int)px, (int)px, (int)f.Np, 1.0, X, px, f.xw, px, 0.0, f.g, px)) return KG_ERR_CUDA;
    k_fac_sym_out<<<grid_for(k * k), 256, 0, f.st>>>(f.g, px, G, k);
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// w_r = fh / *fd * x_r^T M x_r with Y = X M (M k x k, padded into upad)
static int fac_form(const Fac& f, const double* X, int64_t px, int64_t k, const double* M, double fh, const double* fd) {
    k_fac_pad<double><<<grid_for(px * px), 256, 0, f.st>>>(M, k, k, f.upad, px, px, nullptr);
    KG_LAUNCH_CHECK();
    if (!dgemm(f.st, 0, (int)f.Np, (int)px, (int)px, 1.0, X, px, f.upad, px, 0.0, f.y, px)) return KG_ERR_CUDA;
    k_fac_rowform<<<grid_for(f.Np * 32), 256, 0, f.st>>>(f.y, X, f.Np, px, 0, fh, fd, f.w);
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// w_r = fh * x_r^T M^-1 x_r = fh * ||U x_r||^2 with U^T U = M^-1 (prepare, damping 0): Y = X U^T
static int fac_form_inv(const Fac& f, const double* X, int64_t px, int64_t k, const double* M, double fh) {
    int rc = kron_gptq_prepare(M, k, nullptr, 0, KG_F64, 0.0, f.u, nullptr, nullptr, nullptr, f.prep, f.prep_bytes, f.st);
    if (rc) return rc;
    k_fac_merge_status<<<1, 32, 0, f.st>>>(f.status, static_cast<const DevStatus*>(f.prep));
    KG_LAUNCH_CHECK();
    k_fac_pad<double><<<grid_for(px * px), 256, 0, f.st>>>(f.u, k, k, f.upad, px, px, nullptr);
    KG_LAUNCH_CHECK();
    if (!dgemm(f.st, DG_TRANS_B, (int)f.Np, (int)px, (int)px, 1.0, X, px, f.upad, px, 0.0, f.y, px)) return KG_ERR_CUDA;
    k_fac_rowform<<<grid_for(f.Np * 32), 256, 0, f.st>>>(f.y, X, f.Np, px, 1, fh, nullptr, f.w);
    KG_LAUNCH_CHECK();
    return KG_OK;
}

static int factors_impl(const void* a, const void* b, int64_t N, int64_t n, int64_t m, int dtype, int method, int iters,
                        double* A, double* B, void* ws, cudaStream_t st) {
    const FacLayout L = fac_layout(N, n, m);
    unsigned char* base = static_cast<unsigned char*>(ws);
    Fac f{};
    f.st = st;
    f.status = reinterpret_cast<DevStatus*>(base);
    f.y = reinterpret_cast<double*>(base + L.off_y);
    f.xw = reinterpret_cast<double*>(base + L.off_xw);
    f.w = reinterpret_cast<double*>(base + L.off_w);
    f.u = reinterpret_cast<double*>(base + L.off_u);
    f.upad = reinterpret_cast<double*>(base + L.off_upad);
    f.g = reinterpret_cast<double*>(base + L.off_g);
    f.scal = reinterpret_cast<double*>(base + L.off_scal);
    f.prep = base + L.off_prep;
    f.prep_bytes = L.total - L.off_prep;
    f.N = N;
    f.Np = L.Np;
    double* ad = reinterpret_cast<double*>(base + L.off_a);
    double* bd = reinterpret_cast<double*>(base + L.off_b);
    const int64_t np = L.np, mp = L.mp;
    KG_CUDA_TRY(cudaMemsetAsync(f.status, 0, kStatusBytes, st));
    if (dtype == KG_F64) {
        k_fac_pad<double><<<grid_for(L.Np * np), 256, 0, st>>>(static_cast<const double*>(a), N, n, ad, L.Np, np, f.status);
        k_fac_pad<double><<<grid_for(L.Np * mp), 256, 0, st>>>(static_cast<const double*>(b), N, m, bd, L.Np, mp, f.status);
    } else {
        k_fac_pad<float><<<grid_for(L.Np * np), 256, 0, st>>>(static_cast<const float*>(a), N, n, ad, L.Np, np, f.status);
        k_fac_pad<float><<<grid_for(L.Np * mp), 256, 0, st>>>(static_cast<const float*>(b), N, m, bd, L.Np, mp, f.status);
    }
    KG_LAUNCH_CHECK();
    const double invN = 1.0 / (double)N;
    int rc;
    for (int it = 0; it < (method == KG_FACTOR_MARGINAL ? 1 : iters); ++it) {
        if (method == KG_FACTOR_MARGINAL) {
            if (!dgemm(st, DG_TRANS_A, (int)np, (int)np, (int)L.Np, invN, ad, np, ad, np, 0.0, f.g, np)) return KG_ERR_CUDA;
            k_fac_sym_out<<<grid_for(n * n), 256, 0, st>>>(f.g, np, A, n);
            KG_LAUNCH_CHECK();
            if (!dgemm(st, DG_TRANS_A, (int)mp, (int)mp, (int)L.Np, invN, bd, mp, bd, mp, 0.0, f.g, mp)) return KG_ERR_CUDA;
            k_fac_sym_out<<<grid_for(m * m), 256, 0, st>>>(f.g, mp, B, m);
            KG_LAUNCH_CHECK();
            break;
        }
        if (it == 0) {
            k_fac_eye<<<grid_for(m * m), 256, 0, st>>>(B, m);
            KG_LAUNCH_CHECK();
        }
        if (method == KG_FACTOR_FROBENIUS) {
            k_fac_sumsq<<<1, 1024, 0, st>>>(B, m * m, f.scal);
            KG_LAUNCH_CHECK();
            if ((rc = fac_form(f, bd, mp, m, B, invN, f.scal))) return rc;
            if ((rc = fac_gram(f, ad, np, n, A))) return rc;
            k_fac_sumsq<<<1, 1024, 0, st>>>(A, n * n, f.scal + 1);
            KG_LAUNCH_CHECK();
            if ((rc = fac_form(f, ad, np, n, A, invN, f.scal + 1))) return rc;
            if ((rc = fac_gram(f, bd, mp, m, B))) return rc;
        } else {
            if ((rc = fac_form_inv(f, bd, mp, m, B, invN / (double)m))) return rc;
            if ((rc = fac_gram(f, ad, np, n, A))) return rc;
            if ((rc = fac_form_inv(f, ad, np, n, A, invN / (double)n))) return rc;
            if ((rc = fac_gram(f, bd, mp, m, B))) return rc;
        }
    }
    return KG_OK;
}

}  // namespace kg

using namespace kg;

extern "C" size_t kron_gptq_factors_workspace_size(int64_t N, int64_t n, int64_t m) {
    if (N < 1 || n < 1 || m < 1) return 0;
    return fac_layout(N, n, m).total;
}

extern "C" int kron_gptq_factors(const void* a, const void* b, int64_t N, int64_t n, int64_t m, int dtype, int method,
                                 int iters, double* A, double* B, void* ws, size_t ws_bytes, void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (method != KG_FACTOR_MARGINAL && method != KG_FACTOR_FROBENIUS && method != KG_FACTOR_FLIPFLOP)
        return KG_ERR_UNSUPPORTED;
    if (N < 1 || n < 1 || m < 1 || iters < 1 || !a || !b || !A || !B) return KG_ERR_ARG;
    if (n > (int64_t)1 << 17 || m > (int64_t)1 << 17 || N > (int64_t)INT32_MAX) return KG_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (ws_bytes < fac_layout(N, n, m).total) return KG_ERR_WORKSPACE;
    return factors_impl(a, b, N, n, m, dtype, method, iters, A, B, ws, static_cast<cudaStream_t>(stream));
}
