// kg_dgemm.cuh -- general fp64 GEMM on the FP64 tensor path of sm_100a (mma.sync m8n8k4 f64
// through DmmaPipe), for the library's own dense products in fp64: the recursive Cholesky and
// triangular inverse of the factors, the Kronecker factor estimators and the one-sided solve.
//
//     C (M x N) = alpha * op(A) op(B) + beta * C        all matrices row-major
//
// op(A) is M x K: A itself (lda >= K) or, with DG_TRANS_A, the transpose of a K x M matrix A.
// op(B) is K x N: B itself or, with DG_TRANS_B, the transpose of an N x K matrix B.  M, N, K are
// multiples of 64 (callers pad), leading dimensions and base pointers keep 16-byte alignment.
// One CTA of 128 threads computes one 64 x 64 tile of C; the K loop is double-buffered with
// cp.async (DmmaPipe).  Triangular operands skip the 64-tiles of K where they are zero:
//   DG_A_LOWER   op(A)(i, k) = 0 for k > i      (K tiles  <= tile row of C)
//   DG_B_LOWER   op(B)(k, j) = 0 for k < j      (K tiles  >= tile column of C)
//   DG_B_UPPER   op(B)(k, j) = 0 for k > j      (K tiles  <= tile column of C)
//   DG_C_LOWER   only the tiles of C on or below the diagonal are computed (a symmetric update)
// beta == 0 does not read C.
#pragma once

#include "kg_common.cuh"
#include "kg_gemm.cuh"

namespace kg {

enum DgemmFlags {
    DG_TRANS_A = 1,
    DG_TRANS_B = 2,
    DG_A_LOWER = 4,
    DG_B_LOWER = 8,
    DG_B_UPPER = 16,
    DG_C_LOWER = 32,
};

template <bool TA, bool TB>
__global__ void __launch_bounds__(Dmma64::kThreads)
k_dgemm(int M, int N, int K, double alpha, const double* __restrict__ A, int64_t lda, const double* __restrict__ B,
        int64_t ldb, double beta, double* __restrict__ C, int64_t ldc, int flags) {
    using Pipe = DmmaPipe<TA, TB>;
    __shared__ typename Pipe::Smem sm;
    const int bj = blockIdx.x, bi = blockIdx.y;
    if ((flags & DG_C_LOWER) && bj > bi) return;
    int klo = 0, khi = K / 64;
    if (flags & DG_A_LOWER) khi = min(khi, bi + 1);
    if (flags & DG_B_UPPER) khi = min(khi, bj + 1);
    if (flags & DG_B_LOWER) klo = max(klo, bj);
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    if (klo < khi) {
        const int64_t i0 = (int64_t)bi * 64, j0 = (int64_t)bj * 64, k0 = (int64_t)klo * 64;
        const double* a = TA ? A + k0 * lda + i0 : A + i0 * lda + k0;
        const double* b = TB ? B + j0 * ldb + k0 : B + k0 * ldb + j0;
        Pipe::run(acc, sm, (khi - klo) * 64, a, lda, b, ldb);
    }
    double* c = C + (int64_t)bi * 64 * ldc + (int64_t)bj * 64;
    if (beta == 0.0) {
        Dmma64::for_each(acc, [&](int r, int cc, double v) { c[(int64_t)r * ldc + cc] = alpha * v; });
    } else {
        Dmma64::for_each(acc, [&](int r, int cc, double v) {
            double* p = c + (int64_t)r * ldc + cc;
            *p = alpha * v + beta * *p;
        });
    }
}

// Host launcher: returns false for shapes the kernel does not take (not multiples of 64).
static inline bool dgemm(cudaStream_t st, int flags, int M, int N, int K, double alpha, const double* A, int64_t lda,
                         const double* B, int64_t ldb, double beta, double* C, int64_t ldc) {
    if (M <= 0 || N <= 0) return true;
    if ((M | N | K) & 63) return false;
    const dim3 grid(N / 64, M / 64);
    const bool ta = flags & DG_TRANS_A, tb = flags & DG_TRANS_B;
    if (!ta && !tb)
        k_dgemm<false, false><<<grid, Dmma64::kThreads, 0, st>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else if (!ta && tb)
        k_dgemm<false, true><<<grid, Dmma64::kThreads, 0, st>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else if (ta && !tb)
        k_dgemm<true, false><<<grid, Dmma64::kThreads, 0, st>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else
        k_dgemm<true, true><<<grid, Dmma64::kThreads, 0, st>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace kg
