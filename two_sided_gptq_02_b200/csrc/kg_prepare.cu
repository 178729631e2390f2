// kg_prepare.cu -- factors of the two-sided GPTQ solver (fp64).
//
// For a symmetric positive definite factor A (k x k):
//     A_d = A + damp * mean(diag A) * I          ("WaterKron ...", Section 2, Notation)
//     U   = upper triangular with U^T U = A_d^{-1}
// U is RevCholesky(A_d)^{-T} (same Notation paragraph).  With P the index reversal,
// P A_d P = L' L'^T (ordinary lower Cholesky), hence A_d = (P L' P)(P L' P)^T with P L' P
// upper, and U = (P L' P)^{-1} = P L'^{-1} P.  So the GPU computes
//     1. M  = P A_d P                      (copy with reversal and damping, padded to 64)
//     2. L' = Cholesky(M), X = L'^{-1}     (one recursion that halves the block range: factor
//                                           and invert the leading half, update and factor
//                                           the trailing half, then the off-diagonal block of
//                                           the inverse; 64 x 64 leaves in one CTA)
//     3. U[i][j] = X[k-1-i][k-1-j]         (reversal back; strictly lower part zero)
// The Cholesky and the triangular inverse ("FastKron", Section 2.6: inverse and Cholesky as a
// separate O(n^3) step) instead of the three steps of "Cholesky, inverse, Cholesky of the
// inverse"; the result is the same unique factor.  The recursion's sequential depth is the 64
// leaves; every product between them is one DGEMM on the FP64 tensor path (mma.sync m8n8k4 f64,
// kg_dgemm.cuh) over whole half-blocks.
#include <algorithm>
#include <vector>

#include "kg_common.cuh"
#include "kg_dgemm.cuh"
#include "kg_gemm.cuh"
#include "kg_profile.cuh"

namespace kg {

constexpr int NB = 64;

struct PLayout {
    int64_t k, kp, Kb;
    size_t off_scal, off_M, off_X, off_T, total;
};

static PLayout p_layout(int64_t k) {
    PLayout L{};
    L.k = k;
    L.Kb = ceil_div(k, NB);
    L.kp = L.Kb * NB;
    size_t off = kStatusBytes;
    L.off_scal = off; off += 256;
    L.off_M = off;    off = align_up(off + (size_t)(L.kp * L.kp) * 8, 256);
    L.off_X = off;    off = align_up(off + (size_t)(L.kp * L.kp) * 8, 256);
    L.off_T = off;    off = align_up(off + (size_t)(L.kp * L.kp) * 8, 256);
    L.total = off;
    return L;
}

// mean of the diagonal, accumulated in fp64 by one block
template <typename In>
__global__ void k_diag_mean(const In* __restrict__ A, int64_t k, double* out, DevStatus* st) {
    __shared__ double red[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < k; i += 256) s += (double)A[i * k + i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double mval = red[0] / (double)k;
        if (!isfinite(mval)) set_status(st, KG_ERR_NONFINITE, -1);
        *out = mval;
    }
}

// M[i][j] = A_d[k-1-i][k-1-j] for i,j < k (lower triangle source), identity in the pad
template <typename In>
__global__ void k_build_reversed(const In* __restrict__ A, int64_t k, int64_t kp, const double* __restrict__ mean,
                                 double damp, double* __restrict__ M, DevStatus* st) {
    const double dval = damp * (*mean);
    const int64_t total = kp * kp;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = p / kp, j = p % kp;
        double v;
        if (i < k && j < k) {
            const int64_t oi = k - 1 - i, oj = k - 1 - j;
            // read the lower triangle of A and mirror it
            const int64_t a = oi > oj ? oi : oj, b = oi > oj ? oj : oi;
            v = (double)A[a * k + b];
            if (!isfinite(v)) set_status(st, KG_ERR_NONFINITE, (int)(oi * k + oj));
            if (i == j) v += dval;
        } else {
            v = (i == j) ? 1.0 : 0.0;
        }
        M[p] = v;
    }
}

// Leaf of the recursion: the 64 x 64 diagonal block at (o, o).  In place, its lower triangle
// becomes the Cholesky factor L; X[o.., o..] receives L^{-1} (lower, zero above the diagonal).
// One CTA of 256 threads, thread (ty, tx) owning the 4 x 4 block of rows 4ty.., columns 4tx.. in
// registers.  Cholesky, right-looking by columns: the owner of the pivot takes its square root,
// the owners of column c publish L[r][c] = a[r][c] / L[c][c], every thread subtracts
// L[r][c] L[c'][c] from its entries (c < c' <= r).  The inverse by rows: once row t of X is final
// (divided by L[t][t]), every row r > t subtracts L[r][t] X[t][:].  Two barriers a step.
__global__ void __launch_bounds__(256)
k_chol_inv64(double* __restrict__ M, double* __restrict__ X, int64_t kp, int64_t o, int64_t k, DevStatus* st) {
    __shared__ double colv[NB];          // column c of L (Cholesky) / row t of X (inverse)
    __shared__ double Ls[NB][NB + 1];    // L, for the inverse
    __shared__ double rdg[NB];           // 1 / L[c][c], one division per column
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int r0 = 4 * ty, c0 = 4 * tx;
    double* blk = M + o * kp + o;
    double a[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) a[i][j] = (c0 + j <= r0 + i) ? blk[(int64_t)(r0 + i) * kp + c0 + j] : 0.0;
    for (int c = 0; c < NB; ++c) {
        const int cb = c >> 2, cj = c & 3;
        if (tx == cb && ty == cb) {
            double pv = 0.0;   // a[cj][cj], selected with static register indices
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (i == cj && j == cj) pv = a[i][j];
            if (!(pv > 0.0) || !isfinite(pv)) {
                set_status(st, KG_ERR_NOT_PD, (int)(k - 1 - (o + c)));
                pv = 1.0;
            }
            const double d = sqrt(pv);
            Ls[c][c] = d;
            rdg[c] = 1.0 / d;
        }
        __syncthreads();
        const double d = Ls[c][c], rd = rdg[c];
        if (tx == cb) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                double v = 0.0;   // a[i][cj]
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (j == cj) v = a[i][j];
                const int r = r0 + i;
                if (r >= c) {
                    v = (r == c) ? d : v * rd;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (j == cj) a[i][j] = v;
                    colv[r] = v;
                    Ls[r][c] = v;
                }
            }
        }
        __syncthreads();
        // trailing update of the lower triangle right of column c
        if (r0 + 3 > c && c0 + 3 > c) {
            double lr[4], lc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) lr[i] = (r0 + i > c) ? colv[r0 + i] : 0.0;
#pragma unroll
            for (int j = 0; j < 4; ++j) lc[j] = (c0 + j > c) ? colv[c0 + j] : 0.0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (c0 + j <= r0 + i) a[i][j] -= lr[i] * lc[j];
        }
        __syncthreads();
    }
    // L back to the block (lower triangle; the upper triangle of the block is left as it was)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (c0 + j <= r0 + i) blk[(int64_t)(r0 + i) * kp + c0 + j] = a[i][j];
    // inverse: x starts as the identity; row t is divided by L[t][t], then removed from the rows below
    double x[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) x[i][j] = (r0 + i == c0 + j) ? 1.0 : 0.0;
    for (int t = 0; t < NB; ++t) {
        const int tb = t >> 2, ti = t & 3;
        if (ty == tb) {
            const double inv = rdg[t];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i == ti) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        x[i][j] *= inv;
                        colv[c0 + j] = x[i][j];
                    }
                }
        }
        __syncthreads();
        if (r0 + 3 > t && c0 <= t) {
            double xr[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) xr[j] = colv[c0 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + i;
                if (r > t) {
                    const double l = Ls[r][t];
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[i][j] -= l * xr[j];
                }
            }
        }
        __syncthreads();
    }
    double* xb = X + o * kp + o;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) xb[(int64_t)(r0 + i) * kp + c0 + j] = (c0 + j <= r0 + i) ? x[i][j] : 0.0;
}

// dst[r][c] = src[r][c] on an n_r x n_c block (both leading dimension ld)
__global__ void k_copy_block(const double* __restrict__ src, double* __restrict__ dst, int64_t ld, int64_t n_r,
                             int64_t n_c) {
    const int64_t total = n_r * n_c;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = p / n_c, c = p % n_c;
        dst[r * ld + c] = src[r * ld + c];
    }
}

// Recursive Cholesky with inverse of the block [o, o+n) of M (lower triangle, n a multiple of 64):
// afterwards M's lower triangle there holds L and X holds L^{-1}.  With the split n = n1 + n2,
//     (L11, X11) = rec(A11);  L21 = A21 X11^T;  A22 -= L21 L21^T;  (L22, X22) = rec(A22);
//     X21 = -X22 (L21 X11)
// (X11, X22 lower triangular; L21 and then X21 live in T, the product L21 X11 in X's own block).
// Every product is a DGEMM on the FP64 tensor path that skips the zero tiles of the triangles.
static int chol_inv_rec(double* M, double* X, double* T, int64_t kp, int64_t o, int64_t n, int64_t k, DevStatus* st,
                        cudaStream_t s) {
    if (n == NB) {
        KG_PROF(PK_PREPARE, s, k_chol_inv64<<<1, 256, 0, s>>>(M, X, kp, o, k, st));
        KG_LAUNCH_CHECK();
        return KG_OK;
    }
    const int64_t n1 = ceil_div(n / NB, 2) * NB, n2 = n - n1;
    int rc = chol_inv_rec(M, X, T, kp, o, n1, k, st, s);
    if (rc) return rc;
    double* A21 = M + (o + n1) * kp + o;
    double* A22 = M + (o + n1) * kp + o + n1;
    double* X11 = X + o * kp + o;
    double* X21 = X + (o + n1) * kp + o;
    double* X22 = X + (o + n1) * kp + o + n1;
    double* T21 = T + (o + n1) * kp + o;
    bool ok = true;
    {
        ProfScope ps(PK_PREPARE, s);
        // L21 = A21 X11^T: op(B) = X11^T is upper triangular
        ok = ok && dgemm(s, DG_TRANS_B | DG_B_UPPER, (int)n2, (int)n1, (int)n1, 1.0, A21, kp, X11, kp, 0.0, T21, kp);
    }
    {
        ProfScope ps(PK_PREPARE, s);
        // A22 -= L21 L21^T on the lower tiles
        ok = ok && dgemm(s, DG_TRANS_B | DG_C_LOWER, (int)n2, (int)n2, (int)n1, -1.0, T21, kp, T21, kp, 1.0, A22, kp);
    }
    if (!ok) return KG_ERR_CUDA;
    rc = chol_inv_rec(M, X, T, kp, o + n1, n2, k, st, s);
    if (rc) return rc;
    {
        ProfScope ps(PK_PREPARE, s);
        // P = L21 X11 (X11 lower triangular) into X21's place
        ok = ok && dgemm(s, DG_B_LOWER, (int)n2, (int)n1, (int)n1, 1.0, T21, kp, X11, kp, 0.0, X21, kp);
    }
    {
        ProfScope ps(PK_PREPARE, s);
        // X21 = -X22 P (X22 lower triangular) into T, then back into X
        ok = ok && dgemm(s, DG_A_LOWER, (int)n2, (int)n1, (int)n2, -1.0, X22, kp, X21, kp, 0.0, T21, kp);
    }
    if (!ok) return KG_ERR_CUDA;
    KG_PROF(PK_PREPARE, s, k_copy_block<<<148 * 4, 256, 0, s>>>(T21, X21, kp, n2, n1));
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// U[i][j] = X[k-1-i][k-1-j] (j >= i), 0 below the diagonal; optional fp32 copy
__global__ void k_output(const double* __restrict__ X, int64_t k, int64_t kp, double* __restrict__ U, float* __restrict__ U32) {
    const int64_t total = k * k;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = p / k, j = p % k;
        const double v = (j >= i) ? X[(k - 1 - i) * kp + (k - 1 - j)] : 0.0;
        U[p] = v;
        if (U32) U32[p] = (float)v;
    }
}

template <typename In>
static int prepare_one(const In* A, int64_t k, double damp, double* U, float* U32, unsigned char* base,
                       cudaStream_t st) {
    const PLayout L = p_layout(k);
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    double* scal = reinterpret_cast<double*>(base + L.off_scal);
    double* M = reinterpret_cast<double*>(base + L.off_M);
    double* X = reinterpret_cast<double*>(base + L.off_X);
    double* T = reinterpret_cast<double*>(base + L.off_T);
    const int nb = 148 * 4;

    KG_PROF(PK_PREPARE, st, k_diag_mean<In><<<1, 256, 0, st>>>(A, k, scal, status));
    KG_LAUNCH_CHECK();
    KG_PROF(PK_PREPARE, st, k_build_reversed<In><<<nb, 256, 0, st>>>(A, k, L.kp, scal, damp, M, status));
    KG_LAUNCH_CHECK();
    const int rc = chol_inv_rec(M, X, T, L.kp, 0, L.kp, k, status, st);
    if (rc) return rc;
    KG_PROF(PK_PREPARE, st, k_output<<<nb, 256, 0, st>>>(X, k, L.kp, U, U32));
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// the first error of the side region's status word reaches the call's status word
__global__ void k_merge_status(DevStatus* dst, const DevStatus* src) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && src->code != 0) set_status(dst, src->code, src->detail);
}

// Per host thread and device: one non-blocking side stream and two events, created on first use and
// kept for the life of the process, on which the output-side factor is prepared while the input-side
// one runs on the caller's stream.
struct PrepSide {
    int dev = -1;
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

static int prep_side(PrepSide*& out) {
    static thread_local std::vector<PrepSide> sides;
    int dev = 0;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    for (auto& s : sides)
        if (s.dev == dev) {
            out = &s;
            return KG_OK;
        }
    PrepSide s;
    s.dev = dev;
    KG_CUDA_TRY(cudaStreamCreateWithFlags(&s.st, cudaStreamNonBlocking));
    KG_CUDA_TRY(cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming));
    KG_CUDA_TRY(cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming));
    sides.push_back(s);
    out = &sides.back();
    return KG_OK;
}

}  // namespace kg

using namespace kg;

extern "C" size_t kron_gptq_prepare_workspace_size(int64_t k) {
    if (k <= 0) return kStatusBytes;
    return p_layout(k).total;
}

extern "C" int kron_gptq_prepare(const void* A, int64_t n, const void* B, int64_t m, int fac_dtype, double damp,
                                 double* U_A, double* U_B, float* U_A32, float* U_B32, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (fac_dtype != KG_F32 && fac_dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (n < 1 || m < 0 || !(damp >= 0.0) || !A || !U_A) return KG_ERR_ARG;
    if (B && (m < 1 || !U_B)) return KG_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (n > (int64_t)1 << 17 || m > (int64_t)1 << 17) return KG_ERR_UNSUPPORTED;
    const int64_t kmax = B ? std::max(n, m) : n;
    if (ws_bytes < p_layout(kmax).total) return KG_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* base = static_cast<unsigned char*>(ws);
    KG_CUDA_TRY(cudaMemsetAsync(base, 0, kStatusBytes, st));
    auto one = [&](const void* X, int64_t k, double* U, float* U32, unsigned char* b, cudaStream_t s) {
        return fac_dtype == KG_F64 ? prepare_one<double>(static_cast<const double*>(X), k, damp, U, U32, b, s)
                                   : prepare_one<float>(static_cast<const float*>(X), k, damp, U, U32, b, s);
    };
    // Both factors at once when the workspace holds a region for each: B on a side stream that forks
    // from and joins back into the caller's stream, so the call stays one operation on that stream.
    const size_t side_off = align_up(p_layout(n).total, 256);
    if (B && ws_bytes >= side_off + p_layout(m).total) {
        PrepSide* side = nullptr;
        int rc = prep_side(side);
        if (rc) return rc;
        unsigned char* bside = base + side_off;
        KG_CUDA_TRY(cudaMemsetAsync(bside, 0, kStatusBytes, st));
        KG_CUDA_TRY(cudaEventRecord(side->fork, st));
        KG_CUDA_TRY(cudaStreamWaitEvent(side->st, side->fork, 0));
        const int rc_b = one(B, m, U_B, U_B32, bside, side->st);
        // the join is recorded even when the side stream's launches failed, so that the caller's
        // stream never runs ahead of work already queued there
        KG_CUDA_TRY(cudaEventRecord(side->join, side->st));
        rc = rc_b ? rc_b : one(A, n, U_A, U_A32, base, st);
        KG_CUDA_TRY(cudaStreamWaitEvent(st, side->join, 0));
        if (rc) return rc;
        k_merge_status<<<1, 32, 0, st>>>(reinterpret_cast<DevStatus*>(base), reinterpret_cast<const DevStatus*>(bside));
        KG_LAUNCH_CHECK();
        return KG_OK;
    }
    int rc = one(A, n, U_A, U_A32, base, st);
    if (!rc && B) rc = one(B, m, U_B, U_B32, base, st);
    return rc;
}
