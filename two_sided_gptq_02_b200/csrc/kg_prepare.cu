// kg_prepare.cu -- factors of the two-sided GPTQ solver (fp64).
//
// For a symmetric positive definite factor A (k x k):
//     A_d = A + damp * mean(diag A) * I          ("WaterKron ...", Section 2, Notation)
//     U   = upper triangular with U^T U = A_d^{-1}
// U is RevCholesky(A_d)^{-T} (same Notation paragraph).  With P the index reversal,
// P A_d P = L' L'^T (ordinary lower Cholesky), hence A_d = (P L' P)(P L' P)^T with P L' P
// upper, and U = (P L' P)^{-1} = P L'^{-1} P.  So the GPU computes
//     1. M  = P A_d P                      (copy with reversal and damping, padded to 64)
//     2. L' = Cholesky(M)                  (right-looking, 64x64 blocks)
//     3. X  = L'^{-1}                      (blocked lower-triangular inverse)
//     4. U[i][j] = X[k-1-i][k-1-j]         (reversal back; strictly lower part zero)
// Two O(k^3) steps instead of the three of "Cholesky, inverse, Cholesky of the inverse";
// the result is the same unique factor.  Every block product runs on the FP64 tensor path
// (mma.sync m8n8k4 f64) through kg::Dmma64.
#include <algorithm>

#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_profile.cuh"

namespace kg {

constexpr int NB = 64;

struct PLayout {
    int64_t k, kp, Kb;
    size_t off_scal, off_M, off_X, off_Dinv, off_Tmp, total;
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
    L.off_Dinv = off; off = align_up(off + (size_t)(L.kp * NB) * 8, 256);
    L.off_Tmp = off;  off = align_up(off + (size_t)(L.kp * NB) * 8, 256);
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

// Factor the diagonal block M[kb,kb] in place (lower Cholesky) and write its inverse to
// Dinv[kb] (64 x 64, row-major).  One block of 256 threads.
__global__ void __launch_bounds__(256)
k_potrf_diag(double* __restrict__ M, int64_t kp, int kb, int64_t k, double* __restrict__ Dinv, DevStatus* st) {
    __shared__ double Ls[NB][NB + 1];
    const int tid = threadIdx.x;
    double* blk = M + (int64_t)kb * NB * kp + (int64_t)kb * NB;
    for (int idx = tid; idx < NB * NB; idx += 256) {
        const int r = idx / NB, c = idx % NB;
        Ls[r][c] = (c <= r) ? blk[(int64_t)r * kp + c] : 0.0;
    }
    __syncthreads();
    for (int c = 0; c < NB; ++c) {
        if (tid == 0) {
            double pv = Ls[c][c];
            if (!(pv > 0.0) || !isfinite(pv)) {
                const int64_t orig = k - 1 - ((int64_t)kb * NB + c);
                set_status(st, KG_ERR_NOT_PD, (int)orig);
                pv = 1.0;
            }
            Ls[c][c] = sqrt(pv);
        }
        __syncthreads();
        const double d = Ls[c][c];
        for (int r = c + 1 + tid; r < NB; r += 256) Ls[r][c] /= d;
        __syncthreads();
        // trailing update of the lower triangle: Ls[r][cc] -= Ls[r][c] * Ls[cc][c], c < cc <= r
        const int rem = NB - c - 1;
        for (int idx = tid; idx < rem * rem; idx += 256) {
            const int r = c + 1 + idx / rem, cc = c + 1 + idx % rem;
            if (cc <= r) Ls[r][cc] -= Ls[r][c] * Ls[cc][c];
        }
        __syncthreads();
    }
    for (int idx = tid; idx < NB * NB; idx += 256) {
        const int r = idx / NB, c = idx % NB;
        blk[(int64_t)r * kp + c] = (c <= r) ? Ls[r][c] : 0.0;
    }
    // inverse X = L^{-1}, row by row: X[r][c] = (delta_rc - sum_{c<=t<r} L[r][t] X[t][c]) / L[r][r].
    // The strictly lower part of X is kept transposed in the free upper triangle of Ls
    // (Ls[c][r] = X[r][c], c < r); the diagonals live in dg / xd.
    __shared__ double dg[NB], xd[NB];
    if (tid < NB) dg[tid] = Ls[tid][tid];
    __syncthreads();
    for (int r = 0; r < NB; ++r) {
        for (int c = tid; c <= r; c += 256) {
            if (c == r) {
                xd[r] = 1.0 / dg[r];
            } else {
                double s = -Ls[r][c] * xd[c];
                for (int t = c + 1; t < r; ++t) s -= Ls[r][t] * Ls[c][t];
                Ls[c][r] = s / dg[r];
            }
        }
        __syncthreads();
    }
    double* Di = Dinv + (int64_t)kb * NB * NB;
    for (int idx = tid; idx < NB * NB; idx += 256) {
        const int r = idx / NB, c = idx % NB;
        double v = 0.0;
        if (c == r) v = xd[r];
        else if (c < r) v = Ls[c][r];
        Di[(int64_t)r * NB + c] = v;
    }
}

// L[ib,kb] = M[ib,kb] * Dinv[kb]^T for ib = kb+1 .. Kb-1 (in place; each block owns its tile)
__global__ void __launch_bounds__(Dmma64::kThreads)
k_panel(double* __restrict__ M, int64_t kp, int kb, const double* __restrict__ Dinv) {
    using Pipe = DmmaPipe<false, true>;
    __shared__ Pipe::Smem sm;
    const int ib = kb + 1 + blockIdx.x;
    double* tile = M + (int64_t)ib * NB * kp + (int64_t)kb * NB;
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    Pipe::run(acc, sm, NB, tile, kp, Dinv + (int64_t)kb * NB * NB, NB);
    __syncthreads();
    Dmma64::for_each(acc, [&](int r, int c, double v) { tile[(int64_t)r * kp + c] = v; });
}

// M[ib,jb] -= L[ib,kb] L[jb,kb]^T for kb < jb <= ib
__global__ void __launch_bounds__(Dmma64::kThreads)
k_syrk(double* __restrict__ M, int64_t kp, int kb) {
    using Pipe = DmmaPipe<false, true>;
    __shared__ Pipe::Smem sm;
    const int jb = kb + 1 + blockIdx.x;
    const int ib = kb + 1 + blockIdx.y;
    if (jb > ib) return;
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    Pipe::run(acc, sm, NB, M + (int64_t)ib * NB * kp + (int64_t)kb * NB, kp,
              M + (int64_t)jb * NB * kp + (int64_t)kb * NB, kp);
    Dmma64::add_to(acc, M + (int64_t)ib * NB * kp + (int64_t)jb * NB, kp, -1.0);
}

// X[ib,ib] = Dinv[ib] and zero the strictly upper block triangle of X
__global__ void k_x_init(double* __restrict__ X, int64_t kp, const double* __restrict__ Dinv) {
    const int64_t total = kp * kp;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = p / kp, c = p % kp;
        const int64_t rb = r / NB, cb = c / NB;
        double v = 0.0;
        if (rb == cb) v = Dinv[(rb * NB + (r % NB)) * NB + (c % NB)];
        X[p] = v;
    }
}

// Tmp[:, jb] = sum_{kb=jb}^{ib-1} L[ib,kb] X[kb,jb]    for jb < ib
__global__ void __launch_bounds__(Dmma64::kThreads)
k_inv_accum(const double* __restrict__ M, const double* __restrict__ X, int64_t kp, int ib, double* __restrict__ Tmp) {
    using Pipe = DmmaPipe<false, false>;
    __shared__ Pipe::Smem sm;
    const int jb = blockIdx.x;
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    Pipe::run(acc, sm, (ib - jb) * NB, M + (int64_t)ib * NB * kp + (int64_t)jb * NB, kp,
              X + (int64_t)jb * NB * kp + (int64_t)jb * NB, kp);
    double* out = Tmp + (int64_t)jb * NB;
    Dmma64::for_each(acc, [&](int r, int c, double v) { out[(int64_t)r * kp + c] = v; });
}

// X[ib,jb] = -Dinv[ib] * Tmp[:, jb]
__global__ void __launch_bounds__(Dmma64::kThreads)
k_inv_apply(double* __restrict__ X, int64_t kp, int ib, const double* __restrict__ Dinv, const double* __restrict__ Tmp) {
    using Pipe = DmmaPipe<false, false>;
    __shared__ Pipe::Smem sm;
    const int jb = blockIdx.x;
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    Pipe::run(acc, sm, NB, Dinv + (int64_t)ib * NB * NB, NB, Tmp + (int64_t)jb * NB, kp);
    double* out = X + (int64_t)ib * NB * kp + (int64_t)jb * NB;
    Dmma64::for_each(acc, [&](int r, int c, double v) { out[(int64_t)r * kp + c] = -v; });
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
    double* Dinv = reinterpret_cast<double*>(base + L.off_Dinv);
    double* Tmp = reinterpret_cast<double*>(base + L.off_Tmp);
    const int Kb = (int)L.Kb;
    const int nb = 148 * 4;

    KG_PROF(PK_PREPARE, st, k_diag_mean<In><<<1, 256, 0, st>>>(A, k, scal, status));
    KG_LAUNCH_CHECK();
    KG_PROF(PK_PREPARE, st, k_build_reversed<In><<<nb, 256, 0, st>>>(A, k, L.kp, scal, damp, M, status));
    KG_LAUNCH_CHECK();
    for (int kb = 0; kb < Kb; ++kb) {
        KG_PROF(PK_PREPARE, st, k_potrf_diag<<<1, 256, 0, st>>>(M, L.kp, kb, k, Dinv, status));
        KG_LAUNCH_CHECK();
        const int rest = Kb - kb - 1;
        if (rest > 0) {
            KG_PROF(PK_PREPARE, st, k_panel<<<rest, Dmma64::kThreads, 0, st>>>(M, L.kp, kb, Dinv));
            KG_LAUNCH_CHECK();
            KG_PROF(PK_PREPARE, st, k_syrk<<<dim3(rest, rest), Dmma64::kThreads, 0, st>>>(M, L.kp, kb));
            KG_LAUNCH_CHECK();
        }
    }
    KG_PROF(PK_PREPARE, st, k_x_init<<<nb, 256, 0, st>>>(X, L.kp, Dinv));
    KG_LAUNCH_CHECK();
    for (int ib = 1; ib < Kb; ++ib) {
        KG_PROF(PK_PREPARE, st, k_inv_accum<<<ib, Dmma64::kThreads, 0, st>>>(M, X, L.kp, ib, Tmp));
        KG_LAUNCH_CHECK();
        KG_PROF(PK_PREPARE, st, k_inv_apply<<<ib, Dmma64::kThreads, 0, st>>>(X, L.kp, ib, Dinv, Tmp));
        KG_LAUNCH_CHECK();
    }
    KG_PROF(PK_PREPARE, st, k_output<<<nb, 256, 0, st>>>(X, k, L.kp, U, U32));
    KG_LAUNCH_CHECK();
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
    int rc;
    if (fac_dtype == KG_F64) {
        rc = prepare_one<double>(static_cast<const double*>(A), n, damp, U_A, U_A32, base, st);
        if (!rc && B) rc = prepare_one<double>(static_cast<const double*>(B), m, damp, U_B, U_B32, base, st);
    } else {
        rc = prepare_one<float>(static_cast<const float*>(A), n, damp, U_A, U_A32, base, st);
        if (!rc && B) rc = prepare_one<float>(static_cast<const float*>(B), m, damp, U_B, U_B32, base, st);
    }
    return rc;
}
