// kg_rc.cuh -- the row- and column-scaled alphabet on top of the two-sided solver, the
// WaterKron steps, and the empirical entropy of the codes.
//
// Alphabet ("WaterKron and FlipFlop Hessian", Section 2.1): V = beta alpha^T (.) Z with Z
// integer and not clipped; the step of entry (i,j) is s_ij = beta_i alpha_j.  WaterKron
// (same page, Section 3) takes alpha_j proportional to 1/L^(A)_jj = U_A[j,j] and beta_i
// proportional to U_B[i,i].
//
// Change of variables.  Two-sided GPTQ on W with steps s equals two-sided GPTQ with unit steps
// on W' = W (/) (beta alpha^T) under U'_A = D_alpha U_A D_alpha^-1, U'_B = D_beta U_B D_beta^-1:
// dividing the update W~[i',j'] -= U_B[i,i'] E U_A[j,j'] by s_i'j' gives
// W~'[i',j'] -= U'_B[i,i'] E' U'_A[j,j'] with E' = E / s_ij, and U', U have the same diagonals,
// so E' is exactly the solver's error on the scaled problem.  The solve therefore runs unchanged
// on (W', U'_A, U'_B) with unit row scales, a grid too wide to clip and int32 codes, and
// V = s (.) Z, E = s (.) E' afterwards.
#pragma once

#include <math.h>

#include "kg_common.cuh"

namespace kg {

// Every alpha_j and beta_i must be finite and > 0.
template <typename Real>
__global__ void k_rc_check_scales(const Real* __restrict__ alpha, int64_t n, const Real* __restrict__ beta,
                                  int64_t m, DevStatus* status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n + m; k += stride) {
        const Real v = k < n ? alpha[k] : beta[k - n];
        if (!(v > Real(0)) || !isfinite(v)) set_status(status, KG_ERR_NONFINITE, (int)k);
    }
}

// W' = W (/) (beta alpha^T)
template <typename Real>
__global__ void k_rc_scale_w(const Real* __restrict__ W, int64_t m, int64_t n, const Real* __restrict__ alpha,
                             const Real* __restrict__ beta, Real* __restrict__ Wp) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < m * n; p += stride) {
        const int64_t i = p / n, j = p - i * n;
        Wp[p] = W[p] / (beta[i] * alpha[j]);
    }
}

// U' = D_d U D_d^-1 on the upper triangle (the diagonal copied as it is), zero below
template <typename Real>
__global__ void k_rc_scale_u(const Real* __restrict__ U, int64_t k, const Real* __restrict__ d, Real* __restrict__ Up) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < k * k; p += stride) {
        const int64_t r = p / k, c = p - r * k;
        Up[p] = c > r ? U[p] * d[r] / d[c] : (c == r ? U[p] : Real(0));
    }
}

template <typename Real>
__global__ void k_rc_fill(Real* __restrict__ o, int64_t k, Real v) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < k; p += stride) o[p] = v;
}

// V = s (.) Z and E = s (.) E' in place; a code at the grid's bound (it may have been clipped)
// is reported as KG_ERR_RANGE.
template <typename Real>
__global__ void k_rc_finish(const int32_t* __restrict__ Z, int64_t m, int64_t n, const Real* __restrict__ alpha,
                            const Real* __restrict__ beta, Real* __restrict__ V, Real* __restrict__ E, int32_t bound,
                            DevStatus* status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < m * n; p += stride) {
        const int64_t i = p / n, j = p - i * n;
        const int32_t z = Z[p];
        if (z >= bound || z <= -bound) set_status(status, KG_ERR_RANGE, (int)(p < INT32_MAX ? p : INT32_MAX));
        const Real s = beta[i] * alpha[j];
        V[p] = s * (Real)z;
        if (E) E[p] = E[p] * s;
    }
}

// WaterKron steps: alpha_j = sqrt(gamma) U_A[j,j], beta_i = sqrt(gamma) U_B[i,i], so that the step
// of entry (i,j) is gamma U_B[i,i] U_A[j,j] and every error E_ij lies in [-gamma/2, gamma/2].
template <typename Real>
__global__ void k_wk_scales(const Real* __restrict__ UA, int64_t n, const Real* __restrict__ UB, int64_t m,
                            double gamma, Real* __restrict__ alpha, Real* __restrict__ beta) {
    const double r = sqrt(gamma);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n + m; k += stride) {
        if (k < n)
            alpha[k] = (Real)(r * (double)UA[k * n + k]);
        else
            beta[k - n] = (Real)(r * (double)UB[(k - n) * m + (k - n)]);
    }
}

}  // namespace kg
