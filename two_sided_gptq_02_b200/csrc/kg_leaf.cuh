// kg_leaf.cuh -- the in-tile anti-diagonal sweep ("leaf") of the two-sided GPTQ solver.
//
// One CTA per 64x64 tile (I, J) of a tile anti-diagonal, 256 threads, four per tile row.
// In-tile problem ("FastKron: Efficient Quantization with Kronecker-Factored Hessians",
// Sections 2.3-2.4, restated on one tile with a = U_A[J,J], b = U_B[I,I]):
//     w'   = W~[I,J] - b^T R[I,J]                       (external row chain, folded once)
//     r_ij = sum_{k<j} E_ik a[k][j]                      (in-tile row chain)
//     c_ij = sum_{k<i} b[k][i] X_kj,  X_kj = r_kj + E_kj a[j][j]   (in-tile column chain)
//     x    = w'_ij - c_ij - b_ii r_ij,  code = clamp(rint(x / s_i)),  Q = s_i code,
//     E_ij = (x - Q) / (b_ii a_jj)
// Entries with i + j = d are independent; step d handles them all.
//
// Look-ahead.  At step d the thread group of row i handles column j = d - i.  Everything
// entry (i, j) needs except the two newest terms (from (i-1, j) and (i, j-1), both produced at
// step d-1) was computed during step d-1 as pre_x; so the dependent chain of a step is one
// shared-memory load, two FMAs and the rounding.  The dot products for column j+1 run in the
// shadow of that chain: lanes read 16-byte chunks interleaved across the quad (k = VW*q +
// 4*VW*t + u), which with a row stride of 16 (mod 32) words is free of bank conflicts, and the
// U_B column of the row is held in registers.  Chunks beyond the warp's largest index are
// skipped (warp-uniform bounds).
#pragma once

#include "kg_common.cuh"

namespace kg {

template <typename Real>
struct LeafCfg;
template <>
struct LeafCfg<float> {
    static constexpr int VW = 4;    // elements per 16-byte vector
    static constexpr int S = 80;    // row stride (elements): 80 words = 16 (mod 32)
    using V = float4;
};
template <>
struct LeafCfg<double> {
    static constexpr int VW = 2;
    static constexpr int S = 72;    // 144 words = 16 (mod 32)
    using V = double2;
};

template <typename Real>
struct LeafSmem {
    static constexpr int S = LeafCfg<Real>::S;
    Real aT[KG_T][S];   // aT[j][k] = a[k][j]  (zero for k > j)
    Real Es[KG_T][S];   // errors E[i][k]; during set-up b row-major
    Real XT[KG_T][S];   // local X transposed XT[j][k] = X[k][j]; during set-up R row-major
    Real Ws[KG_T][S];   // w', then Q
    Real s[KG_T], invs[KG_T], inva[KG_T], ajj[KG_T];
    int8_t Cs[KG_T][KG_T];
};

template <typename Real>
__device__ __forceinline__ Real leaf_clamp(Real v, Real lo, Real hi) {
    return v < lo ? lo : (v > hi ? hi : v);
}

template <typename Real>
__global__ void __launch_bounds__(256)
k_leaf(int D, int Mt, int Nt, int64_t m, int64_t n, int64_t Np,
       Real* __restrict__ Wt, Real* __restrict__ R, Real* __restrict__ Ebuf,
       const Real* __restrict__ UA, int64_t ldA, const Real* __restrict__ UB, int64_t ldB,
       const Real* __restrict__ sp, int qmin, int qmax,
       int8_t* __restrict__ codes, Real* __restrict__ V, Real* __restrict__ outE) {
    constexpr int T = KG_T;
    constexpr int VW = LeafCfg<Real>::VW;
    constexpr int NC = T / (4 * VW);     // chunks per lane and dot product
    using Vec = typename LeafCfg<Real>::V;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LeafSmem<Real>& sm = *reinterpret_cast<LeafSmem<Real>*>(smem_raw);

    const int Imin = max(0, D - Nt + 1);
    const int I = Imin + blockIdx.x;
    const int J = D - I;
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)I * T, c0 = (int64_t)J * T;

    // ---- load: a^T (masked), b row-major (masked) into Es, R into XT, W~ into Ws
    for (int idx = tid; idx < T * T; idx += 256) {
        const int r = idx / T, c = idx % T;
        const Real av = UA[(c0 + r) * ldA + c0 + c];
        const Real bv = UB[(r0 + r) * ldB + r0 + c];
        sm.aT[c][r] = (c >= r) ? av : Real(0);
        sm.Es[r][c] = (c >= r) ? bv : Real(0);
        sm.XT[r][c] = R[(r0 + r) * Np + c0 + c];
        sm.Ws[r][c] = Wt[(r0 + r) * Np + c0 + c];
    }
    if (tid < T) {
        const Real s = sp[r0 + tid];
        sm.s[tid] = s;
        sm.invs[tid] = Real(1) / s;
    }
    __syncthreads();
    if (tid < T) {
        sm.ajj[tid] = sm.aT[tid][tid];
        sm.inva[tid] = Real(1) / sm.aT[tid][tid];
    }

    // ---- per-row constants; U_B column of the row in registers
    const int i = tid >> 2, q = tid & 3, w = tid >> 5;
    const Real b_ii = sm.Es[i][i];
    const Real b_up = (i > 0) ? sm.Es[i - 1][i] : Real(0);
    const Real invb = Real(1) / b_ii;
    const Real s_i = sm.s[i], invs_i = sm.invs[i];
    Real breg[NC][VW];   // b[k][i] for the lane's k, zero unless k < i-1
#pragma unroll
    for (int t = 0; t < NC; ++t)
#pragma unroll
        for (int u = 0; u < VW; ++u) {
            const int k = VW * q + 4 * VW * t + u;
            breg[t][u] = (k < i - 1) ? sm.Es[k][i] : Real(0);
        }

    // ---- fold the external row chain: w' = W~ - b^T R  (b^T[i][k] = b[k][i] = 0 for k > i)
    {
        const int ty = tid >> 4, tx = tid & 15;
        Real acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = Real(0);
        const int kmax = ty * 4 + 3;
        for (int k = 0; k <= kmax; ++k) {
            Real bv[4], rv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) bv[a] = sm.Es[k][ty * 4 + a];
#pragma unroll
            for (int c = 0; c < 4; ++c) rv[c] = sm.XT[k][tx * 4 + c];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] += bv[a] * rv[c];
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) sm.Ws[ty * 4 + a][tx * 4 + c] -= acc[a][c];
        // Es and XT start the sweep at zero (unvisited entries contribute nothing)
        for (int idx = tid; idx < T * T; idx += 256) {
            sm.Es[idx / T][idx % T] = Real(0);
            sm.XT[idx / T][idx % T] = Real(0);
        }
    }
    __syncthreads();

    // ---- sweep
    const Real fqmin = Real(qmin), fqmax = Real(qmax);
    const int imax_w = 8 * w + 7;
    const int tc = min(NC, (imax_w - 1 + 4 * VW - 1) / (4 * VW));   // chunks with some k < i-1
    Real pre_x = Real(0), r_pre = Real(0), e_prev = Real(0), a_left = Real(0);
    Real inva_j = Real(0), ajj_j = Real(0);
    for (int d = -1; d < 2 * T - 1; ++d) {
        const int j = d - i;
        const bool proc = (j >= 0) && (j < T);
        Real e = Real(0), Q = Real(0), Xv = Real(0), code = Real(0);
        if (proc) {
            const Real x_up = (i > 0) ? sm.XT[j][i - 1] : Real(0);
            const Real t_left = e_prev * a_left;
            const Real x = pre_x - b_up * x_up - b_ii * t_left;
            code = leaf_clamp(rint(x * invs_i), fqmin, fqmax);
            Q = code * s_i;
            e = (x - Q) * invb * inva_j;
            Xv = (r_pre + t_left) + e * ajj_j;
        }
        // look-ahead: everything column j+1 needs except the terms produced at this step
        const int jn = j + 1;
        const int jmax_w = d - 8 * w;                 // largest j in the warp (row 8w)
        if (jmax_w + 1 >= 0 && d - imax_w + 1 < T) {  // some row of the warp precomputes
            Real c = Real(0), r = Real(0);
            const bool pre = (jn >= 0) && (jn < T);
            const int jr = pre ? jn : 0;
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                if (t < tc) {
                    const Vec xv = *reinterpret_cast<const Vec*>(&sm.XT[jr][VW * q + 4 * VW * t]);
                    const Real* xs = reinterpret_cast<const Real*>(&xv);
#pragma unroll
                    for (int u = 0; u < VW; ++u) c += breg[t][u] * xs[u];
                }
            }
            const int tr = min(NC, max(0, (jmax_w + 4 * VW - 1) / (4 * VW)));   // chunks with some k < j
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                if (t < tr) {
                    const Vec ev = *reinterpret_cast<const Vec*>(&sm.Es[i][VW * q + 4 * VW * t]);
                    const Vec av = *reinterpret_cast<const Vec*>(&sm.aT[jr][VW * q + 4 * VW * t]);
                    const Real* es = reinterpret_cast<const Real*>(&ev);
                    const Real* as = reinterpret_cast<const Real*>(&av);
#pragma unroll
                    for (int u = 0; u < VW; ++u) r += es[u] * as[u];
                }
            }
            c += __shfl_xor_sync(0xffffffffu, c, 1);
            c += __shfl_xor_sync(0xffffffffu, c, 2);
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            r += __shfl_xor_sync(0xffffffffu, r, 2);
            if (pre) {
                // E[i][j] is still zero in shared memory here (written below), so r covers k < j
                pre_x = sm.Ws[i][jn] - c - b_ii * r;
                r_pre = r;
                a_left = (jn > 0) ? sm.aT[jn][jn - 1] : Real(0);
                inva_j = sm.inva[jn];
                ajj_j = sm.ajj[jn];
            }
        }
        e_prev = e;
        __syncwarp();
        if (proc && q == 0) {
            sm.Es[i][j] = e;
            sm.XT[j][i] = Xv;
            sm.Ws[i][j] = Q;
            sm.Cs[i][j] = (int8_t)code;
        }
        __syncthreads();
    }

    // ---- write back: codes, V, E; then the complete X = R + local X into R
    for (int idx = tid; idx < T * T; idx += 256) {
        const int r = idx / T, c = idx % T;
        const int64_t gi = r0 + r, gj = c0 + c;
        const Real ev = sm.Es[r][c];
        Ebuf[gi * Np + gj] = ev;
        if (gi < m && gj < n) {
            codes[gi * n + gj] = sm.Cs[r][c];
            V[gi * n + gj] = sm.Ws[r][c];
            if (outE) outE[gi * n + gj] = ev;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < T * T; idx += 256) {
        const int r = idx / T, c = idx % T;
        sm.Ws[r][c] = sm.XT[c][r];
    }
    __syncthreads();
    for (int idx = tid; idx < T * T; idx += 256) {
        const int r = idx / T, c = idx % T;
        const int64_t g = (r0 + r) * Np + c0 + c;
        R[g] = R[g] + sm.Ws[r][c];
    }
}

}  // namespace kg
