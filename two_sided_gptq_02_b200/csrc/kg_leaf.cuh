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
// 4*VW*t + u), which with a row stride of 16 (mod 32) words is free of bank conflicts; all
// chunk loads are issued before any FMA and every chunk has its own accumulator, so the
// products form short independent chains.  The U_B column of the row is held in registers.
#pragma once

#include "kg_common.cuh"
#include "kg_tc.cuh"

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
    Real Rs[KG_T][KG_T + 1];   // R tile as loaded, then the transpose buffer for the final X
                               // (stride 65: column and row walks are both conflict-free)
    Real s[KG_T], invs[KG_T], inva[KG_T], ajj[KG_T];
    int32_t Cs[KG_T][KG_T];   // codes (int32: the unclipped alphabet needs more than 8 bits)
};

// Codes leave as int8 (clipped grids) or int32 (the unclipped alphabet), by the caller's width.
__device__ __forceinline__ void store_code(void* codes, int code_bytes, int64_t idx, int32_t c) {
    if (code_bytes == 1)
        static_cast<int8_t*>(codes)[idx] = (int8_t)c;
    else
        static_cast<int32_t*>(codes)[idx] = c;
}

// Store one 16-byte vector; when a second plane is given (fp32 feeding the 3xTF32 update),
// store the tf32 split instead: hi to dst_hi, the tf32 remainder to dst_lo.
__device__ __forceinline__ void leaf_store_split(float* dst_hi, float* dst_lo, int64_t off, float4 v) {
    if (dst_lo) {
        float4 h, l;
        tc::split_tf32(v.x, h.x, l.x);
        tc::split_tf32(v.y, h.y, l.y);
        tc::split_tf32(v.z, h.z, l.z);
        tc::split_tf32(v.w, h.w, l.w);
        *reinterpret_cast<float4*>(dst_hi + off) = h;
        *reinterpret_cast<float4*>(dst_lo + off) = l;
    } else {
        *reinterpret_cast<float4*>(dst_hi + off) = v;
    }
}
__device__ __forceinline__ void leaf_store_split(double* dst, double*, int64_t off, double2 v) {
    *reinterpret_cast<double2*>(dst + off) = v;
}

template <typename Real>
__device__ __forceinline__ Real leaf_clamp(Real v, Real lo, Real hi) {
    return v < lo ? lo : (v > hi ? hi : v);
}

// Copy four 64x64 tiles of row-major matrices into shared memory with a per-element transform
// store(tile, r, c, x), in PASSES memory round trips: each pass issues its share of the global
// loads of all four tiles before any store.  Threads 0..255 take part.  Tile 0, which the store
// transposes, is taken down its columns (a warp's lanes on consecutive rows), so that the transposed
// stores of a warp land on consecutive words; the others along their rows.
template <typename Real, int PASSES, class Store>
__device__ __forceinline__ void leaf_load_tiles4(const Real* const (&src)[4], const int64_t (&ld)[4], Store store) {
    constexpr int VW = LeafCfg<Real>::VW;
    constexpr int PER_ROW = KG_T / VW;                // vectors per tile row
    constexpr int PER_THREAD = KG_T * PER_ROW / 256;  // per tile: 4 (fp32) or 8 (fp64)
    constexpr int PER_PASS = PER_THREAD / PASSES;
    using Vec = typename LeafCfg<Real>::V;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        Vec v[4][PER_PASS];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < PER_PASS; ++e) {
                const int f = (p * PER_PASS + e) * 256 + threadIdx.x;
                const int r = t == 0 ? f % KG_T : f / PER_ROW, c = (t == 0 ? f / KG_T : f % PER_ROW) * VW;
                v[t][e] = *reinterpret_cast<const Vec*>(src[t] + (int64_t)r * ld[t] + c);
            }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < PER_PASS; ++e) {
                const int f = (p * PER_PASS + e) * 256 + threadIdx.x;
                const int r = t == 0 ? f % KG_T : f / PER_ROW, c = (t == 0 ? f / KG_T : f % PER_ROW) * VW;
                const Real* x = reinterpret_cast<const Real*>(&v[t][e]);
#pragma unroll
                for (int u = 0; u < VW; ++u) store(t, r, c + u, x[u]);
            }
    }
}

template <typename Real>
__global__ void __launch_bounds__(256)
k_leaf(int D, int Mt, int Nt, int64_t m, int64_t n, int64_t Np, int64_t Mp,
       Real* __restrict__ Wt, Real* __restrict__ R, Real* __restrict__ Ebuf, Real* __restrict__ Elo,
       Real* __restrict__ XTg, Real* __restrict__ XTlo,
       const Real* __restrict__ UA, int64_t ldA, const Real* __restrict__ UB, int64_t ldB,
       const Real* __restrict__ sp, int qmin, int qmax,
       void* __restrict__ codes, int code_bytes, Real* __restrict__ V, Real* __restrict__ outE) {
    constexpr int T = KG_T;
    constexpr int VW = LeafCfg<Real>::VW;
    constexpr int NC = T / (4 * VW);     // chunks per lane and dot product
    constexpr int PASSES = (sizeof(Real) == 8) ? 2 : 1;
    using Vec = typename LeafCfg<Real>::V;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LeafSmem<Real>& sm = *reinterpret_cast<LeafSmem<Real>*>(smem_raw);

    const int Imin = max(0, D - Nt + 1);
    const int I = Imin + blockIdx.x;
    const int J = D - I;
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)I * T, c0 = (int64_t)J * T;

    // ---- load: a^T (masked), b row-major (masked) into Es, R into XT (and Rs), W~ into Ws
    //      (after the previous kernel of the stream has finished: programmatic launch)
    grid_dep_launch();
    grid_dep_wait();
    {
        const Real* const src[4] = {UA + c0 * ldA + c0, UB + r0 * ldB + r0, R + r0 * Np + c0, Wt + r0 * Np + c0};
        const int64_t lds[4] = {ldA, ldB, Np, Np};
        leaf_load_tiles4<Real, PASSES>(src, lds, [&](int t, int r, int c, Real x) {
            if (t == 0) {
                sm.aT[c][r] = (c >= r) ? x : Real(0);
            } else if (t == 1) {
                sm.Es[r][c] = (c >= r) ? x : Real(0);
            } else if (t == 2) {
                sm.XT[r][c] = x;
                sm.Rs[r][c] = x;
            } else {
                sm.Ws[r][c] = x;
            }
        });
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
    const int i = tid >> 2, q = tid & 3;
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
        const int ty = tid >> 4, tx = tid & 15;   // rows 4 ty .. 4 ty + 3; columns tx + 16 c (c < 4)
        Real acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = Real(0);
        const int kmax = ty * 4 + 3;
#pragma unroll 4
        for (int k = 0; k <= kmax; ++k) {
            Real bv[4], rv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) bv[a] = sm.Es[k][ty * 4 + a];
#pragma unroll
            for (int c = 0; c < 4; ++c) rv[c] = sm.XT[k][tx + 16 * c];   // 16 lanes on consecutive words
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] += bv[a] * rv[c];
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) sm.Ws[ty * 4 + a][tx + 16 * c] -= acc[a][c];
        // Es and XT start the sweep at zero (unvisited entries contribute nothing)
        for (int idx = tid; idx < T * T; idx += 256) {
            sm.Es[idx / T][idx % T] = Real(0);
            sm.XT[idx / T][idx % T] = Real(0);
        }
    }
    __syncthreads();

    // ---- sweep
    const Real fqmin = Real(qmin), fqmax = Real(qmax);
    Real pre_x = Real(0), r_pre = Real(0), e_prev = Real(0), a_left = Real(0);
    Real inva_j = Real(0), ajj_j = Real(0);
    const int w = tid >> 5;
    // The lane's share of row i of E (k = VW*q + 4*VW*t + u) lives in registers: written by
    // predicated moves when the row produces it, so the row-chain products read only a^T from
    // shared memory.  Shared-memory bandwidth is what bounds a step.
    Real ereg[NC][VW];
#pragma unroll
    for (int t = 0; t < NC; ++t)
#pragma unroll
        for (int u = 0; u < VW; ++u) ereg[t][u] = Real(0);
    // chunks holding some k < i-1 (column chain) are fixed per warp
    const int tc = min(NC, (8 * w + 6 + 4 * VW - 1) / (4 * VW));
    for (int d = -1; d < 2 * T - 1; ++d) {
        const int j = d - i;
        const int jn = j + 1;
        const bool proc = (j >= 0) && (j < T);
        const bool pre = (jn >= 0) && (jn < T);
        const bool warp_pre = (d - 8 * w + 1 >= 0) && (d - (8 * w + 7) + 1 < T);   // warp-uniform
        // chunks holding some k < j (row chain): the warp's largest j is d - 8w
        const int tr = min(NC, max(0, (d - 8 * w + 4 * VW - 1) / (4 * VW)));
        // issue the look-ahead loads first: they do not depend on this step's results
        Vec xv[NC], av[NC];
        Real w_next = Real(0), a_next = Real(0), inva_next = Real(0), ajj_next = Real(0);
        if (warp_pre) {
            const int jr = pre ? jn : 0;
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                if (t < tc) xv[t] = *reinterpret_cast<const Vec*>(&sm.XT[jr][VW * q + 4 * VW * t]);
                if (t < tr) av[t] = *reinterpret_cast<const Vec*>(&sm.aT[jr][VW * q + 4 * VW * t]);
            }
            w_next = sm.Ws[i][jr];
            a_next = (jr > 0) ? sm.aT[jr][jr - 1] : Real(0);
            inva_next = sm.inva[jr];
            ajj_next = sm.ajj[jr];
        }
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
        if (warp_pre) {
            Real cacc[NC], racc[NC];
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                cacc[t] = Real(0);
                racc[t] = Real(0);
                if (t < tc) {
                    const Real* xs = reinterpret_cast<const Real*>(&xv[t]);
#pragma unroll
                    for (int u = 0; u < VW; ++u) cacc[t] += breg[t][u] * xs[u];
                }
                if (t < tr) {
                    const Real* as = reinterpret_cast<const Real*>(&av[t]);
#pragma unroll
                    for (int u = 0; u < VW; ++u) racc[t] += ereg[t][u] * as[u];
                }
            }
#pragma unroll
            for (int h = NC / 2; h > 0; h >>= 1)
#pragma unroll
                for (int t = 0; t < h; ++t) {
                    cacc[t] += cacc[t + h];
                    racc[t] += racc[t + h];
                }
            Real c = cacc[0], r = racc[0];
            c += __shfl_xor_sync(0xffffffffu, c, 1);
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            c += __shfl_xor_sync(0xffffffffu, c, 2);
            r += __shfl_xor_sync(0xffffffffu, r, 2);
            if (pre) {
                // E[i][j] enters ereg only below, so r covers k < j; b[i-1][i] is zero in breg,
                // so c covers k < i-1
                pre_x = w_next - c - b_ii * r;
                r_pre = r;
                a_left = a_next;
                inva_j = inva_next;
                ajj_j = ajj_next;
            }
        }
        e_prev = e;
        if (proc) {   // the lane owning column j keeps E[i][j]
#pragma unroll
            for (int t = 0; t < NC; ++t)
#pragma unroll
                for (int u = 0; u < VW; ++u)
                    if (j == VW * q + 4 * VW * t + u) ereg[t][u] = e;
        }
        __syncwarp();
        if (proc && q == 0) {
            sm.Es[i][j] = e;
            sm.XT[j][i] = Xv;
            sm.Ws[i][j] = Q;
            sm.Cs[i][j] = (int32_t)code;
        }
        __syncthreads();
    }

    // ---- write back: codes, V, E (16-byte stores where the layout allows)
    {
        constexpr int PER_ROW = T / VW;
        for (int f = tid; f < T * PER_ROW; f += 256) {
            const int r = f / PER_ROW, c = (f % PER_ROW) * VW;
            const int64_t gi = r0 + r, gj = c0 + c;
            Vec ev = *reinterpret_cast<const Vec*>(&sm.Es[r][c]);
            leaf_store_split(Ebuf, Elo, gi * Np + gj, ev);
            if (gi < m) {
                const Real* es = reinterpret_cast<const Real*>(&ev);
#pragma unroll
                for (int u = 0; u < VW; ++u) {
                    if (gj + u < n) {
                        store_code(codes, code_bytes, gi * n + gj + u, sm.Cs[r][c + u]);
                        V[gi * n + gj + u] = sm.Ws[r][c + u];
                        if (outE) outE[gi * n + gj + u] = es[u];
                    }
                }
            }
        }
    }
    // ---- the complete X = R + local X: back into R (row-major) and, when the tensor-core
    //      update needs it, into XTg (X transposed, leading dimension Mp), through the stride-65
    //      buffer (independent of the write-back above: no barrier between them)
    for (int idx = tid; idx < T * T; idx += 256) {
        const int c = idx >> 6, r = idx & 63;
        sm.XT[c][r] += sm.Rs[r][c];
    }
    __syncthreads();
    constexpr int PER_ROW = T / VW;
    if (XTg) {
        for (int f = tid; f < T * PER_ROW; f += 256) {
            const int c = f / PER_ROW, r = (f % PER_ROW) * VW;
            leaf_store_split(XTg, XTlo, (c0 + c) * Mp + r0 + r, *reinterpret_cast<const Vec*>(&sm.XT[c][r]));
        }
    }
    for (int idx = tid; idx < T * T; idx += 256) {
        const int c = idx >> 6, r = idx & 63;
        sm.Rs[r][c] = sm.XT[c][r];
    }
    __syncthreads();
    for (int idx = tid; idx < T * T; idx += 256) {
        const int r = idx >> 6, c = idx & 63;
        R[(r0 + r) * Np + c0 + c] = sm.Rs[r][c];
    }
}

}  // namespace kg
