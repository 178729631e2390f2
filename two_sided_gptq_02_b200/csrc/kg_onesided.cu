// kg_onesided.cu -- one-sided GPTQ with recursively batched trailing updates.
//
// "FastKron: Efficient Quantization with Kronecker-Factored Hessians", Section 2.2 (standard
// GPTQ: the columns in order, all rows of a column rounded at once, each error fed forward along
// its row through the upper Cholesky factor U_A of A_d^-1; the case B = I of the two-sided
// algorithm) and Section 2.4 (GPTQ-recursive: solve the first half of the columns, propagate its
// errors to the second half in one batched update, solve the second half).  For column j:
//     c = clamp(rint(x / s_i), qmin, qmax),  Q = s_i c,  E_ij = (x - Q) / U_A[j,j],
//     W~[i, j'] -= E_ij U_A[j, j']   for j' > j.
//
// The columns are cut into 64-wide blocks (the recursion's base case).  A leaf solves one block
// for all rows: one warp per 32 rows, each lane one row held in registers, the 64 columns in
// sequence with the in-block updates applied at once (U_A's block broadcast from shared memory).
// solve(J0, J1) recurses over blocks: solve [J0, mid), then
//     W~[:, mid..J1) -= E[:, J0..mid) U_A[J0..mid, mid..J1)
// -- one dense GEMM on the tensor cores: fp32 on tcgen05 with 3xTF32 (k_gemm_tc32: E and U_A^T
// kept as split tf32 planes, staged by TMA, accumulated in TMEM), fp64 on the FP64 tensor path
// (mma.sync m8n8k4, kg_dgemm.cuh) -- then solve [mid, J1).  Rows never interact, so the leaves
// need no anti-diagonal wavefront and there is no second chain.  W~ and E are padded to a
// multiple of 64 rows (zero rows, which stay zero).
#include <algorithm>
#include <type_traits>
#include <vector>

#include "kg_common.cuh"
#include "kg_dgemm.cuh"
#include "kg_profile.cuh"
#include "kg_push_tc.cuh"

namespace kg {

constexpr int OS_T = 64;      // block width (columns)
constexpr int OS_ROWS = 32;   // rows per leaf CTA (one warp)

template <typename Real>
struct OsSmem {
    Real a[OS_T][OS_T + 1];          // U_A's diagonal block (upper triangle; zero below)
    Real inva[OS_T];                 // 1 / U_A[j,j]
    Real st[OS_ROWS][OS_T + 1];      // W~ tile in, E tile out
    Real vq[OS_ROWS][OS_T + 1];      // Q = s_i c
    int8_t cs[OS_ROWS][OS_T];
};

// W~ = W padded with zero rows and columns to Mp x Np (W must be finite); E (and its lo plane in
// fp32) zero, so that the padded rows stay zero through every update
template <typename Real>
__global__ void k_os_init(const Real* __restrict__ W, int64_t m, int64_t n, int64_t Mp, int64_t Np,
                          Real* __restrict__ Wt, Real* __restrict__ E, Real* __restrict__ Elo, DevStatus* status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < Mp * Np; p += stride) {
        const int64_t i = p / Np, j = p - i * Np;
        Real v = Real(0);
        if (i < m && j < n) {
            v = W[i * n + j];
            if (!isfinite(v)) set_status(status, KG_ERR_NONFINITE, (int)(i * n + j < INT32_MAX ? i * n + j : INT32_MAX));
        }
        Wt[p] = v;
        E[p] = Real(0);
        if (Elo) Elo[p] = Real(0);
    }
}

// row scales finite and > 0, factor diagonal finite and > 0
template <typename Real>
__global__ void k_os_check(const Real* __restrict__ s, int64_t m, const Real* __restrict__ UA, int64_t n,
                           DevStatus* status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < m + n; k += stride) {
        const Real v = k < m ? s[k] : UA[(k - m) * n + (k - m)];
        if (!(v > Real(0)) || !isfinite(v)) set_status(status, KG_ERR_NONFINITE, (int)k);
    }
}

// U_A padded to Np x Np with the identity (padded columns get zero error, never touch real ones)
template <typename Real>
__global__ void k_os_pad(const Real* __restrict__ U, int64_t n, int64_t Np, Real* __restrict__ Up) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < Np * Np; p += stride) {
        const int64_t r = p / Np, c = p - r * Np;
        Up[p] = (r < n && c < n) ? U[r * n + c] : (r == c ? Real(1) : Real(0));
    }
}

// One 64-column block J for 32 rows per CTA.
template <typename Real>
__global__ void __launch_bounds__(OS_ROWS) k_os_leaf(int J, int64_t m, int64_t n, int64_t Np, Real* __restrict__ Wt,
                                                     Real* __restrict__ Ebuf, Real* __restrict__ Elo,
                                                     const Real* __restrict__ UA, int64_t ldA,
                                                     const Real* __restrict__ sp, int qmin, int qmax,
                                                     int8_t* __restrict__ codes, Real* __restrict__ V,
                                                     Real* __restrict__ outE) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    OsSmem<Real>& sm = *reinterpret_cast<OsSmem<Real>*>(smem_raw);
    // 16-byte vectors; every load of a batch is issued before its stores, so a batch costs one
    // memory round trip (rows start on 64-element boundaries: Np, ldA and c0 are multiples of 64)
    using Vec = typename std::conditional<sizeof(Real) == 4, float4, double2>::type;
    constexpr int VW = 16 / sizeof(Real);
    constexpr int VPR = OS_T / VW;                 // vectors per row
    constexpr int BATCH = 16;                      // vectors per thread per batch
    const int lane = threadIdx.x;
    const int64_t r0 = (int64_t)blockIdx.x * OS_ROWS, c0 = (int64_t)J * OS_T;
    {   // W~ tile: OS_ROWS x 64
        constexpr int NV = OS_ROWS * VPR / OS_ROWS;   // vectors per thread
        for (int t0 = 0; t0 < NV; t0 += BATCH) {
            Vec v[BATCH];
#pragma unroll
            for (int t = 0; t < BATCH; ++t) {
                const int idx = lane + OS_ROWS * (t0 + t), r = idx / VPR, cv = idx % VPR;
                v[t] = (r0 + r < m) ? *reinterpret_cast<const Vec*>(Wt + (r0 + r) * Np + c0 + cv * VW) : Vec{};
            }
#pragma unroll
            for (int t = 0; t < BATCH; ++t) {
                const int idx = lane + OS_ROWS * (t0 + t), r = idx / VPR, cv = idx % VPR;
                const Real* x = reinterpret_cast<const Real*>(&v[t]);
#pragma unroll
                for (int u = 0; u < VW; ++u) sm.st[r][cv * VW + u] = x[u];
            }
        }
    }
    {   // U_A's diagonal block, zero below the diagonal
        constexpr int NV = OS_T * VPR / OS_ROWS;
        for (int t0 = 0; t0 < NV; t0 += BATCH) {
            Vec v[BATCH];
#pragma unroll
            for (int t = 0; t < BATCH; ++t) {
                const int idx = lane + OS_ROWS * (t0 + t), r = idx / VPR, cv = idx % VPR;
                v[t] = *reinterpret_cast<const Vec*>(UA + (c0 + r) * ldA + c0 + cv * VW);
            }
#pragma unroll
            for (int t = 0; t < BATCH; ++t) {
                const int idx = lane + OS_ROWS * (t0 + t), r = idx / VPR, cv = idx % VPR;
                const Real* x = reinterpret_cast<const Real*>(&v[t]);
#pragma unroll
                for (int u = 0; u < VW; ++u) {
                    const int c = cv * VW + u;
                    sm.a[r][c] = c >= r ? x[u] : Real(0);
                }
            }
        }
    }
    __syncthreads();
    for (int j = lane; j < OS_T; j += OS_ROWS) sm.inva[j] = Real(1) / sm.a[j][j];
    const int64_t i = r0 + lane;
    const bool live = i < m;
    const Real s = live ? sp[i] : Real(1);
    const Real invs = Real(1) / s;
    const Real fqmin = (Real)qmin, fqmax = (Real)qmax;
    Real w[OS_T];
#pragma unroll
    for (int k = 0; k < OS_T; ++k) w[k] = live ? sm.st[lane][k] : Real(0);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < OS_T; ++j) {
        const Real x = w[j];
        Real c = rint(x * invs);
        c = c < fqmin ? fqmin : (c > fqmax ? fqmax : c);
        const Real Q = c * s;
        const Real e = (x - Q) * sm.inva[j];
        sm.st[lane][j] = e;
        sm.vq[lane][j] = Q;
        sm.cs[lane][j] = (int8_t)c;
#pragma unroll
        for (int k = j + 1; k < OS_T; ++k) w[k] -= e * sm.a[j][k];
    }
    __syncthreads();
    for (int r = 0; r < OS_ROWS; ++r) {
        const int64_t row = r0 + r;
        if (row >= m) break;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            const int64_t col = c0 + c;
            if constexpr (sizeof(Real) == 4) {
                float hi, lo;   // the tensor-core update reads E as tf32 hi + lo planes
                tc::split_tf32(sm.st[r][c], hi, lo);
                Ebuf[row * Np + col] = hi;
                Elo[row * Np + col] = lo;
            } else {
                Ebuf[row * Np + col] = sm.st[r][c];
            }
            if (col < n) {
                codes[row * n + col] = sm.cs[r][c];
                V[row * n + col] = sm.vq[r][c];
                if (outE) outE[row * n + col] = sm.st[r][c];
            }
        }
    }
}

struct OsArgs {
    int64_t m, n, Mp, Np, Nt, ldA;
    void *Wt, *E, *Elo;
    const void* UA;
    const void* sp;
    int qmin, qmax;
    int8_t* codes;
    void* V;
    void* outE;
    cudaStream_t st;
    DevStatus* status;
    const CUtensorMap *mEh, *mEl, *mUh, *mUl;   // fp32: E and U_A^T split planes
};

template <typename Real>
static int os_leaf(const OsArgs& a, int J) {
    ProfScope ps(PK_LEAF, a.st);
    const int grid = (int)ceil_div(a.m, OS_ROWS);
    k_os_leaf<Real><<<grid, OS_ROWS, sizeof(OsSmem<Real>), a.st>>>(
        J, a.m, a.n, a.Np, static_cast<Real*>(a.Wt), static_cast<Real*>(a.E), static_cast<Real*>(a.Elo),
        static_cast<const Real*>(a.UA), a.ldA,
        static_cast<const Real*>(a.sp), a.qmin, a.qmax, a.codes, static_cast<Real*>(a.V), static_cast<Real*>(a.outE));
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// W~[:, mid..J1) -= E[:, J0..mid) U_A[J0..mid, mid..J1) over all Mp rows
template <typename Real>
static int os_update(const OsArgs& a, int J0, int mid, int J1) {
    ProfScope ps(PK_PUSH, a.st);
    const int rows = (int)a.Mp, c0 = mid * OS_T, cols = (J1 - mid) * OS_T, k0 = J0 * OS_T, k1 = mid * OS_T;
    if constexpr (sizeof(Real) == 8) {
        const double* A = static_cast<const double*>(a.E) + k0;
        const double* B = static_cast<const double*>(a.UA) + (int64_t)k0 * a.ldA + c0;
        double* C = static_cast<double*>(a.Wt) + c0;
        return dgemm(a.st, 0, rows, cols, k1 - k0, -1.0, A, a.Np, B, a.ldA, 1.0, C, a.Np) ? KG_OK : KG_ERR_CUDA;
    } else {
        const dim3 grid((unsigned)ceil_div(cols, 128), (unsigned)ceil_div(rows, 128));
        k_gemm_tc32<<<grid, PushCfg<2>::THREADS, PushCfg<2>::SMEM_BYTES, a.st>>>(
            rows, c0, cols, k0, k1, static_cast<float*>(a.Wt), a.Np, *a.mEh, *a.mEl, *a.mUh, *a.mUl, a.status);
        KG_LAUNCH_CHECK();
        return KG_OK;
    }
}

template <typename Real>
static int os_solve(const OsArgs& a, int J0, int J1) {
    if (J1 - J0 == 1) return os_leaf<Real>(a, J0);
    const int mid = (J0 + J1) / 2;
    int rc;
    if ((rc = os_solve<Real>(a, J0, mid))) return rc;
    if ((rc = os_update<Real>(a, J0, mid, J1))) return rc;
    return os_solve<Real>(a, mid, J1);
}

// Workspace: [status][W~ Mp*Np][E Mp*Np][padded U_A Np*Np, when n % 64 != 0]
//            fp32 only: [E lo plane Mp*Np][U_A^T hi Np*Np][U_A^T lo Np*Np]
struct OsLayout {
    int64_t Mp, Np;
    size_t off_wt, off_e, off_ua, off_elo, off_uath, off_uatl, total;
    bool padded;
};

static OsLayout os_layout(int64_t m, int64_t n, size_t es) {
    OsLayout L{};
    L.Mp = ceil_div(m, OS_T) * OS_T;
    L.Np = ceil_div(n, OS_T) * OS_T;
    L.padded = L.Np != n;
    size_t off = kStatusBytes;
    L.off_wt = off;   off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
    L.off_e = off;    off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
    L.off_ua = off;
    if (L.padded) off = align_up(off + (size_t)(L.Np * L.Np) * es, 256);
    L.off_elo = L.off_uath = L.off_uatl = off;
    if (es == 4) {
        L.off_elo = off;  off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
        L.off_uath = off; off = align_up(off + (size_t)(L.Np * L.Np) * es, 256);
        L.off_uatl = off; off = align_up(off + (size_t)(L.Np * L.Np) * es, 256);
    }
    L.total = off;
    return L;
}

template <typename Real>
static int quantize_onesided_impl(const void* W, int64_t m, int64_t n, const void* UA, kg_grid grid, int8_t* codes,
                                  void* V, void* outE, void* ws, cudaStream_t st) {
    const OsLayout L = os_layout(m, n, sizeof(Real));
    unsigned char* base = static_cast<unsigned char*>(ws);
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    OsArgs a{};
    a.m = m; a.n = n; a.Mp = L.Mp; a.Np = L.Np; a.Nt = L.Np / OS_T;
    a.Wt = base + L.off_wt;
    a.E = base + L.off_e;
    a.Elo = sizeof(Real) == 4 ? base + L.off_elo : nullptr;
    a.sp = grid.row_scale;
    a.qmin = grid.qmin; a.qmax = grid.qmax;
    a.codes = codes; a.V = V; a.outE = outE; a.st = st;
    a.status = status;
    const int nb = 148 * 4;
    KG_CUDA_TRY(cudaMemsetAsync(status, 0, kStatusBytes, st));
    {
        ProfScope ps(PK_INIT, st);
        k_os_init<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(W), m, n, L.Mp, L.Np, static_cast<Real*>(a.Wt),
                                            static_cast<Real*>(a.E), static_cast<Real*>(a.Elo), status);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_os_check<Real><<<(int)std::max<int64_t>(1, std::min<int64_t>(nb, ceil_div(m + n, 256))), 256, 0, st>>>(
            static_cast<const Real*>(grid.row_scale), m, static_cast<const Real*>(UA), n, status);
    }
    KG_LAUNCH_CHECK();
    if (L.padded) {
        ProfScope ps(PK_INIT, st);
        k_os_pad<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(UA), n, L.Np, reinterpret_cast<Real*>(base + L.off_ua));
        KG_LAUNCH_CHECK();
        a.UA = base + L.off_ua;
        a.ldA = L.Np;
    } else {
        a.UA = UA;
        a.ldA = n;
    }
    CUtensorMap maps[4];
    if constexpr (sizeof(Real) == 4) {
        float* uath = reinterpret_cast<float*>(base + L.off_uath);
        float* uatl = reinterpret_cast<float*>(base + L.off_uatl);
        {
            ProfScope ps(PK_INIT, st);
            k_transpose_split<<<nb, 256, 0, st>>>(static_cast<const float*>(a.UA), L.Np, a.ldA, uath, uatl);
        }
        KG_LAUNCH_CHECK();
        if (!push_tma_map(&maps[0], static_cast<const float*>(a.E), L.Np, L.Mp) ||
            !push_tma_map(&maps[1], static_cast<const float*>(a.Elo), L.Np, L.Mp) ||
            !push_tma_map(&maps[2], uath, L.Np, L.Np) || !push_tma_map(&maps[3], uatl, L.Np, L.Np))
            return KG_ERR_CUDA;
        a.mEh = &maps[0]; a.mEl = &maps[1]; a.mUh = &maps[2]; a.mUl = &maps[3];
    }
    return os_solve<Real>(a, 0, (int)a.Nt);
}

template <typename Real>
static int os_configure() {
    KG_CUDA_TRY(cudaFuncSetAttribute(k_os_leaf<Real>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sizeof(OsSmem<Real>)));
    if constexpr (sizeof(Real) == 4) {
        KG_CUDA_TRY(cudaFuncSetAttribute(k_gemm_tc32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PushCfg<2>::SMEM_BYTES));
        KG_CUDA_TRY(cudaFuncSetAttribute(k_gemm_tc32, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared));
    }
    return KG_OK;
}

}  // namespace kg

using namespace kg;

extern "C" size_t kron_gptq_quantize_onesided_workspace_size(int64_t m, int64_t n, int dtype) {
    if (m < 0 || n < 0) return 0;
    if (dtype != KG_F32 && dtype != KG_F64) return 0;
    if (m == 0 || n == 0) return kStatusBytes;
    return os_layout(m, n, dtype == KG_F64 ? 8 : 4).total;
}

extern "C" int kron_gptq_quantize_onesided(const void* W, int64_t m, int64_t n, int dtype, const void* U_A,
                                           kg_grid grid, int8_t* out_codes, void* out_V, void* out_E, void* ws,
                                           size_t ws_bytes, void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (m < 0 || n < 0) return KG_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (grid.qmin >= 0 || grid.qmax <= 0 || grid.qmin < -128 || grid.qmax > 127) return KG_ERR_UNSUPPORTED;
    if (m > (int64_t)1 << 20 || n > (int64_t)1 << 20) return KG_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == 0 || n == 0) {
        if (ws_bytes < kStatusBytes) return KG_ERR_WORKSPACE;
        KG_CUDA_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
        return KG_OK;
    }
    if (!W || !U_A || !grid.row_scale || !out_codes || !out_V) return KG_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(U_A) & 15) return KG_ERR_ARG;   // the leaves read U_A in 16-byte vectors
    if (ws_bytes < os_layout(m, n, dtype == KG_F64 ? 8 : 4).total) return KG_ERR_WORKSPACE;
    int rc;
    if (dtype == KG_F64) {
        if ((rc = os_configure<double>())) return rc;
        return quantize_onesided_impl<double>(W, m, n, U_A, grid, out_codes, out_V, out_E, ws, st);
    }
    if ((rc = os_configure<float>())) return rc;
    return quantize_onesided_impl<float>(W, m, n, U_A, grid, out_codes, out_V, out_E, ws, st);
}
