// kg_push_tc.cuh -- fp32 trailing band update on the 5th-generation tensor cores (tcgen05),
// 3xTF32, operands staged by the Tensor Memory Accelerator.
//
// The band update of "FastKron: Efficient Quantization with Kronecker-Factored Hessians",
// Section 2.4 (W -= L^B Delta L^A^T, batched), in its two-chain form:
//   column chain  W~[I,J] -= sum_{I'} U_B[I',I]^T X[I',J]         (I' over band 1 of column J)
//   row chain     R[I,J]  += sum_{J'} E[I,J'] U_A[J',J]            (J' over band 1 of row I)
// Every fp32 operand x is kept as two tf32 planes hi + lo (x = hi + lo to ~22 bits); each product
// is a_hi b_hi + a_hi b_lo + a_lo b_hi, accumulated in fp32 in tensor memory (TMEM).
// Target tiles that share a K range are paired along M: two tiles of one column (column chain)
// or, computing R^T = U_A^T E^T, two tiles of one row (row chain).  One CTA computes one 128 x 64
// block with M=128, N=64, K=8 MMAs.  Both operands are read K-major (k contiguous) from split
// copies the solve keeps for this purpose:
//   row chain     A(m,k) = U_A^T[J*64+m][k],   B(k,n) = E[I*64+n][k]      D[m][n] = dR[n][m]
//   column chain  A(m,k) = U_B^T[I*64+m][k],   B(k,n) = X^T[J*64+n][k]    D[m][n] = dW[m][n]
// Staging: a chunk is 32 K-elements, so each operand row is one 128-byte line; tensor-map loads
// of 64-row x 32-element boxes land in the 128-byte swizzled K-major layout the MMA descriptors
// name (16-byte pieces of row r permuted by r mod 8).  In a CTA of four warps
//   * one producer thread (warp 0) issues the loads of a stage, completing on the stage's "full"
//     mbarrier by transaction count;
//   * one MMA thread (warp 1) waits for a full stage, issues its 12 MMAs and commits them to
//     the stage's "empty" mbarrier, which the producer waits on before refilling it (4 stages);
//   * all four warps meet only at the end, to drain the accumulator from TMEM.
// Every wait is bounded in time and ends early once the solve has recorded an error; before the
// CTA exits it waits (bounded, without early exit) for the loads it issued and the MMAs it
// committed.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_tc.cuh"

namespace kg {

struct PushTc {
    static constexpr int M = 128, N = 64, BK = 32, STAGES = 4, THREADS = 128;
    // one chunk = BK = 32 K-elements = one 128-byte line per operand row
    static constexpr int A_BYTES = M * BK * 4;                         // 16 KB per plane
    static constexpr int B_BYTES = N * BK * 4;                         //  8 KB
    static constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;      // 48 KB
    static constexpr int BOX_BYTES = 64 * BK * 4;                      // one 64-row box of one plane
    // + barriers (full[S], empty[S], done), TMEM slot, counters; + pad to a 1024-byte base
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = 64;
    // 128-byte swizzled K-major layout: rows of 128 bytes, 8-row groups 1024 bytes apart
    static constexpr uint32_t SBO = 1024;
    // about 0.1 s at 2 GHz: far beyond any legitimate wait for one stage of MMAs
    static constexpr long long MAX_WAIT_CYCLES = 200000000LL;
};

// Split operand planes of the tensor-core update (all fp32 values exactly representable as
// tf32).  E* are Mp x Np (row-major), XT* Np x Mp, UAT* Np x Np, UBT* Mp x Mp.
struct SplitOperands {
    const float *E_hi, *E_lo, *XT_hi, *XT_lo, *UAT_hi, *UAT_lo, *UBT_hi, *UBT_lo;
};

// Tensor maps of the eight split planes (2-D, inner dimension = K, box 32 x 64, 128-byte
// swizzle).  E* are Mp x Np, XT* Np x Mp, UAT* Np x Np, UBT* Mp x Mp (rows x inner).
struct PushTmaMaps {
    CUtensorMap E_hi, E_lo, XT_hi, XT_lo, UAT_hi, UAT_lo, UBT_hi, UBT_lo;
};

namespace tc {
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// 2-D tiled bulk tensor load global -> shared, completing on bar; x = inner (K) coordinate in
// elements (a multiple of 32 here, so 16-byte aligned), y = row coordinate
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
}  // namespace tc

__global__ void __launch_bounds__(PushTc::THREADS, 1)
k_push_tc32(int D0, int mid, int D1, int Mt, int Nt, int64_t Np, float* __restrict__ Wt, float* __restrict__ R,
            const __grid_constant__ PushTmaMaps maps, DevStatus* status) {
    constexpr int T = KG_T;
    constexpr int S = PushTc::STAGES;
    extern __shared__ __align__(16) unsigned char smem_tc_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * PushTc::STAGE_BYTES);
    uint64_t* empty = full + S;
    uint64_t* done = empty + S;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
    int* issued_s = reinterpret_cast<int*>(tslot + 1);     // chunks whose loads were issued
    int* consumed_s = issued_s + 1;                         // chunks whose MMAs were issued

    const int chain = blockIdx.z;   // 0: row chain (into R), 1: column chain (into W~)
    int I, J, k0, k1;
    bool two;
    if (chain == 1) {
        J = blockIdx.x;
        if (J >= Nt) return;
        const int ilo = max(0, mid - J), ihi = min(Mt, D1 - J);
        I = ilo + 2 * blockIdx.y;
        if (I >= ihi) return;
        two = (I + 1 < ihi);
        k0 = max(0, D0 - J);
        k1 = min(Mt, mid - J);
    } else {
        I = blockIdx.x;
        if (I >= Mt) return;
        const int jlo = max(0, mid - I), jhi = min(Nt, D1 - I);
        J = jlo + 2 * blockIdx.y;
        if (J >= jhi) return;
        two = (J + 1 < jhi);
        k0 = max(0, D0 - I);
        k1 = min(Nt, mid - I);
    }
    if (k0 >= k1) return;
    // a solve that already failed (time-out, bad input) does no further tensor-core work
    if (*reinterpret_cast<const volatile int*>(&status->code) != 0) return;
    const int nchunks = (k1 - k0) * (T / PushTc::BK);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const CUtensorMap* mAh = (chain == 1) ? &maps.UBT_hi : &maps.UAT_hi;
    const CUtensorMap* mAl = (chain == 1) ? &maps.UBT_lo : &maps.UAT_lo;
    const CUtensorMap* mBh = (chain == 1) ? &maps.XT_hi : &maps.E_hi;
    const CUtensorMap* mBl = (chain == 1) ? &maps.XT_lo : &maps.E_lo;
    const int rowA = (chain == 1) ? I * T : J * T;
    const int rowB = (chain == 1) ? J * T : I * T;
    const uint32_t chunk_bytes = (uint32_t)((two ? 4 : 2) + 2) * PushTc::BOX_BYTES;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(done, 1);
        *issued_s = 0;
        *consumed_s = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // rows 64..127 of A stay zero in every stage when the pair is a single tile
    if (!two) {
        for (int s = 0; s < S; ++s) {
            unsigned char* st = smem + s * PushTc::STAGE_BYTES;
            for (int f = tid; f < PushTc::A_BYTES / 32; f += PushTc::THREADS) {
                const int off = PushTc::A_BYTES / 2 + f * 16;
                *reinterpret_cast<float4*>(st + off) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(st + PushTc::A_BYTES + off) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        tc::fence_proxy_async_smem();
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, PushTc::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // ---- producer
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % S;
            if (c >= S && !tc::mbar_wait(&empty[s], (uint32_t)(((c / S) - 1) & 1), PushTc::MAX_WAIT_CYCLES,
                                         &status->code)) {
                ok = false;
                break;
            }
            unsigned char* st = smem + s * PushTc::STAGE_BYTES;
            const int kx = (k0 * T) + c * PushTc::BK;
            tc::mbar_arrive_expect_tx(&full[s], chunk_bytes);
            tc::tma_load_2d(st, mAh, kx, rowA, &full[s]);
            tc::tma_load_2d(st + PushTc::A_BYTES, mAl, kx, rowA, &full[s]);
            if (two) {
                tc::tma_load_2d(st + PushTc::BOX_BYTES, mAh, kx, rowA + T, &full[s]);
                tc::tma_load_2d(st + PushTc::A_BYTES + PushTc::BOX_BYTES, mAl, kx, rowA + T, &full[s]);
            }
            tc::tma_load_2d(st + 2 * PushTc::A_BYTES, mBh, kx, rowB, &full[s]);
            tc::tma_load_2d(st + 2 * PushTc::A_BYTES + PushTc::B_BYTES, mBl, kx, rowB, &full[s]);
            *reinterpret_cast<volatile int*>(issued_s) = c + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        const uint32_t idesc = tc::idesc_tf32(PushTc::M, PushTc::N, false, false);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % S;
            if (!tc::mbar_wait(&full[s], (uint32_t)((c / S) & 1), PushTc::MAX_WAIT_CYCLES, &status->code)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            unsigned char* st = smem + s * PushTc::STAGE_BYTES;
            const uint32_t sa_hi = tc::smem_u32(st), sa_lo = sa_hi + PushTc::A_BYTES;
            const uint32_t sb_hi = sa_hi + 2 * PushTc::A_BYTES, sb_lo = sb_hi + PushTc::B_BYTES;
#pragma unroll
            for (int ks = 0; ks < PushTc::BK / 8; ++ks) {
                const uint64_t ah = tc::smem_desc_sw128(sa_hi + 32 * ks, PushTc::SBO);
                const uint64_t al = tc::smem_desc_sw128(sa_lo + 32 * ks, PushTc::SBO);
                const uint64_t bh = tc::smem_desc_sw128(sb_hi + 32 * ks, PushTc::SBO);
                const uint64_t bl = tc::smem_desc_sw128(sb_lo + 32 * ks, PushTc::SBO);
                const uint32_t acc0 = (c > 0 || ks > 0) ? 1u : 0u;
                tc::mma_tf32(tbase, al, bh, idesc, acc0);
                tc::mma_tf32(tbase, ah, bl, idesc, 1u);
                tc::mma_tf32(tbase, ah, bh, idesc, 1u);
            }
            tc::mma_commit(&empty[s]);
            *reinterpret_cast<volatile int*>(consumed_s) = c + 1;
        }
        // completes once every MMA this thread issued has finished
        tc::mma_commit(done);
    }
    if (!ok) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    __syncthreads();
    // ---- drain: the MMAs (done) and any loads issued but never consumed, without early exit
    const int never = 0;
    bool drained = tc::mbar_wait(done, 0u, PushTc::MAX_WAIT_CYCLES, &never);
    if (warp == 0 && lane == 0) {
        const int consumed = *reinterpret_cast<volatile int*>(consumed_s);
        const int issued = *reinterpret_cast<volatile int*>(issued_s);
        for (int c = consumed; c < issued; ++c)
            drained &= tc::mbar_wait(&full[c % S], (uint32_t)((c / S) & 1), PushTc::MAX_WAIT_CYCLES, &never);
    }
    const bool all_done = __syncthreads_and(drained) &&
                          *reinterpret_cast<volatile int*>(consumed_s) == nchunks;
    if (!all_done && tid == 0) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    tc::fence_after_sync();
    if (all_done) {
        // The whole 64-column accumulator row of this thread comes out of TMEM first; then all
        // global loads of the read-modify-write are issued before any store, so the update costs
        // one memory round trip rather than one per element.
        const int mrow = warp * 32 + lane;
        const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
        const bool valid = two || mrow < 64;
        float v[PushTc::N];
#pragma unroll
        for (int cb = 0; cb < PushTc::N / 16; ++cb)
            tc::tmem_ld16(trow + cb * 16, *reinterpret_cast<float(*)[16]>(&v[cb * 16]));
        tc::tmem_wait_ld();
        if (valid) {
            if (chain == 1) {
                float4* out = reinterpret_cast<float4*>(Wt + ((int64_t)I * T + mrow) * Np + (int64_t)J * T);
                float4 o[PushTc::N / 4];
#pragma unroll
                for (int q = 0; q < PushTc::N / 4; ++q) o[q] = out[q];
#pragma unroll
                for (int q = 0; q < PushTc::N / 4; ++q) {
                    o[q].x -= v[4 * q + 0];
                    o[q].y -= v[4 * q + 1];
                    o[q].z -= v[4 * q + 2];
                    o[q].w -= v[4 * q + 3];
                    out[q] = o[q];
                }
            } else {
                // D[m][n] = dR[I*64 + n][J*64 + m]: column m of the thread, one row per n
                float* out = R + (int64_t)I * T * Np + (int64_t)J * T + mrow;
                float o[PushTc::N];
#pragma unroll
                for (int q = 0; q < PushTc::N; ++q) o[q] = out[(int64_t)q * Np];
#pragma unroll
                for (int q = 0; q < PushTc::N; ++q) out[(int64_t)q * Np] = o[q] + v[q];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, PushTc::TMEM_COLS);
}

// ---- host: tensor maps.  cuTensorMapEncodeTiled is a driver entry point; it is looked up once
// through the runtime so the library needs no link-time dependency on libcuda.
static PFN_cuTensorMapEncodeTiled_v12000 push_tma_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over a row-major rows x inner fp32 matrix: box 32 (inner) x 64 (rows), 128-byte
// swizzle, zero fill outside.  The base must be 16-byte aligned and inner a multiple of 4.
static bool push_tma_map(CUtensorMap* map, const float* base, int64_t inner, int64_t rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = push_tma_encoder();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (inner & 3) != 0) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)inner * sizeof(float)};
    const cuuint32_t box[2] = {(cuuint32_t)PushTc::BK, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of the eight planes; Np, Mp are the padded layer sizes (multiples of 64).
static bool push_tma_maps(PushTmaMaps* mp, const SplitOperands& op, int64_t Np, int64_t Mp) {
    return push_tma_map(&mp->E_hi, op.E_hi, Np, Mp) && push_tma_map(&mp->E_lo, op.E_lo, Np, Mp) &&
           push_tma_map(&mp->XT_hi, op.XT_hi, Mp, Np) && push_tma_map(&mp->XT_lo, op.XT_lo, Mp, Np) &&
           push_tma_map(&mp->UAT_hi, op.UAT_hi, Np, Np) && push_tma_map(&mp->UAT_lo, op.UAT_lo, Np, Np) &&
           push_tma_map(&mp->UBT_hi, op.UBT_hi, Mp, Mp) && push_tma_map(&mp->UBT_lo, op.UBT_lo, Mp, Mp);
}

// U^T split into tf32 planes: UT_hi[c][r] + UT_lo[c][r] = U[r][c] (k x k, k multiple of 32)
__global__ void k_transpose_split(const float* __restrict__ U, int64_t k, int64_t ld, float* __restrict__ UT_hi,
                                  float* __restrict__ UT_lo) {
    __shared__ float t[32][33];
    const int64_t tiles = k / 32;
    for (int64_t b = blockIdx.x; b < tiles * tiles; b += gridDim.x) {
        const int64_t br = b / tiles, bc = b % tiles;
        const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
        for (int r = ty; r < 32; r += 8) t[r][tx] = U[(br * 32 + r) * ld + bc * 32 + tx];
        __syncthreads();
        for (int r = ty; r < 32; r += 8) {
            float hi, lo;
            tc::split_tf32(t[tx][r], hi, lo);
            const int64_t o = (bc * 32 + r) * k + br * 32 + tx;
            UT_hi[o] = hi;
            UT_lo[o] = lo;
        }
        __syncthreads();
    }
}

}  // namespace kg
