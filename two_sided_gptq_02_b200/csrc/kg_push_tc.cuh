// kg_push_tc.cuh -- fp32 trailing band update on the 5th-generation tensor cores (tcgen05),
// 3xTF32, operands staged by the Tensor Memory Accelerator.
//
// The band update of "FastKron: Efficient Quantization with Kronecker-Factored Hessians",
// Section 2.4 (W -= L^B Delta L^A^T, batched), in its two-chain form:
//   column chain  W~[I,J] -= sum_{I'} U_B[I',I]^T X[I',J]         (I' over band 1 of column J)
//   row chain     R[I,J]  += sum_{J'} E[I,J'] U_A[J',J]            (J' over band 1 of row I)
// Every fp32 operand x is kept as two tf32 planes hi + lo (x = hi + lo to ~22 bits); each product
// is a_hi b_hi + a_hi b_lo + a_lo b_hi, accumulated in fp32 in tensor memory (TMEM).
// One CTA computes a 128 x 128 block with M=128, N=128, K=8 MMAs: two target tiles (M) against
// two operand tiles (N) whose K ranges differ by one tile (adjacent columns of X in the column
// chain; adjacent rows of E in the row chain, which computes R^T = U_A^T E^T).  The CTA runs over
// the union of the two K ranges and loads the operand box of the one tile outside its range from
// beyond the tensor, which the TMA fills with zeros; targets outside the band are not stored.
// Both operands are read K-major (k contiguous) from split copies the solve keeps for this purpose:
//   row chain     A(m,k) = U_A^T[J*64+m][k],   B(k,n) = E[I*64+n][k]      D[m][n] = dR[n][m]
//   column chain  A(m,k) = U_B^T[I*64+m][k],   B(k,n) = X^T[J*64+n][k]    D[m][n] = dW[m][n]
// Staging: a chunk is 32 K-elements, so each operand row is one 128-byte line; tensor-map loads
// of 64-row x 32-element boxes land in the 128-byte swizzled K-major layout the MMA descriptors
// name (16-byte pieces of row r permuted by r mod 8).  In a CTA of four warps
//   * one producer thread (warp 0) issues the loads of a stage, completing on the stage's "full"
//     mbarrier by transaction count;
//   * one MMA thread (warp 1) waits for a full stage, issues its 12 MMAs and commits them to
//     the stage's "empty" mbarrier, which the producer waits on before refilling it (3 stages);
//   * all four warps meet only at the end, to drain the accumulator from TMEM.
// Every wait is bounded in time and ends early once the solve has recorded an error; before the
// CTA exits it waits (bounded, without early exit) for the loads it issued and the MMAs it
// committed.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_tc.cuh"

namespace kg {

// NB operand tiles per CTA (N = 64 NB): NB = 2 pairs two operand tiles whose K ranges differ by
// one tile and runs over their union; NB = 1 (small bands, where the extra tile would double the
// work) takes one operand tile and its exact K range.
// MT target tiles per CTA (M = 64 MT): MT = 2 for bands with several target diagonals; MT = 1 for
// the critical part (one target diagonal: the tile next to a CTA's target never is one).
template <int NB, int MT = 2>
struct PushCfg {
    static constexpr int M = 64 * MT, N = 64 * NB, BK = 32, STAGES = NB == 2 ? 3 : 4, THREADS = 128;
    // chunk = BK = 32 K-elements = one 128-byte line per operand row
    static constexpr int A_BYTES = M * BK * 4;                         // 16 KB (MT = 2) or 8 KB per plane
    static constexpr int B_BYTES = N * BK * 4;                         // 8 KB per plane per operand tile
    static constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
    static constexpr int BOX_BYTES = 64 * BK * 4;                      // one 64-row box of one plane
    static constexpr int CHUNK_BYTES = (2 * MT + 2 * NB) * BOX_BYTES;  // MT target tiles x 2 planes + B
    // + barriers (full[S], empty[S], done), TMEM slot, counters; + pad to a 1024-byte base
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = N;
    // 128-byte swizzled K-major layout: rows of 128 bytes, 8-row groups 1024 bytes apart
    static constexpr uint32_t SBO = 1024;
    // a row coordinate beyond every tensor map (m, n <= 2^20): loads there read zeros
    static constexpr int OOB_ROW = 1 << 21;
    // about 0.1 s at 2 GHz: far beyond any legitimate wait for one stage of MMAs
    static constexpr long long MAX_WAIT_CYCLES = 200000000LL;
};
// the band (in K tiles) from which the update pairs operand tiles
constexpr int PUSH_PAIR_MIN_K = 4;

// Launch shapes of the update of targets on tile diagonals [tgt0, D1) from sources on [D0, mid).
// The variant: pairs of operand tiles (NB = 2, MT = 2) for bands of PUSH_PAIR_MIN_K K tiles or more
// with several target diagonals; one operand and one target tile per CTA (NB = 1, MT = 1, M = 64)
// for a single target diagonal, where beside a target there is never a second one to fill M = 128;
// otherwise one operand tile and a pair of targets (NB = 1, MT = 2).
enum PushVariant { PV_PAIR = 0, PV_SINGLE = 1, PV_NARROW = 2 };
__host__ __device__ inline int push_variant(int D0, int mid, int tgt0, int D1) {
    if (mid - D0 >= PUSH_PAIR_MIN_K && D1 - tgt0 > 1) return PV_PAIR;
    return D1 - tgt0 == 1 ? PV_SINGLE : PV_NARROW;
}
__host__ __device__ inline int push_imax(int a, int b) { return a > b ? a : b; }
__host__ __device__ inline int push_imin(int a, int b) { return a < b ? a : b; }

// Grid (x, y, z = chain) of a launch of the given variant.  PV_PAIR runs in target-major order:
// x = the operand pairs around one target pair (at most (D1 - tgt0 + 2) / 2 + 1 of them), y =
// target pair slots j, from the highest that a CTA with work can take down to the lowest.  The
// other variants: x = operand tile, y = target pair (or the one target) above the band's edge.
inline dim3 push_grid(int variant, int tgt0, int D1, int Mt, int Nt) {
    const int mx = std::max(Mt, Nt);
    if (variant == PV_PAIR) {
        const int gx = (mx + 1) / 2;
        const int j0 = std::max(0, tgt0 - 1 - 2 * (gx - 1)) >> 1;
        const int j1 = (std::min(mx, D1) + 1) >> 1;
        return dim3((D1 - tgt0 + 2) / 2 + 1, std::max(1, j1 - j0), 2);
    }
    if (variant == PV_SINGLE) return dim3(mx, 1, 2);
    return dim3(mx, (D1 - tgt0 + 1) / 2, 2);
}

// The CTA (bx, by) of chain `chain` in a launch of ny target slots (the grid's y): its operand tiles
// b0 .. b0 + NB - 1, its target tiles t0 .. t0 + MT - 1 and its K tiles [k0, k1); false when it has
// no work.
//   chain 1 (column chain, into W~): b = column J (B = X^T rows), t = row I (A = U_B^T rows), K over
//     rows I' of the source band.  chain 0 (row chain, into R, computed transposed): b = row I
//     (B = E rows), t = column J (A = U_A^T rows), K over columns J'.
// Tile (t, b) is a target when t + b lies in [tgt0, D1) (tgt0 >= mid: the band may be updated in
// parts); operand tile b uses K tiles [D0 - b, mid - b).  A CTA runs over the union of its operand
// tiles' K ranges; a B box outside its own tile's range is loaded from beyond the tensor (zeros).
// NB = MT = 2 (target-major order): slot j is a pair of target tiles, t0 = 2j + p where the pair
// starts one below the band edge of operand pair b0 (p = (tgt0 - 1) mod 2), t0 = 2j where that edge
// is clipped to 0; bx walks the operand pairs whose band contains it.  CTAs that run together then
// share their U^T row slab (operand A), the larger operand of a tall or wide layer, instead of each
// reading its own; the CTAs with work are those of the plain (b0, t0) order of the other variants.
// Slots run from the highest j down: only the high slots reach the low operand pairs, whose K ranges
// are the longest, so the longest CTAs start first and the launch ends evenly.
struct PushCta {
    int b0, t0, k0, k1;
};
template <int NB, int MT>
__host__ __device__ inline bool push_cta(int bx, int by, int ny, int chain, int D0, int mid, int tgt0, int D1,
                                         int Mt, int Nt, PushCta& c) {
    const int Bmax = chain ? Nt : Mt, Tmax = chain ? Mt : Nt, Kmax = chain ? Mt : Nt;
    if (NB == 2 && MT == 2) {
        const int gx = (push_imax(Mt, Nt) + 1) / 2;
        const int p = (tgt0 - 1) & 1;
        const int j = (push_imax(0, tgt0 - 1 - 2 * (gx - 1)) >> 1) + (ny - 1 - by);
        const int e = tgt0 - 1 - p - 2 * j;
        c.b0 = 2 * ((e > 0 ? (e + 1) >> 1 : 0) + bx);
        c.t0 = tgt0 - c.b0 - 1 > 0 ? p + 2 * j : 2 * j;
    } else {
        c.b0 = NB * bx;
        c.t0 = push_imax(0, tgt0 - c.b0 - (NB - 1)) + MT * by;
    }
    if (c.b0 >= Bmax) return false;
    const int tlo = push_imax(0, tgt0 - c.b0 - (NB - 1)), thi = push_imin(Tmax, D1 - c.b0);
    if (c.t0 < tlo || c.t0 >= thi) return false;
    c.k0 = push_imax(0, D0 - c.b0 - (NB - 1));
    c.k1 = push_imin(Kmax, mid - c.b0);
    return c.k0 < c.k1;
}

// Split operand planes of the tensor-core update (all fp32 values exactly representable as
// tf32).  E* are Mp x Np (row-major), XT* Np x Mp, UAT* Np x Np, UBT* Mp x Mp.
struct SplitOperands {
    const float *E_hi, *E_lo, *XT_hi, *XT_lo, *UAT_hi, *UAT_lo, *UBT_hi, *UBT_lo;
};

// Tensor maps of the eight split planes (2-D, inner dimension = K, box 32 x 64, 128-byte
// swizzle, zero fill outside).  E* are Mp x Np, XT* Np x Mp, UAT* Np x Np, UBT* Mp x Mp (rows x inner).
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

template <int NB, int MT = 2>
__global__ void __launch_bounds__(PushCfg<NB, MT>::THREADS, 1)
k_push_tc32(int D0, int mid, int tgt0, int D1, int Mt, int Nt, int64_t Np, float* __restrict__ Wt,
            float* __restrict__ R, const __grid_constant__ PushTmaMaps maps, DevStatus* status) {
    using PushTc = PushCfg<NB, MT>;
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

    // which tiles this CTA updates (push_cta)
    const int chain = blockIdx.z;
    const int Bmax = chain ? Nt : Mt, Tmax = chain ? Mt : Nt;
    PushCta cta;
    if (!push_cta<NB, MT>((int)blockIdx.x, (int)blockIdx.y, (int)gridDim.y, chain, D0, mid, tgt0, D1, Mt, Nt, cta))
        return;
    const int b0 = cta.b0, t0 = cta.t0, k0 = cta.k0, k1 = cta.k1;
    grid_dep_launch();
    // set-up below overlaps the end of the previous kernel of the stream (programmatic launch);
    // everything that kernel writes -- the status word included -- is read after grid_dep_wait()
    const int nchunks = (k1 - k0) * (T / PushTc::BK);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const CUtensorMap* mAh = chain ? &maps.UBT_hi : &maps.UAT_hi;
    const CUtensorMap* mAl = chain ? &maps.UBT_lo : &maps.UAT_lo;
    const CUtensorMap* mBh = chain ? &maps.XT_hi : &maps.E_hi;
    const CUtensorMap* mBl = chain ? &maps.XT_lo : &maps.E_lo;

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
    if (warp == 0) {
        tc::tmem_alloc(tslot, PushTc::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;
    grid_dep_wait();
    // a solve that already failed (time-out, bad input) does no further tensor-core work
    const bool failed = *reinterpret_cast<const volatile int*>(&status->code) != 0;
    const int nch = failed ? 0 : nchunks;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // ---- producer
        for (int c = 0; c < nch; ++c) {
            const int s = c % S;
            if (c >= S && !tc::mbar_wait(&empty[s], (uint32_t)(((c / S) - 1) & 1), PushTc::MAX_WAIT_CYCLES,
                                         &status->code)) {
                ok = false;
                break;
            }
            unsigned char* st = smem + s * PushTc::STAGE_BYTES;
            const int kt = k0 + c / (T / PushTc::BK);        // K tile of this chunk
            const int kx = k0 * T + c * PushTc::BK;
            tc::mbar_arrive_expect_tx(&full[s], PushTc::CHUNK_BYTES);
#pragma unroll
            for (int u = 0; u < MT; ++u) {
                tc::tma_load_2d(st + u * PushTc::BOX_BYTES, mAh, kx, (t0 + u) * T, &full[s]);
                tc::tma_load_2d(st + PushTc::A_BYTES + u * PushTc::BOX_BYTES, mAl, kx, (t0 + u) * T, &full[s]);
            }
            unsigned char* sb = st + 2 * PushTc::A_BYTES;
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                // B rows of operand tile b0 + u, or beyond the tensor when kt is outside its K range
                const int b = b0 + u;
                const int rb = (kt >= D0 - b && kt < mid - b) ? b * T : PushTc::OOB_ROW;
                tc::tma_load_2d(sb + u * PushTc::BOX_BYTES, mBh, kx, rb, &full[s]);
                tc::tma_load_2d(sb + PushTc::B_BYTES + u * PushTc::BOX_BYTES, mBl, kx, rb, &full[s]);
            }
            *reinterpret_cast<volatile int*>(issued_s) = c + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        const uint32_t idesc = tc::idesc_tf32(PushTc::M, PushTc::N, false, false);
        for (int c = 0; c < nch; ++c) {
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
                // one MMA covers K = 8, i.e. 32 bytes of every row
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
                          *reinterpret_cast<volatile int*>(consumed_s) == nch;
    if (!all_done && tid == 0) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    tc::fence_after_sync();
    if (all_done && !failed) {
        // Thread mrow owns accumulator row mrow (target tile t = t0 + mrow / 64).  Each 64-column
        // part (operand tile b = b0 + h) comes out of TMEM first; then all global loads of the
        // read-modify-write are issued before any store (one memory round trip).  With M = 128 row m
        // sits in TMEM lane m; with M = 64 (MT = 1) in lane m % 16 + 32 (m / 16), so lanes 16..31
        // of each warp hold no row.
        const int mrow = MT == 2 ? warp * 32 + lane : warp * 16 + lane;
        const bool row_lane = MT == 2 || lane < 16;
        const int t = t0 + (mrow >> 6), r = mrow & 63;
        const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int h = 0; h < NB; ++h) {
            const int b = b0 + h;
            float v[64];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb)
                tc::tmem_ld16(trow + 64 * h + cb * 16, *reinterpret_cast<float(*)[16]>(&v[cb * 16]));
            tc::tmem_wait_ld();
            const bool valid = row_lane && t < Tmax && b < Bmax && t + b >= tgt0 && t + b < D1;
            if (!valid) continue;
            if (chain == 1) {
                float4* out = reinterpret_cast<float4*>(Wt + ((int64_t)t * T + r) * Np + (int64_t)b * T);
                float4 o[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) o[q] = out[q];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    o[q].x -= v[4 * q + 0];
                    o[q].y -= v[4 * q + 1];
                    o[q].z -= v[4 * q + 2];
                    o[q].w -= v[4 * q + 3];
                    out[q] = o[q];
                }
            } else {
                // D[m][n] = dR[b*64 + n][t*64 + r]: column r of target tile t, one row per n
                float* out = R + (int64_t)b * T * Np + (int64_t)t * T + r;
                float o[64];
#pragma unroll
                for (int q = 0; q < 64; ++q) o[q] = out[(int64_t)q * Np];
#pragma unroll
                for (int q = 0; q < 64; ++q) out[(int64_t)q * Np] = o[q] + v[q];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, PushTc::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------
// Rectangular form of the same engine, for the one-sided solve's batched update
// ("FastKron", Section 2.4, GPTQ-recursive):  C[r, c] -= sum_k A(r, k) B(k, c)  over
// rows [0, rows) (a multiple of 64) and columns [c0, c0 + cols) of C (multiples of 64), K over
// [k0, k1) (multiples of 64), with A and B^T given as K-major split tf32 planes:
//     A(r, k)  = mA[r][k]          (e.g. E, rows x K)
//     B(k, c)  = mB[c][k]          (e.g. U_A^T, so B = U_A)
// One CTA takes a 128 x 128 block (two 64-row boxes of A, two of B); boxes past the end of a map
// read zeros, and rows or columns past the block's range are not stored.  Staging, the MMA
// sequence, the bounded waits and the drain are those of k_push_tc32<2>.
static __global__ void __launch_bounds__(PushCfg<2>::THREADS, 1)
k_gemm_tc32(int rows, int c0, int cols, int k0, int k1, float* __restrict__ C, int64_t ldc,
            const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
            const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl, DevStatus* status) {
    using Cfg = PushCfg<2>;
    constexpr int S = Cfg::STAGES;
    extern __shared__ __align__(16) unsigned char smem_tc_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cfg::STAGE_BYTES);
    uint64_t* empty = full + S;
    uint64_t* done = empty + S;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
    int* issued_s = reinterpret_cast<int*>(tslot + 1);
    int* consumed_s = issued_s + 1;

    const int r0 = 128 * blockIdx.y, cb = c0 + 128 * blockIdx.x;
    if (r0 >= rows || cb >= c0 + cols || k0 >= k1) return;
    const int nchunks = (k1 - k0) / Cfg::BK;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    if (warp == 0) {
        tc::tmem_alloc(tslot, Cfg::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;
    const bool failed = *reinterpret_cast<const volatile int*>(&status->code) != 0;
    const int nch = failed ? 0 : nchunks;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // ---- producer: A rows r0, r0 + 64 and B rows (= C columns) cb, cb + 64 of each chunk
        for (int c = 0; c < nch; ++c) {
            const int s = c % S;
            if (c >= S && !tc::mbar_wait(&empty[s], (uint32_t)(((c / S) - 1) & 1), Cfg::MAX_WAIT_CYCLES, &status->code)) {
                ok = false;
                break;
            }
            unsigned char* st = smem + s * Cfg::STAGE_BYTES;
            const int kx = k0 + c * Cfg::BK;
            tc::mbar_arrive_expect_tx(&full[s], Cfg::CHUNK_BYTES);
            tc::tma_load_2d(st, &mAh, kx, r0, &full[s]);
            tc::tma_load_2d(st + Cfg::BOX_BYTES, &mAh, kx, r0 + 64, &full[s]);
            tc::tma_load_2d(st + Cfg::A_BYTES, &mAl, kx, r0, &full[s]);
            tc::tma_load_2d(st + Cfg::A_BYTES + Cfg::BOX_BYTES, &mAl, kx, r0 + 64, &full[s]);
            unsigned char* sb = st + 2 * Cfg::A_BYTES;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                tc::tma_load_2d(sb + u * Cfg::BOX_BYTES, &mBh, kx, cb + 64 * u, &full[s]);
                tc::tma_load_2d(sb + Cfg::B_BYTES + u * Cfg::BOX_BYTES, &mBl, kx, cb + 64 * u, &full[s]);
            }
            *reinterpret_cast<volatile int*>(issued_s) = c + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        const uint32_t idesc = tc::idesc_tf32(Cfg::M, Cfg::N, false, false);
        for (int c = 0; c < nch; ++c) {
            const int s = c % S;
            if (!tc::mbar_wait(&full[s], (uint32_t)((c / S) & 1), Cfg::MAX_WAIT_CYCLES, &status->code)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            unsigned char* st = smem + s * Cfg::STAGE_BYTES;
            const uint32_t sa_hi = tc::smem_u32(st), sa_lo = sa_hi + Cfg::A_BYTES;
            const uint32_t sb_hi = sa_hi + 2 * Cfg::A_BYTES, sb_lo = sb_hi + Cfg::B_BYTES;
#pragma unroll
            for (int ks = 0; ks < Cfg::BK / 8; ++ks) {
                const uint64_t ah = tc::smem_desc_sw128(sa_hi + 32 * ks, Cfg::SBO);
                const uint64_t al = tc::smem_desc_sw128(sa_lo + 32 * ks, Cfg::SBO);
                const uint64_t bh = tc::smem_desc_sw128(sb_hi + 32 * ks, Cfg::SBO);
                const uint64_t bl = tc::smem_desc_sw128(sb_lo + 32 * ks, Cfg::SBO);
                const uint32_t acc0 = (c > 0 || ks > 0) ? 1u : 0u;
                tc::mma_tf32(tbase, al, bh, idesc, acc0);
                tc::mma_tf32(tbase, ah, bl, idesc, 1u);
                tc::mma_tf32(tbase, ah, bh, idesc, 1u);
            }
            tc::mma_commit(&empty[s]);
            *reinterpret_cast<volatile int*>(consumed_s) = c + 1;
        }
        tc::mma_commit(done);
    }
    if (!ok) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    __syncthreads();
    const int never = 0;
    bool drained = tc::mbar_wait(done, 0u, Cfg::MAX_WAIT_CYCLES, &never);
    if (warp == 0 && lane == 0) {
        const int consumed = *reinterpret_cast<volatile int*>(consumed_s);
        const int issued = *reinterpret_cast<volatile int*>(issued_s);
        for (int c = consumed; c < issued; ++c)
            drained &= tc::mbar_wait(&full[c % S], (uint32_t)((c / S) & 1), Cfg::MAX_WAIT_CYCLES, &never);
    }
    const bool all_done = __syncthreads_and(drained) && *reinterpret_cast<volatile int*>(consumed_s) == nch;
    if (!all_done && tid == 0) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    tc::fence_after_sync();
    if (all_done && !failed) {
        // thread mrow owns row r0 + mrow; each 64-column half comes out of TMEM, then its 64 values
        // are read, reduced and stored in one memory round trip
        const int mrow = warp * 32 + lane;
        const int r = r0 + mrow;
        const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float v[64];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tc::tmem_ld16(trow + 64 * h + q * 16, *reinterpret_cast<float(*)[16]>(&v[q * 16]));
            tc::tmem_wait_ld();
            const int cc = cb + 64 * h;
            if (r >= rows || cc >= c0 + cols) continue;
            float4* out = reinterpret_cast<float4*>(C + (int64_t)r * ldc + cc);
            float4 o[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) o[q] = out[q];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                o[q].x -= v[4 * q + 0];
                o[q].y -= v[4 * q + 1];
                o[q].z -= v[4 * q + 2];
                o[q].w -= v[4 * q + 3];
                out[q] = o[q];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, Cfg::TMEM_COLS);
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
    const cuuint32_t box[2] = {(cuuint32_t)PushCfg<1>::BK, 64u};
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
static __global__ void k_transpose_split(const float* __restrict__ U, int64_t k, int64_t ld, float* __restrict__ UT_hi,
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
