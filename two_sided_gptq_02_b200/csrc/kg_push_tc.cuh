// kg_push_tc.cuh -- fp32 trailing band update on the 5th-generation tensor cores (tcgen05),
// 3xTF32: every fp32 operand x is kept as two tf32 planes hi + lo (x = hi + lo to ~22 bits)
// and each product is formed as a_hi b_hi + a_hi b_lo + a_lo b_hi, accumulated in fp32 in
// tensor memory (TMEM).
//
// The band update of "FastKron: Efficient Quantization with Kronecker-Factored Hessians",
// Section 2.4 (W -= L^B Delta L^A^T, batched), in its two-chain form:
//   column chain  W~[I,J] -= sum_{I'} U_B[I',I]^T X[I',J]         (I' over band 1 of column J)
//   row chain     R[I,J]  += sum_{J'} E[I,J'] U_A[J',J]            (J' over band 1 of row I)
// Target tiles that share a K range are paired along M: two tiles of one column (column
// chain) or, computing R^T = U_A^T E^T, two tiles of one row (row chain).  One CTA computes
// one 128 x 64 block with M=128, N=64, K=8 MMAs.  Both operands are read K-major (k
// contiguous) from split copies the solve keeps for this purpose:
//   row chain     A(m,k) = U_A^T[J*64+m][k],   B(k,n) = E[I*64+n][k]      D[m][n] = dR[n][m]
//   column chain  A(m,k) = U_B^T[I*64+m][k],   B(k,n) = X^T[J*64+n][k]    D[m][n] = dW[m][n]
// Staging is a pure copy into the 128-byte swizzled K-major layout of a 4-stage ring: a chunk
// is 32 K-elements, so each operand row is one 128-byte line in global memory and one
// 128-byte row in shared memory, with its 16-byte pieces permuted by the row index (mod 8).
// Eight consecutive lanes copy one row, so every quarter-warp of a 16-byte cp.async reads a
// whole line (one L2 request) and writes 128 distinct bytes (no bank conflict).  One thread
// issues the MMAs of a stage and commits them to that stage's mbarrier, which gates the
// stage's reuse.  All waits are bounded in time and end early once another CTA of the solve
// has recorded an error.
#pragma once

#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_tc.cuh"

namespace kg {

struct PushTc {
    static constexpr int M = 128, N = 64, BK = 32, STAGES = 4, THREADS = 128;
    static constexpr int A_BYTES = M * BK * 4;                         // 16 KB per plane
    static constexpr int B_BYTES = N * BK * 4;                         //  8 KB
    static constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;      // 48 KB
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;  // + barriers, slot, align pad
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

__global__ void __launch_bounds__(PushTc::THREADS)
k_push_tc32(int D0, int mid, int D1, int Mt, int Nt, int64_t Np, int64_t Mp, float* __restrict__ Wt,
            float* __restrict__ R, SplitOperands op, DevStatus* status) {
    constexpr int T = KG_T;
    constexpr int S = PushTc::STAGES;
    extern __shared__ __align__(16) unsigned char smem_tc_raw[];
    // 1024-byte aligned base for the operand stages (the launch reserves the padding)
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + S * PushTc::STAGE_BYTES);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + S * PushTc::STAGE_BYTES + 128);

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
    const int tid = threadIdx.x, warp = tid >> 5;

    // K-major operand rows: A rows start at rowA (128, or 64 when the pair is a single tile),
    // B rows at rowB (64)
    const float* Ahi = (chain == 1) ? op.UBT_hi : op.UAT_hi;
    const float* Alo = (chain == 1) ? op.UBT_lo : op.UAT_lo;
    const float* Bhi = (chain == 1) ? op.XT_hi : op.E_hi;
    const float* Blo = (chain == 1) ? op.XT_lo : op.E_lo;
    const int64_t ld = (chain == 1) ? Mp : Np;
    const int64_t rowA = (chain == 1) ? (int64_t)I * T : (int64_t)J * T;
    const int64_t rowB = (chain == 1) ? (int64_t)J * T : (int64_t)I * T;
    const int64_t kbase0 = (int64_t)k0 * T;
    const int arows = two ? 128 : 64;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) tc::mbar_init(&mbar[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // rows of A beyond a single tile stay zero in every stage
    if (!two) {
        for (int s = 0; s < S; ++s) {
            unsigned char* st = smem + s * PushTc::STAGE_BYTES;
            for (int f = tid; f < PushTc::A_BYTES / 32; f += PushTc::THREADS) {   // rows 64..127 of each plane
                const int off = PushTc::A_BYTES / 2 + f * 16;
                *reinterpret_cast<float4*>(st + off) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(st + PushTc::A_BYTES + off) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tslot, PushTc::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tslot;

    // copy of chunk c into stage s: A = arows x 32, B = 64 x 32, both planes
    auto load_chunk = [&](int c, int s) {
        unsigned char* st = smem + s * PushTc::STAGE_BYTES;
        const int64_t kb = kbase0 + (int64_t)c * PushTc::BK;
        // granule f: row f / 8, 16-byte piece ch = f % 8 of the row's 128 bytes
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int f = it * PushTc::THREADS + tid;
            const int ch = f & 7, mr = f >> 3;
            if (mr < arows) {
                const int off = mr * 128 + ((ch ^ (mr & 7)) << 4);
                const int64_t g = (rowA + mr) * ld + kb + 4 * ch;
                cp_async16(st + off, Ahi + g);
                cp_async16(st + PushTc::A_BYTES + off, Alo + g);
            }
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int f = it * PushTc::THREADS + tid;
            const int ch = f & 7, nr = f >> 3;
            const int off = nr * 128 + ((ch ^ (nr & 7)) << 4);
            const int64_t g = (rowB + nr) * ld + kb + 4 * ch;
            cp_async16(st + 2 * PushTc::A_BYTES + off, Bhi + g);
            cp_async16(st + 2 * PushTc::A_BYTES + PushTc::B_BYTES + off, Blo + g);
        }
    };

    const uint32_t idesc = tc::idesc_tf32(PushTc::M, PushTc::N, false, false);
#pragma unroll
    for (int s = 0; s < S - 1; ++s) {
        if (s < nchunks) load_chunk(s, s);
        cp_async_commit();
    }
    int issued = 0;   // chunks whose MMAs have been issued and committed
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % S;
        cp_async_wait<S - 2>();          // this thread's copies of chunk c have landed
        tc::fence_proxy_async_smem();    // ... and are visible to the tensor core
        __syncthreads();
        if (tid == 0) {
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
            tc::mma_commit(&mbar[s]);
        }
        issued = c + 1;
        // refill the stage chunk c-1 used, once its MMAs are done
        const int cn = c + S - 1;
        if (cn < nchunks) {
            bool freed = true;
            if (c >= 1) freed = tc::mbar_wait(&mbar[(c - 1) % S], ((c - 1) / S) & 1, PushTc::MAX_WAIT_CYCLES,
                                              &status->code);
            if (!__syncthreads_and(freed)) break;
            load_chunk(cn, cn % S);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
    // ---- wait for the last issued commit (it covers every earlier MMA of this thread)
    bool done = true;
    if (issued > 0)
        done = tc::mbar_wait(&mbar[(issued - 1) % S], ((issued - 1) / S) & 1, PushTc::MAX_WAIT_CYCLES,
                             &status->code);
    done = __syncthreads_and(done) && issued == nchunks;
    if (!done && tid == 0) set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    tc::fence_after_sync();
    if (done) {
        const int mrow = warp * 32 + (tid & 31);
        const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
        const bool valid = two || mrow < 64;
#pragma unroll
        for (int cb = 0; cb < PushTc::N / 16; ++cb) {
            float v[16];
            tc::tmem_ld16(trow + cb * 16, v);
            tc::tmem_wait_ld();
            if (valid) {
                if (chain == 1) {
                    float* out = Wt + ((int64_t)I * T + mrow) * Np + (int64_t)J * T + cb * 16;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float4 o = *reinterpret_cast<float4*>(out + 4 * q);
                        o.x -= v[4 * q + 0];
                        o.y -= v[4 * q + 1];
                        o.z -= v[4 * q + 2];
                        o.w -= v[4 * q + 3];
                        *reinterpret_cast<float4*>(out + 4 * q) = o;
                    }
                } else {
                    // D[m][n] = dR[I*64 + n][J*64 + m]
                    float* out = R + ((int64_t)I * T + cb * 16) * Np + (int64_t)J * T + mrow;
#pragma unroll
                    for (int q = 0; q < 16; ++q) out[(int64_t)q * Np] += v[q];
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, PushTc::TMEM_COLS);
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
