// kg_gemm.cuh -- 64x64 output-tile GEMM engines used by the trailing updates, the factor
// preparation and the loss.
//
//   Dmma64  : fp64, 128 threads (4 warps, 2x2 warp tiles of 32x32), mma.sync m8n8k4 f64
//             (the FP64 tensor path of sm_100a; tcgen05 has no f64 kind).
//
// Dmma64 takes loader functors so that each caller decides where the operands come from
// (row-major, transposed, computed on the fly):
//   la(k0, As) fills As[r][kk] = A(r, k0+kk)
//   lb(k0, Bs) fills Bs[kk][c] = B(k0+kk, c)
// and accumulates acc += A(0:64, 0:K) * B(0:K, 0:64).  K must be a multiple of BK.
// DmmaPipe is the same arithmetic with cp.async double-buffered staging of plain copies.
#pragma once

#include "kg_common.cuh"

namespace kg {

// ------------------------------------------------------------------------------ fp64
struct Dmma64 {
    static constexpr int BM = 64, BN = 64, BK = 16;
    static constexpr int SA = BK + 4;   // row stride of As (doubles): conflict-free fragment loads
    static constexpr int SB = BN + 4;   // row stride of Bs
    static constexpr int kThreads = 128;
    struct Smem {
        double As[BM][SA];
        double Bs[BK][SB];
    };
    struct Acc {
        double c[4][4][2];
    };

    __device__ static __forceinline__ void zero(Acc& a) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) a.c[i][j][0] = a.c[i][j][1] = 0.0;
    }

    __device__ static __forceinline__ void mma(double& d0, double& d1, double a, double b) {
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
                     : "+d"(d0), "+d"(d1)
                     : "d"(a), "d"(b));
    }

    template <class LA, class LB>
    __device__ static __forceinline__ void run(Acc& acc, Smem& sm, int K, LA la, LB lb) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
        for (int k0 = 0; k0 < K; k0 += BK) {
            __syncthreads();
            la(k0, sm.As);
            lb(k0, sm.Bs);
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < BK; kk += 4) {
                double a[4], b[4];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) a[mi] = sm.As[wm + mi * 8 + (lane >> 2)][kk + (lane & 3)];
#pragma unroll
                for (int ni = 0; ni < 4; ++ni) b[ni] = sm.Bs[kk + (lane & 3)][wn + ni * 8 + (lane >> 2)];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni) mma(acc.c[mi][ni][0], acc.c[mi][ni][1], a[mi], b[ni]);
            }
        }
    }

    // f(row, col, value) for every accumulator element owned by this thread
    template <class F>
    __device__ static __forceinline__ void for_each(const Acc& acc, F f) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
                const int r = wm + mi * 8 + (lane >> 2);
                const int c = wn + ni * 8 + 2 * (lane & 3);
                f(r, c, acc.c[mi][ni][0]);
                f(r, c + 1, acc.c[mi][ni][1]);
            }
    }
    // out[r][c] += sign * acc[r][c] on a 64 x 64 tile (row-major, leading dimension ld, 16-byte
    // aligned rows).  All loads are issued before any store: one memory round trip in total.
    __device__ static __forceinline__ void add_to(const Acc& acc, double* out, int64_t ld, double sign) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
        double2 o[4][4];
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
                const int r = wm + mi * 8 + (lane >> 2);
                const int c = wn + ni * 8 + 2 * (lane & 3);
                o[mi][ni] = *reinterpret_cast<const double2*>(out + (int64_t)r * ld + c);
            }
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
                const int r = wm + mi * 8 + (lane >> 2);
                const int c = wn + ni * 8 + 2 * (lane & 3);
                o[mi][ni].x += sign * acc.c[mi][ni][0];
                o[mi][ni].y += sign * acc.c[mi][ni][1];
                *reinterpret_cast<double2*>(out + (int64_t)r * ld + c) = o[mi][ni];
            }
    }
};

// g(row, col, a, b) over two accumulators with the same layout
template <class F>
__device__ static __forceinline__ void dmma_for_each2(const Dmma64::Acc& x, const Dmma64::Acc& y, F f) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            const int r = wm + mi * 8 + (lane >> 2);
            const int c = wn + ni * 8 + 2 * (lane & 3);
            f(r, c, x.c[mi][ni][0], y.c[mi][ni][0]);
            f(r, c + 1, x.c[mi][ni][1], y.c[mi][ni][1]);
        }
}

// Loader helpers for Dmma64 (128 threads).  Row-major source with leading dimension ld.
// A(r,k) = src[(r0 + r) * ld + k0 + k]
struct LdA_RowMajor64 {
    const double* src; int64_t ld;
    __device__ void operator()(int k0, double (*As)[Dmma64::SA]) const {
        for (int idx = threadIdx.x; idx < Dmma64::BM * Dmma64::BK; idx += Dmma64::kThreads) {
            const int r = idx / Dmma64::BK, k = idx % Dmma64::BK;
            As[r][k] = src[(int64_t)r * ld + k0 + k];
        }
    }
};
// A(r,k) = src[(k0 + k) * ld + r]   (A is stored transposed, K x 64)
struct LdA_Trans64 {
    const double* src; int64_t ld;
    __device__ void operator()(int k0, double (*As)[Dmma64::SA]) const {
        for (int idx = threadIdx.x; idx < Dmma64::BM * Dmma64::BK; idx += Dmma64::kThreads) {
            const int k = idx / Dmma64::BM, r = idx % Dmma64::BM;
            As[r][k] = src[(int64_t)(k0 + k) * ld + r];
        }
    }
};
// B(k,c) = src[(k0 + k) * ld + c]
struct LdB_RowMajor64 {
    const double* src; int64_t ld;
    __device__ void operator()(int k0, double (*Bs)[Dmma64::SB]) const {
        for (int idx = threadIdx.x; idx < Dmma64::BK * Dmma64::BN; idx += Dmma64::kThreads) {
            const int k = idx / Dmma64::BN, c = idx % Dmma64::BN;
            Bs[k][c] = src[(int64_t)(k0 + k) * ld + c];
        }
    }
};
// B(k,c) = src[c * ld + k0 + k]   (B is stored transposed, 64 x K)
struct LdB_Trans64 {
    const double* src; int64_t ld;
    __device__ void operator()(int k0, double (*Bs)[Dmma64::SB]) const {
        for (int idx = threadIdx.x; idx < Dmma64::BK * Dmma64::BN; idx += Dmma64::kThreads) {
            const int c = idx / Dmma64::BK, k = idx % Dmma64::BK;
            Bs[k][c] = src[(int64_t)c * ld + k0 + k];
        }
    }
};

// ------------------------------------------------------------------------------ fp64, pipelined
// Same warp tiling and mma.sync m8n8k4 f64 as Dmma64, but the operands are plain copies of
// global memory staged with cp.async (16-byte granules) into two shared-memory stages, so the
// copy of chunk k+1 overlaps the MMAs of chunk k.
//   A_KM: A is stored K x 64 (A(r,k) = A[k*lda + r]) instead of 64 x K (A[r*lda + k]).
//   B_T : B is stored 64 x K (B(k,c) = B[c*ldb + k]) instead of K x 64 (B[k*ldb + c]).
// All source rows must start on 16-byte boundaries (ld and offsets even).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <bool A_KM, bool B_T>
struct DmmaPipe {
    static constexpr int BK = 16, STAGES = 2, kThreads = 128;
    static constexpr int SR = BK + 4;      // stride of a 64 x BK stage (row per output row/column)
    static constexpr int SK = 64 + 4;      // stride of a BK x 64 stage (row per k)
    static constexpr int A_ELEMS = A_KM ? BK * SK : 64 * SR;
    static constexpr int B_ELEMS = B_T ? 64 * SR : BK * SK;
    struct Smem {
        __align__(16) double a[STAGES][A_ELEMS];
        __align__(16) double b[STAGES][B_ELEMS];
    };

    __device__ static __forceinline__ void load(Smem& sm, int s, const double* A, int64_t lda, const double* B,
                                                int64_t ldb, int k0) {
        const int tid = threadIdx.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {   // 64 x 16 doubles = 512 granules of 16 bytes
            const int f = e * kThreads + tid;
            if (!A_KM) {
                const int r = f >> 3, c = (f & 7) * 2;
                cp_async16(&sm.a[s][r * SR + c], A + (int64_t)r * lda + k0 + c);
            } else {
                const int k = f >> 5, r = (f & 31) * 2;
                cp_async16(&sm.a[s][k * SK + r], A + (int64_t)(k0 + k) * lda + r);
            }
            if (!B_T) {
                const int k = f >> 5, c = (f & 31) * 2;
                cp_async16(&sm.b[s][k * SK + c], B + (int64_t)(k0 + k) * ldb + c);
            } else {
                const int c = f >> 3, k = (f & 7) * 2;
                cp_async16(&sm.b[s][c * SR + k], B + (int64_t)c * ldb + k0 + k);
            }
        }
    }

    __device__ static __forceinline__ void run(Dmma64::Acc& acc, Smem& sm, int K, const double* A, int64_t lda,
                                               const double* B, int64_t ldb) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
        const int nk = K / BK;
        load(sm, 0, A, lda, B, ldb, 0);
        cp_async_commit();
        for (int c = 0; c < nk; ++c) {
            if (c + 1 < nk) {
                load(sm, (c + 1) & 1, A, lda, B, ldb, (c + 1) * BK);
                cp_async_commit();
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();
            const double* as = sm.a[c & 1];
            const double* bs = sm.b[c & 1];
#pragma unroll
            for (int kk = 0; kk < BK; kk += 4) {
                double a[4], b[4];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    const int r = wm + mi * 8 + (lane >> 2), k = kk + (lane & 3);
                    a[mi] = A_KM ? as[k * SK + r] : as[r * SR + k];
                }
#pragma unroll
                for (int ni = 0; ni < 4; ++ni) {
                    const int cc = wn + ni * 8 + (lane >> 2), k = kk + (lane & 3);
                    b[ni] = B_T ? bs[cc * SR + k] : bs[k * SK + cc];
                }
#pragma unroll
                for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni) Dmma64::mma(acc.c[mi][ni][0], acc.c[mi][ni][1], a[mi], b[ni]);
            }
            __syncthreads();
        }
    }
};

}  // namespace kg
