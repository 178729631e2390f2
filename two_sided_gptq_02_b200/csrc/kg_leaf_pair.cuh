// kg_leaf_pair.cuh -- two consecutive tile anti-diagonals (D and D+1) in one launch, fp32.
//
// Same in-tile problem and roles as k_leaf_ws (kg_leaf_ws.cuh).  What is new is that the tiles of
// D+1 start while those of D are still sweeping, and take over the update from D to D+1 that would
// otherwise be a launch of its own between two leaves ("FastKron", Sections 2.3-2.5: a tile needs
// from its left neighbour L = (I, J-1) only the rows of E_L and from its upper neighbour
// U = (I-1, J) only the columns of the complete X_U, as they complete):
//   * row chain    RT[i][j] = sum_k E_L[i][k] U_A[J-1,J][k][j]     (row i of E_L: L's step i+63)
//   * column chain CT[i][j] = sum_k U_B[I-1,I][k][i] X_U[k][j]     (column j of X_U: U's step 63+j)
// RT enters the tile's row chain (the helpers add it to r', so it also reaches the X the in-tile
// column chain uses) and CT its column chain (the helpers subtract it from P); the rounding warp is
// unchanged.  The R the pushes of earlier diagonals accumulated is still folded once up front.
//
// Roles come from an atomic ticket per diagonal: the first tickets solve the tiles of D, the rest
// those of D+1, so a CTA that waits only ever waits on CTAs that are already running.  A warp
// beyond the leaf's (the 18th):
//   * in a tile of D (publisher): after step idx+63 it writes row idx of E, and column idx of the
//     complete X (X_local + R) as row idx, into the tile's own W~ and R regions (nobody reads
//     those once the tile has loaded them) and then, with a release at GPU scope, the tile's
//     progress word (D << 8) | (idx + 1);
//   * in a tile of D+1 (loader): it waits (bounded) for its neighbours' progress words, reads up
//     to PAIR_BATCH new rows / columns at once, forms those rows of RT / columns of CT from
//     U_A[J-1,J] / U_B[I-1,I] held in shared memory (every row of the batch in registers, k
//     outer, each sum in k order 0..63), and releases them to the helpers through a count in
//     shared memory.
// Every wait is bounded in time; on expiry the CTA records a time-out and leaves.
//
// Not part of the default build: kg_quantize.cu uses it only when compiled with
// KG_EXPERIMENTAL_PAIR (and KG_PAIR_TIMELINE adds per-CTA timestamps).  Its first form, with one
// row per fence and the loaders forming rows one at a time, passed every fp32 parity test with the
// solve scheduled in pairs, but took 10.2 ms for a 4096 x 4096 layer against 8.4; this form
// (batched register-blocked loaders, X's columns exchanged as rows, pitch-69 RT / CT, backed-off
// shared-memory waits) has not been run yet.
#pragma once

#include <cstddef>

#include "kg_common.cuh"
#include "kg_leaf.cuh"
#include "kg_leaf_ws.cuh"
#include "kg_tc.cuh"

namespace kg {

#ifdef KG_PAIR_TIMELINE
// Per-CTA timeline of the paired launches of one solve (%globaltimer, ns): launch slot D/2 mod
// KG_PAIR_TL_SLOTS, CTA < KG_PAIR_TL_CTAS, 8 words: start, sweep start, sweep end, loader waits
// (row, column), helper waits, role * 1000 + tile, end.  Read with kron_gptq_debug_pair_timeline.
constexpr int KG_PAIR_TL_SLOTS = 96, KG_PAIR_TL_CTAS = 160;
__device__ unsigned long long g_pair_tl[KG_PAIR_TL_SLOTS * KG_PAIR_TL_CTAS * 8];
__device__ __forceinline__ unsigned long long pair_gtime() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
#define KG_PAIR_TL(...) __VA_ARGS__
#else
#define KG_PAIR_TL(...)
#endif
constexpr int PAIR_THREADS = WS_THREADS + 64;   // + two warps: publisher (D) / loaders (D+1)
constexpr int PAIR_BATCH = 8;                    // rows / columns a loader fetches per round trip

struct LeafPairSmem {
    LeafWsSmem ws;                 // the leaf's own buffers (same layout as k_leaf_ws)
    float nb[2][KG_T][KG_T + 1];   // U_A[J-1,J] (nb[0][k][j]) and U_B[I-1,I] (nb[1][k][i])
    // pitch 69 (= 5 mod 32): the eight rows of a helper warp read RT[i][d-i] / CT[i][d-i] on
    // distinct banks, and a loader's column writes CT[lane][c] stay conflict-free
    float RT[KG_T][KG_T + 5];      // row-chain term from L
    float CT[KG_T][KG_T + 5];      // column-chain term from U
    // stg[w][k][b]: element k of the b-th row (column) of a batch, so one float4 broadcast read
    // serves four rows of the batch
    alignas(16) float stg[2][KG_T][PAIR_BATCH];
    uint32_t pub_steps;            // steps published and seen by a helper (monotonic)
    uint32_t rt_ready, ct_ready;   // rows of RT / columns of CT complete
    int role, tile;
};
// the loaders read and write stg as float4
static_assert(offsetof(LeafPairSmem, stg) % 16 == 0, "stg must be 16-byte aligned");

__device__ __forceinline__ uint32_t pair_ld_acquire_cta(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(tc::smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void pair_st_release_cta(uint32_t* p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(tc::smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int pair_ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void pair_st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *cnt >= target (shared memory, one lane); false on time-out or abort.
__device__ __forceinline__ bool pair_wait_smem(const uint32_t* cnt, uint32_t target, const int* abort) {
    if (pair_ld_acquire_cta(cnt) >= target) return true;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(20);
        if (pair_ld_acquire_cta(cnt) >= target) return true;
        if (*reinterpret_cast<const volatile int*>(abort) != 0) return false;
        if (clock64() - t0 > WS_MAX_WAIT_CYCLES) return false;
    }
}

// Bounded wait until the progress word of a tile of diagonal D reports at least `need` rows and
// columns (global memory, one lane).  Returns the count it saw (>= need), or -1 on time-out/abort.
__device__ __forceinline__ int pair_wait_prog(const int* prog, int D, int need, const int* abort) {
    auto count = [&](int v) { return (v >> 8) == D ? (v & 255) : 0; };
    int c = count(pair_ld_acquire_gpu(prog));
    if (c >= need) return c;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(32);
        c = count(pair_ld_acquire_gpu(prog));
        if (c >= need) return c;
        if (*reinterpret_cast<const volatile int*>(abort) != 0) return -1;
        if (clock64() - t0 > WS_MAX_WAIT_CYCLES) return -1;
    }
}


// Grid: tiles of D first (in ticket order), then tiles of D+1; PAIR_THREADS threads.
// tickets[0] counts this launch's tickets (zero before it); prog[I] is the progress word of the
// tile of D in tile row I.
__global__ void __launch_bounds__(PAIR_THREADS, 1)
k_leaf_pair(int D, int Mt, int Nt, int64_t m, int64_t n, int64_t Np, int64_t Mp, float* __restrict__ Wt,
            float* __restrict__ R, float* __restrict__ Ebuf, float* __restrict__ Elo, float* __restrict__ XTg,
            float* __restrict__ XTlo, const float* __restrict__ UA, int64_t ldA, const float* __restrict__ UB,
            int64_t ldB, const float* __restrict__ sp, int qmin, int qmax, void* __restrict__ codes, int code_bytes,
            float* __restrict__ V, float* __restrict__ outE, DevStatus* status, int* __restrict__ tickets,
            int* __restrict__ prog) {
    constexpr int T = KG_T;
    constexpr int VW = 4;
    constexpr int NC = T / (4 * VW);
    constexpr int A = WS_AHEAD;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LeafPairSmem& P = *reinterpret_cast<LeafPairSmem*>(smem_raw);
    LeafWsSmem& sm = P.ws;
    const int tid = threadIdx.x;
    const bool helper = tid < WS_HELPERS;
    const bool extra = tid >= WS_THREADS;   // publisher (tiles of D) / loader (tiles of D+1)
    const int lane = tid & 31;

    // ---- role from the ticket
    const int nA = min(D, Mt - 1) - max(0, D - Nt + 1) + 1;
    KG_PAIR_TL(__shared__ unsigned long long tl_wait[3];)
    if (tid == 0) {
        const int t = atomicAdd(tickets, 1);
        P.role = t < nA ? 0 : 1;
        P.tile = t < nA ? t : t - nA;
        KG_PAIR_TL(tl_wait[0] = tl_wait[1] = tl_wait[2] = 0;)
    }
    KG_PAIR_TL(unsigned long long* tl = blockIdx.x < (unsigned)KG_PAIR_TL_CTAS
                   ? g_pair_tl + ((size_t)(D / 2 % KG_PAIR_TL_SLOTS) * KG_PAIR_TL_CTAS + blockIdx.x) * 8
                   : nullptr;
               if (tid == 0 && tl) tl[0] = pair_gtime();)
    __syncthreads();
    const int role = P.role;                 // 0: tile of D, 1: tile of D+1
    const int Dt = D + role;
    const int I = max(0, Dt - Nt + 1) + P.tile;
    const int J = Dt - I;
    const bool hasL = role == 1 && J >= 1;   // left neighbour (I, J-1) on D
    const bool hasU = role == 1 && I >= 1;   // upper neighbour (I-1, J) on D
    grid_dep_launch();
    const int64_t r0 = (int64_t)I * T, c0 = (int64_t)J * T;

    // ---- load (as k_leaf_ws) plus, for a tile of D+1, the off-diagonal factor blocks
    if (tid == 0) {
        sm.abort_flag = 0;
        for (int c = 0; c < 3; ++c)
            for (int k = c; k < 3; ++k) sm.colc[c][k] = 0.f;
        P.pub_steps = 0;
        P.rt_ready = hasL ? 0u : (uint32_t)T;
        P.ct_ready = hasU ? 0u : (uint32_t)T;
    }
    if (helper) {
        // U_A[J-1,J] and U_B[I-1,I] do not depend on earlier kernels: they load first
        if (role == 1) {
            const float* nsrc[2] = {UA + (c0 - T) * ldA + c0, UB + (r0 - T) * ldB + r0};
            const int64_t nld[2] = {ldA, ldB};
            const bool nhas[2] = {hasL, hasU};
            float4 v[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const int e = (f & 1) * WS_HELPERS + tid, blk = f >> 1;
                v[f] = nhas[blk] ? *reinterpret_cast<const float4*>(nsrc[blk] + (int64_t)(e >> 4) * nld[blk] + (e & 15) * 4)
                                 : float4{};
            }
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const int e = (f & 1) * WS_HELPERS + tid, blk = f >> 1;
                const int r = e >> 4, c4 = (e & 15) * 4;
                const float* x = reinterpret_cast<const float*>(&v[f]);
#pragma unroll
                for (int u = 0; u < 4; ++u) P.nb[blk][r][c4 + u] = x[u];
            }
        }
        const float* src[4] = {UA + c0 * ldA + c0, UB + r0 * ldB + r0, R + r0 * Np + c0, Wt + r0 * Np + c0};
        const int64_t lds[4] = {ldA, ldB, Np, Np};
        float4 v[8];
#pragma unroll
        for (int f = 0; f < 8; ++f) {
            if (f == 4) grid_dep_wait();
            const int e = (f & 1) * WS_HELPERS + tid, tile = f >> 1;
            v[f] = *reinterpret_cast<const float4*>(src[tile] + (int64_t)(e >> 4) * lds[tile] + (e & 15) * 4);
        }
#pragma unroll
        for (int f = 0; f < 8; ++f) {
            const int e = (f & 1) * WS_HELPERS + tid, tile = f >> 1;
            const int r = e >> 4, c4 = (e & 15) * 4;
            const float* x = reinterpret_cast<const float*>(&v[f]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c4 + u;
                if (tile == 0) {
                    sm.aT[c][r] = (r <= c - A) ? x[u] : 0.f;
                    if (r == c) {
                        sm.colc[c][4] = x[u];
                        sm.colc[c][3] = 1.f / x[u];
                    } else if (r == c - 1) {
                        sm.colc[c][0] = x[u];
                    } else if (r == c - 2) {
                        sm.colc[c][1] = x[u];
                    } else if (r == c - 3) {
                        sm.colc[c][2] = x[u];
                    }
                } else if (tile == 1) {
                    sm.Es[r][c] = (c >= r) ? x[u] : 0.f;
                } else if (tile == 2) {
                    sm.XT[r][c] = x[u];
                    sm.Rs[r][c] = x[u];
                } else {
                    sm.Ws[r][c] = x[u];
                }
            }
        }
        if (tid < T) {
            const float s = sp[r0 + tid];
            sm.s[tid] = s;
            sm.invs[tid] = 1.f / s;
        }
    }
    if (tid == 0) {
        for (int k = 0; k < WS_RING; ++k) {
            tc::mbar_init(&sm.cbar[k], 32);
            tc::mbar_init(&sm.hbar[k], T);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int idx = tid; idx < T * T; idx += PAIR_THREADS) {
        P.RT[idx / T][idx % T] = 0.f;
        P.CT[idx / T][idx % T] = 0.f;
    }
    __syncthreads();

    // ---- per-row constants (as k_leaf_ws)
    const int ht = tid & 255, g = tid >> 8;
    const int i = ht >> 2, q = ht & 3;
    float breg[NC][VW];
#pragma unroll
    for (int t = 0; t < NC; ++t)
#pragma unroll
        for (int u = 0; u < VW; ++u) {
            const int k = VW * q + 4 * VW * t + u;
            breg[t][u] = (helper && k <= i - A) ? sm.Es[k][i] : 0.f;
        }
    float bii[2], b1[2], b2[2], b3[2], sr[2], isr[2], ib[2];
    if (!helper && !extra) {
        const int l = tid & 31;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int ir = 2 * l + r;
            bii[r] = sm.Es[ir][ir];
            b1[r] = (ir >= 1) ? sm.Es[ir - 1][ir] : 0.f;
            b2[r] = (ir >= 2) ? sm.Es[ir - 2][ir] : 0.f;
            b3[r] = (ir >= 3) ? sm.Es[ir - 3][ir] : 0.f;
            sr[r] = sm.s[ir];
            isr[r] = sm.invs[ir];
            ib[r] = 1.f / bii[r];
        }
    }

    // ---- fold of the known row chain: w' = W~ - b^T R (as k_leaf_ws)
    {
        const int ty = tid >> 4, tx = tid & 15;
        float acc[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
        if (helper) {
            const int kmax = ty * 2 + 1;
#pragma unroll 4
            for (int k = 0; k <= kmax; ++k) {
                const float2 bv = *reinterpret_cast<const float2*>(&sm.Es[k][ty * 2]);
                const float4 rv = *reinterpret_cast<const float4*>(&sm.XT[k][tx * 4]);
                acc[0][0] += bv.x * rv.x; acc[0][1] += bv.x * rv.y; acc[0][2] += bv.x * rv.z; acc[0][3] += bv.x * rv.w;
                acc[1][0] += bv.y * rv.x; acc[1][1] += bv.y * rv.y; acc[1][2] += bv.y * rv.z; acc[1][3] += bv.y * rv.w;
            }
        }
        __syncthreads();
        if (helper) {
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) sm.Ws[ty * 2 + a][tx * 4 + c] -= acc[a][c];
        }
        for (int idx = tid; idx < T * T; idx += PAIR_THREADS) {
            sm.Es[idx / T][idx % T] = 0.f;
            sm.XT[idx / T][idx % T] = 0.f;
        }
    }
    __syncthreads();

    // ---- sweep
    KG_PAIR_TL(if (tid == 0 && tl) {
        tl[1] = pair_gtime();
        tl[6] = (unsigned long long)(P.role * 1000 + P.tile);
    })
    const float fqmin = (float)qmin, fqmax = (float)qmax;
    bool ok = true;
    if (extra) {
        const int xw = (tid - WS_THREADS) >> 5;   // 0 or 1
        if (role == 0) {
            // publisher (first extra warp): rows of E and columns of the complete X are final after
            // step idx+63; each round writes all that became final, then one fence and one release
            if (xw == 0) {
                for (int done = 0; done < T && ok;) {
                    int avail = 0;
                    if (lane == 0) {
                        avail = pair_wait_smem(&P.pub_steps, (uint32_t)(done + T), &sm.abort_flag)
                                    ? min(T, (int)pair_ld_acquire_cta(&P.pub_steps) - (T - 1))
                                    : -1;
                    }
                    avail = __shfl_sync(0xffffffffu, avail, 0);
                    if (avail < 0) {
                        ok = false;
                        break;
                    }
                    for (int idx = done; idx < avail; ++idx) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int c = lane + 32 * h;
                            Wt[(r0 + idx) * Np + c0 + c] = sm.Es[idx][c];
                            // column idx of X stored as row idx of the tile's R region
                            R[(r0 + idx) * Np + c0 + c] = sm.XT[idx][c] + sm.Rs[c][idx];
                        }
                    }
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) pair_st_release_gpu(&prog[I], (D << 8) | avail);
                    done = avail;
                }
            }
        } else if (xw == 0 ? hasL : hasU) {
            // loaders: warp 0 turns rows of E_L into rows of RT, warp 1 columns of X_U into columns
            // of CT; each fetches what became available (up to PAIR_BATCH) in one round trip
            const int* pw = xw == 0 ? &prog[I] : &prog[I - 1];
            for (int done = 0; done < T && ok;) {
                int avail = 0;
                KG_PAIR_TL(const unsigned long long tw0 = pair_gtime();)
                if (lane == 0) avail = pair_wait_prog(pw, D, done + 1, &sm.abort_flag);
                KG_PAIR_TL(if (lane == 0) atomicAdd(&tl_wait[xw], pair_gtime() - tw0);)
                avail = __shfl_sync(0xffffffffu, avail, 0);
                if (avail < 0) {
                    ok = false;
                    break;
                }
                const int cnt = min(avail - done, PAIR_BATCH);
                float v0[PAIR_BATCH], v1[PAIR_BATCH];
                if (xw == 0) {
#pragma unroll
                    for (int b = 0; b < PAIR_BATCH; ++b) {
                        const float* src = Wt + (r0 + done + b) * Np + (c0 - T);
                        v0[b] = b < cnt ? __ldcg(src + lane) : 0.f;
                        v1[b] = b < cnt ? __ldcg(src + lane + 32) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int b = 0; b < PAIR_BATCH; ++b) {
                        // column done + b of X_U, stored by U's publisher as a row of U's R region
                        const float* src = R + (r0 - T + done + b) * Np + c0;
                        v0[b] = b < cnt ? __ldcg(src + lane) : 0.f;
                        v1[b] = b < cnt ? __ldcg(src + lane + 32) : 0.f;
                    }
                }
#pragma unroll
                for (int b4 = 0; b4 < PAIR_BATCH; b4 += 4) {
                    *reinterpret_cast<float4*>(&P.stg[xw][lane][b4]) = make_float4(v0[b4], v0[b4 + 1], v0[b4 + 2], v0[b4 + 3]);
                    *reinterpret_cast<float4*>(&P.stg[xw][lane + 32][b4]) =
                        make_float4(v1[b4], v1[b4 + 1], v1[b4 + 2], v1[b4 + 3]);
                }
                __syncwarp();
                // acc[b] = (element lane, element lane + 32) of row / column b; the k order of every
                // sum is 0..63 as before, so the results are unchanged
                float2 acc[PAIR_BATCH];
#pragma unroll
                for (int b = 0; b < PAIR_BATCH; ++b) acc[b] = make_float2(0.f, 0.f);
#pragma unroll 4
                for (int k = 0; k < T; ++k) {
                    const float2 nk = make_float2(P.nb[xw][k][lane], P.nb[xw][k][lane + 32]);
#pragma unroll
                    for (int b4 = 0; b4 < PAIR_BATCH; b4 += 4) {
                        const float4 x = *reinterpret_cast<const float4*>(&P.stg[xw][k][b4]);
                        acc[b4 + 0] = __ffma2_rn(make_float2(x.x, x.x), nk, acc[b4 + 0]);
                        acc[b4 + 1] = __ffma2_rn(make_float2(x.y, x.y), nk, acc[b4 + 1]);
                        acc[b4 + 2] = __ffma2_rn(make_float2(x.z, x.z), nk, acc[b4 + 2]);
                        acc[b4 + 3] = __ffma2_rn(make_float2(x.w, x.w), nk, acc[b4 + 3]);
                    }
                }
#pragma unroll
                for (int b = 0; b < PAIR_BATCH; ++b) {
                    if (b < cnt) {
                        if (xw == 0) {
                            P.RT[done + b][lane] = acc[b].x;
                            P.RT[done + b][lane + 32] = acc[b].y;
                        } else {
                            P.CT[lane][done + b] = acc[b].x;
                            P.CT[lane + 32][done + b] = acc[b].y;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) pair_st_release_cta(xw == 0 ? &P.rt_ready : &P.ct_ready, (uint32_t)(done + cnt));
                done += cnt;
            }
        }
    } else if (!helper) {
        ok = ws_round_warp(sm, bii, b1, b2, b3, sr, isr, ib, fqmin, fqmax);
        __threadfence_block();   // every lane's stores of every step before the final count
        __syncwarp();
        if (lane == 0) atomicMax(&P.pub_steps, (uint32_t)(2 * T - 1));
    } else {
        const int wq = ht >> 5;   // rows 8 wq .. 8 wq + 7 of this warp
        bool all_ready = role == 0;   // every row of RT and column of CT is in
        for (int d = g; d < 2 * T - 1; d += WS_GROUPS) {
            if (d >= A) {
                const int dp = d - A;
                bool w_ok = true;
                if ((tid & 31) == 0) {
                    w_ok = tc::mbar_wait(&sm.cbar[dp % WS_RING], (uint32_t)((dp / WS_RING) & 1), WS_MAX_WAIT_CYCLES,
                                         &sm.abort_flag);
                    if (w_ok && (tid & 255) == 0) {   // steps up to dp are published: tell the publisher
                        __threadfence_block();
                        atomicMax(&P.pub_steps, (uint32_t)(dp + 1));
                    }
                }
                __syncwarp();
                w_ok = __shfl_sync(0xffffffffu, (int)w_ok, 0) != 0;
                if (!w_ok) {
                    ok = false;
                    break;
                }
            }
            float rt = 0.f, ct = 0.f;
            const int j = d - i;
            const bool active = (unsigned)j < (unsigned)T;
            const int jr = active ? j : 0;
            if (!all_ready) {
                // the neighbours' terms of this warp's entries must be ready
                const bool wact = d - 8 * wq >= 0 && d - 8 * wq - 7 < T;
                bool w_ok = true;
                KG_PAIR_TL(const unsigned long long th0 = pair_gtime();)
                if (wact && (tid & 31) == 0) {
                    const uint32_t need_r = (uint32_t)(min(8 * wq + 7, d) + 1);
                    const uint32_t need_c = (uint32_t)(min(d - 8 * wq, T - 1) + 1);
                    w_ok = pair_wait_smem(&P.rt_ready, need_r, &sm.abort_flag) &&
                           pair_wait_smem(&P.ct_ready, need_c, &sm.abort_flag);
                    KG_PAIR_TL(if (tid == 0) atomicAdd(&tl_wait[2], pair_gtime() - th0);)
                }
                int done_all = 0;
                if ((tid & 31) == 0)
                    done_all = pair_ld_acquire_cta(&P.rt_ready) >= (uint32_t)T && pair_ld_acquire_cta(&P.ct_ready) >= (uint32_t)T;
                __syncwarp();
                w_ok = __shfl_sync(0xffffffffu, (int)w_ok, 0) != 0;
                all_ready = __shfl_sync(0xffffffffu, done_all, 0) != 0;
                if (!w_ok) {
                    ok = false;
                    break;
                }
            }
            if (role == 1 && active) {
                rt = P.RT[i][jr];
                ct = P.CT[i][jr];
            }
            float4 xv[NC], av[NC], ev[NC];
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                const int k0 = VW * q + 4 * VW * t;
                const bool pc = active && k0 <= i - A;
                const bool pr = active && k0 <= j - A;
                xv[t] = pc ? *reinterpret_cast<const float4*>(&sm.XT[jr][k0]) : float4{};
                av[t] = pr ? *reinterpret_cast<const float4*>(&sm.aT[jr][k0]) : float4{};
                ev[t] = pr ? *reinterpret_cast<const float4*>(&sm.Es[i][k0]) : float4{};
            }
            const float w = active ? sm.Ws[i][jr] : 0.f;
            float c, r;
            ws_dots(breg, xv, av, ev, c, r);
            c += __shfl_xor_sync(0xffffffffu, c, 1);
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            c += __shfl_xor_sync(0xffffffffu, c, 2);
            r += __shfl_xor_sync(0xffffffffu, r, 2);
            if (active && q == 0) {
                sm.pre[d % WS_RING][i][0] = (w - c) - ct;
                sm.pre[d % WS_RING][i][1] = r + rt;
            }
            if (q == 0) tc::mbar_arrive(&sm.hbar[d % WS_RING]);
        }
    }
    if (!ok) {
        sm.abort_flag = 1;
        set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    }
    __syncthreads();
    KG_PAIR_TL(if (tid == 0 && tl) {
        tl[2] = pair_gtime();
        tl[3] = tl_wait[0];
        tl[4] = tl_wait[1];
        tl[5] = tl_wait[2];
    })
    if (*reinterpret_cast<volatile int*>(&sm.abort_flag) != 0) return;

    // ---- write back (as k_leaf_ws)
    constexpr int PER_ROW = T / VW;
    if (helper) {
        for (int f = tid; f < T * PER_ROW; f += WS_HELPERS) {
            const int rr = f / PER_ROW, cc = (f % PER_ROW) * VW;
            const int64_t gi = r0 + rr, gj = c0 + cc;
            const float4 evv = *reinterpret_cast<const float4*>(&sm.Es[rr][cc]);
            leaf_store_split(Ebuf, Elo, gi * Np + gj, evv);
            if (gi < m) {
                const float* es = reinterpret_cast<const float*>(&evv);
#pragma unroll
                for (int u = 0; u < VW; ++u) {
                    if (gj + u < n) {
                        store_code(codes, code_bytes, gi * n + gj + u, sm.Cs[rr][cc + u]);
                        V[gi * n + gj + u] = (float)sm.Cs[rr][cc + u] * sm.s[rr];
                        if (outE) outE[gi * n + gj + u] = es[u];
                    }
                }
            }
        }
    }
    for (int idx = tid; idx < T * T; idx += PAIR_THREADS) {
        const int cc = idx >> 6, rr = idx & 63;
        sm.XT[cc][rr] += sm.Rs[rr][cc];
    }
    __syncthreads();
    if (helper && XTg) {
        for (int f = tid; f < T * PER_ROW; f += WS_HELPERS) {
            const int cc = f / PER_ROW, rr = (f % PER_ROW) * VW;
            leaf_store_split(XTg, XTlo, (c0 + cc) * Mp + r0 + rr, *reinterpret_cast<const float4*>(&sm.XT[cc][rr]));
        }
    }
    KG_PAIR_TL(__syncthreads(); if (tid == 0 && tl) tl[7] = pair_gtime();)
}
}  // namespace kg
