// kg_leaf_ws.cuh -- the fp32 in-tile sweep ("leaf") with warp specialisation.
//
// Same in-tile problem as k_leaf in kg_leaf.cuh ("FastKron: Efficient Quantization with
// Kronecker-Factored Hessians", Sections 2.3-2.4, restated on one tile with a = U_A[J,J],
// b = U_B[I,I]):
//     w'   = W~[I,J] - b^T R[I,J]
//     r_ij = sum_{k<j} E_ik a[k][j],   c_ij = sum_{k<i} b[k][i] X_kj,   X_kj = r_kj + E_kj a[j][j]
//     x    = w'_ij - c_ij - b_ii r_ij,  code = clamp(rint(x / s_i)),  Q = s_i code,
//     E_ij = (x - Q) / (b_ii a_jj)
// and the same outputs, but the 127 steps of the sweep are split between roles:
//   * the rounding warp (warp 16) owns rows 2l and 2l+1 in lane l.  For entry (i, j) at step d
//     it takes the helpers' partial sums
//         P  = w'_ij - sum_{k<=i-6} b[k][i] X[k][j],     r' = sum_{k<=j-6} E[i][k] a[k][j]
//     and adds the ten newest terms itself: X of rows i-1..i-5 in column j and E of row i in
//     columns j-1..j-5 (made at steps d-1..d-5; X of row i-1 is the lane's own other row or one
//     shuffle away).  Only the terms of step d-1 are on its dependent chain.  It publishes E, X
//     and the code of every entry to shared memory.
//   * four groups of four helper warps (two threads per row) take the steps in turn: the group of
//     step d starts as soon as step d-6 is published, so each group has four rounding steps to
//     deliver (P, r') into an eight-slot ring.  A helper thread reads one column of X, one column
//     of a and one row of E in 16-byte chunks (k = 4q + 8t + u, the row's two threads interleaved)
//     and multiplies with packed fp32x2 FMAs; the row's U_B column stays in registers.  Reads of
//     entries published concurrently meet a zero coefficient (b and a are masked to k <= i-6 and
//     k <= j-6), so they cannot change a sum.
// Hand-off goes through mbarriers, one phase per pair of steps (steps 2p and 2p+1): the rounding
// warp arrives once it has published both, the helpers of both steps arrive on the pair's other
// barrier (128 arrivals; the last, unpaired step arrives twice), so each side waits once per two
// steps.  Arrival releases the writer's shared-memory stores, a waiting warp sleeps in try_wait,
// every wait is bounded in time, and on expiry the CTA records a time-out and skips the rest.  Each warp leaves as a whole: a helper warp takes lane
// 0's verdict; a rounding lane whose wait gives up raises the abort flag and skips its later
// waits, but still runs every step, so the warp's shuffles stay converged, and the warp votes
// once, after the last step.  The helpers of step s wait for the pair holding step s-6; the
// rounding warp waits for the pair of steps 2p, 2p+1 while it runs step 2p-1, and the helpers of
// those steps wait only for pair p-3, published after step 2p-5, so neither side waits on the other
// in a cycle.  No barrier slot (eight pairs) is reused before its previous phase was seen by every
// waiter: the rounding warp cannot start the steps of pair p+3 before the helpers waiting on pair p
// are done, long before it publishes pair p+8 into that slot again; the (P, r') slot of step s is
// refilled (for step s+8) only after step s+2 is published, and the rounding warp read it during
// step s-1.
#pragma once

#include "kg_common.cuh"
#include "kg_leaf.cuh"
#include "kg_tc.cuh"

namespace kg {

constexpr int WS_AHEAD = 6;                                  // helpers run this many steps ahead
constexpr int WS_RING = 8;                                   // slots of the (P, r') ring
constexpr int WS_GROUPS = 4;                                 // helper groups, taking steps in turn
constexpr int WS_TPR = 2;                                    // helper threads per row
constexpr int WS_GTHREADS = KG_T * WS_TPR;                   // threads per group (four warps)
constexpr int WS_HELPERS = WS_GTHREADS * WS_GROUPS;
constexpr int WS_THREADS = WS_HELPERS + 32;                  // + the rounding warp
#ifndef KG_TEST_HANDOFF_FAULT
constexpr long long WS_MAX_WAIT_CYCLES = 50000000LL;         // ~25 ms: far beyond any hand-off
#else
// Test build only (python -m two_sided_gptq_02_b200.build --define KG_TEST_HANDOFF_FAULT --out ...):
// a shorter limit, and a device switch that makes the helpers of row 0 in the first leaf (tile
// anti-diagonal 0) withhold their arrival for step 5, so that the rounding warp's bounded wait on
// that slot runs out.  The wait then gives up, the CTA raises its abort flag, every other wait of
// the CTA ends at its next check of the flag, and the leaf records KG_ERR_TIMEOUT and returns.
// Nothing faults or traps: the kernel only skips work.  The default build contains none of this.
constexpr long long WS_MAX_WAIT_CYCLES = 4000000LL;          // ~2 ms
__device__ int g_test_handoff_fault;
#endif

struct LeafWsSmem {
    static constexpr int S = LeafCfg<float>::S;
    float aT[KG_T][S];             // aT[j][k] = a[k][j] for k <= j - WS_AHEAD, else 0
    float Es[KG_T][S];             // errors E[i][k]; during set-up b row-major
    float XT[KG_T][S];             // XT[j][k] = X[k][j]; during set-up R row-major
    float Ws[KG_T][S];             // w'
    float Rs[KG_T][KG_T + 1];      // R tile as loaded, added to the local X at the end
                                   // (stride 65: the column walk is conflict-free)
    float colc[KG_T][8];           // column j: a[j-1][j] .. a[j-5][j], 1/a[j][j], a[j][j], unused
    float pre[WS_RING][KG_T][2];   // (P, r') of row i for step d, slot d % WS_RING
    float s[KG_T], invs[KG_T];
    int32_t Cs[KG_T][KG_T];        // codes (int32: the unclipped alphabet needs more than 8 bits)
    // near field (set-up only): the operands of the updates from the two adjacent tiles of the
    // previous tile anti-diagonal, each k-major ([k][row]) so that a thread reads four rows of one
    // k in one 16-byte load
    float Nel[KG_T][68];           // E of tile (I, J-1), transposed: [k][i] = E[i][k]
    float Nxu[KG_T][68];           // X of tile (I-1, J): [k][j]
    float Na[KG_T][68];            // U_A[J-1, J] block: [k][j]
    float Nb[KG_T][68];            // U_B[I-1, I] block: [k][i]
    uint64_t cbar[WS_RING];        // step d published (32 arrivals)
    uint64_t hbar[WS_RING];        // (P, r') of step d written (one arrival per row)
    int abort_flag;
};

// partial dots of one helper lane: c = sum breg * xv, r = sum ev * av over its NC chunks of 4 k
template <int NC>
__device__ __forceinline__ void ws_dots(const float (&breg)[NC][4], const float4 (&xv)[NC], const float4 (&av)[NC],
                                        const float4 (&ev)[NC], float& c, float& r) {
    float2 c0 = make_float2(0.f, 0.f), c1 = c0, r0 = c0, r1 = c0;
#pragma unroll
    for (int t = 0; t < NC; ++t) {
        c0 = __ffma2_rn(make_float2(breg[t][0], breg[t][1]), make_float2(xv[t].x, xv[t].y), c0);
        c1 = __ffma2_rn(make_float2(breg[t][2], breg[t][3]), make_float2(xv[t].z, xv[t].w), c1);
        r0 = __ffma2_rn(make_float2(ev[t].x, ev[t].y), make_float2(av[t].x, av[t].y), r0);
        r1 = __ffma2_rn(make_float2(ev[t].z, ev[t].w), make_float2(av[t].z, av[t].w), r1);
    }
    c = (c0.x + c0.y) + (c1.x + c1.y);
    r = (r0.x + r0.y) + (r1.x + r1.y);
}

// column constants of j: a1 .. a5, 1/ajj, ajj (and one unused word)
__device__ __forceinline__ void ws_ldcol(const float* p, float (&o)[8]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    const float4 u = *reinterpret_cast<const float4*>(p + 4);
    o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
    o[4] = u.x; o[5] = u.y; o[6] = u.z; o[7] = u.w;
}

// The rounding warp: lane l owns rows 2l (r = 0) and 2l+1 (r = 1).  The inputs of step d + 1
// (the helpers' (P, r') and the column constants) are loaded into one of two register sets while
// step d runs on the other; the step loop is unrolled by two so that the sets swap roles without a
// copy (a copy at the end of the step would wait for the loads it copies).
struct WsStepIn {
    float pre[4];      // (P, r') of rows 2l and 2l + 1
    float col[2][8];   // column constants of each row's column
};

// The helpers leave out the WS_AHEAD - 1 = 5 newest terms of each chain; the rounding warp adds
// them: E of its row in columns j-1 .. j-5 (its own, 1..5 steps old) and X of rows i-1 .. i-5 in
// column j.  Row i - k (k >= 1) of column j was made k steps ago by lane l - o, o = ceil((k - r)/2),
// as that lane's row of parity (r - k) & 1 (for r = 1, k = 1: the lane's own even row).  Each step
// the lane takes, by shuffle, the new X of lane l-1 (both rows), l-2 (both) and l-3 (odd row) and
// keeps them as long as they are needed: H<o><p>[t] is the X of row 2(l-o)+p made t steps ago.
__device__ __forceinline__ bool ws_round_warp(LeafWsSmem& sm, const float (&bii)[2], const float (&bk)[2][6],
                                              const float (&sr)[2], const float (&isr)[2], const float (&ib)[2],
                                              float fqmin, float fqmax) {
    constexpr int T = KG_T, NSTEP = 2 * KG_T - 1;
    const int l = threadIdx.x & 31;
    bool ok = true;   // this lane's waits so far
    auto load_step = [&](int d, WsStepIn& in) {
        // the helpers' sums arrive per pair of steps: wait once, before the pair's first step
        const int pr = d >> 1;
        if ((d & 1) == 0 && ok &&
            !tc::mbar_wait(&sm.hbar[pr % WS_RING], (uint32_t)((pr / WS_RING) & 1), WS_MAX_WAIT_CYCLES,
                           &sm.abort_flag)) {
            ok = false;
            sm.abort_flag = 1;   // wakes the helpers and the other lanes out of their waits
        }
        const float4 p = *reinterpret_cast<const float4*>(&sm.pre[d % WS_RING][2 * l][0]);
        in.pre[0] = p.x; in.pre[1] = p.y; in.pre[2] = p.z; in.pre[3] = p.w;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int j = d - 2 * l - r;
            ws_ldcol(&sm.colc[(unsigned)j < (unsigned)T ? j : 0][0], in.col[r]);
        }
    };
    float eh[2][6];   // eh[r][k]: own E of row r, k steps ago (k = 1..5)
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int k = 0; k < 6; ++k) eh[r][k] = 0.f;
    float H11[3] = {0.f, 0.f, 0.f}, H10[4] = {0.f, 0.f, 0.f, 0.f};
    float H21[5] = {0.f, 0.f, 0.f, 0.f, 0.f}, H20[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float H31[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float xe_1 = 0.f;   // own X of row 2l, 1 step ago
    auto step = [&](int d, const WsStepIn& cur, WsStepIn& nxt) {
        // prefetch the next step's inputs; the helpers are normally ahead
        if (d + 1 < NSTEP) load_step(d + 1, nxt);
        float e[2], X[2], code[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            // X[i-k][j], k = 1..5
            const float xm1 = r ? xe_1 : H11[1];
            const float xm2 = r ? H11[2] : H10[2];
            const float xm3 = r ? H10[3] : H21[3];
            const float xm4 = r ? H21[4] : H20[4];
            const float xm5 = r ? H20[5] : H31[5];
            const float* a = cur.col[r];
            const float P = cur.pre[2 * r], rh = cur.pre[2 * r + 1];
            // terms known before this step's chain starts
            const float rp = (((rh + eh[r][5] * a[4]) + eh[r][4] * a[3]) + eh[r][3] * a[2]) + eh[r][2] * a[1];
            const float base =
                ((((P - bk[r][5] * xm5) - bk[r][4] * xm4) - bk[r][3] * xm3) - bk[r][2] * xm2) - bii[r] * rp;
            // the chain: E[i][j-1] and X[i-1][j] were made at step d-1
            const float t1 = eh[r][1] * a[0];
            const float x = (base - bii[r] * t1) - bk[r][1] * xm1;
            code[r] = leaf_clamp(rintf(x * isr[r]), fqmin, fqmax);
            const float Q = code[r] * sr[r];
            e[r] = (x - Q) * (ib[r] * a[5]);
            X[r] = (rp + t1) + e[r] * a[6];
            const int j = d - 2 * l - r;
            if ((unsigned)j >= (unsigned)T) {
                e[r] = 0.f;
                X[r] = 0.f;
            }
        }
        const float n11 = __shfl_up_sync(0xffffffffu, X[1], 1);
        const float n10 = __shfl_up_sync(0xffffffffu, X[0], 1);
        const float n21 = __shfl_up_sync(0xffffffffu, X[1], 2);
        const float n20 = __shfl_up_sync(0xffffffffu, X[0], 2);
        const float n31 = __shfl_up_sync(0xffffffffu, X[1], 3);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = 2 * l + r, j = d - i;
            if ((unsigned)j < (unsigned)T) {
                sm.Es[i][j] = e[r];
                sm.XT[j][i] = X[r];
                sm.Cs[i][j] = (int32_t)code[r];
            }
        }
        if ((d & 1) == 1 || d == NSTEP - 1) tc::mbar_arrive(&sm.cbar[(d >> 1) % WS_RING]);
#pragma unroll
        for (int t = 2; t > 1; --t) H11[t] = H11[t - 1];
        H11[1] = n11;
#pragma unroll
        for (int t = 3; t > 1; --t) H10[t] = H10[t - 1];
        H10[1] = n10;
#pragma unroll
        for (int t = 4; t > 1; --t) H21[t] = H21[t - 1];
        H21[1] = n21;
#pragma unroll
        for (int t = 5; t > 1; --t) H20[t] = H20[t - 1];
        H20[1] = n20;
#pragma unroll
        for (int t = 5; t > 1; --t) H31[t] = H31[t - 1];
        H31[1] = n31;
        xe_1 = X[0];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int k = 5; k > 1; --k) eh[r][k] = eh[r][k - 1];
            eh[r][1] = e[r];
        }
    };
    WsStepIn s0, s1;
    load_step(0, s0);
    int d = 0;
    for (; d + 1 < NSTEP; d += 2) {
        step(d, s0, s1);
        step(d + 1, s1, s0);
    }
    step(d, s0, s1);   // NSTEP is odd: the last step
    return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(WS_THREADS, 1)
k_leaf_ws(int D, int Mt, int Nt, int64_t m, int64_t n, int64_t Np, int64_t Mp, float* __restrict__ Wt,
          float* __restrict__ R, float* __restrict__ Ebuf, float* __restrict__ Elo, float* __restrict__ XTg,
          float* __restrict__ XTlo, const float* __restrict__ UA, int64_t ldA, const float* __restrict__ UB,
          int64_t ldB, const float* __restrict__ sp, int qmin, int qmax, void* __restrict__ codes, int code_bytes,
          float* __restrict__ V, float* __restrict__ outE, DevStatus* status) {
    constexpr int T = KG_T;
    constexpr int VW = 4;
    constexpr int NC = T / (WS_TPR * VW);   // chunks per lane and dot product
    constexpr int A = WS_AHEAD;
    constexpr int PER_ROW_Z = T / VW;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LeafWsSmem& sm = *reinterpret_cast<LeafWsSmem*>(smem_raw);

    const int Imin = max(0, D - Nt + 1);
    const int I = Imin + blockIdx.x;
    const int J = D - I;
    const int tid = threadIdx.x;
    const bool helper = tid < WS_HELPERS;
    grid_dep_launch();
    const int64_t r0 = (int64_t)I * T, c0 = (int64_t)J * T;

    // ---- load: a^T (masked to k <= j-4) and the column constants, b row-major (masked) into
    //      Es, R into XT, W~ into Ws
    if (tid == 0) {
        sm.abort_flag = 0;
        for (int c = 0; c < WS_AHEAD - 1; ++c)
            for (int k = c; k < WS_AHEAD - 1; ++k) sm.colc[c][k] = 0.f;   // a[j-k-1][j] with j-k-1 < 0
    }
    // the adjacent tiles of the previous tile anti-diagonal: (I, J-1) sends its errors along the row
    // chain, (I-1, J) its X down the column chain
    const bool has_left = J > 0, has_up = I > 0;
    if (helper) {
        // the four tiles in one memory round trip: 512 threads x 8 float4.  The factor blocks a
        // (threads 0-255) and b (threads 256-511) as one 4 x 4 block per thread, a read down its
        // columns so that the transposed 16-byte stores of a quarter-warp land on distinct banks; R
        // and W~ as two float4 each.
        const float* src[4] = {UA + c0 * ldA + c0, UB + r0 * ldB + r0, R + r0 * Np + c0, Wt + r0 * Np + c0};
        const int64_t lds[4] = {ldA, ldB, Np, Np};
        const int fq = tid & 255, fa = tid < 256;
        const int fk = fa ? 4 * (fq & 15) : 4 * (fq >> 4);   // first row of the block
        const int fj = fa ? 4 * (fq >> 4) : 4 * (fq & 15);   // first column
        const float* fsrc = fa ? UA + c0 * ldA + c0 : UB + r0 * ldB + r0;
        const int64_t fld = fa ? ldA : ldB;
        // with the factor blocks of the near field: U_A[J-1, J] and U_B[I-1, I]
        float4 v[8], nf[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) {
            const int e = (f & 1) * WS_HELPERS + tid;
            const bool on = f < 2 ? has_left : has_up;
            const float* p = f < 2 ? UA + (c0 - T) * ldA + c0 : UB + (r0 - T) * ldB + r0;
            const int64_t ld = f < 2 ? ldA : ldB;
            nf[f] = on ? *reinterpret_cast<const float4*>(p + (int64_t)(e >> 4) * ld + (e & 15) * 4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int f = 0; f < 8; ++f) {
            // the factor tiles (f < 4) do not depend on earlier kernels of the solve: they load while
            // the previous kernel finishes; R and W~ (f >= 4) only after it has
            if (f == 4) grid_dep_wait();
            if (f < 4) {
                v[f] = *reinterpret_cast<const float4*>(fsrc + (int64_t)(fk + f) * fld + fj);
            } else {
                const int e = (f & 1) * WS_HELPERS + tid, tile = f >> 1;   // e: vector index in the tile
                v[f] = *reinterpret_cast<const float4*>(src[tile] + (int64_t)(e >> 4) * lds[tile] + (e & 15) * 4);
            }
        }
        // the near-field sources, written by the previous leaf: E of (I, J-1) (threads 0-255) and X^T of
        // (I-1, J) (threads 256-511), each as its two tf32 planes (hi + lo is the value to within 2^-22
        // relative).  A thread takes a 4 x 4 block (rows 4 (q >> 4) .., columns 4 (q & 15) ..) and
        // stores it transposed, so that both land k-major.
        const int q = tid & 255;
        const bool xside = tid >= 256, on = xside ? has_up : has_left;
        const float* hi = xside ? XTg + c0 * Mp + (r0 - T) : Ebuf + r0 * Np + (c0 - T);
        const float* lo = xside ? XTlo + c0 * Mp + (r0 - T) : Elo + r0 * Np + (c0 - T);
        const int64_t ldn = xside ? Mp : Np;
        float4 ns[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t off = (int64_t)(4 * (q >> 4) + u) * ldn + 4 * (q & 15);
            ns[u] = on ? *reinterpret_cast<const float4*>(hi + off) : make_float4(0.f, 0.f, 0.f, 0.f);
            ns[u + 4] = on ? *reinterpret_cast<const float4*>(lo + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int f = 0; f < 4; ++f) {
            const int e = (f & 1) * WS_HELPERS + tid, r = e >> 4, c4 = (e & 15) * 4;
            float* dst = f < 2 ? &sm.Na[r][c4] : &sm.Nb[r][c4];
            *reinterpret_cast<float4*>(dst) = nf[f];
        }
        {
            float blk[4][4];   // blk[u][w] = value at (row 4 (q >> 4) + u, column 4 (q & 15) + w)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                blk[u][0] = ns[u].x + ns[u + 4].x;
                blk[u][1] = ns[u].y + ns[u + 4].y;
                blk[u][2] = ns[u].z + ns[u + 4].z;
                blk[u][3] = ns[u].w + ns[u + 4].w;
            }
            float(*dstT)[68] = xside ? sm.Nxu : sm.Nel;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                *reinterpret_cast<float4*>(&dstT[4 * (q & 15) + w][4 * (q >> 4)]) =
                    make_float4(blk[0][w], blk[1][w], blk[2][w], blk[3][w]);
        }
        if (fa) {   // a: transposed, masked to k <= j - WS_AHEAD; the column constants
#pragma unroll
            for (int w = 0; w < 4; ++w) {   // v[u] = a[fk + u][fj .. fj + 3]
                const int c = fj + w;
                float o[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = fk + u;
                    const float x = w == 0 ? v[u].x : w == 1 ? v[u].y : w == 2 ? v[u].z : v[u].w;
                    o[u] = (r <= c - A) ? x : 0.f;
                    if (r == c) {
                        sm.colc[c][6] = x;
                        sm.colc[c][5] = 1.f / x;
                    } else if (r < c && r >= c - (WS_AHEAD - 1)) {
                        sm.colc[c][c - 1 - r] = x;   // a[c-k-1][c] at k = c - 1 - r
                    }
                }
                *reinterpret_cast<float4*>(&sm.aT[c][fk]) = make_float4(o[0], o[1], o[2], o[3]);
            }
        } else {   // b row-major, masked to the upper triangle
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = fk + u;
                const float4 x = v[u];
                *reinterpret_cast<float4*>(&sm.Es[r][fj]) =
                    make_float4(fj >= r ? x.x : 0.f, fj + 1 >= r ? x.y : 0.f, fj + 2 >= r ? x.z : 0.f,
                                fj + 3 >= r ? x.w : 0.f);
            }
        }
#pragma unroll
        for (int f = 4; f < 8; ++f) {
            const int e = (f & 1) * WS_HELPERS + tid, tile = f >> 1;
            const int r = e >> 4, c4 = (e & 15) * 4;
            const float* x = reinterpret_cast<const float*>(&v[f]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c4 + u;
                if (tile == 2) {   // R: for the fold (XT) and kept for the final X (Rs)
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
            tc::mbar_init(&sm.hbar[k], 2 * T);   // both steps of a pair, one arrival per row each
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // ---- near field: the updates from the adjacent tiles of tile anti-diagonal D - 1, which no
    //      update kernel carries:
    //        R  += E[I, J-1] U_A[J-1, J]          (threads 0-255)
    //        W~ -= U_B[I-1, I]^T X[I-1, J]        (threads 256-511)
    //      fp32, a 4 x 4 block per thread: rows 4 (q >> 4) .., columns 4 (q & 15) ..
    if (helper) {
        const int q = tid & 255, i0 = 4 * (q >> 4), j0 = 4 * (q & 15);
        const bool xside = tid >= 256;
        if (xside ? has_up : has_left) {
            float2 acc[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = make_float2(0.f, 0.f);
            const float(*A)[68] = xside ? sm.Nb : sm.Nel;   // [k][i]
            const float(*B)[68] = xside ? sm.Nxu : sm.Na;   // [k][j]
#pragma unroll 8
            for (int k = 0; k < T; ++k) {
                const float4 av = *reinterpret_cast<const float4*>(&A[k][i0]);
                const float4 bv = *reinterpret_cast<const float4*>(&B[k][j0]);
                const float2 b01 = make_float2(bv.x, bv.y), b23 = make_float2(bv.z, bv.w);
                const float ar[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc[u][0] = __ffma2_rn(make_float2(ar[u], ar[u]), b01, acc[u][0]);
                    acc[u][1] = __ffma2_rn(make_float2(ar[u], ar[u]), b23, acc[u][1]);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float o[4] = {acc[u][0].x, acc[u][0].y, acc[u][1].x, acc[u][1].y};
                if (xside) {
                    float4 wv = *reinterpret_cast<float4*>(&sm.Ws[i0 + u][j0]);
                    wv.x -= o[0]; wv.y -= o[1]; wv.z -= o[2]; wv.w -= o[3];
                    *reinterpret_cast<float4*>(&sm.Ws[i0 + u][j0]) = wv;
                } else {
                    float4 rv = *reinterpret_cast<float4*>(&sm.XT[i0 + u][j0]);   // R row-major in set-up
                    rv.x += o[0]; rv.y += o[1]; rv.z += o[2]; rv.w += o[3];
                    *reinterpret_cast<float4*>(&sm.XT[i0 + u][j0]) = rv;
#pragma unroll
                    for (int w = 0; w < 4; ++w) sm.Rs[i0 + u][j0 + w] += o[w];
                }
            }
        }
    }
    __syncthreads();

    // ---- per-row constants.  Helpers: U_B column of the row for k <= i-4 in registers.
    //      Rounding warp: b_ii, b[i-1][i], b[i-2][i], b[i-3][i], s_i for its two rows.
    const int ht = tid % WS_GTHREADS, g = tid / WS_GTHREADS;
    const int i = ht / WS_TPR, q = ht % WS_TPR;
    float breg[NC][VW];
#pragma unroll
    for (int t = 0; t < NC; ++t)
#pragma unroll
        for (int u = 0; u < VW; ++u) {
            const int k = VW * q + WS_TPR * VW * t + u;
            breg[t][u] = (helper && k <= i - A) ? sm.Es[k][i] : 0.f;
        }
    float bii[2], bk[2][6], sr[2], isr[2], ib[2];
    if (!helper) {
        const int l = tid & 31;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int ir = 2 * l + r;
            bii[r] = sm.Es[ir][ir];
            bk[r][0] = 0.f;
#pragma unroll
            for (int k = 1; k < 6; ++k) bk[r][k] = (ir >= k) ? sm.Es[ir - k][ir] : 0.f;
            sr[r] = sm.s[ir];
            isr[r] = sm.invs[ir];
            ib[r] = 1.f / bii[r];
        }
    }

    // ---- fold the external row chain: w' = W~ - b^T R  (b^T[i][k] = b[k][i] = 0 for k > i);
    //      512 threads, a 2 x 4 block each
    {
        const int ty = tid >> 4, tx = tid & 15;   // rows 2 ty, 2 ty + 1; columns 4 tx .. 4 tx + 3
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
        // Es and XT start the sweep at zero (unvisited entries contribute nothing)
        for (int idx = tid; idx < T * T / VW; idx += WS_THREADS) {
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(&sm.Es[idx / PER_ROW_Z][(idx % PER_ROW_Z) * VW]) = z;
            *reinterpret_cast<float4*>(&sm.XT[idx / PER_ROW_Z][(idx % PER_ROW_Z) * VW]) = z;
        }
    }
    __syncthreads();

    // ---- sweep
    const float fqmin = (float)qmin, fqmax = (float)qmax;
    bool ok = true;
    if (!helper) {
        ok = ws_round_warp(sm, bii, bk, sr, isr, ib, fqmin, fqmax);
    } else {
        for (int d = g; d < 2 * T - 1; d += WS_GROUPS) {
            if (d >= A) {
                // step d needs everything published up to step d-4; lane 0 waits for the warp
                const int dp = (d - A) >> 1;   // the pair holding step d - A
                bool w_ok = true;
                if ((tid & 31) == 0)
                    w_ok = tc::mbar_wait(&sm.cbar[dp % WS_RING], (uint32_t)((dp / WS_RING) & 1), WS_MAX_WAIT_CYCLES,
                                         &sm.abort_flag);
                __syncwarp();   // orders lane 0's acquire before the other lanes' reads
                w_ok = __shfl_sync(0xffffffffu, (int)w_ok, 0) != 0;
                if (!w_ok) {
                    ok = false;
                    break;
                }
            }
            const int j = d - i;
            const bool active = (unsigned)j < (unsigned)T;
            const int jr = active ? j : 0;
            float4 xv[NC], av[NC], ev[NC];
#pragma unroll
            for (int t = 0; t < NC; ++t) {
                const int k0 = VW * q + WS_TPR * VW * t;
                const bool pc = active && k0 <= i - A;
                const bool pr = active && k0 <= j - A;
                xv[t] = pc ? *reinterpret_cast<const float4*>(&sm.XT[jr][k0]) : float4{};
                av[t] = pr ? *reinterpret_cast<const float4*>(&sm.aT[jr][k0]) : float4{};
                ev[t] = pr ? *reinterpret_cast<const float4*>(&sm.Es[i][k0]) : float4{};
            }
            const float w = active ? sm.Ws[i][jr] : 0.f;
            float c, r;
            ws_dots(breg, xv, av, ev, c, r);
#pragma unroll
            for (int o = 1; o < WS_TPR; o <<= 1) {
                c += __shfl_xor_sync(0xffffffffu, c, o);
                r += __shfl_xor_sync(0xffffffffu, r, o);
            }
            if (active && q == 0) {
                sm.pre[d % WS_RING][i][0] = w - c;
                sm.pre[d % WS_RING][i][1] = r;
            }
#ifdef KG_TEST_HANDOFF_FAULT
            const bool withhold = g_test_handoff_fault != 0 && D == 0 && i == 0 && d == 5;
#else
            constexpr bool withhold = false;
#endif
            if (q == 0 && !withhold) {
                tc::mbar_arrive(&sm.hbar[(d >> 1) % WS_RING]);
                // the last step has no partner: it completes its pair's phase alone
                if (d == 2 * T - 2) tc::mbar_arrive(&sm.hbar[(d >> 1) % WS_RING]);
            }
        }
    }
    if (!ok) {
        sm.abort_flag = 1;   // wakes the other role out of its waits
        set_status(status, KG_ERR_TIMEOUT, (int)blockIdx.x);
    }
    __syncthreads();
    if (*reinterpret_cast<volatile int*>(&sm.abort_flag) != 0) return;

    // ---- write back: codes, V = s_i code, E (16-byte stores where the layout allows)
    constexpr int PER_ROW = T / VW;
    if (helper) {
        // whole 4-entry runs of codes, V and E go out as one store each when the run lies inside the
        // matrix and its addresses are aligned (the output pointers need not be)
        const bool vec_ok = (n & 3) == 0 && ((reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(outE)) & 15) == 0 &&
                            (reinterpret_cast<uintptr_t>(codes) & (code_bytes == 1 ? 3 : 15)) == 0;
        for (int f = tid; f < T * PER_ROW; f += WS_HELPERS) {
            const int rr = f / PER_ROW, cc = (f % PER_ROW) * VW;
            const int64_t gi = r0 + rr, gj = c0 + cc;
            const float4 evv = *reinterpret_cast<const float4*>(&sm.Es[rr][cc]);
            leaf_store_split(Ebuf, Elo, gi * Np + gj, evv);
            if (gi < m) {
                const int4 cv = *reinterpret_cast<const int4*>(&sm.Cs[rr][cc]);
                const float sv = sm.s[rr];
                const int64_t o = gi * n + gj;
                if (vec_ok && gj + VW <= n) {
                    if (code_bytes == 1)
                        *reinterpret_cast<char4*>(static_cast<int8_t*>(codes) + o) =
                            make_char4((signed char)cv.x, (signed char)cv.y, (signed char)cv.z, (signed char)cv.w);
                    else
                        *reinterpret_cast<int4*>(static_cast<int32_t*>(codes) + o) = cv;
                    *reinterpret_cast<float4*>(V + o) =
                        make_float4((float)cv.x * sv, (float)cv.y * sv, (float)cv.z * sv, (float)cv.w * sv);
                    if (outE) *reinterpret_cast<float4*>(outE + o) = evv;
                } else {
                    const float* es = reinterpret_cast<const float*>(&evv);
                    const int* cs = reinterpret_cast<const int*>(&cv);
#pragma unroll
                    for (int u = 0; u < VW; ++u) {
                        if (gj + u < n) {
                            store_code(codes, code_bytes, o + u, cs[u]);
                            V[o + u] = (float)cs[u] * sv;
                            if (outE) outE[o + u] = es[u];
                        }
                    }
                }
            }
        }
        // ---- the complete X = R + local X into XTg (X transposed, leading dimension Mp, split for the
        //      tensor-core update).  The updates read a solved tile's X only from there, so R itself is
        //      not written back.
        if (XTg) {
            for (int f = tid; f < T * PER_ROW; f += WS_HELPERS) {
                const int cc = f / PER_ROW, rr = (f % PER_ROW) * VW;
                float4 x = *reinterpret_cast<const float4*>(&sm.XT[cc][rr]);
                x.x += sm.Rs[rr][cc];
                x.y += sm.Rs[rr + 1][cc];
                x.z += sm.Rs[rr + 2][cc];
                x.w += sm.Rs[rr + 3][cc];
                leaf_store_split(XTg, XTlo, (c0 + cc) * Mp + r0 + rr, x);
            }
        }
    }
}

}  // namespace kg
