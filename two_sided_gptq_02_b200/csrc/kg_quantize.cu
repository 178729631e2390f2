// kg_quantize.cu -- two-sided GPTQ rounding (FastKron / BaKron) on 64x64 tiles.
//
// Algorithm ("FastKron: Efficient Quantization with Kronecker-Factored Hessians",
// Sections 2.2-2.5).  Entry (i,j) is rounded once every entry to its top-left has pushed
// its error; the error E_ij = (x - Q)/(U_B[i,i] U_A[j,j]) reaches entry (i',j') as
// U_B[i,i'] E_ij U_A[j,j'] (i' >= i, j' >= j).  The update factors through two chains,
// which is the associativity of the batched update W -= U_B^T E U_A (Section 2.4):
//     row chain     R[i,j] = sum_{j'<j} E[i,j'] U_A[j',j]          (along a row)
//                   X[i,j] = R[i,j] + E[i,j] U_A[j,j]              (complete once (i,j) is done)
//     column chain  C[i,j] = sum_{i'<i} U_B[i',i] X[i',j]          (down a column)
//     x_ij = W_ij - C_ij - U_B[i,i] R_ij .
// Only complete values are pushed (E along rows, X down columns), so every source/target
// pair costs one multiply-add and the total work is mn(m+n)/2 multiply-adds whatever the
// batching.
//
// Tiles.  W is cut into 64x64 tiles; tile (I,J) lies on tile anti-diagonal D = I + J.
// Tiles of one tile anti-diagonal are independent (Section 2.3).  The schedule is the
// recursion of Section 2.5 applied to ranges of tile anti-diagonals:
//     solve(D0, D1): if one diagonal: leaf(D0)
//                    else solve(D0, mid); push(D0 | mid | D1); solve(mid, D1)
// leaf(D)  -- every tile on D runs the in-tile anti-diagonal sweep (one CTA per tile);
// push     -- the band of tiles [D0, mid) sends its errors to the band [mid, D1): for each
//             target tile (I,J) in [mid, D1)
//               R[I,J]  += sum_{J': I+J' in [D0,mid)} E[I,J'] U_A[J',J]       (row chain)
//               W~[I,J] -= sum_{I': I'+J in [D0,mid)} U_B[I',I]^T X[I',J]     (column chain)
//             Both are dense GEMMs over contiguous K ranges.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "kg_blas.cuh"
#include "kg_common.cuh"
#include "kg_gemm.cuh"
#include "kg_leaf.cuh"
#include "kg_leaf_ws.cuh"
#include "kg_profile.cuh"
#include "kg_push_tc.cuh"
#include "kg_rc.cuh"

namespace kg {

constexpr int T = KG_T;

// ---------------------------------------------------------------------------------------
// Workspace layout (all offsets 256-byte aligned):
//   [status 256B][Wt Mp*Np][R Mp*Np][E Mp*Np][scale Mp][UApad Np*Np][UBpad Mp*Mp]
// Wt holds W minus the column chain, R holds the row chain of unsolved tiles.  The update reads
// a solved tile's complete X from R in fp64 and from the split X^T planes (below) in fp32, so
// only the fp64 leaf writes it back into R.  The padded factors exist only when m or n is not a multiple of 64; the pad
// is the identity, so padded entries have zero error and never touch real ones.
// ---------------------------------------------------------------------------------------
struct QLayout {
    int64_t m, n, Mt, Nt, Mp, Np;
    bool padded;
    size_t es;
    size_t off_wt, off_r, off_e, off_s, off_ua, off_ub;
    size_t off_elo, off_uat, off_uatlo, off_ubt, off_ubtlo, off_xt, off_xtlo, total;
};

static QLayout q_layout(int64_t m, int64_t n, size_t es) {
    QLayout L{};
    L.m = m; L.n = n; L.es = es;
    L.Mt = ceil_div(m, T); L.Nt = ceil_div(n, T);
    L.Mp = L.Mt * T; L.Np = L.Nt * T;
    L.padded = (L.Mp != m) || (L.Np != n);
    size_t off = kStatusBytes;
    L.off_wt = off; off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
    L.off_r = off;  off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
    L.off_e = off;  off = align_up(off + (size_t)(L.Mp * L.Np) * es, 256);
    L.off_s = off;  off = align_up(off + (size_t)L.Mp * es, 256);
    L.off_ua = off;
    if (L.padded) {
        off = align_up(off + (size_t)(L.Np * L.Np) * es, 256);
        L.off_ub = off;
        off = align_up(off + (size_t)(L.Mp * L.Mp) * es, 256);
    } else {
        L.off_ub = off;
    }
    L.off_elo = L.off_uat = L.off_uatlo = L.off_ubt = L.off_ubtlo = L.off_xt = L.off_xtlo = off;
    if (es == 4) {
        // the tensor-core update reads every operand K-major and pre-split into tf32 planes:
        // E (the E buffer above holds its hi plane), U_A^T, U_B^T and X^T
        auto plane = [&](size_t& o, int64_t elems) { o = off; off = align_up(off + (size_t)elems * es, 256); };
        plane(L.off_elo, L.Mp * L.Np);
        plane(L.off_uat, L.Np * L.Np);
        plane(L.off_uatlo, L.Np * L.Np);
        plane(L.off_ubt, L.Mp * L.Mp);
        plane(L.off_ubtlo, L.Mp * L.Mp);
        plane(L.off_xt, L.Np * L.Mp);
        plane(L.off_xtlo, L.Np * L.Mp);
    }
    L.total = off;
    return L;
}

// ------------------------------------------------------------------------------ init
template <typename Real>
__global__ void k_init_w(const Real* __restrict__ W, int64_t m, int64_t n, int64_t Np, int64_t Mp,
                         Real* __restrict__ Wt, Real* __restrict__ R, DevStatus* st) {
    const int64_t total = Mp * Np;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = p / Np, j = p % Np;
        Real v = Real(0);
        if (i < m && j < n) {
            v = W[i * n + j];
            if (!isfinite(v)) set_status(st, KG_ERR_NONFINITE, (int)(i * n + j));
        }
        Wt[p] = v;
        R[p] = Real(0);
    }
}

template <typename Real>
__global__ void k_init_scale(const Real* __restrict__ s, int64_t m, int64_t Mp, Real* __restrict__ sp,
                             DevStatus* st) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < Mp; i += (int64_t)gridDim.x * blockDim.x) {
        Real v = Real(1);
        if (i < m) {
            v = s[i];
            if (!isfinite(v) || !(v > Real(0))) { set_status(st, KG_ERR_NONFINITE, (int)i); v = Real(1); }
        }
        sp[i] = v;
    }
}

// Copy an upper-triangular factor into a padded buffer with identity padding, zeroing the
// strictly lower triangle; also validates the diagonal.
template <typename Real>
__global__ void k_pad_factor(const Real* __restrict__ U, int64_t k, int64_t kp, Real* __restrict__ Up,
                             DevStatus* st) {
    const int64_t total = kp * kp;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < total; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = p / kp, c = p % kp;
        Real v = Real(0);
        if (r < k && c < k) {
            if (c >= r) v = U[r * k + c];
        } else if (r == c) {
            v = Real(1);
        }
        Up[p] = v;
    }
}

template <typename Real>
__global__ void k_check_diag2(const Real* __restrict__ UA, int64_t n, const Real* __restrict__ UB, int64_t m,
                              DevStatus* st) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n || i < m; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < n) {
            const Real d = UA[i * n + i];
            if (!isfinite(d) || !(d > Real(0))) set_status(st, KG_ERR_NONFINITE, (int)i);
        }
        if (i < m) {
            const Real d = UB[i * m + i];
            if (!isfinite(d) || !(d > Real(0))) set_status(st, KG_ERR_NONFINITE, (int)i);
        }
    }
}

// ------------------------------------------------------------------------------ push
// Sources: diagonals [D0, mid); targets: diagonals [tgt0, D1) with tgt0 >= mid (a band may be
// updated in parts).  Grid: x = position along a target diagonal, y = target diagonal offset from
// tgt0, z = chain (0: row chain into R, 1: column chain into W~).
__global__ void __launch_bounds__(Dmma64::kThreads)
k_push_f64(int D0, int mid, int tgt0, int Mt, int Nt, int64_t Np,
           double* __restrict__ Wt, double* __restrict__ R, const double* __restrict__ E,
           const double* __restrict__ UA, int64_t ldA, const double* __restrict__ UB, int64_t ldB) {
    using PipeRow = DmmaPipe<false, false>;   // A = rows of E,  B = rows of U_A
    using PipeCol = DmmaPipe<true, false>;    // A = U_B (stored K x 64), B = rows of X
    constexpr size_t kSmem = sizeof(PipeRow::Smem) > sizeof(PipeCol::Smem) ? sizeof(PipeRow::Smem)
                                                                            : sizeof(PipeCol::Smem);
    __shared__ __align__(16) unsigned char smem[kSmem];
    const int D = tgt0 + blockIdx.y;
    const int I = max(0, D - Nt + 1) + blockIdx.x;
    if (I > min(D, Mt - 1)) return;
    const int J = D - I;
    grid_dep_launch();
    grid_dep_wait();   // programmatic launch: the previous kernel's writes are visible from here
    Dmma64::Acc acc;
    Dmma64::zero(acc);
    if (blockIdx.z == 0) {
        const int k0 = max(0, D0 - I), k1 = min(Nt, mid - I);
        if (k0 >= k1) return;
        PipeRow::run(acc, *reinterpret_cast<PipeRow::Smem*>(smem), (k1 - k0) * T,
                     E + (int64_t)I * T * Np + (int64_t)k0 * T, Np, UA + (int64_t)k0 * T * ldA + (int64_t)J * T, ldA);
        Dmma64::add_to(acc, R + (int64_t)I * T * Np + (int64_t)J * T, Np, 1.0);
    } else {
        const int k0 = max(0, D0 - J), k1 = min(Mt, mid - J);
        if (k0 >= k1) return;
        PipeCol::run(acc, *reinterpret_cast<PipeCol::Smem*>(smem), (k1 - k0) * T,
                     UB + (int64_t)k0 * T * ldB + (int64_t)I * T, ldB, R + (int64_t)k0 * T * Np + (int64_t)J * T, Np);
        Dmma64::add_to(acc, Wt + (int64_t)I * T * Np + (int64_t)J * T, Np, -1.0);
    }
}

// ------------------------------------------------------------------------------ driver
template <typename Real>
struct QArgs {
    QLayout L;
    Real *Wt, *R, *E, *sp;
    const Real *UA, *UB;
    int64_t ldA, ldB;
    int qmin, qmax;
    void* codes;
    int code_bytes;   // 1: int8 codes, 4: int32 codes
    Real* V;
    Real* outE;
    cudaStream_t st;
    DevStatus* status;
    // split K-major operand planes of the tensor-core path (fp32 only; null otherwise)
    Real *Elo, *XT, *XTlo, *UAT, *UATlo, *UBT, *UBTlo;
    // their tensor maps (fp32 only)
    const PushTmaMaps* maps;
};

// Launch with programmatic stream serialization when pdl is set: the kernel may start while the
// previous kernel of the stream finishes, and waits for it inside (grid_dep_wait).
template <typename... KArgs, typename... Args>
static int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                    Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // the stream's priority on the launch itself, so that it survives stream capture into a graph
    // (a captured kernel node does not inherit the priority of the stream it was captured from)
    int prio = 0;
    if (cudaStreamGetPriority(st, &prio) != cudaSuccess) return KG_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributePriority;
    attr[0].val.priority = prio;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? KG_OK : KG_ERR_CUDA;
}

template <typename Real>
static int launch_leaf(const QArgs<Real>& a, int D, cudaStream_t st) {
    const int Mt = (int)a.L.Mt, Nt = (int)a.L.Nt;
    const int Imin = std::max(0, D - Nt + 1), Imax = std::min(D, Mt - 1);
    const int ntiles = Imax - Imin + 1;
    ProfScope ps(PK_LEAF, st);
    if constexpr (sizeof(Real) == 4) {
        return launch_k(k_leaf_ws, dim3(ntiles), dim3(WS_THREADS), sizeof(LeafWsSmem), st, true, D, Mt, Nt, a.L.m,
                        a.L.n, a.L.Np, a.L.Mp, a.Wt, a.R, a.E, a.Elo, a.XT, a.XTlo, a.UA, a.ldA, a.UB, a.ldB, a.sp,
                        a.qmin, a.qmax, a.codes, a.code_bytes, a.V, a.outE, a.status);
    } else {
        return launch_k(k_leaf<Real>, dim3(ntiles), dim3(256), sizeof(LeafSmem<Real>), st, true, D, Mt, Nt, a.L.m,
                        a.L.n, a.L.Np, a.L.Mp, a.Wt, a.R, a.E, a.Elo, a.XT, a.XTlo, a.UA, a.ldA, a.UB, a.ldB, a.sp,
                        a.qmin, a.qmax, a.codes, a.code_bytes, a.V, a.outE);
    }
}


// Update of the targets on diagonals [tgt0, D1) from the sources on diagonals [D0, mid).
static int launch_push(const QArgs<double>& a, int D0, int mid, int tgt0, int D1, cudaStream_t st, bool pdl) {
    const int Mt = (int)a.L.Mt, Nt = (int)a.L.Nt;
    ProfScope ps(PK_PUSH, st);
    return launch_k(k_push_f64, dim3(std::min(Mt, Nt), D1 - tgt0, 2), dim3(Dmma64::kThreads), 0, st, pdl, D0, mid,
                    tgt0, Mt, Nt, a.L.Np, a.Wt, a.R, (const double*)a.E, a.UA, a.ldA, a.UB, a.ldB);
}
static int launch_push(const QArgs<float>& a, int D0, int mid, int tgt0, int D1, cudaStream_t st, bool pdl) {
    const int Mt = (int)a.L.Mt, Nt = (int)a.L.Nt;
    // one CTA per (operand tiles) x (target tiles), the variant, grid and CTA order of push_variant,
    // push_grid and push_cta
    ProfScope ps(PK_PUSH, st);
    const int v = push_variant(D0, mid, tgt0, D1);
    const dim3 grid = push_grid(v, tgt0, D1, Mt, Nt);
    if (v == PV_PAIR)
        return launch_k(k_push_tc32<2>, grid, dim3(PushCfg<2>::THREADS), PushCfg<2>::SMEM_BYTES, st, pdl, D0, mid,
                        tgt0, D1, Mt, Nt, a.L.Np, a.Wt, a.R, *a.maps, a.status);
    if (v == PV_SINGLE)
        return launch_k(k_push_tc32<1, 1>, grid, dim3(PushCfg<1, 1>::THREADS), PushCfg<1, 1>::SMEM_BYTES, st, pdl,
                        D0, mid, tgt0, D1, Mt, Nt, a.L.Np, a.Wt, a.R, *a.maps, a.status);
    return launch_k(k_push_tc32<1>, grid, dim3(PushCfg<1>::THREADS), PushCfg<1>::SMEM_BYTES, st, pdl, D0, mid, tgt0,
                    D1, Mt, Nt, a.L.Np, a.Wt, a.R, *a.maps, a.status);
}

// ---------------------------------------------------------------------------------------
// Schedule.  The recursion fixes which update carries each (source, target) pair of tile
// anti-diagonals: push(D0 | mid | D1) sends sources [D0, mid) to targets [mid, D1).  Its parts are
// needed at different times, so each push is cut into pieces; a piece (sources [s0, s1), targets
// [t0, t1)) may start once leaf s1 - 1 is done and is due when leaf t0 starts.  The source range is
// first halved from the old end while it is wider than kUrgentK: each half [a, h) goes to all the
// targets at once and is free after leaf h - 1, long before it is due (background stream).  The last
// chunk [c, mid), at most kUrgentK wide, is cut by target:
//   near  source mid-1 -> target mid: the adjacent tiles only; the fp32 leaf of mid computes it in
//         its set-up, in fp64 an update on the critical stream runs it between leaves mid-1 and mid;
//   far   sources [c, mid-1) -> target mid: free one leaf before it is due, beside leaf mid-1;
//   next  sources [c, mid) -> target mid+1: likewise beside leaf mid;     (both: urgent stream)
//   rest  sources [c, mid) -> targets [mid+2, D1), in pieces of 2, 4, 8, ... target diagonals, each
//         due at the leaf of its first target (soon stream).
// Streams, by priority: critical and urgent at the device's greatest, soon in the middle,
// background at the least, so that waiting blocks of the critical path start first on the SMs the
// leaves leave idle.
// Hazards: a piece waits for the leaf that completes its sources (an event per leaf on the critical
// stream) and for the latest piece of any other stream that targets one of its diagonals (tracked
// per diagonal and stream); a stream runs its own pieces in order.  Every piece that targets
// diagonal d is free by leaf d-2, so it is issued before the near piece and the leaf of d, which
// wait for it; nothing targets d after that.  Every wait binds to an event recorded by work issued earlier, so
// the waits cannot form a cycle.  The caller's stream forks the streams at the start and waits for
// all of them at the end (on the error path too).
// ---------------------------------------------------------------------------------------
enum SchedStream : int { SS_CRIT = 0, SS_URGENT = 1, SS_SOON = 2, SS_BACK = 3, SS_COUNT = 4 };
constexpr int kUrgentK = 4;   // widest source range of the last chunk, in tile anti-diagonals

struct Piece {
    int s0, s1;   // sources: tile anti-diagonals [s0, s1)
    int t0, t1;   // targets: tile anti-diagonals [t0, t1)
    int stream;
};

// The pieces of push(D0 | mid | D1) other than the near one, each appended to free_at[the leaf
// after which it may start].
static void push_pieces(int D0, int mid, int D1, std::vector<std::vector<Piece>>& free_at) {
    int c = D0;
    while (mid - c > kUrgentK) {
        const int h = (c + mid) / 2;
        free_at[h - 1].push_back(Piece{c, h, mid, D1, SS_BACK});
        c = h;
    }
    if (c < mid - 1) free_at[mid - 2].push_back(Piece{c, mid - 1, mid, mid + 1, SS_URGENT});    // far
    if (mid + 1 < D1) free_at[mid - 1].push_back(Piece{c, mid, mid + 1, mid + 2, SS_URGENT});   // next
    for (int t0 = mid + 2, w = 2; t0 < D1; t0 += w, w *= 2)                                     // rest
        free_at[mid - 1].push_back(Piece{c, mid, t0, std::min(D1, t0 + w), SS_SOON});
}

static void plan_pieces(int D0, int D1, std::vector<std::vector<Piece>>& free_at) {
    if (D1 - D0 <= 1) return;
    const int mid = (D0 + D1) / 2;
    plan_pieces(D0, mid, free_at);
    push_pieces(D0, mid, D1, free_at);
    plan_pieces(mid, D1, free_at);
}

// Per host thread and device: a few sets of the four streams with their events, created on first
// use and kept for the life of the process (a thread that exits leaves its slots allocated; nothing
// is destroyed at exit, when the CUDA runtime may already be gone).  Calls take them in turn, so
// that solves in flight at the same time on different caller streams (several layers at once) run
// side by side; two calls that share a slot only serialise.
static constexpr int kSchedSlots = 8;
static constexpr int kSchedEvents = 64;   // ring of events per stream, and one for the leaves
struct SchedSlot {
    cudaStream_t s[SS_COUNT] = {};
    cudaEvent_t fork = nullptr;
    cudaEvent_t join[SS_COUNT] = {};
    std::vector<cudaEvent_t> ev[SS_COUNT];
    std::vector<cudaEvent_t> leaf_ev;
};
struct SchedPool {
    int dev = -1;
    unsigned next = 0;
    std::vector<SchedSlot> slots;
};

static int sched_slot(SchedSlot*& out) {
    static thread_local std::vector<SchedPool> pools;
    int dev = 0;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    SchedPool* pool = nullptr;
    for (auto& p : pools)
        if (p.dev == dev) pool = &p;
    if (!pool) {
        int least = 0, greatest = 0;
        KG_CUDA_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
        SchedPool p;
        p.dev = dev;
        p.slots.resize(kSchedSlots);
        auto mk = [](cudaEvent_t* e) { return cudaEventCreateWithFlags(e, cudaEventDisableTiming); };
        for (auto& sl : p.slots) {
            for (int k = 0; k < SS_COUNT; ++k) {
                const int prio = k == SS_BACK ? least : k == SS_SOON ? (least + greatest) / 2 : greatest;
                KG_CUDA_TRY(cudaStreamCreateWithPriority(&sl.s[k], cudaStreamNonBlocking, prio));
                KG_CUDA_TRY(mk(&sl.join[k]));
                sl.ev[k].resize(kSchedEvents);
                for (auto& e : sl.ev[k]) KG_CUDA_TRY(mk(&e));
            }
            KG_CUDA_TRY(mk(&sl.fork));
            sl.leaf_ev.resize(kSchedEvents);
            for (auto& e : sl.leaf_ev) KG_CUDA_TRY(mk(&e));
        }
        pools.push_back(std::move(p));
        pool = &pools.back();
    }
    out = &pool->slots[pool->next++ % pool->slots.size()];
    return KG_OK;
}

struct Sched {
    SchedSlot* sl;
    int seq[SS_COUNT] = {-1, -1, -1, -1};              // latest piece per stream
    int waited[SS_COUNT][SS_COUNT];                    // [S][o]: latest piece of o that S waits for
    int leaf_waited[SS_COUNT] = {-1, -1, -1, -1};      // latest leaf that S waits for
    std::vector<std::array<int, SS_COUNT>> pending;    // per diagonal: latest piece per stream on it
};

// Stream S is about to write targets [t0, t1): wait for the latest piece of every other stream
// that targets one of them.  A ring slot may since have been re-recorded by a later piece of the
// same stream; the wait then covers that one too, which is only conservative.
static int sched_hazards(Sched& s, int S, int t0, int t1) {
    for (int o = 0; o < SS_COUNT; ++o) {
        if (o == S) continue;
        int need = -1;
        for (int t = t0; t < t1; ++t) need = std::max(need, s.pending[t][o]);
        if (need > s.waited[S][o]) {
            KG_CUDA_TRY(cudaStreamWaitEvent(s.sl->s[S], s.sl->ev[o][need % kSchedEvents], 0));
            s.waited[S][o] = need;
        }
    }
    return KG_OK;
}

template <typename Real>
static int sched_piece(const QArgs<Real>& a, Sched& s, const Piece& p) {
    const int S = p.stream;
    int rc;
    if (p.s1 - 1 > s.leaf_waited[S]) {
        KG_CUDA_TRY(cudaStreamWaitEvent(s.sl->s[S], s.sl->leaf_ev[(p.s1 - 1) % kSchedEvents], 0));
        s.leaf_waited[S] = p.s1 - 1;
    }
    if ((rc = sched_hazards(s, S, p.t0, p.t1))) return rc;
    if ((rc = launch_push(a, p.s0, p.s1, p.t0, p.t1, s.sl->s[S], false))) return rc;
    const int q = ++s.seq[S];
    KG_CUDA_TRY(cudaEventRecord(s.sl->ev[S][q % kSchedEvents], s.sl->s[S]));
    for (int t = p.t0; t < p.t1; ++t) s.pending[t][S] = q;
    return KG_OK;
}

// The order in which the solve issues its work: for every leaf L, the near piece of L (L > 0), the
// leaf itself (a Piece with stream -1 and s0 = s1 = t0 = L, t1 = L + 1), then the pieces that leaf
// L frees, earliest due first.
static std::vector<Piece> issue_order(int ndiag) {
    std::vector<std::vector<Piece>> free_at(ndiag);
    plan_pieces(0, ndiag, free_at);
    std::vector<Piece> order;
    for (int L = 0; L < ndiag; ++L) {
        if (L > 0) order.push_back(Piece{L - 1, L, L, L + 1, SS_CRIT});
        order.push_back(Piece{L, L, L, L + 1, -1});
        std::stable_sort(free_at[L].begin(), free_at[L].end(),
                         [](const Piece& x, const Piece& y) { return x.t0 < y.t0; });
        order.insert(order.end(), free_at[L].begin(), free_at[L].end());
    }
    return order;
}

template <typename Real>
static int solve_leaves(const QArgs<Real>& a, Sched& s, int ndiag) {
    const std::vector<Piece> order = issue_order(ndiag);
    cudaStream_t crit = s.sl->s[SS_CRIT];
    int rc;
    for (size_t k = 0; k < order.size(); ++k) {
        const Piece& p = order[k];
        if (p.stream == SS_CRIT) {
            // near piece: the fp32 leaf computes it itself in its set-up; in fp64 an update kernel
            // runs it just before the leaf (both launched back to back, programmatic launch)
            if constexpr (sizeof(Real) == 8) {
                if ((rc = sched_hazards(s, SS_CRIT, p.t0, p.t1))) return rc;
                if ((rc = launch_push(a, p.s0, p.s1, p.t0, p.t1, crit, true))) return rc;
            }
        } else if (p.stream < 0) {
            const int L = p.t0;
            if ((rc = sched_hazards(s, SS_CRIT, L, L + 1))) return rc;
            if ((rc = launch_leaf(a, L, crit))) return rc;
            if (k + 1 < order.size() && order[k + 1].stream > 0)   // pieces freed by this leaf follow
                KG_CUDA_TRY(cudaEventRecord(s.sl->leaf_ev[L % kSchedEvents], crit));
        } else if ((rc = sched_piece(a, s, p))) {
            return rc;
        }
    }
    return KG_OK;
}

template <typename Real>
static int solve_all(const QArgs<Real>& a, int ndiag) {
    SchedSlot* slot = nullptr;
    int rc = sched_slot(slot);
    if (rc) return rc;
    Sched s;
    s.sl = slot;
    for (auto& w : s.waited)
        for (int& x : w) x = -1;
    s.pending.assign(ndiag + 1, std::array<int, SS_COUNT>{-1, -1, -1, -1});
    KG_CUDA_TRY(cudaEventRecord(slot->fork, a.st));
    for (int k = 0; k < SS_COUNT; ++k) KG_CUDA_TRY(cudaStreamWaitEvent(slot->s[k], slot->fork, 0));
    rc = solve_leaves(a, s, ndiag);
    // join: the caller's stream waits for all of them (also on the error path, so that no stream runs
    // past the caller's view of the solve)
    for (int k = 0; k < SS_COUNT; ++k) {
        KG_CUDA_TRY(cudaEventRecord(slot->join[k], slot->s[k]));
        KG_CUDA_TRY(cudaStreamWaitEvent(a.st, slot->join[k], 0));
    }
    return rc;
}

template <typename Real>
static int solve_antidiagonal(const QArgs<Real>& a, int ndiag, unsigned char* extra);

// codes: int8 (code_bytes 1) or int32 (code_bytes 4).  reset_status: clear the status word first;
// a caller that ran checks of its own into it before the solve passes false.  anti_extra: when
// given, the solve is the non-recursive anti-diagonal baseline (fp64) with its extra workspace.
template <typename Real>
static int quantize_impl(const void* W, int64_t m, int64_t n, const void* UA_, const void* UB_, kg_grid grid,
                         void* codes, int code_bytes, void* V, void* outE, void* ws, size_t ws_bytes,
                         cudaStream_t st, bool reset_status = true, unsigned char* anti_extra = nullptr) {
    const QLayout L = q_layout(m, n, sizeof(Real));
    if (ws_bytes < L.total) return KG_ERR_WORKSPACE;
    unsigned char* base = static_cast<unsigned char*>(ws);
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    QArgs<Real> a;
    a.L = L;
    a.Wt = reinterpret_cast<Real*>(base + L.off_wt);
    a.R = reinterpret_cast<Real*>(base + L.off_r);
    a.E = reinterpret_cast<Real*>(base + L.off_e);
    a.sp = reinterpret_cast<Real*>(base + L.off_s);
    a.qmin = grid.qmin; a.qmax = grid.qmax;
    a.codes = codes;
    a.code_bytes = code_bytes;
    a.V = static_cast<Real*>(V);
    a.outE = static_cast<Real*>(outE);
    a.st = st;
    a.status = status;

    if (reset_status) KG_CUDA_TRY(cudaMemsetAsync(status, 0, kStatusBytes, st));
    const int nb = 148 * 4;
    {
        ProfScope ps(PK_INIT, st);
        k_init_w<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(W), m, n, L.Np, L.Mp, a.Wt, a.R, status);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_init_scale<Real><<<std::max<int64_t>(1, std::min<int64_t>(nb, ceil_div(L.Mp, 256))), 256, 0, st>>>(
            static_cast<const Real*>(grid.row_scale), m, L.Mp, a.sp, status);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_check_diag2<Real><<<std::max<int64_t>(1, ceil_div(std::max(m, n), 256)), 256, 0, st>>>(
            static_cast<const Real*>(UA_), n, static_cast<const Real*>(UB_), m, status);
    }
    KG_LAUNCH_CHECK();
    if (L.padded) {
        Real* UAp = reinterpret_cast<Real*>(base + L.off_ua);
        Real* UBp = reinterpret_cast<Real*>(base + L.off_ub);
        {
            ProfScope ps(PK_INIT, st);
            k_pad_factor<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(UA_), n, L.Np, UAp, status);
        }
        KG_LAUNCH_CHECK();
        {
            ProfScope ps(PK_INIT, st);
            k_pad_factor<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(UB_), m, L.Mp, UBp, status);
        }
        KG_LAUNCH_CHECK();
        a.UA = UAp; a.ldA = L.Np;
        a.UB = UBp; a.ldB = L.Mp;
    } else {
        a.UA = static_cast<const Real*>(UA_); a.ldA = n;
        a.UB = static_cast<const Real*>(UB_); a.ldB = m;
    }
    a.Elo = a.XT = a.XTlo = a.UAT = a.UATlo = a.UBT = a.UBTlo = nullptr;
    a.maps = nullptr;
    PushTmaMaps maps;
    if (sizeof(Real) == 4) {
        a.Elo = reinterpret_cast<Real*>(base + L.off_elo);
        a.UAT = reinterpret_cast<Real*>(base + L.off_uat);
        a.UATlo = reinterpret_cast<Real*>(base + L.off_uatlo);
        a.UBT = reinterpret_cast<Real*>(base + L.off_ubt);
        a.UBTlo = reinterpret_cast<Real*>(base + L.off_ubtlo);
        a.XT = reinterpret_cast<Real*>(base + L.off_xt);
        a.XTlo = reinterpret_cast<Real*>(base + L.off_xtlo);
        const SplitOperands op{reinterpret_cast<const float*>(a.E), reinterpret_cast<const float*>(a.Elo),
                               reinterpret_cast<const float*>(a.XT), reinterpret_cast<const float*>(a.XTlo),
                               reinterpret_cast<const float*>(a.UAT), reinterpret_cast<const float*>(a.UATlo),
                               reinterpret_cast<const float*>(a.UBT), reinterpret_cast<const float*>(a.UBTlo)};
        if (!push_tma_maps(&maps, op, L.Np, L.Mp)) return KG_ERR_CUDA;
        a.maps = &maps;
        {
            ProfScope ps(PK_INIT, st);
            k_transpose_split<<<nb, 256, 0, st>>>(reinterpret_cast<const float*>(a.UA), L.Np, a.ldA,
                                                  reinterpret_cast<float*>(a.UAT), reinterpret_cast<float*>(a.UATlo));
        }
        KG_LAUNCH_CHECK();
        {
            ProfScope ps(PK_INIT, st);
            k_transpose_split<<<nb, 256, 0, st>>>(reinterpret_cast<const float*>(a.UB), L.Mp, a.ldB,
                                                  reinterpret_cast<float*>(a.UBT), reinterpret_cast<float*>(a.UBTlo));
        }
        KG_LAUNCH_CHECK();
    }
    if (anti_extra) return solve_antidiagonal(a, (int)(L.Mt + L.Nt - 1), anti_extra);
    return solve_all(a, (int)(L.Mt + L.Nt - 1));
}

// Kernel attributes are per device: configure each device once (guarded by a mutex).
static std::mutex g_cfg_mu;
static bool g_cfg_done[2][256] = {};

template <typename Real>
static int configure_leaf() {
    const int idx = sizeof(Real) == 8 ? 1 : 0;
    int dev = 0;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 256) return KG_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_cfg_mu);
    if (!g_cfg_done[idx][dev]) {
        // The solve alternates leaf and update launches.  All of them ask for the largest
        // shared-memory carveout, so the SMs never switch their L1 / shared split between two
        // launches of one solve.
        if (idx == 0) {
            KG_CUDA_TRY(cudaFuncSetAttribute(k_leaf_ws, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sizeof(LeafWsSmem)));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_leaf_ws, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             PushCfg<1>::SMEM_BYTES));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<1>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             PushCfg<1, 1>::SMEM_BYTES));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<1, 1>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             PushCfg<2>::SMEM_BYTES));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_tc32<2>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
        } else {
            KG_CUDA_TRY(cudaFuncSetAttribute(k_leaf<double>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sizeof(LeafSmem<double>)));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_leaf<double>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
            KG_CUDA_TRY(cudaFuncSetAttribute(k_push_f64, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared));
        }
        g_cfg_done[idx][dev] = true;
    }
    return KG_OK;
}

}  // namespace kg

using namespace kg;

extern "C" size_t kron_gptq_quantize_workspace_size(int64_t m, int64_t n, int dtype) {
    if (m < 0 || n < 0) return 0;
    if (dtype != KG_F32 && dtype != KG_F64) return 0;
    if (m == 0 || n == 0) return kStatusBytes;
    return q_layout(m, n, dtype == KG_F64 ? 8 : 4).total;
}

// ---------------------------------------------------------------------------------------
// Replays.  A solve is a few hundred launches on five streams.  The leaves' launches wait on events
// of the piece streams, and such a wait keeps a leaf from starting early while the previous leaf
// finishes; captured into a CUDA graph, the same work keeps its programmatic edges beside the
// ordinary ones (4096^2 fp32: 7.14 -> 6.71 ms a solve, bit-identical results).  So
// kron_gptq_quantize (and kron_gptq_quantize_rc, whose solve is the same) replays a captured graph
// when the same arguments come back on the same device:
// the first call with a given set runs directly, the second is captured (on a stream of the
// library's own: the caller's may be the legacy default stream, which cannot capture) and launched
// on the caller's stream, later ones replay it there.  fp32 only (the fp64 solve, whose leaves take
// twice as long, measured 14.12 ms direct and 14.46 ms replayed), and not when the caller's stream
// is capturing already (its capture gets the plain launches), while the event profiler is on, or for
// layers of more than kGraphMaxDiag tile anti-diagonals (14336x4096: a replay measured 4 % slower
// than direct launches).
// KRON_GPTQ_GRAPHS=0 in the environment turns replays off.  Each host thread keeps its own cache of
// at most kGraphCache entries (the least recently used is dropped first); nothing is destroyed at
// thread or process exit, when the CUDA runtime may already be gone.
// ---------------------------------------------------------------------------------------
constexpr int kGraphMaxDiag = 160;
constexpr int kGraphCache = 32;

// Every argument that shapes a call's launches, as words (zero-filled first: compared bytewise).
struct GraphKey {
    uint64_t w[16];
};
struct GraphEntry {
    GraphKey key;
    cudaGraphExec_t exec;   // null: seen once, or capture not possible for this key
    bool no_graph;
    int64_t launches[PK_COUNT];
    uint64_t last_use;
};

static bool graphs_allowed() {
    static const bool on = [] {
        const char* e = std::getenv("KRON_GPTQ_GRAPHS");
        return !(e && e[0] == '0');
    }();
    return on;
}

// Run a call whose launches run(s) issues on stream s: directly, or as a replay of the graph captured
// the second time the same key came, per the rules above.  eligible: the call's own conditions
// (dtype and size) allow a replay.
template <class Run>
static int run_replayed(GraphKey key, bool eligible, cudaStream_t st, Run run) {
    if (!eligible || !graphs_allowed() || prof_timing()) return run(st);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    KG_CUDA_TRY(cudaStreamIsCapturing(st, &cap));
    if (cap != cudaStreamCaptureStatusNone) return run(st);
    int dev = 0;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    key.w[15] = (uint64_t)dev;

    static thread_local std::vector<GraphEntry> cache;
    static thread_local uint64_t clock = 0;
    GraphEntry* e = nullptr;
    for (auto& c : cache)
        if (std::memcmp(&c.key, &key, sizeof(key)) == 0) e = &c;
    if (!e) {   // first call with these arguments: run it directly and remember it
        if ((int)cache.size() >= kGraphCache) {
            auto lru = std::min_element(cache.begin(), cache.end(), [](const GraphEntry& x, const GraphEntry& y) {
                return x.last_use < y.last_use;
            });
            if (lru->exec) {
                // a replay of it may still run on some stream: let the device finish before destroying it
                KG_CUDA_TRY(cudaDeviceSynchronize());
                cudaGraphExecDestroy(lru->exec);
            }
            cache.erase(lru);
        }
        GraphEntry fresh;
        std::memset(&fresh, 0, sizeof(fresh));
        fresh.key = key;
        fresh.last_use = ++clock;
        cache.push_back(fresh);
        return run(st);
    }
    e->last_use = ++clock;
    if (e->exec) {   // replay
        KG_CUDA_TRY(cudaGraphLaunch(e->exec, st));
        prof_add(e->launches);
        return KG_OK;
    }
    if (e->no_graph) return run(st);

    // second call: capture on the library's capture stream, then launch on the caller's
    static thread_local std::vector<std::pair<int, cudaStream_t>> cap_streams;   // per device
    cudaStream_t cs = nullptr;
    for (auto& d : cap_streams)
        if (d.first == dev) cs = d.second;
    if (!cs) {
        KG_CUDA_TRY(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
        cap_streams.emplace_back(dev, cs);
    }
    int64_t before[PK_COUNT], after[PK_COUNT];
    prof_counts(before);
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        (void)cudaGetLastError();
        e->no_graph = true;
        return run(st);
    }
    const int rc = run(cs);
    cudaGraph_t graph = nullptr;
    const cudaError_t end = cudaStreamEndCapture(cs, &graph);
    prof_counts(after);
    for (int k = 0; k < PK_COUNT; ++k) e->launches[k] = after[k] - before[k];
    cudaGraphExec_t exec = nullptr;
    const bool ok = rc == KG_OK && end == cudaSuccess && graph &&
                    cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    if (!ok) {   // nothing ran: take the captured launches back out of the counts and run directly
        (void)cudaGetLastError();
        int64_t back[PK_COUNT];
        for (int k = 0; k < PK_COUNT; ++k) back[k] = -e->launches[k];
        prof_add(back);
        e->no_graph = true;
        if (rc != KG_OK) return rc;
        return run(st);
    }
    e->exec = exec;
    KG_CUDA_TRY(cudaGraphLaunch(exec, st));   // the captured launches were counted once already
    return KG_OK;
}

static uint64_t kw(const void* p) { return (uint64_t)reinterpret_cast<uintptr_t>(p); }

static int quantize_direct(const void* W, int64_t m, int64_t n, int dtype, const void* U_A, const void* U_B,
                           kg_grid grid, int8_t* out_codes, void* out_V, void* out_E, void* ws, size_t ws_bytes,
                           cudaStream_t st) {
    if (dtype == KG_F64) {
        int rc = configure_leaf<double>();
        if (rc) return rc;
        return quantize_impl<double>(W, m, n, U_A, U_B, grid, out_codes, 1, out_V, out_E, ws, ws_bytes, st);
    }
    int rc = configure_leaf<float>();
    if (rc) return rc;
    return quantize_impl<float>(W, m, n, U_A, U_B, grid, out_codes, 1, out_V, out_E, ws, ws_bytes, st);
}

extern "C" int kron_gptq_quantize(const void* W, int64_t m, int64_t n, int dtype, const void* U_A,
                                  const void* U_B, kg_grid grid, int8_t* out_codes, void* out_V, void* out_E,
                                  void* ws, size_t ws_bytes, void* stream) {
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
    if (!W || !U_A || !U_B || !grid.row_scale || !out_codes || !out_V) return KG_ERR_ARG;
    if (ws_bytes < q_layout(m, n, dtype == KG_F64 ? 8 : 4).total) return KG_ERR_WORKSPACE;

    const int64_t ndiag = ceil_div(m, (int64_t)KG_T) + ceil_div(n, (int64_t)KG_T) - 1;
    GraphKey key;
    std::memset(&key, 0, sizeof(key));
    const uint64_t w[] = {1, kw(W), kw(U_A), kw(U_B), kw(grid.row_scale), kw(out_codes), kw(out_V), kw(out_E),
                          kw(ws), (uint64_t)m, (uint64_t)n, (uint64_t)ws_bytes, (uint64_t)dtype,
                          (uint64_t)(uint32_t)grid.qmin, (uint64_t)(uint32_t)grid.qmax};
    std::memcpy(key.w, w, sizeof(w));
    return run_replayed(key, dtype == KG_F32 && ndiag <= kGraphMaxDiag, st, [&](cudaStream_t s) {
        return quantize_direct(W, m, n, dtype, U_A, U_B, grid, out_codes, out_V, out_E, ws, ws_bytes, s);
    });
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of kron_gptq_quantize.
//
// Some callers cannot hand the library a workspace: code that runs inside a host framework
// whose allocator owns all device memory and forbids direct cudaMalloc, or a service path that
// must not allocate after start-up (cudaMalloc may synchronize the whole device).  For them the
// scratch lives in a fixed file-scope device array, KG_NOALLOC_SCRATCH_BYTES large, which every
// GPU that loads the library keeps until the process exits.  In host code the array's name is
// only a host-side stand-in, so its device address is fetched with cudaGetSymbolAddress, once
// per device, with that device current, on the first call made on that device.  All calls share
// the array: each call re-initialises everything it reads (status word, W~, R, scales), and calls
// whose executions overlap on a GPU race on it.
// ---------------------------------------------------------------------------------------
#include <mutex>

namespace kg {

static_assert(KG_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");
static __device__ __align__(256) unsigned char g_noalloc_scratch[KG_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

// Device address of the scratch array on the current device (looked up once per device).
static int noalloc_scratch(void** out) {
    int dev = -1;
    KG_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return KG_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KG_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return KG_OK;
}

}  // namespace kg

extern "C" int kron_gptq_quantize_noalloc(const void* W, int64_t m, int64_t n, int dtype, const void* U_A,
                                          const void* U_B, kg_grid grid, int8_t* out_codes, void* out_V,
                                          void* out_E, int* dev_status, void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (m < 0 || n < 0) return KG_ERR_ARG;
    if (grid.qmin >= 0 || grid.qmax <= 0 || grid.qmin < -128 || grid.qmax > 127) return KG_ERR_UNSUPPORTED;
    if (m > (int64_t)1 << 20 || n > (int64_t)1 << 20) return KG_ERR_UNSUPPORTED;
    const size_t need = (m == 0 || n == 0) ? kStatusBytes : q_layout(m, n, dtype == KG_F64 ? 8 : 4).total;
    if (need > (size_t)KG_NOALLOC_SCRATCH_BYTES) return KG_ERR_WORKSPACE;
    if (m != 0 && n != 0 && (!W || !U_A || !U_B || !grid.row_scale || !out_codes || !out_V)) return KG_ERR_ARG;
    void* scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == 0 || n == 0) {
        KG_CUDA_TRY(cudaMemsetAsync(scratch, 0, kStatusBytes, st));
    } else if (dtype == KG_F64) {
        rc = configure_leaf<double>();
        if (!rc) rc = quantize_impl<double>(W, m, n, U_A, U_B, grid, out_codes, 1, out_V, out_E, scratch,
                                            (size_t)KG_NOALLOC_SCRATCH_BYTES, st);
    } else {
        rc = configure_leaf<float>();
        if (!rc) rc = quantize_impl<float>(W, m, n, U_A, U_B, grid, out_codes, 1, out_V, out_E, scratch,
                                           (size_t)KG_NOALLOC_SCRATCH_BYTES, st);
    }
    if (rc) return rc;
    if (dev_status) KG_CUDA_TRY(cudaMemcpyAsync(dev_status, scratch, sizeof(int), cudaMemcpyDeviceToDevice, st));
    return KG_OK;
}

// ---------------------------------------------------------------------------------------
// Row- and column-scaled alphabet with unclipped integers (kg_rc.cuh): the same solve on the
// rescaled problem.  Workspace: [the solve's workspace (status word first)][W' m*n][U'_A n*n]
// [U'_B m*m][unit row scales m], each part 256-byte aligned.
// ---------------------------------------------------------------------------------------
namespace kg {

struct RcLayout {
    size_t off_w, off_ua, off_ub, off_one, total;
};

static RcLayout rc_layout(int64_t m, int64_t n, size_t es) {
    RcLayout R{};
    size_t off = q_layout(m, n, es).total;
    R.off_w = off;   off = align_up(off + (size_t)(m * n) * es, 256);
    R.off_ua = off;  off = align_up(off + (size_t)(n * n) * es, 256);
    R.off_ub = off;  off = align_up(off + (size_t)(m * m) * es, 256);
    R.off_one = off; off = align_up(off + (size_t)m * es, 256);
    R.total = off;
    return R;
}

// largest |code| the unclipped alphabet represents: fp32 keeps every integer of the step up to
// 2^24; the margin leaves the rounding of x / s exact in the last bits that matter
template <typename Real>
constexpr int32_t rc_bound() { return sizeof(Real) == 4 ? (1 << 22) : (1 << 30); }

template <typename Real>
static int quantize_rc_impl(const void* W, int64_t m, int64_t n, const void* UA, const void* UB, const void* alpha,
                            const void* beta, int32_t* Z, void* V, void* E, void* ws, cudaStream_t st) {
    const RcLayout R = rc_layout(m, n, sizeof(Real));
    unsigned char* base = static_cast<unsigned char*>(ws);
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    Real* Wp = reinterpret_cast<Real*>(base + R.off_w);
    Real* UAp = reinterpret_cast<Real*>(base + R.off_ua);
    Real* UBp = reinterpret_cast<Real*>(base + R.off_ub);
    Real* one = reinterpret_cast<Real*>(base + R.off_one);
    const Real* al = static_cast<const Real*>(alpha);
    const Real* be = static_cast<const Real*>(beta);
    const int nb = 148 * 4;
    KG_CUDA_TRY(cudaMemsetAsync(status, 0, kStatusBytes, st));
    {
        ProfScope ps(PK_INIT, st);
        k_rc_check_scales<Real><<<nb, 256, 0, st>>>(al, n, be, m, status);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_rc_scale_w<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(W), m, n, al, be, Wp);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_rc_scale_u<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(UA), n, al, UAp);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_rc_scale_u<Real><<<nb, 256, 0, st>>>(static_cast<const Real*>(UB), m, be, UBp);
    }
    KG_LAUNCH_CHECK();
    {
        ProfScope ps(PK_INIT, st);
        k_rc_fill<Real><<<std::max<int64_t>(1, std::min<int64_t>(nb, ceil_div(m, 256))), 256, 0, st>>>(one, m, Real(1));
    }
    KG_LAUNCH_CHECK();
    const kg_grid grid{-rc_bound<Real>(), rc_bound<Real>(), one};
    int rc = quantize_impl<Real>(Wp, m, n, UAp, UBp, grid, Z, 4, V, E, ws, q_layout(m, n, sizeof(Real)).total, st,
                                 false);
    if (rc) return rc;
    {
        ProfScope ps(PK_INIT, st);
        k_rc_finish<Real><<<nb, 256, 0, st>>>(Z, m, n, al, be, static_cast<Real*>(V), static_cast<Real*>(E),
                                              rc_bound<Real>(), status);
    }
    KG_LAUNCH_CHECK();
    return KG_OK;
}

}  // namespace kg

extern "C" size_t kron_gptq_quantize_rc_workspace_size(int64_t m, int64_t n, int dtype) {
    if (m < 0 || n < 0) return 0;
    if (dtype != KG_F32 && dtype != KG_F64) return 0;
    if (m == 0 || n == 0) return kStatusBytes;
    return rc_layout(m, n, dtype == KG_F64 ? 8 : 4).total;
}

extern "C" int kron_gptq_quantize_rc(const void* W, int64_t m, int64_t n, int dtype, const void* U_A,
                                     const void* U_B, const void* alpha, const void* beta, int32_t* out_Z,
                                     void* out_V, void* out_E, void* ws, size_t ws_bytes, void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (m < 0 || n < 0) return KG_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (m > (int64_t)1 << 20 || n > (int64_t)1 << 20) return KG_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == 0 || n == 0) {
        if (ws_bytes < kStatusBytes) return KG_ERR_WORKSPACE;
        KG_CUDA_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
        return KG_OK;
    }
    if (!W || !U_A || !U_B || !alpha || !beta || !out_Z || !out_V) return KG_ERR_ARG;
    if (ws_bytes < rc_layout(m, n, dtype == KG_F64 ? 8 : 4).total) return KG_ERR_WORKSPACE;
    const int64_t ndiag = ceil_div(m, (int64_t)KG_T) + ceil_div(n, (int64_t)KG_T) - 1;
    GraphKey key;   // replayed as kron_gptq_quantize is
    std::memset(&key, 0, sizeof(key));
    const uint64_t w[] = {2, kw(W), kw(U_A), kw(U_B), kw(alpha), kw(beta), kw(out_Z), kw(out_V), kw(out_E),
                          kw(ws), (uint64_t)m, (uint64_t)n, (uint64_t)ws_bytes, (uint64_t)dtype};
    std::memcpy(key.w, w, sizeof(w));
    return run_replayed(key, dtype == KG_F32 && ndiag <= kGraphMaxDiag, st, [&](cudaStream_t s) {
        if (dtype == KG_F64) {
            int rc = configure_leaf<double>();
            if (rc) return rc;
            return quantize_rc_impl<double>(W, m, n, U_A, U_B, alpha, beta, out_Z, out_V, out_E, ws, s);
        }
        int rc = configure_leaf<float>();
        if (rc) return rc;
        return quantize_rc_impl<float>(W, m, n, U_A, U_B, alpha, beta, out_Z, out_V, out_E, ws, s);
    });
}

extern "C" int kron_gptq_waterkron_scales(const void* U_A, int64_t n, const void* U_B, int64_t m, int dtype,
                                          double gamma, void* alpha, void* beta, void* stream) {
    if (dtype != KG_F32 && dtype != KG_F64) return KG_ERR_UNSUPPORTED;
    if (m < 0 || n < 0 || !(gamma > 0.0) || !std::isfinite(gamma)) return KG_ERR_ARG;
    if (m + n == 0) return KG_OK;
    if ((n > 0 && (!U_A || !alpha)) || (m > 0 && (!U_B || !beta))) return KG_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int nb = (int)std::max<int64_t>(1, std::min<int64_t>(148 * 4, ceil_div(m + n, 256)));
    if (dtype == KG_F64)
        k_wk_scales<double><<<nb, 256, 0, st>>>(static_cast<const double*>(U_A), n, static_cast<const double*>(U_B),
                                                m, gamma, static_cast<double*>(alpha), static_cast<double*>(beta));
    else
        k_wk_scales<float><<<nb, 256, 0, st>>>(static_cast<const float*>(U_A), n, static_cast<const float*>(U_B), m,
                                               gamma, static_cast<float*>(alpha), static_cast<float*>(beta));
    KG_LAUNCH_CHECK();
    return KG_OK;
}

// ---------------------------------------------------------------------------------------
// The non-recursive anti-diagonal algorithm ("FastKron", Section 2.3, FastKron-antidiagonal; the
// scheme of YAQA): after each tile anti-diagonal D is solved, its errors reach the whole matrix at
// once through the dense product  W~ -= U_B^T Delta_D U_A,  Delta_D = E on the tiles of D and zero
// elsewhere.  Every step costs two full GEMMs, O(mn(m+n)), so the total is quartic; it exists as
// the baseline the recursion is measured against.  fp64 only.  The leaves are the solver's own:
// the row-chain buffer R stays zero (every cross-tile contribution is already in W~), so a leaf
// propagates only its own tile's errors, which the dense product then applies a second time to
// entries the leaf has finished -- entries nobody reads again.
// ---------------------------------------------------------------------------------------
namespace kg {

constexpr size_t ANTI_BLAS_WS = 32u << 20;

static size_t anti_extra_bytes(int64_t m, int64_t n) {
    const QLayout L = q_layout(m, n, 8);
    return 2 * align_up((size_t)(L.Mp * L.Np) * 8, 256) + ANTI_BLAS_WS;
}

// Delta = E on the tiles of anti-diagonal D, zero elsewhere (Mp x Np, row-major like E)
__global__ void k_anti_delta(const double* __restrict__ E, int D, int64_t Mp, int64_t Np, double* __restrict__ Dl) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < Mp * Np; p += stride) {
        const int64_t i = p / Np, j = p - i * Np;
        Dl[p] = (i / KG_T + j / KG_T == D) ? E[p] : 0.0;
    }
}

template <typename Real>
static int solve_antidiagonal(const QArgs<Real>& a, int ndiag, unsigned char* extra) {
    if constexpr (sizeof(Real) != 8) {
        return KG_ERR_UNSUPPORTED;
    } else {
        const int64_t Mp = a.L.Mp, Np = a.L.Np;
        double* Dl = reinterpret_cast<double*>(extra);
        double* T = reinterpret_cast<double*>(extra + align_up((size_t)(Mp * Np) * 8, 256));
        void* bws = extra + 2 * align_up((size_t)(Mp * Np) * 8, 256);
        cublasHandle_t h;
        int rc = blas_handle(&h);
        if (!rc) rc = blas_bind(h, a.st, bws, ANTI_BLAS_WS);
        if (rc) return rc;
        const double one = 1.0, zero = 0.0, minus_one = -1.0;
        const int nb = 148 * 4;
        for (int D = 0; D < ndiag; ++D) {
            if ((rc = launch_leaf(a, D, a.st))) return rc;
            if (D + 1 == ndiag) break;
            {
                ProfScope ps(PK_PUSH, a.st);
                k_anti_delta<<<nb, 256, 0, a.st>>>(a.E, D, Mp, Np, Dl);
                KG_LAUNCH_CHECK();
                // T = Delta U_A:  column-major T^T = U_A^T Delta^T (row-major storage read as its transpose)
                if (cublasDgemm(h, CUBLAS_OP_N, CUBLAS_OP_N, (int)Np, (int)Mp, (int)Np, &one, a.UA, (int)a.ldA, Dl,
                                (int)Np, &zero, T, (int)Np) != CUBLAS_STATUS_SUCCESS)
                    return KG_ERR_CUDA;
                // W~ -= U_B^T T:  column-major W~^T -= T^T U_B
                if (cublasDgemm(h, CUBLAS_OP_N, CUBLAS_OP_T, (int)Np, (int)Mp, (int)Mp, &minus_one, T, (int)Np, a.UB,
                                (int)a.ldB, &one, a.Wt, (int)Np) != CUBLAS_STATUS_SUCCESS)
                    return KG_ERR_CUDA;
            }
        }
        return KG_OK;
    }
}

}  // namespace kg

extern "C" size_t kron_gptq_quantize_antidiagonal_workspace_size(int64_t m, int64_t n) {
    if (m < 0 || n < 0) return 0;
    if (m == 0 || n == 0) return kStatusBytes;
    return q_layout(m, n, 8).total + anti_extra_bytes(m, n);
}

extern "C" int kron_gptq_quantize_antidiagonal(const void* W, int64_t m, int64_t n, const void* U_A, const void* U_B,
                                               kg_grid grid, int8_t* out_codes, void* out_V, void* out_E, void* ws,
                                               size_t ws_bytes, void* stream) {
    if (m < 0 || n < 0) return KG_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return KG_ERR_ARG;
    if (grid.qmin >= 0 || grid.qmax <= 0 || grid.qmin < -128 || grid.qmax > 127) return KG_ERR_UNSUPPORTED;
    if (m > (int64_t)1 << 17 || n > (int64_t)1 << 17) return KG_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == 0 || n == 0) {
        if (ws_bytes < kStatusBytes) return KG_ERR_WORKSPACE;
        KG_CUDA_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
        return KG_OK;
    }
    if (!W || !U_A || !U_B || !grid.row_scale || !out_codes || !out_V) return KG_ERR_ARG;
    const size_t qbytes = q_layout(m, n, 8).total;
    if (ws_bytes < qbytes + anti_extra_bytes(m, n)) return KG_ERR_WORKSPACE;
    int rc = configure_leaf<double>();
    if (rc) return rc;
    return quantize_impl<double>(W, m, n, U_A, U_B, grid, out_codes, 1, out_V, out_E, ws, qbytes, st, true,
                                 static_cast<unsigned char*>(ws) + qbytes);
}

#ifdef KG_TEST_HANDOFF_FAULT
// Test build only: switch the withheld hand-off of kg_leaf_ws.cuh on (1) or off (0) on the
// current device.  0 on success, KG_ERR_CUDA otherwise.  Not part of the C ABI of the default
// library, which does not contain it.
extern "C" __attribute__((visibility("default"))) int kron_gptq_debug_handoff_fault(int on) {
    const int v = on ? 1 : 0;
    return cudaMemcpyToSymbol(kg::g_test_handoff_fault, &v, sizeof(v)) == cudaSuccess ? 0 : KG_ERR_CUDA;
}
#endif

extern "C" int kron_gptq_schedule_plan(int ndiag, int* out, int max_pieces) {
    if (ndiag < 1 || max_pieces < 0) return KG_ERR_ARG;
    int count = 0;
    for (const Piece& p : issue_order(ndiag)) {
        if (p.stream < 0) continue;
        if (out && count < max_pieces) {
            int* o = out + 5 * (int64_t)count;
            o[0] = p.s0; o[1] = p.s1; o[2] = p.t0; o[3] = p.t1; o[4] = p.stream;
        }
        ++count;
    }
    return count;
}
