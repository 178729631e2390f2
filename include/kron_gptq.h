/*
 * kron_gptq.h -- C ABI of the two-sided (Kronecker-factored) GPTQ library for NVIDIA B200.
 *
 * The library rounds one weight matrix W (m x n; row i = output channel, column j = input
 * channel) onto a per-row scaled integer grid, minimizing the proxy loss
 *     D_{A,B} = || B^{1/2} (V - W) A^{1/2} ||_F^2 = vec(V-W)^T (A (x) B) vec(V-W)
 * with the two-sided GPTQ rounding rule (Babai nearest plane on vec(W) under the Gram matrix
 * A (x) B).  Sources, by page title and section:
 *   - "FastKron: Efficient Quantization with Kronecker-Factored Hessians" (later "BaKron"),
 *     Section 2.1 (notation, quantize instead of round, clipping), Section 2.2 (the
 *     vectorized algorithm and D_{A,B}), Sections 2.3-2.5 (anti-diagonal parallelism and the
 *     recursive divide-and-conquer that give O(m+n) steps and O(mn(m+n)) work), Section 2.6
 *     (inverse and Cholesky as a separate step).
 *   - "WaterKron and FlipFlop Hessian ...", Section 2 (Notation: Cholesky, RevCholesky,
 *     damping), Section 2.1 (the scaled integer alphabet).
 *   - "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding" (abstract): the same rounded matrix.
 *
 * Conventions for every call:
 *   - All matrices are dense, row-major, contiguous, in DEVICE memory owned by the caller.
 *     The library never allocates or frees device memory: each call takes a caller-owned
 *     workspace of at least the size the matching *_workspace_size() function returns.  The one
 *     exception: quantize_antidiagonal, the quartic baseline kept as a yardstick, hands its dense
 *     products to cuBLAS; it creates one cuBLAS handle per host thread and device on first use,
 *     and cuBLAS allocates its own small device state then (its GEMM workspace is inside ws).
 *     Handles live until the process exits, also those of threads that have ended, so make
 *     that call from long-lived threads.  Every other product runs in the library's own
 *     kernels.
 *   - Calls are asynchronous on the given CUDA stream (passed as void*, a cudaStream_t;
 *     NULL = the legacy default stream).  Errors the host can see (bad arguments,
 *     unsupported options, a failed launch) are returned at once and nothing is launched
 *     after them.  Errors only the device can see (a factor that is not positive definite,
 *     non-finite input, a device wait that ran out) are written to a status word inside the
 *     workspace; kron_gptq_sync_status() synchronizes the stream and returns it.
 *   - The recursive two-sided solves (quantize, quantize_noalloc, quantize_rc) run on four
 *     internal streams (the leaves on one, the update pieces on the others by when they are due;
 *     kron_gptq_schedule_plan lists them), forked from the caller's stream at the start; the
 *     caller's stream waits for all four at the end, so each call stays one asynchronous
 *     operation on the caller's stream.  For this each host thread keeps, per device, eight sets
 *     of four non-blocking streams with their events (host-side driver objects, no device
 *     buffers), created on the first call and kept until the process exits.  Solves in flight on
 *     several caller streams at once want more than CUDA's default eight hardware connections
 *     (CUDA_DEVICE_MAX_CONNECTIONS, set before the CUDA context exists; the Python binding defaults
 *     it to 32): seven 4096-to-14336-wide layers in flight took 0.087 s with 8 and 0.072 s with 32.
 *   - Concurrent calls on different streams need distinct workspaces.
 *   - Status codes: 0 = success, negative = error (see kg_status).
 */
#ifndef KRON_GPTQ_H
#define KRON_GPTQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KG_API __attribute__((visibility("default")))
#else
#define KG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kg_status {
    KG_OK = 0,
    KG_ERR_ARG = -1,          /* null pointer, negative size, bad grid, misaligned pointer */
    KG_ERR_UNSUPPORTED = -2,  /* dtype or grid the library does not implement */
    KG_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed, or (fp32) the driver
                                 could not encode the tensor maps of the update operands */
    KG_ERR_WORKSPACE = -4,    /* workspace smaller than *_workspace_size() */
    KG_ERR_NOT_PD = -5,       /* (device) a Cholesky pivot was not positive */
    KG_ERR_NONFINITE = -6,    /* (device) NaN/Inf in W, in the scales or in a factor diagonal */
    KG_ERR_TIMEOUT = -7,      /* (device) a bounded device-side wait ran out */
    KG_ERR_RANGE = -8         /* (device) an unclipped code reached the representable bound, or
                                 the codes span more values than the entropy workspace has bins */
} kg_status;

typedef enum kg_dtype {
    KG_F32 = 1,   /* float32: the solve runs in fp32 with 3xTF32 tensor-core updates */
    KG_F64 = 2    /* float64: the exact path, fp64 throughout */
} kg_dtype;

/* Quantization grid: codes are integers in [qmin, qmax] (qmin < 0 < qmax, both within
 * int8), the value of a code c in row i is row_scale[i] * c.  row_scale is a device array
 * of m entries with the dtype of the solve ("WaterKron", Section 2.1: V = beta alpha^T (.) Z
 * with per-row beta and alpha = 1; "FastKron", Section 2.1: integers may be clipped). */
typedef struct kg_grid {
    int qmin;
    int qmax;
    const void* row_scale;
} kg_grid;

/* Library version (major*10000 + minor*100 + patch). */
KG_API int kron_gptq_version(void);

/* Human-readable name of a status code (static string, never NULL). */
KG_API const char* kron_gptq_status_string(int status);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_prepare -- factors for the solver.
 *   For each of A (n x n, input side) and B (m x m, output side):
 *     A_d = A + damp * mean(diag A) * I             (damping, "WaterKron" Sec. 2 Notation)
 *     U_A = upper-triangular factor with U_A^T U_A = A_d^{-1}
 *   U_A equals RevCholesky(A_d)^{-T}; its transpose is the lower Cholesky factor of
 *   A_d^{-1} that the error feedback of "FastKron" Sec. 2.4 uses.  Computed in fp64 by a
 *   recursion that computes the reversed Cholesky factor of A_d and its inverse together.
 * Arguments:
 *   A, B      device, symmetric positive (semi)definite, row-major; dtype fac_dtype
 *             (KG_F32 is promoted to fp64).  The full matrix is read; only its lower
 *             triangle enters the factorization (symmetry is assumed, not checked).
 *   n, m      sizes (>= 1).  B may be NULL with m >= 1 to skip the output side.
 *   damp      relative damping (>= 0); pass 0 if A, B are already damped.
 *   U_A, U_B  device outputs, fp64, n x n and m x m; the strictly lower triangle is zeroed.
 *   U_A32, U_B32  optional fp32 copies of the same factors (NULL to skip).
 *   ws        device workspace, 256-byte aligned, of at least
 *             kron_gptq_prepare_workspace_size(max(n, m)) bytes.  With
 *             kron_gptq_prepare_workspace_size(n) + kron_gptq_prepare_workspace_size(m) bytes or
 *             more, B's factor is prepared on an internal side stream (one per host thread and
 *             device, created on first use and kept until exit) at the same time as A's; the call
 *             still forks from and joins back into `stream`.
 * Device errors: KG_ERR_NOT_PD when a pivot of A_d or B_d is not positive (the outputs are
 *   then unspecified), KG_ERR_NONFINITE for NaN/Inf input.
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_prepare_workspace_size(int64_t k);
KG_API int kron_gptq_prepare(const void* A, int64_t n, const void* B, int64_t m, int fac_dtype,
                             double damp, double* U_A, double* U_B, float* U_A32, float* U_B32,
                             void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_quantize -- two-sided GPTQ rounding of W ("FastKron" Sec. 2.2-2.5).
 *   Produces the codes of the naive algorithm: every entry is visited after all entries to
 *   its top-left (any such order gives the same result); for entry (i,j) with current value x:
 *       c = clamp(rint(x / s_i), qmin, qmax),  Q = s_i c,
 *       E_ij = (x - Q) / (U_B[i,i] U_A[j,j]),
 *       W[i',j'] -= U_B[i,i'] E_ij U_A[j,j']   for i' >= i, j' >= j, (i',j') != (i,j).
 *   Computed as a sweep over anti-diagonals of 64x64 tiles with recursive divide-and-
 *   conquer batching of the trailing updates over ranges of tile anti-diagonals.
 *   Rounding is round-half-to-even; in fp64 the codes equal the definition's except at
 *   entries whose pre-rounding value lies within rounding noise of a half-integer.
 * Arguments:
 *   W         device, m x n, dtype (KG_F32 or KG_F64); not modified.
 *   U_A, U_B  device, n x n and m x m upper-triangular factors (as from prepare), dtype
 *             matching the solve (the fp32 copies for KG_F32).  Lower triangles are ignored.
 *   grid      qmin/qmax with -128 <= qmin < 0 < qmax <= 127; row_scale: device, m entries
 *             of dtype, each finite and > 0 (kron_gptq_row_scales computes max|W_i|/qmax).
 *   out_codes device, m x n int8.
 *   out_V     device, m x n, dtype: V = row_scale[i] * code.
 *   out_E     optional device, m x n, dtype: the scaled errors E (NULL to skip).  They
 *             satisfy V - W = -U_B^T E U_A and sum(E^2) = D_{A_d,B_d}.
 *   ws        kron_gptq_quantize_workspace_size(m, n, dtype) bytes, 256-byte aligned.
 * m == 0 or n == 0 is a no-op returning KG_OK.
 * Replays (fp32, up to 160 tile anti-diagonals, i.e. ceil(m/64) + ceil(n/64) <= 161): the second
 *   call on a host thread with the same arguments (every pointer, size, dtype and grid) on the same
 *   device captures the solve into a CUDA graph on a stream of the library's own and launches it on
 *   `stream`; later such calls replay it (4096^2: 7.15 -> 6.85 ms a solve, the same results).  The
 *   graph reads the buffers' contents when it runs, so new values under the same pointers are fine.
 *   Not while `stream` is capturing or the event profiler is on; KRON_GPTQ_GRAPHS=0 in the
 *   environment turns replays off.  A thread caches up to 32 graphs; evicting one synchronizes the
 *   device first.
 * Device errors: KG_ERR_NONFINITE (NaN/Inf in W or scales, non-positive scale or factor
 *   diagonal), KG_ERR_TIMEOUT (a bounded device-side wait ran out: the hand-off between the
 *   warps of a leaf, or the load / MMA pipeline of an update).
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_quantize_workspace_size(int64_t m, int64_t n, int dtype);
KG_API int kron_gptq_quantize(const void* W, int64_t m, int64_t n, int dtype,
                       const void* U_A, const void* U_B, kg_grid grid,
                       int8_t* out_codes, void* out_V, void* out_E,
                       void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_loss -- proxy loss D_{A_d,B_d} = tr((V - W) A_d (V - W)^T B_d)
 *   = vec(V-W)^T (A_d (x) B_d) vec(V-W)   ("FastKron" Sec. 2.2), accumulated in fp64.
 *   A_d, B_d are damped exactly as in prepare (same damp).  For the output of quantize it
 *   equals the sum of E^2 up to rounding.
 * Arguments: W, V device m x n of dtype; A (n x n), B (m x m) device, dtype fac_dtype;
 *   out_loss device pointer to one double; ws of kron_gptq_loss_workspace_size(m, n) bytes.
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_loss_workspace_size(int64_t m, int64_t n);
KG_API int kron_gptq_loss(const void* W, const void* V, int64_t m, int64_t n, int dtype,
                   const void* A, const void* B, int fac_dtype, double damp,
                   double* out_loss, void* ws, size_t ws_bytes, void* stream);

/* Per-row scales s_i = max_j |W_ij| / qmax (1 for an all-zero row), chosen from the
 * original W before any update ("WaterKron" Sec. 2.4: scales are chosen up front).
 * W device m x n of dtype; out_scale device, m entries of dtype. */
KG_API int kron_gptq_row_scales(const void* W, int64_t m, int64_t n, int dtype, int qmax,
                         void* out_scale, void* stream);

/* Synchronize `stream` and return the device status word of the call that used `ws`
 * (KG_OK or a negative device error), or KG_ERR_CUDA if the synchronization failed. */
KG_API int kron_gptq_sync_status(const void* ws, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_quantize_noalloc -- kron_gptq_quantize without a caller workspace.
 *   The paper has no counterpart: this is a deployment variant for callers that cannot
 *   allocate device memory -- code running inside a host framework whose allocator owns all
 *   device memory and forbids direct cudaMalloc, or a service path that must not allocate
 *   after start-up (cudaMalloc may synchronize the device).  It runs exactly the same kernels
 *   as kron_gptq_quantize, with the scratch in a fixed device array of
 *   KG_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the library holds
 *   until the process exits.  It allocates nothing: no cudaMalloc, no cudaFree.
 * Arguments: as kron_gptq_quantize, without ws/ws_bytes, plus
 *   dev_status  optional device pointer to one int that receives the device status word of
 *               this call (KG_OK or a negative device error) in stream order; NULL to skip.
 * Limits and behaviour:
 *   - Problems whose scratch (kron_gptq_quantize_workspace_size(m, n, dtype)) exceeds
 *     KG_NOALLOC_SCRATCH_BYTES are rejected with KG_ERR_WORKSPACE before anything is launched
 *     (for a square layer about 40 bytes per weight in fp32, which keeps split copies of the
 *     operands for the tensor cores, and 24 in fp64: fp32 fits e.g. 896 x 896, fp64 e.g.
 *     1024 x 1024).
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current).  The first call from each host thread on a device also creates
 *     the internal streams and events that every recursive solve uses (eight sets of four streams;
 *     host-side driver objects, no device buffers; see the conventions above).  Make both first
 *     calls before any stream capture.
 *   - All calls share the one array and each call re-initialises what it reads; calls whose
 *     executions overlap on the same GPU (different streams, threads) race on it.
 * --------------------------------------------------------------------------------------- */
#define KG_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
KG_API int kron_gptq_quantize_noalloc(const void* W, int64_t m, int64_t n, int dtype,
                                      const void* U_A, const void* U_B, kg_grid grid,
                                      int8_t* out_codes, void* out_V, void* out_E,
                                      int* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_quantize_rc -- two-sided GPTQ on the row- and column-scaled alphabet with unclipped
 *   integers ("WaterKron and FlipFlop Hessian", Section 2.1: V = beta alpha^T (.) Z, Z integer
 *   and not clipped, the scales chosen up front and handed to the algorithm).  For entry (i,j)
 *   with current value x and step s_ij = beta_i alpha_j:
 *       z = rint(x / s_ij),  Q = s_ij z,  E_ij = (x - Q) / (U_B[i,i] U_A[j,j]),
 *   then the same update as kron_gptq_quantize.  Computed by the same solve on the rescaled
 *   problem W (/) (beta alpha^T) with factors D_alpha U_A D_alpha^-1, D_beta U_B D_beta^-1 (the
 *   two are the same algorithm: dividing every update by the target's step turns one into the
 *   other), then V = s (.) Z and E = s (.) E'.
 * Arguments:
 *   W, U_A, U_B, dtype, m, n   as kron_gptq_quantize.
 *   alpha     device, n entries of dtype, each finite and > 0 (column steps).
 *   beta      device, m entries of dtype, each finite and > 0 (row steps).
 *   out_Z     device, m x n int32 codes.
 *   out_V     device, m x n, dtype: V = beta_i alpha_j Z_ij.
 *   out_E     optional device, m x n, dtype (NULL to skip): V - W = -U_B^T E U_A.
 *   ws        kron_gptq_quantize_rc_workspace_size(m, n, dtype) bytes, 256-byte aligned; its
 *             first 256 bytes are the status word (kron_gptq_sync_status).
 * The codes are unclipped up to |Z| < 2^22 in fp32 (where fp32 still holds every integer of the
 * step) and |Z| < 2^30 in fp64; a code at that bound raises KG_ERR_RANGE.
 * m == 0 or n == 0 is a no-op returning KG_OK.
 * Device errors: KG_ERR_NONFINITE (NaN/Inf in W, a step not finite and > 0, a factor diagonal
 *   not > 0), KG_ERR_RANGE, KG_ERR_TIMEOUT.
 * Replays: as kron_gptq_quantize (fp32, up to 160 tile anti-diagonals, same arguments again).
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_quantize_rc_workspace_size(int64_t m, int64_t n, int dtype);
KG_API int kron_gptq_quantize_rc(const void* W, int64_t m, int64_t n, int dtype,
                                 const void* U_A, const void* U_B, const void* alpha, const void* beta,
                                 int32_t* out_Z, void* out_V, void* out_E,
                                 void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_waterkron_scales -- the WaterKron steps ("WaterKron and FlipFlop Hessian",
 *   Section 3: alpha_j proportional to 1/L^(A)_jj and beta_i to 1/L^(B)_ii, where L is the
 *   reverse Cholesky factor, so 1/L^(A)_jj = U_A[j,j]).  One knob gamma > 0 sets both constants:
 *       alpha_j = sqrt(gamma) U_A[j,j],   beta_i = sqrt(gamma) U_B[i,i],
 *   so the step of entry (i,j) is gamma U_B[i,i] U_A[j,j] and every error E_ij of
 *   kron_gptq_quantize_rc lies in [-gamma/2, gamma/2].
 * Arguments: U_A (n x n), U_B (m x m) device factors of dtype; alpha (n), beta (m) device
 *   outputs of dtype.  gamma must be finite and > 0 (else KG_ERR_ARG).
 * --------------------------------------------------------------------------------------- */
KG_API int kron_gptq_waterkron_scales(const void* U_A, int64_t n, const void* U_B, int64_t m, int dtype,
                                      double gamma, void* alpha, void* beta, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_code_entropy -- empirical entropy of integer codes in bits per entry, the memory
 *   cost of Z under a good entropy coder ("WaterKron and FlipFlop Hessian", Section 2.1):
 *       H = -sum_z (c_z / N) log2(c_z / N),  c_z = number of entries equal to z.
 * Arguments:
 *   Z         device, count int32 codes (count < 2^32).
 *   out_bits  device, one double (written in stream order; NaN when the range does not fit).
 *   ws        kron_gptq_code_entropy_workspace_size(max_bins) bytes, 256-byte aligned: room for
 *             max_bins distinct values between min(Z) and max(Z); status word first.
 * Device errors: KG_ERR_RANGE when max(Z) - min(Z) + 1 exceeds the workspace's bins.
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_code_entropy_workspace_size(int64_t max_bins);
KG_API int kron_gptq_code_entropy(const int32_t* Z, int64_t count, double* out_bits,
                                  void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_quantize_onesided -- standard (one-sided) GPTQ with recursively batched updates
 *   ("FastKron", Section 2.2: GPTQ, the case B = I of the two-sided algorithm; Section 2.4:
 *   GPTQ-recursive, solve the first half of the columns, propagate its errors to the second half
 *   in one batched update, solve the second half).  For column j in order, all rows at once:
 *       c = clamp(rint(x / s_i), qmin, qmax),  Q = s_i c,  E_ij = (x - Q) / U_A[j,j],
 *       W[i, j'] -= E_ij U_A[j, j']   for j' > j.
 *   The result equals kron_gptq_quantize with U_B = I (up to rounding ties).  The recursion stops
 *   at 64-column blocks; each batched update is one dense GEMM on the tensor cores in the
 *   library's own kernels (fp32: tcgen05 with 3xTF32 split operands; fp64: the FP64 mma path).
 * Arguments: W (m x n), U_A (n x n, 16-byte aligned), grid, out_codes (int8), out_V, out_E
 *   (optional): as kron_gptq_quantize.  ws: kron_gptq_quantize_onesided_workspace_size(m, n, dtype) bytes,
 *   256-byte aligned, status word first.
 * m == 0 or n == 0 is a no-op returning KG_OK.
 * Device errors: KG_ERR_NONFINITE (NaN/Inf in W, a scale or a diagonal entry of U_A not > 0).
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_quantize_onesided_workspace_size(int64_t m, int64_t n, int dtype);
KG_API int kron_gptq_quantize_onesided(const void* W, int64_t m, int64_t n, int dtype,
                                       const void* U_A, kg_grid grid,
                                       int8_t* out_codes, void* out_V, void* out_E,
                                       void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_factors -- Kronecker factors A (n x n), B (m x m) with A (x) B ~ H = E[a a^T (x) b b^T]
 *   from N samples: a_k the input of the linear unit (length n), b_k the gradient at its output
 *   (length m) ("FastKron", Section 3.2 and Appendix E.2; "WaterKron and FlipFlop Hessian",
 *   Table 1 and Section 5).  E is the sample mean.
 *     KG_FACTOR_MARGINAL:  A = E[a a^T], B = E[b b^T].
 *     KG_FACTOR_FROBENIUS: from B = I, repeat: A = E[(b^T B b) a a^T] / ||B||_F^2,
 *                          B = E[(a^T A a) b b^T] / ||A||_F^2  (least squares on ||H - A (x) B||_F).
 *     KG_FACTOR_FLIPFLOP:  from B = I, repeat: A = E[(b^T B^-1 b) a a^T] / m,
 *                          B = E[(a^T A^-1 a) b b^T] / n.
 *   iters (>= 1) is the number of (A, B) updates of the two alternating methods.  Computed in
 *   fp64: the library's own DGEMMs on the FP64 tensor path and its own prepare for A^-1, B^-1.
 * Arguments:
 *   a, b      device, row-major N x n and N x m, dtype KG_F32 (promoted) or KG_F64.
 *   A, B      device fp64 outputs, n x n and m x m, symmetric.
 *   ws        kron_gptq_factors_workspace_size(N, n, m) bytes, 256-byte aligned, status first.
 * Device errors: KG_ERR_NONFINITE (NaN/Inf in a or b), KG_ERR_NOT_PD (FlipFlop: an iterate that is
 *   not positive definite, e.g. fewer samples than n or m).
 * --------------------------------------------------------------------------------------- */
typedef enum kg_factor_method {
    KG_FACTOR_MARGINAL = 0,
    KG_FACTOR_FROBENIUS = 1,
    KG_FACTOR_FLIPFLOP = 2
} kg_factor_method;
KG_API size_t kron_gptq_factors_workspace_size(int64_t N, int64_t n, int64_t m);
KG_API int kron_gptq_factors(const void* a, const void* b, int64_t N, int64_t n, int64_t m, int dtype,
                             int method, int iters, double* A, double* B,
                             void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_quantize_antidiagonal -- the non-recursive anti-diagonal algorithm ("FastKron",
 *   Section 2.3, FastKron-antidiagonal; the scheme YAQA uses): the tile anti-diagonals are solved in
 *   order, and after each one its errors reach the whole matrix through the dense product
 *   W -= U_B^T Delta U_A (Delta = the errors of that anti-diagonal).  Same outputs as
 *   kron_gptq_quantize (equal codes up to rounding ties: the FastKron variants are equivalent,
 *   Section 2.5), at O(mn(m+n)) work per anti-diagonal -- quartic in total.  A baseline to measure
 *   the recursion against; fp64 only, dense products in cuBLAS (DGEMM) with a workspace slice.
 * Arguments: as kron_gptq_quantize with dtype KG_F64; m, n <= 2^17.
 *   ws: kron_gptq_quantize_antidiagonal_workspace_size(m, n) bytes, 256-byte aligned.
 * --------------------------------------------------------------------------------------- */
KG_API size_t kron_gptq_quantize_antidiagonal_workspace_size(int64_t m, int64_t n);
KG_API int kron_gptq_quantize_antidiagonal(const void* W, int64_t m, int64_t n,
                                           const void* U_A, const void* U_B, kg_grid grid,
                                           int8_t* out_codes, void* out_V, void* out_E,
                                           void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Diagnostics (tracing).  The library counts every kernel launch by kind:
 *   0 init/validation, 1 in-tile sweep (leaf), 2 trailing band update (push),
 *   3 factor preparation, 4 loss and scales, 5 reserved (no launch of this kind).
 * kron_gptq_profile_enable(1) additionally brackets each launch with a pair of CUDA events
 * recorded on the launch's own stream (the events are host-side resources; no device
 * memory is allocated).  kron_gptq_profile_read() waits for the recorded events, adds
 * their elapsed times per kind, and copies the counters (launches[k], ms[k] for
 * k < nkinds; either pointer may be NULL); reset != 0 clears them afterwards.
 * Not meant for production timing loops: the events add host work per launch.
 * --------------------------------------------------------------------------------------- */
KG_API void kron_gptq_profile_enable(int enable);
KG_API int kron_gptq_profile_read(int64_t* launches, double* ms, int nkinds, int reset);

/* ---------------------------------------------------------------------------------------
 * kron_gptq_schedule_plan -- the update pieces kron_gptq_quantize (and _rc, _noalloc) issues for
 *   ndiag tile anti-diagonals (ndiag = ceil(m/64) + ceil(n/64) - 1), in issue order; host only, no
 *   device call.  The recursion of "FastKron" Section 2.5 fixes which update carries each (source,
 *   target) pair of tile anti-diagonals; the solve cuts each update into pieces by when they are
 *   needed.  Piece k is out[5k .. 5k+4] = {s0, s1, t0, t1, stream}: sources [s0, s1) to targets
 *   [t0, t1); stream 0 = critical (the near piece s1 = t0 issued just before leaf t0), 1 = urgent,
 *   2 = soon, 3 = background.  Writes at most max_pieces pieces (out may be NULL) and returns the
 *   total count, or
 *   KG_ERR_ARG for ndiag < 1 or max_pieces < 0.
 * --------------------------------------------------------------------------------------- */
KG_API int kron_gptq_schedule_plan(int ndiag, int* out, int max_pieces);

#ifdef __cplusplus
}
#endif

#endif /* KRON_GPTQ_H */
