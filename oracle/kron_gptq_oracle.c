/*
 * kron_gptq_oracle.c -- the CPU oracle for two-sided (Kronecker-factored) GPTQ.
 *
 * TEST INFRASTRUCTURE.  This file is the plain, slow, obviously correct statement of
 * what the CUDA library computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * Everything is float64, single threaded, row-major, with no blocking and no reordering
 * beyond what the definitions state.  Sources (page title, section):
 *
 *  [WK]  "WaterKron and FlipFlop Hessian: Information-Theoretically Grounded Quantization
 *         with Kronecker-Factored Hessians", Section 2 (Notation), Section 2.1 (Alphabet),
 *         Section 3 (the vectorized problem: W-hat = vecop(W)^T, A-hat = A (x) B).
 *  [FK]  "FastKron: Efficient Quantization with Kronecker-Factored Hessians" (later
 *         "BaKron"), Section 2.1 (notation, quantize replaces round, clipping allowed),
 *         Section 2.2 (FastKron-naive = GPTQ on vecop(W) with Hessian A (x) B, loss
 *         D_{A,B}), Section 2.3 (updates only reach entries to the bottom-right),
 *         Section 2.6 (inverse and Cholesky are a separate O(n^3) step).
 *  [G2D] "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding" (abstract): GPTQ is Babai's
 *         nearest-plane algorithm; the two-sided case is the 1-D algorithm applied
 *         verbatim to the vectorized matrix with a Kronecker Gram matrix.
 *
 * Conventions fixed here (the pages' printed algorithms were lost; these are the
 * plainest readings the prose supports):
 *  - W is m x n (row i = output channel, column j = input channel); A is n x n (input
 *    side), B is m x m (output side); vecop is column-major, so entry (i,j) has vector
 *    index p = j*m + i and the Gram matrix is kron(A, B) in that index order [WK Sec. 2].
 *  - U_A is the upper-triangular Cholesky factor of A_d^{-1} (U_A^T U_A = A_d^{-1}),
 *    U_B likewise; kron(U_A, U_B) is then the upper Cholesky factor of kron(A_d,B_d)^{-1}.
 *  - damping: A_d = A + damp * mean(diag A) * I, each factor with its own mean [WK Sec. 2
 *    allows adding a small multiple of the identity to each factor].
 *  - quantize(x) = s_i * clamp(rint(x / s_i), qmin, qmax), rint = round half to even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_NOT_FORCED INT32_MIN

/* ------------------------------------------------------------------------------------
 * Factor preparation [WK Sec. 2 Notation; FK Sec. 2.6: the inverse of each factor and a
 * Cholesky factorisation of it are a separate step before the rounding].  Four textbook steps,
 * in this order:
 *   1. A_d = A + damp * mean(diag A) * I
 *   2. L   = Cholesky(A_d)               (lower, L L^T = A_d)
 *   3. A_d^{-1} = L^{-T} L^{-1}          (via the inverse of L by forward substitution)
 *   4. U   = upper Cholesky of A_d^{-1}  (U^T U = A_d^{-1})
 * Returns 0, or -1 when a pivot of step 2 or step 4 is not positive.
 * ------------------------------------------------------------------------------------ */
int ora_prepare(const double* A, int64_t n, double damp, double* U, double* Ad_out)
{
    double* Ad = (double*)malloc(sizeof(double) * n * n);
    double* L = (double*)calloc((size_t)(n * n), sizeof(double));
    double* Li = (double*)calloc((size_t)(n * n), sizeof(double));
    double* Ai = (double*)malloc(sizeof(double) * n * n);
    int rc = 0;
    if (!Ad || !L || !Li || !Ai) { rc = -2; goto done; }

    double md = 0.0;
    for (int64_t i = 0; i < n; ++i) md += A[i * n + i];
    md /= (double)n;
    for (int64_t i = 0; i < n * n; ++i) Ad[i] = A[i];
    for (int64_t i = 0; i < n; ++i) Ad[i * n + i] += damp * md;
    if (Ad_out) memcpy(Ad_out, Ad, sizeof(double) * n * n);

    /* 2. Cholesky-Banachiewicz, row by row */
    for (int64_t i = 0; i < n; ++i) {
        for (int64_t j = 0; j <= i; ++j) {
            double s = Ad[i * n + j];
            for (int64_t k = 0; k < j; ++k) s -= L[i * n + k] * L[j * n + k];
            if (i == j) {
                if (!(s > 0.0)) { rc = -1; goto done; }
                L[i * n + i] = sqrt(s);
            } else {
                L[i * n + j] = s / L[j * n + j];
            }
        }
    }
    /* 3a. L^{-1}: solve L x = e_c column by column (forward substitution) */
    for (int64_t c = 0; c < n; ++c) {
        for (int64_t i = c; i < n; ++i) {
            double s = (i == c) ? 1.0 : 0.0;
            for (int64_t k = c; k < i; ++k) s -= L[i * n + k] * Li[k * n + c];
            Li[i * n + c] = s / L[i * n + i];
        }
    }
    /* 3b. A_d^{-1} = (L^{-1})^T (L^{-1}) */
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double s = 0.0;
            for (int64_t k = (i > j ? i : j); k < n; ++k) s += Li[k * n + i] * Li[k * n + j];
            Ai[i * n + j] = s;
        }
    /* 4. upper Cholesky U^T U = A_d^{-1}, row by row of U */
    memset(U, 0, sizeof(double) * n * n);
    for (int64_t i = 0; i < n; ++i) {
        double s = Ai[i * n + i];
        for (int64_t k = 0; k < i; ++k) s -= U[k * n + i] * U[k * n + i];
        if (!(s > 0.0)) { rc = -1; goto done; }
        double uii = sqrt(s);
        U[i * n + i] = uii;
        for (int64_t j = i + 1; j < n; ++j) {
            double t = Ai[i * n + j];
            for (int64_t k = 0; k < i; ++k) t -= U[k * n + i] * U[k * n + j];
            U[i * n + j] = t / uii;
        }
    }
done:
    free(Ad); free(L); free(Li); free(Ai);
    return rc;
}

/* Per-row scale s_i = max_j |W_ij| / qmax; an all-zero row gets scale 1 so that its
 * codes are 0.  The scales are chosen up front from the original W, before any update
 * [WK Sec. 2.4: the scales are fixed before the rounding starts and passed in]. */
void ora_row_scales(const double* W, int64_t m, int64_t n, int qmax, double* s)
{
    for (int64_t i = 0; i < m; ++i) {
        double mx = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double a = fabs(W[i * n + j]);
            if (a > mx) mx = a;
        }
        s[i] = (mx > 0.0) ? mx / (double)qmax : 1.0;
    }
}

static double ora_clamp(double c, int qmin, int qmax)
{
    if (c < (double)qmin) return (double)qmin;
    if (c > (double)qmax) return (double)qmax;
    return c;
}

/* A pre-rounding value t = x/s is a boundary value when it lies within tol of a
 * half-integer and both neighbouring grid points are inside [qmin, qmax]. */
static int ora_is_boundary(double t, double tol, int qmin, int qmax)
{
    double f = floor(t);
    if (f < (double)qmin || f + 1.0 > (double)qmax) return 0;
    return fabs(t - (f + 0.5)) < tol;
}

/* ------------------------------------------------------------------------------------
 * Two-sided GPTQ by definition [FK Sec. 2.2; G2D abstract; WK Sec. 3]: standard GPTQ on
 * the vector vecop(W) with Gram kron(A_d, B_d), written in matrix coordinates.  Entries
 * are visited in vecop order (column j outer, row i inner).  For entry (i,j):
 *     x = W~[i,j];  c = clamp(rint(x/s_i));  Q = s_i c;
 *     e = (x - Q) / (U_B[i,i] U_A[j,j]);
 *     W~[i',j'] -= U_B[i,i'] * e * U_A[j,j']   for all i' >= i, j' >= j, (i',j') != (i,j)
 * which is row p of kron(U_A, U_B) applied to the vector error -- the update touches only
 * entries to the bottom-right [FK Sec. 2.3].
 *
 * forced (nullable, m*n): a code other than ORA_NOT_FORCED replaces the rounding decision
 * at that entry (used by the parity tests to absorb a decision taken at a rounding tie).
 * tmin (nullable, m*n): receives x/s_i for every entry (pre-rounding value in grid units).
 * Returns the number of boundary entries (|x/s - half-integer| < tol, unclipped).
 * ------------------------------------------------------------------------------------ */
int64_t ora_quantize_naive(const double* W, int64_t m, int64_t n,
                           const double* UA, const double* UB, const double* s,
                           int qmin, int qmax, const int32_t* forced, double tol,
                           int32_t* codes, double* V, double* E, double* tpre, uint8_t* bflag)
{
    double* Wt = (double*)malloc(sizeof(double) * (size_t)(m * n));
    if (!Wt) return -1;
    memcpy(Wt, W, sizeof(double) * (size_t)(m * n));
    int64_t nb = 0;
    for (int64_t j = 0; j < n; ++j) {
        for (int64_t i = 0; i < m; ++i) {
            const int64_t p = i * n + j;
            const double x = Wt[p];
            const double t = x / s[i];
            double c;
            if (forced && forced[p] != ORA_NOT_FORCED) c = (double)forced[p];
            else c = ora_clamp(rint(t), qmin, qmax);
            const int b = ora_is_boundary(t, tol, qmin, qmax);
            nb += b;
            if (bflag) bflag[p] = (uint8_t)b;
            if (tpre) tpre[p] = t;
            const double q = s[i] * c;
            const double e = (x - q) / (UB[i * m + i] * UA[j * n + j]);
            codes[p] = (int32_t)c;
            V[p] = q;
            if (E) E[p] = e;
            for (int64_t ip = i; ip < m; ++ip) {
                const double be = UB[i * m + ip] * e;
                if (be == 0.0) continue;
                double* row = Wt + ip * n;
                for (int64_t jp = j; jp < n; ++jp) {
                    if (ip == i && jp == j) continue;
                    row[jp] -= be * UA[j * n + jp];
                }
            }
        }
    }
    free(Wt);
    return nb;
}

/* ------------------------------------------------------------------------------------
 * The same algorithm on the row- and column-scaled alphabet with unbounded integers
 * [WK Sec. 2.1: V = beta alpha^T (.) Z with Z integer and not clipped; the scales are
 * chosen up front and handed to the algorithm].  Entry (i,j) has grid step
 * s_ij = beta_i * alpha_j:
 *     x = W~[i,j];  z = rint(x / s_ij);  Q = s_ij z;  e = (x - Q) / (U_B[i,i] U_A[j,j]);
 * followed by the same bottom-right update as ora_quantize_naive.  Codes are int64.
 * forced (nullable): a code other than INT64_MIN replaces the decision at that entry.
 * Returns the number of boundary entries (|x/s_ij - half-integer| < tol).
 * ------------------------------------------------------------------------------------ */
int64_t ora_quantize_rc(const double* W, int64_t m, int64_t n,
                        const double* UA, const double* UB, const double* alpha, const double* beta,
                        const int64_t* forced, double tol,
                        int64_t* codes, double* V, double* E, double* tpre, uint8_t* bflag)
{
    double* Wt = (double*)malloc(sizeof(double) * (size_t)(m * n));
    if (!Wt) return -1;
    memcpy(Wt, W, sizeof(double) * (size_t)(m * n));
    int64_t nb = 0;
    for (int64_t j = 0; j < n; ++j) {
        for (int64_t i = 0; i < m; ++i) {
            const int64_t p = i * n + j;
            const double x = Wt[p];
            const double sij = beta[i] * alpha[j];
            const double t = x / sij;
            double z;
            if (forced && forced[p] != INT64_MIN) z = (double)forced[p];
            else z = rint(t);
            const double f = floor(t);
            const int b = fabs(t - (f + 0.5)) < tol;
            nb += b;
            if (bflag) bflag[p] = (uint8_t)b;
            if (tpre) tpre[p] = t;
            const double q = sij * z;
            const double e = (x - q) / (UB[i * m + i] * UA[j * n + j]);
            codes[p] = (int64_t)z;
            V[p] = q;
            if (E) E[p] = e;
            for (int64_t ip = i; ip < m; ++ip) {
                const double be = UB[i * m + ip] * e;
                if (be == 0.0) continue;
                double* row = Wt + ip * n;
                for (int64_t jp = j; jp < n; ++jp) {
                    if (ip == i && jp == j) continue;
                    row[jp] -= be * UA[j * n + jp];
                }
            }
        }
    }
    free(Wt);
    return nb;
}

/* ------------------------------------------------------------------------------------
 * Standard one-sided GPTQ [FK Sec. 2.2, "Algorithm 1"; WK Sec. 2.2]: columns in order,
 * all rows of a column rounded at once, error fed forward along the row through the
 * upper Cholesky factor U of A_d^{-1}.  The scale is given per entry (S, m x n) so that
 * the same routine also serves the transposed problem.
 * ------------------------------------------------------------------------------------ */
void ora_quantize_onesided(const double* W, int64_t m, int64_t n, const double* U,
                           const double* S, int qmin, int qmax,
                           int32_t* codes, double* V, double* E)
{
    double* Wt = (double*)malloc(sizeof(double) * (size_t)(m * n));
    memcpy(Wt, W, sizeof(double) * (size_t)(m * n));
    for (int64_t j = 0; j < n; ++j) {
        for (int64_t i = 0; i < m; ++i) {
            const int64_t p = i * n + j;
            const double x = Wt[p];
            const double c = ora_clamp(rint(x / S[p]), qmin, qmax);
            const double q = S[p] * c;
            const double e = (x - q) / U[j * n + j];
            codes[p] = (int32_t)c;
            V[p] = q;
            if (E) E[p] = e;
            for (int64_t jp = j + 1; jp < n; ++jp) Wt[i * n + jp] -= e * U[j * n + jp];
        }
    }
    free(Wt);
}

/* Round to nearest on the grid, no error feedback [FK Sec. 1: the baseline that GPTQ-style
 * error feedback improves on]; per-entry scale S. */
void ora_rtn(const double* W, int64_t m, int64_t n, const double* S, int qmin, int qmax,
             int32_t* codes, double* V)
{
    for (int64_t p = 0; p < m * n; ++p) {
        const double c = ora_clamp(rint(W[p] / S[p]), qmin, qmax);
        codes[p] = (int32_t)c;
        V[p] = S[p] * c;
    }
}

/* Proxy loss D_{A,B} = vec(V-W)^T (A_d (x) B_d) vec(V-W) = tr((V-W) A_d (V-W)^T B_d)
 * [FK Sec. 2.2; WK Sec. 2.3], accumulated in long double:
 *     loss = sum_{i,j} (D A_d)_{ij} (B_d D)_{ij},  D = V - W. */
double ora_loss(const double* W, const double* V, const double* Ad, const double* Bd,
                int64_t m, int64_t n)
{
    double* D = (double*)malloc(sizeof(double) * (size_t)(m * n));
    for (int64_t p = 0; p < m * n; ++p) D[p] = V[p] - W[p];
    long double acc = 0.0L;
    for (int64_t i = 0; i < m; ++i) {
        for (int64_t j = 0; j < n; ++j) {
            long double da = 0.0L, bd = 0.0L;
            for (int64_t k = 0; k < n; ++k) da += (long double)D[i * n + k] * Ad[k * n + j];
            for (int64_t k = 0; k < m; ++k) bd += (long double)Bd[i * m + k] * D[k * n + j];
            acc += da * bd;
        }
    }
    free(D);
    return (double)acc;
}

/* ------------------------------------------------------------------------------------
 * The cubic CPU baseline: the same algorithm in its two-chain form, entry by entry over the
 * anti-diagonals d = i + j, the entries of one anti-diagonal in parallel (OpenMP) -- no tiles,
 * no batching.  Two-chain reading of the batched update W -= U_B^T E U_A ("FastKron",
 * Sections 2.3-2.4): the error of entry (i,j) enters later entries of its row through
 *     R[i][j'] += E_ij U_A[j][j']                       (j' > j, the row chain)
 * and, once (i,j) is solved, its complete X_ij = R[i][j] + E_ij U_A[j][j] enters later entries of
 * its column through
 *     W~[i'][j] -= U_B[i][i'] X_ij                       (i' > i, the column chain),
 * so that x = W~[i][j] - U_B[i][i] R[i][j].  Work mn(m+n)/2 multiply-adds; the entries of one
 * anti-diagonal write disjoint rows of R and disjoint columns of W~ (kept transposed, WT[j][i]).
 * Rounding as in ora_quantize_naive.  Returns 0, or -1 when memory runs out.
 * ------------------------------------------------------------------------------------ */
int ora_quantize_cubic(const double* W, int64_t m, int64_t n,
                       const double* UA, const double* UB, const double* s,
                       int qmin, int qmax, int32_t* codes, double* V, double* E)
{
    double* WT = (double*)malloc(sizeof(double) * (size_t)(m * n));
    double* R = (double*)calloc((size_t)(m * n), sizeof(double));
    if (!WT || !R) { free(WT); free(R); return -1; }
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) WT[j * m + i] = W[i * n + j];
    for (int64_t d = 0; d < m + n - 1; ++d) {
        const int64_t i0 = d - n + 1 > 0 ? d - n + 1 : 0;
        const int64_t i1 = d < m - 1 ? d : m - 1;
#pragma omp parallel for schedule(static)
        for (int64_t i = i0; i <= i1; ++i) {
            const int64_t j = d - i;
            const int64_t p = i * n + j;
            const double* ra = UA + j * n;             /* row j of U_A */
            const double* rb = UB + i * m;             /* row i of U_B */
            double* rr = R + i * n;                    /* row i of R */
            double* wc = WT + j * m;                   /* column j of W~ */
            const double x = wc[i] - rb[i] * rr[j];
            const double c = ora_clamp(rint(x / s[i]), qmin, qmax);
            const double q = s[i] * c;
            const double e = (x - q) / (rb[i] * ra[j]);
            codes[p] = (int32_t)c;
            V[p] = q;
            if (E) E[p] = e;
            const double X = rr[j] + e * ra[j];
            for (int64_t jp = j + 1; jp < n; ++jp) rr[jp] += e * ra[jp];
            for (int64_t ip = i + 1; ip < m; ++ip) wc[ip] -= rb[ip] * X;
        }
    }
    free(WT);
    free(R);
    return 0;
}

/* threads the OpenMP loops of ora_quantize_cubic use */
#include <omp.h>
int ora_threads(void) { return omp_get_max_threads(); }
