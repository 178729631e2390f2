"""Companion forms of the oracle (numpy, float64).  TEST INFRASTRUCTURE.

* ``literal_vec``: the two-sided problem written literally as 1-D GPTQ on the vector
  vecop(W) of length mn with the (mn) x (mn) Gram matrix kron(A_d, B_d)
  ("WaterKron and FlipFlop Hessian", Section 3: W-hat = vecop(W)^T, A-hat = A (x) B;
  "FastKron", Section 2.2).  Tiny sizes only: it forms and inverts the (mn)^2 matrix.
* ``prepare_lapack``: the same four prepare steps as the C oracle (damp, Cholesky,
  inverse, upper Cholesky of the inverse) with numpy's LAPACK routines as the steps;
  used where the textbook C loops would take minutes.
* ``literal_vec_entry``: the same with a step per coordinate and unclipped integers.
* ``certificate`` / ``certificate_rc``: a check of a solver's output that holds at any size.  The
  recurrences of two-sided GPTQ imply V - W = -U_B^T E U_A exactly (each update adds a
  column of kron(U_A,U_B)^T times the scaled error), and every code is the rounding of
  the value W~ = V + E * (u_B u_A^T) the entry had when it was visited (u = diag U).
  By triangularity these two facts determine (codes, E) uniquely, ties aside.
"""
from __future__ import annotations

import numpy as np


def damped(A, damp: float):
    A = np.asarray(A, dtype=np.float64)
    return A + damp * np.mean(np.diag(A)) * np.eye(A.shape[0])


def prepare_lapack(A, damp: float):
    """Upper U with U^T U = A_d^{-1}: numpy Cholesky, inverse via the Cholesky factor,
    then Cholesky of the inverse (transposed to the upper factor)."""
    Ad = damped(A, damp)
    L = np.linalg.cholesky(Ad)
    Li = np.linalg.inv(L)
    Ai = Li.T @ Li
    Ai = 0.5 * (Ai + Ai.T)
    return np.linalg.cholesky(Ai).T.copy()


def literal_vec(W, Ad, Bd, s, qmin: int, qmax: int, forced=None):
    """1-D GPTQ on w = vecop(W) with Gram H = kron(Ad, Bd), index p = j*m + i.

    K = upper Cholesky of H^{-1};  for p in order: c = clamp(rint(w_p/s)), q = s c,
    e_p = (w_p - q)/K_pp,  w_{p+1:} -= e_p K_{p,p+1:}.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    H = np.kron(np.asarray(Ad, dtype=np.float64), np.asarray(Bd, dtype=np.float64))
    Hi = np.linalg.inv(H)
    Hi = 0.5 * (Hi + Hi.T)
    K = np.linalg.cholesky(Hi).T
    w = W.T.reshape(-1).copy()          # column-major vectorization
    svec = np.tile(np.asarray(s, dtype=np.float64), n)
    N = m * n
    c = np.zeros(N, dtype=np.int64)
    q = np.zeros(N)
    e = np.zeros(N)
    for p in range(N):
        x = w[p]
        if forced is not None and forced[p % m, p // m] != -(2 ** 31):
            cp = forced[p % m, p // m]
        else:
            cp = min(max(np.rint(x / svec[p]), qmin), qmax)
        c[p] = cp
        q[p] = svec[p] * cp
        e[p] = (x - q[p]) / K[p, p]
        w[p + 1:] -= e[p] * K[p, p + 1:]
    unvec = lambda v: v.reshape(n, m).T.copy()
    return dict(codes=unvec(c).astype(np.int32), V=unvec(q), E=unvec(e), K=K)


def literal_vec_entry(W, Ad, Bd, S):
    """1-D GPTQ on w = vecop(W) with Gram kron(Ad, Bd) and a step per coordinate
    (S, m x n), integers not clipped ("WaterKron and FlipFlop Hessian", Sections 2.1 and 3:
    alpha-hat = alpha (x) beta on the vectorized problem)."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    H = np.kron(np.asarray(Ad, dtype=np.float64), np.asarray(Bd, dtype=np.float64))
    Hi = np.linalg.inv(H)
    Hi = 0.5 * (Hi + Hi.T)
    K = np.linalg.cholesky(Hi).T
    w = W.T.reshape(-1).copy()
    svec = np.asarray(S, dtype=np.float64).T.reshape(-1)
    N = m * n
    c = np.zeros(N, dtype=np.int64)
    q = np.zeros(N)
    e = np.zeros(N)
    for p in range(N):
        x = w[p]
        c[p] = np.rint(x / svec[p])
        q[p] = svec[p] * c[p]
        e[p] = (x - q[p]) / K[p, p]
        w[p + 1:] -= e[p] * K[p, p + 1:]
    unvec = lambda v: v.reshape(n, m).T.copy()
    return dict(codes=unvec(c), V=unvec(q), E=unvec(e), K=K)


def certificate_rc(W, UA, UB, alpha, beta, codes, V, E, rows=None, tol: float = 1e-9):
    """The certificate for the row- and column-scaled alphabet: (1) V - W + U_B^T E U_A = 0,
    (2) codes = rint(W~ / (beta_i alpha_j)), (3) |W~ - V| <= step / 2, with
    W~ = V + E * (u_B u_A^T)."""
    W = np.asarray(W, dtype=np.float64)
    UA = np.asarray(UA, dtype=np.float64)
    UB = np.asarray(UB, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    codes = np.asarray(codes)
    m, n = W.shape
    if rows is None:
        rows = np.arange(m)
        corr = UB.T @ E @ UA
    else:
        rows = np.asarray(rows)
        corr = np.stack([(UB[: i + 1, i] @ E[: i + 1, :]) @ UA for i in rows])
    resid = V[rows] - W[rows] + corr
    scale = max(np.abs(W[rows]).max(), 1e-300)
    uB = np.diag(UB)[rows]
    uA = np.diag(UA)
    Wt = V[rows] + E[rows] * (uB[:, None] * uA[None, :])
    step = beta[rows, None] * alpha[None, :]
    t = Wt / step
    f = np.floor(t)
    tie = np.abs(t - (f + 0.5)) < tol
    mism = (np.rint(t) != codes[rows]) & ~tie
    half = np.abs(Wt - V[rows]) > (0.5 + tol) * step
    return dict(resid_abs=float(np.abs(resid).max()), resid_rel=float(np.abs(resid).max() / scale),
                code_mismatch=int(mism.sum()), halfstep_violations=int(half.sum()), rows=len(rows))


def certificate(W, UA, UB, s, qmin: int, qmax: int, codes, V, E, rows=None, tol: float = 1e-9):
    """Check (1) V - W + U_B^T E U_A = 0, (2) codes = clamp(rint(W~/s)) with
    W~ = V + E*(u_B u_A^T), (3) |W~ - Q| <= s/2 where unclipped.

    ``rows``: optional row indices (sampled check at large sizes).
    Returns a dict with the residual (absolute, and relative to max|W| of the rows),
    the number of code mismatches away from rounding ties, and half-step violations.
    """
    W = np.asarray(W, dtype=np.float64)
    UA = np.asarray(UA, dtype=np.float64)
    UB = np.asarray(UB, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    codes = np.asarray(codes)
    m, n = W.shape
    if rows is None:
        rows = np.arange(m)
        corr = UB.T @ E @ UA
    else:
        rows = np.asarray(rows)
        corr = np.stack([(UB[: i + 1, i] @ E[: i + 1, :]) @ UA for i in rows])
    resid = V[rows] - W[rows] + corr
    scale = max(np.abs(W[rows]).max(), 1e-300)
    uB = np.diag(UB)[rows]
    uA = np.diag(UA)
    Wt = V[rows] + E[rows] * (uB[:, None] * uA[None, :])
    t = Wt / s[rows, None]
    c_re = np.clip(np.rint(t), qmin, qmax)
    f = np.floor(t)
    tie = (np.abs(t - (f + 0.5)) < tol) & (f >= qmin) & (f + 1 <= qmax)
    mism = (c_re != codes[rows]) & ~tie
    unclipped = (np.rint(t) >= qmin) & (np.rint(t) <= qmax)
    half = np.abs(Wt - V[rows]) > (0.5 + tol) * s[rows, None]
    return dict(resid_abs=float(np.abs(resid).max()), resid_rel=float(np.abs(resid).max() / scale),
                code_mismatch=int(mism.sum()), halfstep_violations=int((half & unclipped).sum()),
                rows=len(rows))
