"""Kronecker factors A (n x n), B (m x m) of H = E[a a^T (x) b b^T] from samples.  TEST INFRASTRUCTURE.

Samples a_k (input of the linear unit, length n) and b_k (gradient at its output, length m),
k = 1..N; E is the sample mean ("FastKron", Section 3.2 and Appendix E.2: the Hessian is an
expectation of Kronecker products, not itself one; "WaterKron and FlipFlop Hessian", Table 1 and
Section 5).  Three approximations H ~ A (x) B, all float64:

  * Marginal (independence):  A = E[a a^T],  B = E[b b^T].
  * Frobenius (alternating least squares on ||H - A (x) B||_F, a power iteration): with B fixed
    the best A is E[(b^T B b) a a^T] / ||B||_F^2, and with A fixed the best B is
    E[(a^T A a) b b^T] / ||A||_F^2.
  * FlipFlop (the same alternation with the reciprocal weighting, the Gaussian flip-flop):
    A = E[(b^T B^-1 b) a a^T] / m,  B = E[(a^T A^-1 a) b b^T] / n.
Both iterations start from B = I (Table 1 starts them from the identity); one iteration
updates A, then B.  The normalisations (a reading: the pages' displayed formulas were lost) fix
only the split of a common scale between A and B, which two-sided GPTQ does not see.

Parity status: pinned in tests/test_oracle_pins.py -- an exactly Kronecker H (a factorial sample
design) is reproduced by all three; Frobenius reaches the Van Loan-Pitsianis optimum (numpy SVD
of the rearranged H); FlipFlop is a local minimum of the scale-free mismatch
tr(H (A (x) B)^-1) |A (x) B|^(1/mn) / (mn); scale covariance.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def hessian(a, b):
    """H = mean_k kron(a_k a_k^T, b_k b_k^T), (nm) x (nm); tiny sizes only."""
    a, b = _f64(a), _f64(b)
    N = a.shape[0]
    H = np.zeros((a.shape[1] * b.shape[1],) * 2)
    for k in range(N):
        H += np.kron(np.outer(a[k], a[k]), np.outer(b[k], b[k]))
    return H / N


def _weighted_gram(x, w):
    return (x.T * w) @ x / x.shape[0]


def marginal(a, b):
    a, b = _f64(a), _f64(b)
    return _weighted_gram(a, np.ones(a.shape[0])), _weighted_gram(b, np.ones(b.shape[0]))


def frobenius(a, b, iters: int = 1):
    a, b = _f64(a), _f64(b)
    B = np.eye(b.shape[1])
    A = None
    for _ in range(iters):
        w = np.einsum("ki,ij,kj->k", b, B, b)
        A = _weighted_gram(a, w) / np.sum(B * B)
        v = np.einsum("ki,ij,kj->k", a, A, a)
        B = _weighted_gram(b, v) / np.sum(A * A)
    return A, B


def flipflop(a, b, iters: int = 1):
    a, b = _f64(a), _f64(b)
    n, m = a.shape[1], b.shape[1]
    B = np.eye(m)
    A = None
    for _ in range(iters):
        w = np.einsum("ki,ij,kj->k", b, np.linalg.inv(B), b)
        A = _weighted_gram(a, w) / m
        v = np.einsum("ki,ij,kj->k", a, np.linalg.inv(A), a)
        B = _weighted_gram(b, v) / n
    return A, B


def rearrange(H, n: int, m: int):
    """Van Loan-Pitsianis rearrangement: R[(i1,j1), (i2,j2)] = H[(i1,i2), (j1,j2)] in kron(A, B)
    block indexing (A n x n, B m x m), so that ||H - A (x) B||_F = ||R - vec(A) vec(B)^T||_F."""
    return H.reshape(n, m, n, m).transpose(0, 2, 1, 3).reshape(n * n, m * m)


def mismatch(H, A, B):
    """Scale-free mismatch tr(H (A (x) B)^-1) |A (x) B|^(1/mn) / (mn)."""
    n, m = A.shape[0], B.shape[0]
    K = np.kron(A, B)
    sign, logdet = np.linalg.slogdet(K)
    return float(np.trace(H @ np.linalg.inv(K)) * np.exp(logdet / (n * m)) / (n * m))
