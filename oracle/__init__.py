"""CPU oracle for two-sided (Kronecker-factored) GPTQ.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It shares no code with the CUDA library
(``two_sided_gptq_02_b200``) and never calls it; the product never imports it.

Contents
  * ``kron_gptq_oracle.c`` (built to ``_build/liboracle.so``): float64 textbook prepare,
    the naive entry-by-entry two-sided GPTQ (the definition), one-sided GPTQ, RTN and
    the trace-form proxy loss.
  * ``literal.py``: the literal (mn) x (mn) vectorized GPTQ on kron(A_d, B_d) for tiny
    sizes, the LAPACK (numpy) form of prepare, and the certificate checker.
  * ``parity.py``: comparison of a candidate's codes with the oracle under the
    boundary rule (a decision taken at a rounding tie is absorbed and counted).

Parity status of each function (what pins it, in tests/test_oracle_pins.py):
  prepare         pinned: numpy LAPACK Cholesky/inverse, U^T U A_d = I, Kronecker
                  factor identity, log-determinant identity.
  quantize_naive  pinned: literal vectorized form (4x4, 6x5, ...), A=B=I and diagonal
                  factors reduce to RTN, B=I reduces to one-sided GPTQ, A=I reduces to
                  one-sided GPTQ of W^T, transpose symmetry, leading-block invariance,
                  loss identity, error bound, certificate.
  quantize_onesided  pinned: the vectorized form with B=I, RTN when A is diagonal.
  quantize_cubic  pinned: equals quantize_naive (codes exactly away from ties, E to 1e-9) on
                  ragged shapes; a plain reorganisation of the same sums (the CPU baseline).
  loss            pinned: closed forms (sum E^2) and numpy einsum of the definition.
  quantize_rc     pinned: literal vectorized form with a per-entry step (4x4, 6x5, ...),
                  A=B=I reduces to per-entry rounding, alpha=1 / beta=s equals
                  quantize_naive on an unclipped grid, certificate, |E| <= gamma/2 for the
                  WaterKron steps.
  waterkron_scales  the formula itself (one line); pinned through the |E| <= gamma/2 bound
                  and the high-rate distortion mn gamma^2 / 12.
  code_entropy_bits pinned: closed forms (uniform over 2^k symbols gives k bits, a constant
                  gives 0, a two-point law gives its binary entropy).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kron_gptq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
NOT_FORCED = -(2 ** 31)

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.ora_prepare.argtypes = [P, I64, ctypes.c_double, P, P]
            lib.ora_prepare.restype = ctypes.c_int
            lib.ora_row_scales.argtypes = [P, I64, I64, ctypes.c_int, P]
            lib.ora_row_scales.restype = None
            lib.ora_quantize_naive.argtypes = [P, I64, I64, P, P, P, ctypes.c_int, ctypes.c_int, P,
                                               ctypes.c_double, P, P, P, P, P]
            lib.ora_quantize_naive.restype = I64
            lib.ora_quantize_rc.argtypes = [P, I64, I64, P, P, P, P, P, ctypes.c_double, P, P, P, P, P]
            lib.ora_quantize_rc.restype = I64
            lib.ora_quantize_cubic.argtypes = [P, I64, I64, P, P, P, ctypes.c_int, ctypes.c_int, P, P, P]
            lib.ora_quantize_cubic.restype = ctypes.c_int
            lib.ora_threads.argtypes = []
            lib.ora_threads.restype = ctypes.c_int
            lib.ora_quantize_onesided.argtypes = [P, I64, I64, P, P, ctypes.c_int, ctypes.c_int, P, P, P]
            lib.ora_quantize_onesided.restype = None
            lib.ora_rtn.argtypes = [P, I64, I64, P, ctypes.c_int, ctypes.c_int, P, P]
            lib.ora_rtn.restype = None
            lib.ora_loss.argtypes = [P, P, P, P, I64, I64]
            lib.ora_loss.restype = ctypes.c_double
            _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


class OracleNotPD(ValueError):
    pass


def prepare(A, damp: float, *, return_damped: bool = False):
    """U with U^T U = (A + damp*mean(diag A)*I)^{-1}, upper triangular (float64)."""
    A = _f64(A)
    n = A.shape[0]
    U = np.zeros((n, n), dtype=np.float64)
    Ad = np.zeros((n, n), dtype=np.float64)
    rc = _load().ora_prepare(_ptr(A), n, float(damp), _ptr(U), _ptr(Ad))
    if rc == -1:
        raise OracleNotPD("factor is not positive definite")
    if rc != 0:
        raise MemoryError("oracle prepare: allocation failed")
    return (U, Ad) if return_damped else U


def row_scales(W, qmax: int):
    W = _f64(W)
    m, n = W.shape
    s = np.zeros(m, dtype=np.float64)
    _load().ora_row_scales(_ptr(W), m, n, int(qmax), _ptr(s))
    return s


def quantize_naive(W, UA, UB, s, qmin: int, qmax: int, *, forced=None, tol: float = 1e-9):
    """Two-sided GPTQ by definition.  Returns dict(codes, V, E, t, boundary, n_boundary)."""
    W, UA, UB, s = _f64(W), _f64(UA), _f64(UB), _f64(s)
    m, n = W.shape
    assert UA.shape == (n, n) and UB.shape == (m, m) and s.shape == (m,)
    codes = np.zeros((m, n), dtype=np.int32)
    V = np.zeros((m, n), dtype=np.float64)
    E = np.zeros((m, n), dtype=np.float64)
    t = np.zeros((m, n), dtype=np.float64)
    bflag = np.zeros((m, n), dtype=np.uint8)
    f = None
    if forced is not None:
        f = np.ascontiguousarray(forced, dtype=np.int32)
        assert f.shape == (m, n)
    nb = _load().ora_quantize_naive(_ptr(W), m, n, _ptr(UA), _ptr(UB), _ptr(s), int(qmin), int(qmax),
                                    _ptr(f), float(tol), _ptr(codes), _ptr(V), _ptr(E), _ptr(t), _ptr(bflag))
    if nb < 0:
        raise MemoryError("oracle quantize: allocation failed")
    return dict(codes=codes, V=V, E=E, t=t, boundary=bflag.astype(bool), n_boundary=int(nb))


def quantize_cubic(W, UA, UB, s, qmin: int, qmax: int):
    """The cubic CPU baseline: the two-chain form over anti-diagonals, OpenMP over each one's
    entries (all host cores).  Returns dict(codes, V, E)."""
    W, UA, UB, s = _f64(W), _f64(UA), _f64(UB), _f64(s)
    m, n = W.shape
    codes = np.zeros((m, n), dtype=np.int32)
    V = np.zeros((m, n), dtype=np.float64)
    E = np.zeros((m, n), dtype=np.float64)
    if _load().ora_quantize_cubic(_ptr(W), m, n, _ptr(UA), _ptr(UB), _ptr(s), int(qmin), int(qmax), _ptr(codes),
                                  _ptr(V), _ptr(E)) != 0:
        raise MemoryError("oracle quantize_cubic: allocation failed")
    return dict(codes=codes, V=V, E=E)


def cubic_threads() -> int:
    return int(_load().ora_threads())


NOT_FORCED_64 = -(2 ** 63)


def quantize_rc(W, UA, UB, alpha, beta, *, forced=None, tol: float = 1e-9):
    """Two-sided GPTQ by definition on the alphabet V = beta alpha^T (.) Z, Z unbounded
    ("WaterKron and FlipFlop Hessian", Section 2.1).  Returns dict(codes (int64), V, E, t,
    boundary, n_boundary); ``forced`` uses NOT_FORCED_64 for entries left to the rounding."""
    W, UA, UB, alpha, beta = _f64(W), _f64(UA), _f64(UB), _f64(alpha), _f64(beta)
    m, n = W.shape
    assert UA.shape == (n, n) and UB.shape == (m, m) and alpha.shape == (n,) and beta.shape == (m,)
    codes = np.zeros((m, n), dtype=np.int64)
    V = np.zeros((m, n), dtype=np.float64)
    E = np.zeros((m, n), dtype=np.float64)
    t = np.zeros((m, n), dtype=np.float64)
    bflag = np.zeros((m, n), dtype=np.uint8)
    f = None
    if forced is not None:
        f = np.ascontiguousarray(forced, dtype=np.int64)
        assert f.shape == (m, n)
    nb = _load().ora_quantize_rc(_ptr(W), m, n, _ptr(UA), _ptr(UB), _ptr(alpha), _ptr(beta), _ptr(f),
                                 float(tol), _ptr(codes), _ptr(V), _ptr(E), _ptr(t), _ptr(bflag))
    if nb < 0:
        raise MemoryError("oracle quantize_rc: allocation failed")
    return dict(codes=codes, V=V, E=E, t=t, boundary=bflag.astype(bool), n_boundary=int(nb))


def waterkron_scales(UA, UB, gamma: float):
    """WaterKron steps ("WaterKron and FlipFlop Hessian", Section 3): alpha_j proportional to
    1 / L^(A)_jj = U_A[j,j] and beta_i proportional to U_B[i,i].  One knob gamma > 0 sets
    both constants (alpha = sqrt(gamma) diag U_A, beta = sqrt(gamma) diag U_B), so that the
    step of entry (i,j) is gamma U_B[i,i] U_A[j,j] and every error E_ij = (x - Q)/(U_B[i,i]
    U_A[j,j]) lies in [-gamma/2, gamma/2]."""
    r = np.sqrt(float(gamma))
    return r * np.diag(_f64(UA)).copy(), r * np.diag(_f64(UB)).copy()


def code_entropy_bits(Z) -> float:
    """Empirical (plug-in) entropy of the integer entries of Z in bits per entry: the
    memory cost of Z under a good entropy coder ("WaterKron and FlipFlop Hessian",
    Section 2.1).  H = -sum_z p_z log2 p_z with p_z the frequency of value z."""
    Z = np.asarray(Z).reshape(-1)
    if Z.size == 0:
        return 0.0
    _, counts = np.unique(Z, return_counts=True)
    p = counts.astype(np.float64) / Z.size
    return float(-(p * np.log2(p)).sum())


def quantize_onesided(W, U, S, qmin: int, qmax: int):
    """Standard GPTQ with per-entry scale S (m x n).  Returns dict(codes, V, E)."""
    W, U, S = _f64(W), _f64(U), _f64(S)
    m, n = W.shape
    codes = np.zeros((m, n), dtype=np.int32)
    V = np.zeros((m, n), dtype=np.float64)
    E = np.zeros((m, n), dtype=np.float64)
    _load().ora_quantize_onesided(_ptr(W), m, n, _ptr(U), _ptr(S), int(qmin), int(qmax),
                                  _ptr(codes), _ptr(V), _ptr(E))
    return dict(codes=codes, V=V, E=E)


def rtn(W, S, qmin: int, qmax: int):
    W, S = _f64(W), _f64(S)
    m, n = W.shape
    codes = np.zeros((m, n), dtype=np.int32)
    V = np.zeros((m, n), dtype=np.float64)
    _load().ora_rtn(_ptr(W), m, n, _ptr(S), int(qmin), int(qmax), _ptr(codes), _ptr(V))
    return dict(codes=codes, V=V)


def loss(W, V, Ad, Bd) -> float:
    W, V, Ad, Bd = _f64(W), _f64(V), _f64(Ad), _f64(Bd)
    m, n = W.shape
    return float(_load().ora_loss(_ptr(W), _ptr(V), _ptr(Ad), _ptr(Bd), m, n))


from .literal import (  # noqa: E402,F401
    certificate,
    certificate_rc,
    damped,
    literal_vec,
    literal_vec_entry,
    prepare_lapack,
)
from .parity import compare_with_oracle, compare_with_oracle_rc  # noqa: E402,F401
