"""ctypes binding of libkrongptq.so (see include/kron_gptq.h for the contract)."""
from __future__ import annotations

import ctypes
import os
import threading

import torch

KG_F32 = 1
KG_F64 = 2
_ERRORS = {
    -1: "KG_ERR_ARG", -2: "KG_ERR_UNSUPPORTED", -3: "KG_ERR_CUDA", -4: "KG_ERR_WORKSPACE",
    -5: "KG_ERR_NOT_PD", -6: "KG_ERR_NONFINITE", -7: "KG_ERR_TIMEOUT", -8: "KG_ERR_RANGE",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None


class KGError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        self.name = _ERRORS.get(self.code, "KG_ERR_UNKNOWN")
        super().__init__(f"{where}: {self.name} ({self.code})")


class _Grid(ctypes.Structure):
    _fields_ = [("qmin", ctypes.c_int), ("qmax", ctypes.c_int), ("row_scale", ctypes.c_void_p)]


def lib_path() -> str:
    """The in-tree library, or the build that KRON_GPTQ_LIB names (a variant built with --out)."""
    return os.environ.get("KRON_GPTQ_LIB") or os.path.join(_HERE, "libkrongptq.so")


def load_library():
    """Load the CUDA library; raise ImportError (no fallback) if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m two_sided_gptq_02_b200.build` "
                              "(there is no CPU fallback)")
        L = ctypes.CDLL(path)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        L.kron_gptq_version.restype = I
        L.kron_gptq_status_string.argtypes = [I]
        L.kron_gptq_status_string.restype = ctypes.c_char_p
        L.kron_gptq_prepare_workspace_size.argtypes = [I64]
        L.kron_gptq_prepare_workspace_size.restype = SZ
        L.kron_gptq_prepare.argtypes = [P, I64, P, I64, I, ctypes.c_double, P, P, P, P, P, SZ, P]
        L.kron_gptq_prepare.restype = I
        L.kron_gptq_quantize_workspace_size.argtypes = [I64, I64, I]
        L.kron_gptq_quantize_workspace_size.restype = SZ
        L.kron_gptq_quantize.argtypes = [P, I64, I64, I, P, P, _Grid, P, P, P, P, SZ, P]
        L.kron_gptq_quantize.restype = I
        L.kron_gptq_loss_workspace_size.argtypes = [I64, I64]
        L.kron_gptq_loss_workspace_size.restype = SZ
        L.kron_gptq_loss.argtypes = [P, P, I64, I64, I, P, P, I, ctypes.c_double, P, P, SZ, P]
        L.kron_gptq_loss.restype = I
        L.kron_gptq_row_scales.argtypes = [P, I64, I64, I, I, P, P]
        L.kron_gptq_row_scales.restype = I
        L.kron_gptq_sync_status.argtypes = [P, P]
        L.kron_gptq_sync_status.restype = I
        L.kron_gptq_quantize_noalloc.argtypes = [P, I64, I64, I, P, P, _Grid, P, P, P, P, P]
        L.kron_gptq_quantize_noalloc.restype = I
        L.kron_gptq_quantize_rc_workspace_size.argtypes = [I64, I64, I]
        L.kron_gptq_quantize_rc_workspace_size.restype = SZ
        L.kron_gptq_quantize_rc.argtypes = [P, I64, I64, I, P, P, P, P, P, P, P, P, SZ, P]
        L.kron_gptq_quantize_rc.restype = I
        L.kron_gptq_waterkron_scales.argtypes = [P, I64, P, I64, I, ctypes.c_double, P, P, P]
        L.kron_gptq_waterkron_scales.restype = I
        L.kron_gptq_code_entropy_workspace_size.argtypes = [I64]
        L.kron_gptq_code_entropy_workspace_size.restype = SZ
        L.kron_gptq_code_entropy.argtypes = [P, I64, P, P, SZ, P]
        L.kron_gptq_code_entropy.restype = I
        L.kron_gptq_quantize_onesided_workspace_size.argtypes = [I64, I64, I]
        L.kron_gptq_quantize_onesided_workspace_size.restype = SZ
        L.kron_gptq_quantize_onesided.argtypes = [P, I64, I64, I, P, _Grid, P, P, P, P, SZ, P]
        L.kron_gptq_quantize_onesided.restype = I
        L.kron_gptq_factors_workspace_size.argtypes = [I64, I64, I64]
        L.kron_gptq_factors_workspace_size.restype = SZ
        L.kron_gptq_factors.argtypes = [P, P, I64, I64, I64, I, I, I, P, P, P, SZ, P]
        L.kron_gptq_factors.restype = I
        L.kron_gptq_quantize_antidiagonal_workspace_size.argtypes = [I64, I64]
        L.kron_gptq_quantize_antidiagonal_workspace_size.restype = SZ
        L.kron_gptq_quantize_antidiagonal.argtypes = [P, I64, I64, P, P, _Grid, P, P, P, P, SZ, P]
        L.kron_gptq_quantize_antidiagonal.restype = I
        L.kron_gptq_profile_enable.argtypes = [I]
        L.kron_gptq_profile_enable.restype = None
        L.kron_gptq_profile_read.argtypes = [P, P, I, I]
        L.kron_gptq_profile_read.restype = I
        L.kron_gptq_schedule_plan.argtypes = [I, P, I]
        L.kron_gptq_schedule_plan.restype = I
        _lib = L
        return L


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KG_F32
    if t.dtype == torch.float64:
        return KG_F64
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or float64)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_dev(*ts):
    """Every tensor on the current CUDA device and contiguous: the library launches on the current
    device and takes bare pointers, so a tensor elsewhere would be read through a wrong address."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices ({dev} and {t.device})")
    if dev is not None and dev.index is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"tensors live on {dev} but the current device is cuda:{torch.cuda.current_device()}; "
                         "call under torch.cuda.device(...)")


def _check_tensor(name: str, t, dtype: torch.dtype, shape: tuple) -> None:
    """dtype and shape of one argument; the kernels index by the sizes passed beside the pointers."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_solve_args(W, U_A, U_B, row_scale, dtype=None) -> tuple[int, int]:
    """W (m, n), U_A (n, n), U_B (m, m) (skipped when None), row_scale (m,), all of W's dtype
    (or `dtype`).  Returns (m, n)."""
    if W.dim() != 2:
        raise ValueError(f"W must be a matrix, got shape {tuple(W.shape)}")
    m, n = W.shape
    dtype = W.dtype if dtype is None else dtype
    if dtype not in (torch.float32, torch.float64):
        raise TypeError(f"unsupported dtype {dtype} (float32 or float64)")
    _check_tensor("W", W, dtype, (m, n))
    _check_tensor("U_A", U_A, dtype, (n, n))
    if U_B is not None:
        _check_tensor("U_B", U_B, dtype, (m, m))
    _check_tensor("row_scale", row_scale, dtype, (m,))
    return int(m), int(n)


def _raise(rc: int, where: str):
    if rc != 0:
        raise KGError(rc, where)


def _workspace(nbytes: int, device) -> torch.Tensor:
    # the caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


PROFILE_KINDS = ("init", "leaf", "push", "prepare", "loss", "solve")


def kron_gptq_profile_enable(enable: bool) -> None:
    load_library().kron_gptq_profile_enable(1 if enable else 0)


def kron_gptq_profile_read(reset: bool = False) -> dict:
    """{kind: (launches, milliseconds)}; waits for the recorded events."""
    n = len(PROFILE_KINDS)
    launches = (ctypes.c_int64 * n)()
    ms = (ctypes.c_double * n)()
    _raise(load_library().kron_gptq_profile_read(ctypes.cast(launches, ctypes.c_void_p),
                                                 ctypes.cast(ms, ctypes.c_void_p), n, 1 if reset else 0),
           "kron_gptq_profile_read")
    return {k: (int(launches[i]), float(ms[i])) for i, k in enumerate(PROFILE_KINDS)}


SCHEDULE_STREAMS = ("critical", "urgent", "soon", "background")


def kron_gptq_schedule_plan(ndiag: int) -> list:
    """The update pieces of a solve over ndiag tile anti-diagonals, in issue order:
    [(s0, s1, t0, t1, stream)] with sources [s0, s1), targets [t0, t1) and stream an index into
    SCHEDULE_STREAMS.  Host only."""
    L = load_library()
    count = L.kron_gptq_schedule_plan(int(ndiag), None, 0)
    _raise(min(count, 0), "kron_gptq_schedule_plan")
    buf = (ctypes.c_int * (5 * max(count, 1)))()
    got = L.kron_gptq_schedule_plan(int(ndiag), ctypes.cast(buf, ctypes.c_void_p), count)
    _raise(min(got, 0), "kron_gptq_schedule_plan")
    return [tuple(buf[5 * k:5 * k + 5]) for k in range(count)]


def kron_gptq_version() -> int:
    return load_library().kron_gptq_version()


def kron_gptq_status_string(code: int) -> str:
    return load_library().kron_gptq_status_string(int(code)).decode()


def kron_gptq_sync_status(ws: torch.Tensor, stream=None) -> int:
    return load_library().kron_gptq_sync_status(_ptr(ws), _stream(stream))


def kron_gptq_prepare(A: torch.Tensor, B: torch.Tensor | None, damp: float, *, fp32_copies: bool = True,
                      stream=None, check: bool = True):
    """U_A (n x n) and U_B (m x m), upper triangular, U^T U = (X + damp*mean(diag X)*I)^{-1}.

    Returns (U_A, U_B, U_A32, U_B32); U_B* are None when B is None.
    """
    if A.dtype not in (torch.float32, torch.float64):
        raise TypeError(f"unsupported dtype {A.dtype} (float32 or float64)")
    if B is not None and B.dtype != A.dtype:
        raise TypeError("A and B must share a dtype")
    n = A.shape[0]
    m = B.shape[0] if B is not None else 0
    _check_tensor("A", A, A.dtype, (n, n))
    if B is not None:
        _check_tensor("B", B, A.dtype, (m, m))
    _check_dev(A, B)
    L = load_library()
    dev = A.device
    UA = torch.empty(n, n, dtype=torch.float64, device=dev)
    UB = torch.empty(m, m, dtype=torch.float64, device=dev) if B is not None else None
    UA32 = torch.empty(n, n, dtype=torch.float32, device=dev) if fp32_copies else None
    UB32 = torch.empty(m, m, dtype=torch.float32, device=dev) if (fp32_copies and B is not None) else None
    # a region per factor: the library then prepares the two factors side by side
    ws_bytes = L.kron_gptq_prepare_workspace_size(n) + (L.kron_gptq_prepare_workspace_size(m) if B is not None else 0)
    ws = _workspace(ws_bytes, dev)
    rc = L.kron_gptq_prepare(_ptr(A), n, _ptr(B), m, _dtype_code(A), float(damp), _ptr(UA), _ptr(UB),
                             _ptr(UA32), _ptr(UB32), _ptr(ws), ws.numel(), _stream(stream))
    _raise(rc, "kron_gptq_prepare")
    if check:
        _raise(L.kron_gptq_sync_status(_ptr(ws), _stream(stream)), "kron_gptq_prepare (device)")
    return UA, UB, UA32, UB32


def quantize_workspace_bytes(m: int, n: int, dtype: torch.dtype) -> int:
    code = KG_F64 if dtype == torch.float64 else KG_F32
    return int(load_library().kron_gptq_quantize_workspace_size(int(m), int(n), code))


class Quantizer:
    """Reusable workspace and outputs for repeated solves of one shape (no allocation per call)."""

    def __init__(self, m: int, n: int, dtype: torch.dtype, device, *, want_E: bool = False):
        self.m, self.n, self.dtype = int(m), int(n), dtype
        self.code = KG_F64 if dtype == torch.float64 else KG_F32
        L = load_library()
        self.ws = _workspace(L.kron_gptq_quantize_workspace_size(self.m, self.n, self.code), device)
        self.codes = torch.empty(self.m, self.n, dtype=torch.int8, device=device)
        self.V = torch.empty(self.m, self.n, dtype=dtype, device=device)
        self.E = torch.empty(self.m, self.n, dtype=dtype, device=device) if want_E else None

    def run(self, W, U_A, U_B, row_scale, qmin: int, qmax: int, stream=None) -> None:
        """Enqueue one solve on `stream`; does not synchronize."""
        if _check_solve_args(W, U_A, U_B, row_scale, self.dtype) != (self.m, self.n):
            raise ValueError(f"W must have shape {(self.m, self.n)}, got {tuple(W.shape)}")
        _check_tensor("U_B", U_B, self.dtype, (self.m, self.m))
        _check_dev(W, U_A, U_B, row_scale, self.codes)
        L = load_library()
        grid = _Grid(int(qmin), int(qmax), row_scale.data_ptr())
        rc = L.kron_gptq_quantize(_ptr(W), self.m, self.n, self.code, _ptr(U_A), _ptr(U_B), grid,
                                  _ptr(self.codes), _ptr(self.V), _ptr(self.E), _ptr(self.ws), self.ws.numel(),
                                  _stream(stream))
        _raise(rc, "kron_gptq_quantize")

    def status(self, stream=None) -> int:
        return kron_gptq_sync_status(self.ws, stream)


def kron_gptq_quantize(W, U_A, U_B, qmin: int, qmax: int, row_scale, *, want_E: bool = False, stream=None,
                       check: bool = True):
    """Two-sided GPTQ of W.  Returns (codes int8, V, E or None)."""
    q = Quantizer(W.shape[0], W.shape[1], W.dtype, W.device, want_E=want_E)
    q.run(W, U_A, U_B, row_scale, qmin, qmax, stream=stream)
    if check:
        _raise(q.status(stream), "kron_gptq_quantize (device)")
    return q.codes, q.V, q.E


def kron_gptq_quantize_noalloc(W, U_A, U_B, qmin: int, qmax: int, row_scale, codes, V, E=None, dev_status=None,
                               *, stream=None) -> None:
    """Allocation-free solve into caller-provided outputs (codes int8, V, optional E, optional
    one-int device status).  The library uses its fixed internal scratch array instead of a
    workspace; see include/kron_gptq.h for the size limit and the sharing rules."""
    m, n = _check_solve_args(W, U_A, U_B, row_scale)
    _check_tensor("U_B", U_B, W.dtype, (m, m))
    _check_tensor("codes", codes, torch.int8, (m, n))
    _check_tensor("V", V, W.dtype, (m, n))
    if E is not None:
        _check_tensor("E", E, W.dtype, (m, n))
    if dev_status is not None and (dev_status.dtype != torch.int32 or dev_status.numel() < 1):
        raise TypeError("dev_status must be an int32 tensor with at least one element")
    _check_dev(W, U_A, U_B, row_scale, codes, V, E, dev_status)
    L = load_library()
    grid = _Grid(int(qmin), int(qmax), row_scale.data_ptr())
    rc = L.kron_gptq_quantize_noalloc(_ptr(W), m, n, _dtype_code(W), _ptr(U_A), _ptr(U_B), grid, _ptr(codes),
                                      _ptr(V), _ptr(E), _ptr(dev_status), _stream(stream))
    _raise(rc, "kron_gptq_quantize_noalloc")


def kron_gptq_loss(W, V, A, B, damp: float, *, stream=None) -> float:
    """tr((V-W) A_d (V-W)^T B_d) with A_d, B_d damped as in prepare (fp64 accumulation)."""
    if W.dim() != 2:
        raise ValueError(f"W must be a matrix, got shape {tuple(W.shape)}")
    m, n = W.shape
    _check_tensor("V", V, W.dtype, (m, n))
    if A.dtype not in (torch.float32, torch.float64):
        raise TypeError(f"unsupported factor dtype {A.dtype}")
    _check_tensor("A", A, A.dtype, (n, n))
    _check_tensor("B", B, A.dtype, (m, m))
    _check_dev(W, V, A, B)
    L = load_library()
    out = torch.zeros(1, dtype=torch.float64, device=W.device)
    ws = _workspace(L.kron_gptq_loss_workspace_size(m, n), W.device)
    rc = L.kron_gptq_loss(_ptr(W), _ptr(V), m, n, _dtype_code(W), _ptr(A), _ptr(B), _dtype_code(A), float(damp),
                          _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _raise(rc, "kron_gptq_loss")
    _raise(L.kron_gptq_sync_status(_ptr(ws), _stream(stream)), "kron_gptq_loss (device)")
    return float(out.item())


def kron_gptq_row_scales(W, qmax: int, *, stream=None):
    if W.dim() != 2:
        raise ValueError(f"W must be a matrix, got shape {tuple(W.shape)}")
    _check_dev(W)
    L = load_library()
    m, n = W.shape
    s = torch.empty(m, dtype=W.dtype, device=W.device)
    _raise(L.kron_gptq_row_scales(_ptr(W), m, n, _dtype_code(W), int(qmax), _ptr(s), _stream(stream)),
           "kron_gptq_row_scales")
    return s


class RcQuantizer:
    """Reusable workspace and outputs for repeated solves of one shape on the row- and
    column-scaled alphabet with unclipped int32 codes (kron_gptq_quantize_rc)."""

    def __init__(self, m: int, n: int, dtype: torch.dtype, device, *, want_E: bool = False):
        self.m, self.n, self.dtype = int(m), int(n), dtype
        self.code = KG_F64 if dtype == torch.float64 else KG_F32
        L = load_library()
        self.ws = _workspace(L.kron_gptq_quantize_rc_workspace_size(self.m, self.n, self.code), device)
        self.Z = torch.empty(self.m, self.n, dtype=torch.int32, device=device)
        self.V = torch.empty(self.m, self.n, dtype=dtype, device=device)
        self.E = torch.empty(self.m, self.n, dtype=dtype, device=device) if want_E else None

    def run(self, W, U_A, U_B, alpha, beta, stream=None) -> None:
        """Enqueue one solve on `stream`; does not synchronize."""
        if _check_solve_args(W, U_A, U_B, beta, self.dtype) != (self.m, self.n):
            raise ValueError(f"W must have shape {(self.m, self.n)}, got {tuple(W.shape)}")
        _check_tensor("U_B", U_B, self.dtype, (self.m, self.m))
        _check_tensor("alpha", alpha, self.dtype, (self.n,))
        _check_dev(W, U_A, U_B, alpha, beta, self.Z)
        L = load_library()
        rc = L.kron_gptq_quantize_rc(_ptr(W), self.m, self.n, self.code, _ptr(U_A), _ptr(U_B), _ptr(alpha),
                                     _ptr(beta), _ptr(self.Z), _ptr(self.V), _ptr(self.E), _ptr(self.ws),
                                     self.ws.numel(), _stream(stream))
        _raise(rc, "kron_gptq_quantize_rc")

    def status(self, stream=None) -> int:
        return kron_gptq_sync_status(self.ws, stream)


def kron_gptq_quantize_rc(W, U_A, U_B, alpha, beta, *, want_E: bool = False, stream=None, check: bool = True):
    """Two-sided GPTQ of W on the alphabet V = beta alpha^T (.) Z, Z unclipped.
    Returns (Z int32, V, E or None)."""
    q = RcQuantizer(W.shape[0], W.shape[1], W.dtype, W.device, want_E=want_E)
    q.run(W, U_A, U_B, alpha, beta, stream=stream)
    if check:
        _raise(q.status(stream), "kron_gptq_quantize_rc (device)")
    return q.Z, q.V, q.E


def kron_gptq_waterkron_scales(U_A, U_B, gamma: float, *, stream=None):
    """WaterKron steps: alpha = sqrt(gamma) diag(U_A), beta = sqrt(gamma) diag(U_B)."""
    if U_A.dtype != U_B.dtype:
        raise TypeError("U_A and U_B must share a dtype")
    n, m = U_A.shape[0], U_B.shape[0]
    _check_tensor("U_A", U_A, U_A.dtype, (n, n))
    _check_tensor("U_B", U_B, U_A.dtype, (m, m))
    _check_dev(U_A, U_B)
    L = load_library()
    alpha = torch.empty(n, dtype=U_A.dtype, device=U_A.device)
    beta = torch.empty(m, dtype=U_B.dtype, device=U_B.device)
    _raise(L.kron_gptq_waterkron_scales(_ptr(U_A), n, _ptr(U_B), m, _dtype_code(U_A), float(gamma), _ptr(alpha),
                                        _ptr(beta), _stream(stream)), "kron_gptq_waterkron_scales")
    return alpha, beta


ENTROPY_MAX_BINS = (1 << 23) + 1   # every code of the fp32 unclipped alphabet (|Z| < 2^22)


def kron_gptq_code_entropy(Z, *, max_bins: int = ENTROPY_MAX_BINS, stream=None) -> float:
    """Empirical entropy of the int32 codes Z in bits per entry."""
    L = load_library()
    _check_dev(Z)
    if Z.dtype != torch.int32:
        raise TypeError("Z must be int32")
    out = torch.empty(1, dtype=torch.float64, device=Z.device)
    ws = _workspace(L.kron_gptq_code_entropy_workspace_size(int(max_bins)), Z.device)
    _raise(L.kron_gptq_code_entropy(_ptr(Z), Z.numel(), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "kron_gptq_code_entropy")
    _raise(L.kron_gptq_sync_status(_ptr(ws), _stream(stream)), "kron_gptq_code_entropy (device)")
    return float(out.item())


class OnesidedQuantizer:
    """Reusable workspace and outputs for repeated one-sided GPTQ solves of one shape
    (kron_gptq_quantize_onesided)."""

    def __init__(self, m: int, n: int, dtype: torch.dtype, device, *, want_E: bool = False):
        self.m, self.n, self.dtype = int(m), int(n), dtype
        self.code = KG_F64 if dtype == torch.float64 else KG_F32
        L = load_library()
        self.ws = _workspace(L.kron_gptq_quantize_onesided_workspace_size(self.m, self.n, self.code), device)
        self.codes = torch.empty(self.m, self.n, dtype=torch.int8, device=device)
        self.V = torch.empty(self.m, self.n, dtype=dtype, device=device)
        self.E = torch.empty(self.m, self.n, dtype=dtype, device=device) if want_E else None

    def run(self, W, U_A, row_scale, qmin: int, qmax: int, stream=None) -> None:
        if _check_solve_args(W, U_A, None, row_scale, self.dtype) != (self.m, self.n):
            raise ValueError(f"W must have shape {(self.m, self.n)}, got {tuple(W.shape)}")
        _check_dev(W, U_A, row_scale, self.codes)
        L = load_library()
        grid = _Grid(int(qmin), int(qmax), row_scale.data_ptr())
        rc = L.kron_gptq_quantize_onesided(_ptr(W), self.m, self.n, self.code, _ptr(U_A), grid, _ptr(self.codes),
                                           _ptr(self.V), _ptr(self.E), _ptr(self.ws), self.ws.numel(),
                                           _stream(stream))
        _raise(rc, "kron_gptq_quantize_onesided")

    def status(self, stream=None) -> int:
        return kron_gptq_sync_status(self.ws, stream)


def kron_gptq_quantize_onesided(W, U_A, qmin: int, qmax: int, row_scale, *, want_E: bool = False, stream=None,
                                check: bool = True):
    """One-sided GPTQ of W (the case B = I).  Returns (codes int8, V, E or None)."""
    q = OnesidedQuantizer(W.shape[0], W.shape[1], W.dtype, W.device, want_E=want_E)
    q.run(W, U_A, row_scale, qmin, qmax, stream=stream)
    if check:
        _raise(q.status(stream), "kron_gptq_quantize_onesided (device)")
    return q.codes, q.V, q.E


FACTOR_METHODS = {"marginal": 0, "frobenius": 1, "flipflop": 2}


def kron_gptq_factors(a, b, method: str = "flipflop", iters: int = 2, *, stream=None, check: bool = True):
    """Kronecker factors (A n x n, B m x m, fp64) of E[a a^T (x) b b^T] from samples a (N x n) and
    b (N x m): "marginal", "frobenius" or "flipflop" (iters alternating updates from B = I)."""
    if a.dtype != b.dtype:
        raise TypeError("a and b must share a dtype")
    if a.dtype not in (torch.float32, torch.float64):
        raise TypeError(f"unsupported dtype {a.dtype} (float32 or float64)")
    if a.dim() != 2 or b.dim() != 2:
        raise ValueError("a and b must be matrices (samples x channels)")
    N, n = a.shape
    if b.shape[0] != N:
        raise ValueError("a and b need the same number of samples")
    m = b.shape[1]
    if method not in FACTOR_METHODS:
        raise ValueError(f"method must be one of {sorted(FACTOR_METHODS)}")
    _check_dev(a, b)
    L = load_library()
    A = torch.empty(n, n, dtype=torch.float64, device=a.device)
    B = torch.empty(m, m, dtype=torch.float64, device=a.device)
    ws = _workspace(L.kron_gptq_factors_workspace_size(N, n, m), a.device)
    rc = L.kron_gptq_factors(_ptr(a), _ptr(b), N, n, m, _dtype_code(a), FACTOR_METHODS[method], int(iters), _ptr(A),
                             _ptr(B), _ptr(ws), ws.numel(), _stream(stream))
    _raise(rc, "kron_gptq_factors")
    if check:
        _raise(L.kron_gptq_sync_status(_ptr(ws), _stream(stream)), "kron_gptq_factors (device)")
    return A, B


def kron_gptq_quantize_antidiagonal(W, U_A, U_B, qmin: int, qmax: int, row_scale, *, want_E: bool = False,
                                    stream=None, check: bool = True):
    """The non-recursive anti-diagonal baseline (quartic work; fp64).  Same outputs as
    kron_gptq_quantize: (codes int8, V, E or None)."""
    if W.dtype != torch.float64:
        raise TypeError("the anti-diagonal baseline runs in fp64")
    m, n = _check_solve_args(W, U_A, U_B, row_scale)
    _check_tensor("U_B", U_B, W.dtype, (m, m))
    _check_dev(W, U_A, U_B, row_scale)
    L = load_library()
    ws = _workspace(L.kron_gptq_quantize_antidiagonal_workspace_size(m, n), W.device)
    codes = torch.empty(m, n, dtype=torch.int8, device=W.device)
    V = torch.empty(m, n, dtype=W.dtype, device=W.device)
    E = torch.empty(m, n, dtype=W.dtype, device=W.device) if want_E else None
    grid = _Grid(int(qmin), int(qmax), row_scale.data_ptr())
    rc = L.kron_gptq_quantize_antidiagonal(_ptr(W), m, n, _ptr(U_A), _ptr(U_B), grid, _ptr(codes), _ptr(V), _ptr(E),
                                           _ptr(ws), ws.numel(), _stream(stream))
    _raise(rc, "kron_gptq_quantize_antidiagonal")
    if check:
        _raise(L.kron_gptq_sync_status(_ptr(ws), _stream(stream)), "kron_gptq_quantize_antidiagonal (device)")
    return codes, V, E
