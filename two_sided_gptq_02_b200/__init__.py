"""Two-sided (Kronecker-factored) GPTQ on NVIDIA B200 -- Python binding.

Thin ctypes binding of the C ABI in ``include/kron_gptq.h`` (library ``libkrongptq.so``,
built in-tree by ``python -m two_sided_gptq_02_b200.build``).  Every step of the solve runs
in the library's CUDA kernels; this module only marshals arguments.  PyTorch provides
device memory and streams.  There is no CPU fallback: if the library is missing the import
of the binding fails with an error that says how to build it.

Public functions mirror the C names:
    kron_gptq_prepare(A, B, damp)          -> U_A, U_B (fp64) and fp32 copies
    kron_gptq_quantize(W, U_A, U_B, ...)   -> codes (int8), V, E
    kron_gptq_loss(W, V, A, B, damp)       -> float
    kron_gptq_row_scales(W, qmax)          -> per-row scales
    kron_gptq_quantize_rc(W, U_A, U_B, alpha, beta) -> Z (int32), V, E  (row- and column-scaled
                                              alphabet, unclipped codes)
    kron_gptq_waterkron_scales(U_A, U_B, gamma)     -> alpha, beta (WaterKron steps)
    kron_gptq_code_entropy(Z)                       -> bits per entry
    kron_gptq_quantize_onesided(W, U_A, ...)        -> codes (int8), V, E  (one-sided GPTQ, B = I)
    kron_gptq_factors(a, b, method, iters)          -> A, B (Kronecker factors from samples)
    kron_gptq_quantize_antidiagonal(W, U_A, U_B, ...) -> codes, V, E (quartic baseline, fp64)
    kron_gptq_sync_status(ws, stream)      -> device status word
    kron_gptq_schedule_plan(ndiag)         -> the solve's update pieces (host only)
"""
from __future__ import annotations

import os as _os

# Every recursive solve runs on four internal streams; with the default eight hardware connections
# the streams of concurrent solves share queues and serialise.  Takes effect only if set before the
# process creates its CUDA context (importing this package first does that); a value already in the
# environment wins.
_os.environ.setdefault("CUDA_DEVICE_MAX_CONNECTIONS", "32")

from ._lib import (  # noqa: E402,F401
    KG_F32,
    KG_F64,
    KGError,
    Quantizer,
    RcQuantizer,
    OnesidedQuantizer,
    PROFILE_KINDS,
    SCHEDULE_STREAMS,
    kron_gptq_loss,
    kron_gptq_profile_enable,
    kron_gptq_profile_read,
    kron_gptq_prepare,
    kron_gptq_quantize,
    kron_gptq_quantize_noalloc,
    kron_gptq_quantize_rc,
    kron_gptq_quantize_onesided,
    kron_gptq_factors,
    kron_gptq_quantize_antidiagonal,
    kron_gptq_code_entropy,
    kron_gptq_waterkron_scales,
    kron_gptq_row_scales,
    kron_gptq_schedule_plan,
    kron_gptq_status_string,
    kron_gptq_sync_status,
    kron_gptq_version,
    lib_path,
    load_library,
    quantize_workspace_bytes,
)
