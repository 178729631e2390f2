"""The allocation-free entry point kron_gptq_quantize_noalloc (needs a B200).

It exists for callers that cannot allocate device memory -- code inside a host framework whose
allocator owns the device memory, or a service path that must not call cudaMalloc after
start-up.  It runs the same kernels as kron_gptq_quantize but keeps its scratch in a fixed
device array inside the library, so its output must match the workspace entry point's
exactly (same kernels, same launch shapes, same inputs), on two calls in a row (the second
call finds the first call's leftovers in the shared array and must not be affected by them),
the second one on a stream of its own, and the device's free memory must not change across
them.

This file is collected last on purpose, so a failure here cannot hide other failures in a
run that stops at the first one.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import small_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


@pytest.mark.parametrize("dtype,m,n", [(torch.float64, 300, 200), (torch.float32, 320, 256),
                                       (torch.float32, 768, 768), (torch.float64, 1024, 1024)])
def test_noalloc_matches_workspace_entry_point(kg, dtype, m, n):
    spec, (W, A, B) = small_layer(m, n, 17, bits=3)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    UA = oracle.prepare_lapack(A, 0.01)
    UB = oracle.prepare_lapack(B, 0.01)
    npd = np.float64 if dtype == torch.float64 else np.float32
    Wt = torch.from_numpy(W.astype(npd)).cuda()
    UAt = torch.from_numpy(UA.astype(npd)).cuda()
    UBt = torch.from_numpy(UB.astype(npd)).cuda()
    st = kg.kron_gptq_row_scales(Wt, spec.qmax)
    ref_codes, ref_V, ref_E = kg.kron_gptq_quantize(Wt, UAt, UBt, spec.qmin, spec.qmax, st, want_E=True)
    outs = [(torch.empty((m, n), dtype=torch.int8, device="cuda"), torch.empty((m, n), dtype=dtype, device="cuda"),
             torch.empty((m, n), dtype=dtype, device="cuda"), torch.empty((1,), dtype=torch.int32, device="cuda"))
            for _ in range(2)]
    side = torch.cuda.Stream()
    # a warm-up call loads the kernels and creates the library's per-thread streams and events
    kg.kron_gptq_quantize_noalloc(Wt, UAt, UBt, spec.qmin, spec.qmax, st, *outs[0])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for k, (codes, V, E, status) in enumerate(outs):
        codes.fill_(99)
        V.fill_(float("nan"))
        E.fill_(float("nan"))
        status.fill_(-99)
        # the second call runs on a stream of its own, after the first
        stream = side if k == 1 else None
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream())
        kg.kron_gptq_quantize_noalloc(Wt, UAt, UBt, spec.qmin, spec.qmax, st, codes, V, E, status, stream=stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(codes, ref_codes)
        assert torch.equal(V, ref_V)
        assert torch.equal(E, ref_E)
    # nothing was allocated on the device by the two calls
    assert torch.cuda.mem_get_info()[0] == free_before


def test_noalloc_rejects_oversize_before_launch(kg):
    L = kg.load_library()
    from two_sided_gptq_02_b200._lib import _Grid
    t = torch.zeros(16, dtype=torch.float64, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    # 4096 x 4096 fp64 needs about 400 MB of scratch: rejected with KG_ERR_WORKSPACE
    rc = L.kron_gptq_quantize_noalloc(p, 4096, 4096, 2, p, p, _Grid(-4, 3, t.data_ptr()), p, p, None, None, None)
    assert rc == -4
