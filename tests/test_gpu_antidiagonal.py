"""The non-recursive anti-diagonal baseline (kron_gptq_quantize_antidiagonal, "FastKron" Section 2.3)
against the oracle and against the recursive solve.  Needs a B200.

The FastKron variants compute the same codes ("FastKron", Section 2.5), so the bar is the fp64 one
of the main solver: codes equal to the naive oracle's except entries within 1e-9 grid steps of a
tie (oracle.compare_with_oracle), and equal to kron_gptq_quantize's on a full 1024 x 1024 layer.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import layer_inputs, small_layer, workload

pytestmark = pytest.mark.gpu

DAMP = 0.01


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


@pytest.mark.parametrize("m,n,bits,seed", [(6, 5, 4, 0), (128, 128, 4, 1), (127, 129, 3, 2), (200, 70, 4, 3),
                                           (65, 200, 3, 4)])
def test_fp64_full_oracle(kg, m, n, bits, seed):
    spec, (W, A, B) = small_layer(m, n, seed, bits=bits)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    UA, UB = oracle.prepare_lapack(A, DAMP), oracle.prepare_lapack(B, DAMP)
    s = oracle.row_scales(W, spec.qmax)
    codes, V, E = kg.kron_gptq_quantize_antidiagonal(torch.from_numpy(W).cuda(), torch.from_numpy(UA).cuda(),
                                                     torch.from_numpy(UB).cuda(), spec.qmin, spec.qmax,
                                                     torch.from_numpy(s).cuda(), want_E=True)
    res = oracle.compare_with_oracle(codes.cpu().numpy(), W, UA, UB, s, spec.qmin, spec.qmax, tol=1e-9)
    assert res["ok"], {k: res[k] for k in res if k != "oracle"}
    lo = np.sum(res["oracle"]["E"] ** 2)
    assert abs(float((E.double() ** 2).sum()) - lo) <= 1e-9 * lo


def test_equals_the_recursive_solve(kg):
    spec = workload("sq1024")[0]
    W, A, B = layer_inputs(spec, device="cuda")
    UA, UB, _, _ = kg.kron_gptq_prepare(A, B, DAMP)
    s = kg.kron_gptq_row_scales(W, spec.qmax)
    c1, V1, E1 = kg.kron_gptq_quantize(W, UA, UB, spec.qmin, spec.qmax, s, want_E=True)
    c2, V2, E2 = kg.kron_gptq_quantize_antidiagonal(W, UA, UB, spec.qmin, spec.qmax, s, want_E=True)
    mism = float((c1 != c2).double().mean())
    assert mism <= 1e-5, mism
    if mism == 0:
        torch.testing.assert_close(E2, E1, rtol=1e-8, atol=1e-10 * float(E1.abs().max()))
