"""Parity of the one-sided fast path (kron_gptq_quantize_onesided: GPTQ with recursively batched
updates, "FastKron" Sections 2.2 and 2.4) with the CPU oracle.  Needs a B200.

One-sided GPTQ is the two-sided algorithm with B = I (pinned in the oracle's tests), so the exact
fp64 bar uses the naive oracle with U_B = I and its tie rule (oracle.compare_with_oracle).  Bars:
  * fp64: codes equal except entries within 1e-9 grid steps of a tie; E within 1e-9 relative;
    equal to the GPU's two-sided solve with U_B = I.
  * fp32 (leaf in fp32, batched updates as fp32-accurate tensor-core GEMMs): >= 99.5 % of codes
    equal to the fp64 oracle on the leading 256 x 256 block; the certificate with B = I on sampled
    rows to (m + n) 2^-24.
Rows never interact and columns run in order, so a leading block depends only on leading data.
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


def _case(W, A, qmax, dtype):
    UA = oracle.prepare_lapack(A, DAMP)
    npd = np.float64 if dtype == torch.float64 else np.float32
    Wr, UAr = W.astype(npd), UA.astype(npd)
    s = oracle.row_scales(Wr.astype(np.float64), qmax).astype(npd)
    return dict(W=Wr.astype(np.float64), UA=UAr.astype(np.float64), s=s.astype(np.float64),
                Wt=torch.from_numpy(Wr).cuda(), UAt=torch.from_numpy(UAr).cuda(), st=torch.from_numpy(s).cuda())


def _run(kg, c, qmin, qmax):
    codes, V, E = kg.kron_gptq_quantize_onesided(c["Wt"], c["UAt"], qmin, qmax, c["st"], want_E=True)
    torch.cuda.synchronize()
    return codes.cpu().numpy().astype(np.int32), V.cpu().double().numpy(), E.cpu().double().numpy()


@pytest.mark.parametrize("m,n,bits,seed", [(1, 1, 4, 0), (6, 5, 4, 1), (128, 128, 4, 2), (127, 129, 3, 3),
                                           (200, 70, 4, 4), (65, 200, 3, 5), (33, 300, 2, 6)])
def test_fp64_full_oracle(kg, m, n, bits, seed):
    spec, (W, A, B) = small_layer(m, n, seed, bits=bits)
    c = _case(W.numpy(), A.numpy(), spec.qmax, torch.float64)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    res = oracle.compare_with_oracle(codes, c["W"], c["UA"], np.eye(m), c["s"], spec.qmin, spec.qmax, tol=1e-9)
    assert res["ok"], {k: res[k] for k in res if k != "oracle"}
    o = res["oracle"]
    if not res["flips"]:
        np.testing.assert_array_equal(V, o["V"])
        np.testing.assert_allclose(E, o["E"], rtol=1e-9, atol=1e-12 * max(np.abs(o["E"]).max(), 1e-300))
    one = oracle.quantize_onesided(c["W"], c["UA"], np.repeat(c["s"][:, None], n, 1), spec.qmin, spec.qmax)
    if not res["flips"]:
        np.testing.assert_array_equal(codes, one["codes"])


def test_fp64_equals_two_sided_with_identity_B(kg):
    spec = workload("sq1024")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, spec.qmax, torch.float64)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    eye = torch.eye(spec.m, dtype=torch.float64, device="cuda")
    c2, V2, E2 = kg.kron_gptq_quantize(c["Wt"], c["UAt"], eye, spec.qmin, spec.qmax, c["st"], want_E=True)
    mism = np.mean(codes != c2.cpu().numpy())
    assert mism <= 1e-5, mism
    if mism == 0:
        np.testing.assert_allclose(E, E2.cpu().numpy(), rtol=1e-9, atol=1e-12 * np.abs(E).max())


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_sq1024_leading_block_and_certificate(kg, dtype):
    spec = workload("sq1024")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, spec.qmax, dtype)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    mb = 256
    o = oracle.quantize_onesided(c["W"][:mb, :mb], c["UA"][:mb, :mb], np.repeat(c["s"][:mb, None], mb, 1),
                                 spec.qmin, spec.qmax)
    agree = np.mean(codes[:mb, :mb] == o["codes"])
    assert agree >= (0.995 if dtype == torch.float32 else 0.9999), agree
    rows = np.unique(np.linspace(0, spec.m - 1, 16).astype(int))
    cert = oracle.certificate(c["W"], c["UA"], np.eye(spec.m), c["s"], spec.qmin, spec.qmax, codes, V, E,
                              rows=rows, tol=1e-4 if dtype == torch.float32 else 1e-9)
    bound = (spec.m + spec.n) * 2.0 ** -24 if dtype == torch.float32 else 1e-12
    assert cert["resid_rel"] < bound, cert
    assert cert["code_mismatch"] <= 1e-3 * len(rows) * spec.n, cert


def test_fp32_deterministic_repeat(kg):
    spec = workload("sq1024")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, spec.qmax, torch.float32)
    first = _run(kg, c, spec.qmin, spec.qmax)
    again = _run(kg, c, spec.qmin, spec.qmax)
    np.testing.assert_array_equal(first[0], again[0])
    np.testing.assert_array_equal(first[1], again[1])


def test_errors_and_empty(kg):
    spec, (W, A, B) = small_layer(70, 90, 8)
    c = _case(W.numpy(), A.numpy(), spec.qmax, torch.float64)
    Wt = c["Wt"].clone()
    Wt[3, 4] = float("inf")
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize_onesided(Wt, c["UAt"], spec.qmin, spec.qmax, c["st"])
    assert ei.value.name == "KG_ERR_NONFINITE"
    s = c["st"].clone()
    s[5] = -1.0
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize_onesided(c["Wt"], c["UAt"], spec.qmin, spec.qmax, s)
    assert ei.value.name == "KG_ERR_NONFINITE"
    codes, V, E = kg.kron_gptq_quantize_onesided(c["Wt"], c["UAt"], spec.qmin, spec.qmax, c["st"])
    assert codes.shape == (70, 90)
    W0 = torch.zeros(0, 16, dtype=torch.float64, device="cuda")
    codes, V, E = kg.kron_gptq_quantize_onesided(W0, torch.eye(16, dtype=torch.float64, device="cuda"), -4, 3,
                                                 torch.zeros(0, dtype=torch.float64, device="cuda"))
    assert codes.numel() == 0
