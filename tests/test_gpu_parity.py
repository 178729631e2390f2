"""Parity of the CUDA path (through the C ABI) with the CPU oracle.  Needs a B200.

Bars (stated for the two-sided GPTQ solver):
  * fp64 path: codes identical to the oracle's except at entries whose pre-rounding value
    lies within 1e-9 grid steps of a half-integer (absorbed and counted by
    oracle.compare_with_oracle); proxy loss within 1e-9 relative.
  * fp32 path (3xTF32-class accuracy): on layers the oracle finishes (and on the leading
    blocks of the large ones) >= 99.5 % of codes equal to the fp64 oracle's; at full size the
    certificate, >= 99.5 % equal codes on the leading 1024 x 1024 block and the proxy loss within
    FP32_LOSS_BAR of the fp64 path's -- a bar set from a perturbation control (see the comment
    above test_full_size_fp32_vs_fp64_and_certificate).
Both sides always quantize identical inputs: the factors come from the oracle side (LAPACK
prepare) and are rounded to the solve dtype before either side sees them.
Full-size cases are checked on the leading 256 x 256 block (which depends only on leading
data, "FastKron" Section 2.3) and by the certificate on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import LayerSpec, layer_inputs, small_layer, workload

pytestmark = pytest.mark.gpu

DAMP = 0.01


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


def _inputs(spec: LayerSpec, device="cpu"):
    W, A, B = layer_inputs(spec, device=device)
    return W.cpu().numpy(), A.cpu().numpy(), B.cpu().numpy()


def _case(W, A, B, qmax, dtype):
    """Oracle-side factors and scales, rounded to the solve dtype; float64 views for the oracle."""
    UA = oracle.prepare_lapack(A, DAMP)
    UB = oracle.prepare_lapack(B, DAMP)
    npd = np.float64 if dtype == torch.float64 else np.float32
    Wr, UAr, UBr = W.astype(npd), UA.astype(npd), UB.astype(npd)
    s = oracle.row_scales(Wr.astype(np.float64), qmax).astype(npd)
    return dict(W=Wr.astype(np.float64), UA=UAr.astype(np.float64), UB=UBr.astype(np.float64),
                s=s.astype(np.float64), Wt=torch.from_numpy(Wr).cuda(), UAt=torch.from_numpy(UAr).cuda(),
                UBt=torch.from_numpy(UBr).cuda(), st=torch.from_numpy(s).cuda(),
                Ad=oracle.damped(A, DAMP), Bd=oracle.damped(B, DAMP))


def _run(kg, c, qmin, qmax, want_E=True):
    codes, V, E = kg.kron_gptq_quantize(c["Wt"], c["UAt"], c["UBt"], qmin, qmax, c["st"], want_E=want_E)
    torch.cuda.synchronize()
    return codes.cpu().numpy().astype(np.int32), V.cpu().double().numpy(), (E.cpu().double().numpy() if E is not None else None)


def _assert_fp64_parity(codes, W, UA, UB, s, qmin, qmax):
    res = oracle.compare_with_oracle(codes, W, UA, UB, s, qmin, qmax, tol=1e-9)
    assert res["ok"], {k: res[k] for k in res if k != "oracle"}
    return res


# ------------------------------------------------------------------------------ prepare
@pytest.mark.parametrize("k,seed", [(1, 1), (64, 2), (100, 3), (128, 4), (1024, 5)])
def test_prepare_matches_lapack(kg, k, seed):
    _, (W, A, B) = small_layer(8, k, seed)
    A = A.numpy()
    UA, _, UA32, _ = kg.kron_gptq_prepare(torch.from_numpy(A).cuda(), None, DAMP)
    ref = oracle.prepare_lapack(A, DAMP)
    got = UA.cpu().numpy()
    assert np.all(np.tril(got, -1) == 0)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-9, err
    np.testing.assert_array_equal(UA32.cpu().numpy(), got.astype(np.float32))


def test_prepare_fp32_input_and_both_sides(kg):
    spec = workload("ref128")[0]
    W, A, B = _inputs(spec)
    UA, UB, _, _ = kg.kron_gptq_prepare(torch.from_numpy(A).float().cuda(), torch.from_numpy(B).float().cuda(), DAMP)
    refA = oracle.prepare_lapack(A.astype(np.float32).astype(np.float64), DAMP)
    refB = oracle.prepare_lapack(B.astype(np.float32).astype(np.float64), DAMP)
    assert np.abs(UA.cpu().numpy() - refA).max() / np.abs(refA).max() < 1e-9
    assert np.abs(UB.cpu().numpy() - refB).max() / np.abs(refB).max() < 1e-9


def test_prepare_full_size_residual(kg):
    spec = workload("sq4096")[0]
    W, A, B = layer_inputs(spec, device="cuda")
    UA, UB, _, _ = kg.kron_gptq_prepare(A, B, DAMP)
    for U, M in ((UA, A), (UB, B)):
        Md = M + DAMP * M.diagonal().mean() * torch.eye(M.shape[0], dtype=M.dtype, device=M.device)
        cols = torch.arange(0, M.shape[0], 257, device=M.device)
        # U^T U A_d = I  checked on sampled columns (independent torch fp64 products)
        R = U.T @ (U @ Md[:, cols])
        Iref = torch.eye(M.shape[0], dtype=M.dtype, device=M.device)[:, cols]
        assert (R - Iref).abs().max().item() < 1e-6


def test_prepare_not_pd(kg):
    A = torch.diag(torch.tensor([1.0, 2.0, -0.5, 3.0], dtype=torch.float64)).cuda()
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_prepare(A, None, 0.0)
    assert ei.value.name == "KG_ERR_NOT_PD"


# ------------------------------------------------------------------------------ small, full oracle
def test_ref128_fp64_full_oracle(kg):
    spec = workload("ref128")[0]
    W, A, B = _inputs(spec)
    c = _case(W, A, B, spec.qmax, torch.float64)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    res = _assert_fp64_parity(codes, c["W"], c["UA"], c["UB"], c["s"], spec.qmin, spec.qmax)
    o = res["oracle"]
    lo = np.sum(o["E"] ** 2)
    assert abs(np.sum(E ** 2) - lo) <= 1e-9 * lo
    if not res["flips"]:
        np.testing.assert_array_equal(V, o["V"])
        np.testing.assert_allclose(E, o["E"], rtol=1e-9, atol=1e-12 * np.abs(o["E"]).max())
    lk = kg.kron_gptq_loss(c["Wt"], torch.from_numpy(V).cuda(), torch.from_numpy(A).cuda(),
                           torch.from_numpy(B).cuda(), DAMP)
    assert abs(lk - oracle.loss(c["W"], V, c["Ad"], c["Bd"])) <= 1e-9 * abs(lk)
    assert abs(lk - lo) <= 1e-8 * lo


def test_ref128_fp32(kg):
    spec = workload("ref128")[0]
    W, A, B = _inputs(spec)
    c = _case(W, A, B, spec.qmax, torch.float32)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    o = oracle.quantize_naive(c["W"], c["UA"], c["UB"], c["s"], spec.qmin, spec.qmax)
    agree = np.mean(codes == o["codes"])
    assert agree >= 0.995, agree
    lo = oracle.loss(c["W"], o["V"], c["Ad"], c["Bd"])
    lg = oracle.loss(c["W"], V, c["Ad"], c["Bd"])
    assert abs(lg - lo) <= 1e-3 * lo


@pytest.mark.parametrize("m,n,bits,seed", [(1, 1, 4, 0), (1, 64, 3, 1), (64, 1, 3, 2), (6, 5, 4, 3),
                                           (127, 129, 3, 4), (33, 65, 2, 5), (200, 70, 4, 6), (65, 200, 3, 7)])
def test_ragged_fp64_full_oracle(kg, m, n, bits, seed):
    spec, (W, A, B) = small_layer(m, n, seed, bits=bits)
    c = _case(W.numpy(), A.numpy(), B.numpy(), spec.qmax, torch.float64)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    res = _assert_fp64_parity(codes, c["W"], c["UA"], c["UB"], c["s"], spec.qmin, spec.qmax)
    lo = np.sum(res["oracle"]["E"] ** 2)
    # when every code reproduces W exactly (e.g. one column) E is pure rounding noise
    assert abs(np.sum(E ** 2) - lo) <= 1e-9 * lo + 1e-20


@pytest.mark.parametrize("m,n", [(127, 129), (200, 70)])
def test_ragged_fp32(kg, m, n):
    spec, (W, A, B) = small_layer(m, n, 11, bits=3)
    c = _case(W.numpy(), A.numpy(), B.numpy(), spec.qmax, torch.float32)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    o = oracle.quantize_naive(c["W"], c["UA"], c["UB"], c["s"], spec.qmin, spec.qmax)
    assert np.mean(codes == o["codes"]) >= 0.995


# ------------------------------------------------------------------------------ larger layers
def _leading_block_and_certificate(kg, spec, dtype, block=256, n_rows=24, device="cuda"):
    W, A, B = _inputs(spec, device=device)
    c = _case(W, A, B, spec.qmax, dtype)
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    mb, nb = min(block, spec.m), min(block, spec.n)
    args = (c["W"][:mb, :nb], c["UA"][:nb, :nb], c["UB"][:mb, :mb], c["s"][:mb], spec.qmin, spec.qmax)
    if dtype == torch.float64:
        _assert_fp64_parity(codes[:mb, :nb], *args)
        tol, rtol_res = 1e-9, 1e-10
    else:
        o = oracle.quantize_naive(*args)
        assert np.mean(codes[:mb, :nb] == o["codes"]) >= 0.995
        tol, rtol_res = 1e-4, 1e-4
    rows = np.unique(np.linspace(0, spec.m - 1, n_rows).astype(int))
    cert = oracle.certificate(c["W"], c["UA"], c["UB"], c["s"], spec.qmin, spec.qmax, codes, V, E, rows=rows, tol=tol)
    assert cert["resid_rel"] < rtol_res, cert
    assert cert["code_mismatch"] <= (0 if dtype == torch.float64 else 0.001 * len(rows) * spec.n), cert
    return c, codes, V, E


def test_sq1024_fp32_two_sided(kg):
    _leading_block_and_certificate(kg, workload("sq1024")[0], torch.float32)


def test_sq1024_fp64_two_sided(kg):
    _leading_block_and_certificate(kg, workload("sq1024")[0], torch.float64)


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_sq1024_identity_B_equals_onesided(kg, dtype):
    spec = workload("sq1024_onesided")[0]
    W, A, B = _inputs(spec)
    c = _case(W, A, B, spec.qmax, dtype)
    # B = I is damped to (1 + damp) I: U_B is diagonal, so there is no coupling across rows
    assert np.array_equal(c["UB"], np.diag(np.diag(c["UB"])))
    codes, V, E = _run(kg, c, spec.qmin, spec.qmax)
    one = oracle.quantize_onesided(c["W"], c["UA"], np.repeat(c["s"][:, None], spec.n, 1), spec.qmin, spec.qmax)
    agree = np.mean(codes == one["codes"])
    if dtype == torch.float64:
        assert agree == 1.0, agree
    else:
        assert agree >= 0.995, agree


@pytest.mark.parametrize("name", ["sq4096_2bit", "sq4096_4bit"])
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_sq4096(kg, name, dtype):
    _leading_block_and_certificate(kg, workload(name)[0], dtype)


# The fp32 bar at full size, set from a perturbation control (the reading is stated with its
# numbers in the design notes).  Two-sided GPTQ is a sequence of m*n rounding decisions in which
# one flipped decision changes every later entry to its bottom-right ("FastKron" Section 2.3), so
# the codes of two exact solves drift apart as soon as the inputs differ at all.  The control ran
# the fp64 path on W perturbed by delta * s_i * N(0,1) with delta = 1e-8, 1e-7 and 1e-6 grid steps
# (3 seeds each, sq4096, ffn_up and ffn_down): at delta = 1e-7 -- some 30x below the fp32 path's own
# median noise on the value it rounds, 3e-6 grid steps -- only 71-81 % of all codes stayed equal,
# every leading 1024 x 1024 block kept >= 99.6 %, and the proxy loss moved by up to 2.3e-3 relative
# (RMS 1.1e-3 over the 18 runs at delta = 1e-7 and 1e-6).  So no floating-point solve that is not
# bit-identical to the oracle can promise 99.5 % equal codes over the whole matrix, and a loss bar of
# 1e-3 lies inside the problem's own spread.  The fp32 bar is therefore: the certificate of the
# fp32 solution; >= 99.5 % equal codes on the leading 1024 x 1024 block (the control's minimum);
# and a proxy loss within FP32_LOSS_BAR = 4.5 control RMS of the fp64 loss.  The test re-runs two
# control perturbations (delta = 1e-7) and reports them beside the fp32 figures.
FP32_LOSS_BAR = 5e-3
CONTROL_DELTA = 1e-7


@pytest.mark.parametrize("name", ["sq4096", "ffn_up", "ffn_down"])
def test_full_size_fp32_vs_fp64_and_certificate(kg, name):
    """Full-size layers: no quartic oracle at this size.  Both paths quantize identical
    (fp32-rounded) inputs.  Checked: the certificate of each path on sampled rows; the leading
    1024 x 1024 block of codes agrees on >= 99.5 %; the proxy loss of the fp32 solution (fp64 loss
    kernel) is within FP32_LOSS_BAR of the fp64 one.  Full-matrix agreement and the loss deviation
    are reported next to the same figures for two fp64 solves of W perturbed by 1e-7 grid steps."""
    spec = workload(name)[0]
    W, A, B = layer_inputs(spec, device="cuda")
    UA, UB, UA32, UB32 = kg.kron_gptq_prepare(A, B, DAMP)
    W32 = W.float().contiguous()
    s32 = kg.kron_gptq_row_scales(W32, spec.qmax)
    c32, V32, E32 = kg.kron_gptq_quantize(W32, UA32, UB32, spec.qmin, spec.qmax, s32, want_E=True)
    W64, UA64, UB64, s64 = W32.double(), UA32.double(), UB32.double(), s32.double()
    c64, V64, E64 = kg.kron_gptq_quantize(W64, UA64, UB64, spec.qmin, spec.qmax, s64, want_E=True)
    k = 1024
    agree_lead = (c32[:k, :k] == c64[:k, :k]).float().mean().item()
    agree_full = (c32 == c64).float().mean().item()
    l64 = kg.kron_gptq_loss(W64, V64, A, B, DAMP)
    l32 = kg.kron_gptq_loss(W64, V32.double(), A, B, DAMP)
    rel32 = (l32 - l64) / l64
    control = []
    for seed in (100, 101):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        Wp = W64 + CONTROL_DELTA * s64[:, None] * torch.randn(W64.shape, generator=g, device="cuda",
                                                             dtype=torch.float64)
        cp, Vp, _ = kg.kron_gptq_quantize(Wp, UA64, UB64, spec.qmin, spec.qmax, s64)
        lp = kg.kron_gptq_loss(W64, Vp, A, B, DAMP)
        control.append({"agree_full": round((cp == c64).float().mean().item(), 4),
                        "agree_lead": round((cp[:k, :k] == c64[:k, :k]).float().mean().item(), 4),
                        "loss_rel": float(f"{(lp - l64) / l64:.3e}")})
        del Wp, cp, Vp
    report = {"layer": name, "fp32_agree_full": round(agree_full, 4), "fp32_agree_lead1024": round(agree_lead, 4),
              "fp32_loss_rel": float(f"{rel32:.3e}"), "fp64_loss": l64,
              f"fp64_control_delta{CONTROL_DELTA:g}": control}
    print(report)
    assert agree_lead >= 0.995, report
    assert abs(rel32) <= FP32_LOSS_BAR, report
    rows = np.unique(np.linspace(0, spec.m - 1, 6).astype(int))
    args = (W64.cpu().numpy(), UA64.cpu().numpy(), UB64.cpu().numpy(), s64.cpu().numpy(), spec.qmin, spec.qmax)
    cert = oracle.certificate(*args, c64.cpu().numpy(), V64.cpu().numpy(), E64.cpu().numpy(), rows=rows)
    assert cert["resid_rel"] < 1e-10 and cert["code_mismatch"] == 0, cert
    cert32 = oracle.certificate(*args, c32.cpu().numpy(), V32.double().cpu().numpy(), E32.double().cpu().numpy(),
                                rows=rows, tol=1e-4)
    assert cert32["resid_rel"] < 1e-4 and cert32["code_mismatch"] <= 1e-3 * len(rows) * spec.n, cert32


def test_fp64_perturbation_control(kg):
    """The control behind the fp32 bar, on the 4096 x 4096 layer: exact (fp64) solves of W and of W
    perturbed by 1e-7 grid steps keep the leading 256 x 256 block of codes unchanged (it sees few
    decisions before it) but differ on more than 5 % of all codes, because each flipped decision
    changes the entries to its bottom-right ("FastKron" Section 2.3)."""
    spec = workload("sq4096")[0]
    W, A, B = layer_inputs(spec, device="cuda")
    UA, UB, _, _ = kg.kron_gptq_prepare(A, B, DAMP)
    s = kg.kron_gptq_row_scales(W, spec.qmax)
    c0, _, _ = kg.kron_gptq_quantize(W, UA, UB, spec.qmin, spec.qmax, s)
    g = torch.Generator(device="cuda")
    g.manual_seed(102)
    Wp = W + CONTROL_DELTA * s[:, None] * torch.randn(W.shape, generator=g, device="cuda", dtype=torch.float64)
    cp, _, _ = kg.kron_gptq_quantize(Wp, UA, UB, spec.qmin, spec.qmax, s)
    lead = (cp[:256, :256] == c0[:256, :256]).float().mean().item()
    full = (cp == c0).float().mean().item()
    print({"control_lead256": lead, "control_full": full})
    assert lead == 1.0, lead
    assert full < 0.95, full


# ------------------------------------------------------------------------------ edge cases, errors
def test_empty_is_noop(kg):
    W = torch.zeros(0, 8, dtype=torch.float64, device="cuda")
    codes, V, E = kg.kron_gptq_quantize(W, torch.eye(8, dtype=torch.float64, device="cuda"),
                                        torch.zeros(0, 0, dtype=torch.float64, device="cuda"), -4, 3,
                                        torch.zeros(0, dtype=torch.float64, device="cuda"))
    assert codes.numel() == 0


def test_nonfinite_input_is_reported(kg):
    spec, (W, A, B) = small_layer(70, 70, 3)
    c = _case(W.numpy(), A.numpy(), B.numpy(), spec.qmax, torch.float64)
    Wt = c["Wt"].clone()
    Wt[5, 9] = float("nan")
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize(Wt, c["UAt"], c["UBt"], spec.qmin, spec.qmax, c["st"])
    assert ei.value.name == "KG_ERR_NONFINITE"
    # the context stays usable
    codes, V, E = kg.kron_gptq_quantize(c["Wt"], c["UAt"], c["UBt"], spec.qmin, spec.qmax, c["st"])
    assert codes.shape == (70, 70)


def test_bad_scale_is_reported(kg):
    spec, (W, A, B) = small_layer(64, 64, 4)
    c = _case(W.numpy(), A.numpy(), B.numpy(), spec.qmax, torch.float32)
    s = c["st"].clone()
    s[3] = 0.0
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize(c["Wt"], c["UAt"], c["UBt"], spec.qmin, spec.qmax, s)
    assert ei.value.name == "KG_ERR_NONFINITE"


def test_deterministic_repeat(kg):
    spec = workload("sq1024")[0]
    W, A, B = _inputs(spec)
    c = _case(W, A, B, spec.qmax, torch.float32)
    first = _run(kg, c, spec.qmin, spec.qmax)
    for _ in range(3):
        again = _run(kg, c, spec.qmin, spec.qmax)
        np.testing.assert_array_equal(first[0], again[0])
        np.testing.assert_array_equal(first[1], again[1])


def test_row_scales_match_oracle(kg):
    spec, (W, A, B) = small_layer(77, 300, 9)
    for dt in (torch.float64, torch.float32):
        Wt = W.to(dt).cuda()
        Wt[3] = 0.0
        s = kg.kron_gptq_row_scales(Wt, 7).cpu().double().numpy()
        ref = oracle.row_scales(Wt.cpu().double().numpy(), 7)
        np.testing.assert_allclose(s, ref, rtol=1e-6 if dt == torch.float32 else 0)


def test_loss_kernel_matches_oracle(kg):
    spec, (W, A, B) = small_layer(90, 130, 10)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    rng = np.random.default_rng(0)
    V = W + 0.05 * rng.standard_normal(W.shape)
    ref = oracle.loss(W, V, oracle.damped(A, DAMP), oracle.damped(B, DAMP))
    got = kg.kron_gptq_loss(torch.from_numpy(W).cuda(), torch.from_numpy(V).cuda(), torch.from_numpy(A).cuda(),
                            torch.from_numpy(B).cuda(), DAMP)
    assert abs(got - ref) <= 1e-10 * abs(ref)
