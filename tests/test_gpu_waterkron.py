"""Parity of the row- and column-scaled alphabet (kron_gptq_quantize_rc), the WaterKron steps
and the code entropy with the CPU oracle.  Needs a B200.

The alphabet is V = beta alpha^T (.) Z with Z integer and not clipped ("WaterKron and FlipFlop
Hessian", Section 2.1); WaterKron takes alpha ~ diag U_A and beta ~ diag U_B (Section 3).
Bars, as for the row-scaled solver:
  * fp64: codes identical to oracle.quantize_rc except at entries within 1e-9 steps of a
    half-integer (absorbed and counted by oracle.compare_with_oracle_rc); V equal where the
    codes are; E within 1e-9 relative; the steps equal the oracle's bit for bit.
  * fp32 (3xTF32-class updates): the certificate holds with the recursive-summation bound
    (m + n) 2^-24 and every |E| <= gamma/2; distortion sum E^2 within 1 % and rate (entropy of Z)
    within 0.02 bits of the fp64 oracle's; >= 95 % of codes equal.  The unclipped steps are fine
    (codes up to ~900): a pre-rounding value within fp32 noise of a half-integer flips, and a flip
    moves every later entry to its bottom-right ("FastKron", Section 2.3), so agreement with the
    fp64 oracle is a statistical property here (fp64 oracle runs with 2e-5 relative noise on W
    agree on 99.0-99.9 % of codes), unlike the 3-bit grid of the row-scaled tests.
  * entropy: the kernel's plug-in estimate equals numpy's on the same codes to 1e-12 bits.
Inputs come from the same seeded generator as every other test; the factors from the oracle
side (LAPACK prepare), rounded to the solve dtype before either side sees them.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import layer_inputs, small_layer, workload

pytestmark = pytest.mark.gpu

DAMP = 0.01
GAMMA = 0.02          # about 4.7 bits per entry on the 128 x 128 layer, codes up to ~900


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


def _case(W, A, B, dtype, steps="waterkron", gamma=GAMMA, seed=0):
    UA = oracle.prepare_lapack(A, DAMP)
    UB = oracle.prepare_lapack(B, DAMP)
    npd = np.float64 if dtype == torch.float64 else np.float32
    Wr, UAr, UBr = W.astype(npd), UA.astype(npd), UB.astype(npd)
    m, n = W.shape
    if steps == "waterkron":
        al, be = oracle.waterkron_scales(UAr.astype(np.float64), UBr.astype(np.float64), gamma)
    else:
        rng = np.random.default_rng(seed)
        al = 0.02 * np.exp(0.5 * rng.standard_normal(n))
        be = np.exp(0.5 * rng.standard_normal(m))
    al, be = al.astype(npd), be.astype(npd)
    return dict(W=Wr.astype(np.float64), UA=UAr.astype(np.float64), UB=UBr.astype(np.float64),
                al=al.astype(np.float64), be=be.astype(np.float64),
                Wt=torch.from_numpy(Wr).cuda(), UAt=torch.from_numpy(UAr).cuda(), UBt=torch.from_numpy(UBr).cuda(),
                alt=torch.from_numpy(al).cuda(), bet=torch.from_numpy(be).cuda(),
                Ad=oracle.damped(A, DAMP), Bd=oracle.damped(B, DAMP))


def _run(kg, c, want_E=True):
    Z, V, E = kg.kron_gptq_quantize_rc(c["Wt"], c["UAt"], c["UBt"], c["alt"], c["bet"], want_E=want_E)
    torch.cuda.synchronize()
    return Z.cpu().numpy().astype(np.int64), V.cpu().double().numpy(), \
        (E.cpu().double().numpy() if E is not None else None)


def _assert_fp64_parity(Z, c):
    res = oracle.compare_with_oracle_rc(Z, c["W"], c["UA"], c["UB"], c["al"], c["be"], tol=1e-9)
    assert res["ok"], {k: res[k] for k in res if k != "oracle"}
    return res


# ------------------------------------------------------------------------------ fp64, full oracle
def test_waterkron_scales_match_oracle(kg):
    spec = workload("ref128")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, B, torch.float64)
    al, be = kg.kron_gptq_waterkron_scales(c["UAt"], c["UBt"], GAMMA)
    np.testing.assert_array_equal(al.cpu().numpy(), c["al"])
    np.testing.assert_array_equal(be.cpu().numpy(), c["be"])
    c32 = _case(W, A, B, torch.float32)
    al32, be32 = kg.kron_gptq_waterkron_scales(c32["UAt"], c32["UBt"], GAMMA)
    np.testing.assert_array_equal(al32.cpu().numpy(), c32["al"].astype(np.float32))
    with pytest.raises(kg.KGError):
        kg.kron_gptq_waterkron_scales(c["UAt"], c["UBt"], -1.0)


def test_ref128_fp64_waterkron_full_oracle(kg):
    spec = workload("ref128")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, B, torch.float64)
    Z, V, E = _run(kg, c)
    res = _assert_fp64_parity(Z, c)
    o = res["oracle"]
    assert np.abs(Z).max() > 127            # beyond any clipped int8 grid
    if not res["flips"]:
        np.testing.assert_array_equal(V, o["V"])
        np.testing.assert_allclose(E, o["E"], rtol=1e-9, atol=1e-11 * GAMMA)
    assert np.abs(E).max() <= 0.5 * GAMMA * (1 + 1e-9)
    lo = np.sum(o["E"] ** 2)
    assert abs(np.sum(E ** 2) - lo) <= 1e-9 * lo
    h = kg.kron_gptq_code_entropy(torch.from_numpy(Z.astype(np.int32)).cuda())
    assert h == pytest.approx(oracle.code_entropy_bits(o["codes"]), abs=1e-12)


@pytest.mark.parametrize("m,n,seed", [(1, 1, 0), (6, 5, 1), (127, 129, 2), (200, 70, 3), (65, 200, 4)])
def test_ragged_fp64_free_steps_full_oracle(kg, m, n, seed):
    spec, (W, A, B) = small_layer(m, n, seed)
    c = _case(W.numpy(), A.numpy(), B.numpy(), torch.float64, steps="free", seed=seed)
    Z, V, E = _run(kg, c)
    res = _assert_fp64_parity(Z, c)
    lo = np.sum(res["oracle"]["E"] ** 2)
    assert abs(np.sum(E ** 2) - lo) <= 1e-9 * lo + 1e-20
    cert = oracle.certificate_rc(c["W"], c["UA"], c["UB"], c["al"], c["be"], Z, V, E)
    assert cert["resid_rel"] < 1e-12 and cert["code_mismatch"] == 0 and cert["halfstep_violations"] == 0


def test_unit_column_steps_equal_the_row_scaled_solver(kg):
    # alpha = 1, beta = row scales on a grid that never clips: the clipped-grid solver and the
    # unclipped one compute the same algorithm
    spec, (W, A, B) = small_layer(130, 90, 5, bits=4)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    UA = torch.from_numpy(oracle.prepare_lapack(A, DAMP)).cuda()
    UB = torch.from_numpy(oracle.prepare_lapack(B, DAMP)).cuda()
    Wt = torch.from_numpy(W).cuda()
    s = kg.kron_gptq_row_scales(Wt, 7)            # max |W_i| / 7: row codes stay in [-8, 7] or near
    codes, V, E = kg.kron_gptq_quantize(Wt, UA, UB, -128, 127, s, want_E=True)
    Z, Vr, Er = kg.kron_gptq_quantize_rc(Wt, UA, UB, torch.ones(90, dtype=torch.float64, device="cuda"), s,
                                         want_E=True)
    assert int(codes.abs().max()) < 127
    np.testing.assert_array_equal(Z.cpu().numpy(), codes.cpu().numpy().astype(np.int32))
    np.testing.assert_allclose(Vr.cpu().numpy(), V.cpu().numpy(), rtol=0, atol=0)
    Ec = E.cpu().numpy()
    np.testing.assert_allclose(Er.cpu().numpy(), Ec, rtol=1e-10, atol=1e-10 * np.abs(Ec).max())


# ------------------------------------------------------------------------------ fp32
@pytest.mark.parametrize("m,n", [(128, 128), (127, 129), (200, 70)])
def test_fp32_waterkron_vs_fp64_oracle(kg, m, n):
    spec, (W, A, B) = small_layer(m, n, 21)
    c = _case(W.numpy(), A.numpy(), B.numpy(), torch.float32)
    Z, V, E = _run(kg, c)
    o = oracle.quantize_rc(c["W"], c["UA"], c["UB"], c["al"], c["be"])
    assert np.mean(Z == o["codes"]) >= 0.95
    assert np.abs(E).max() <= 0.5 * GAMMA * (1 + 1e-5)
    assert abs(np.sum(E ** 2) / np.sum(o["E"] ** 2) - 1.0) < 0.01
    assert abs(oracle.code_entropy_bits(Z) - oracle.code_entropy_bits(o["codes"])) < 0.02
    cert = oracle.certificate_rc(c["W"], c["UA"], c["UB"], c["al"], c["be"], Z, V, E, tol=1e-4)
    assert cert["resid_rel"] < (m + n) * 2.0 ** -24, cert
    assert cert["code_mismatch"] <= 1e-3 * m * n, cert


def test_sq1024_fp32_waterkron_leading_block_certificate_entropy(kg):
    spec = workload("sq1024")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, B, torch.float32)
    Z, V, E = _run(kg, c)
    mb = 256
    al, be = oracle.waterkron_scales(c["UA"][:mb, :mb], c["UB"][:mb, :mb], GAMMA)
    np.testing.assert_allclose(al, c["al"][:mb], rtol=1e-6)
    o = oracle.quantize_rc(c["W"][:mb, :mb], c["UA"][:mb, :mb], c["UB"][:mb, :mb], c["al"][:mb], c["be"][:mb])
    assert np.mean(Z[:mb, :mb] == o["codes"]) >= 0.95
    assert abs(np.sum(E[:mb, :mb] ** 2) / np.sum(o["E"] ** 2) - 1.0) < 0.01
    assert np.abs(E).max() <= 0.5 * GAMMA * (1 + 1e-5)
    rows = np.unique(np.linspace(0, spec.m - 1, 12).astype(int))
    cert = oracle.certificate_rc(c["W"], c["UA"], c["UB"], c["al"], c["be"], Z, V, E, rows=rows, tol=1e-4)
    assert cert["resid_rel"] < (spec.m + spec.n) * 2.0 ** -24, cert
    assert cert["code_mismatch"] <= 1e-3 * len(rows) * spec.n, cert
    # high rate: mean E^2 close to gamma^2 / 12
    assert abs(np.mean(E ** 2) / (GAMMA ** 2 / 12) - 1.0) < 0.02
    Zt = torch.from_numpy(Z.astype(np.int32)).cuda()
    assert kg.kron_gptq_code_entropy(Zt) == pytest.approx(oracle.code_entropy_bits(Z), abs=1e-12)


def test_fp32_repeat_and_concurrent_streams_are_deterministic(kg):
    spec = workload("sq1024")[0]
    W, A, B = [x.numpy() for x in layer_inputs(spec)]
    c = _case(W, A, B, torch.float32)
    first = _run(kg, c)
    qs = [kg.RcQuantizer(spec.m, spec.n, torch.float32, "cuda", want_E=True) for _ in range(3)]
    streams = [torch.cuda.Stream() for _ in qs]
    torch.cuda.synchronize()
    for q, st in zip(qs, streams):
        q.run(c["Wt"], c["UAt"], c["UBt"], c["alt"], c["bet"], stream=st)
    torch.cuda.synchronize()
    for q, st in zip(qs, streams):
        assert q.status(st) == 0
        np.testing.assert_array_equal(q.Z.cpu().numpy(), first[0])
        np.testing.assert_array_equal(q.V.cpu().double().numpy(), first[1])


# ------------------------------------------------------------------------------ entropy kernel
@pytest.mark.parametrize("lo,hi,count,seed", [(0, 0, 1000, 0), (-3, 3, 100000, 1), (-20000, 20000, 300000, 2),
                                              (5, 9000, 777, 3), (-(2 ** 22) + 1, 2 ** 22 - 1, 50000, 4)])
def test_entropy_kernel_matches_numpy(kg, lo, hi, count, seed):
    rng = np.random.default_rng(seed)
    z = np.rint(rng.laplace(0.5 * (lo + hi), max(1.0, 0.1 * (hi - lo)), count)).clip(lo, hi).astype(np.int32)
    h = kg.kron_gptq_code_entropy(torch.from_numpy(z).cuda())
    assert h == pytest.approx(oracle.code_entropy_bits(z), abs=1e-12)


def test_entropy_empty_and_range_error(kg):
    assert kg.kron_gptq_code_entropy(torch.zeros(0, dtype=torch.int32, device="cuda")) == 0.0
    z = torch.tensor([0, 100, 5000], dtype=torch.int32, device="cuda")
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_code_entropy(z, max_bins=1000)
    assert ei.value.name == "KG_ERR_RANGE"
    assert kg.kron_gptq_code_entropy(z, max_bins=5001) == pytest.approx(np.log2(3), abs=1e-12)


# ------------------------------------------------------------------------------ edge cases, errors
def test_rc_empty_is_noop(kg):
    W = torch.zeros(0, 8, dtype=torch.float64, device="cuda")
    Z, V, E = kg.kron_gptq_quantize_rc(W, torch.eye(8, dtype=torch.float64, device="cuda"),
                                       torch.zeros(0, 0, dtype=torch.float64, device="cuda"),
                                       torch.ones(8, dtype=torch.float64, device="cuda"),
                                       torch.zeros(0, dtype=torch.float64, device="cuda"))
    assert Z.numel() == 0


def test_rc_bad_step_is_reported(kg):
    spec, (W, A, B) = small_layer(70, 66, 6)
    c = _case(W.numpy(), A.numpy(), B.numpy(), torch.float64)
    al = c["alt"].clone()
    al[7] = 0.0
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize_rc(c["Wt"], c["UAt"], c["UBt"], al, c["bet"])
    assert ei.value.name == "KG_ERR_NONFINITE"
    Z, V, E = kg.kron_gptq_quantize_rc(c["Wt"], c["UAt"], c["UBt"], c["alt"], c["bet"])   # context usable
    assert Z.shape == (70, 66)


def test_rc_code_beyond_fp32_range_is_reported(kg):
    spec, (W, A, B) = small_layer(64, 64, 7)
    c = _case(W.numpy(), A.numpy(), B.numpy(), torch.float32, gamma=1e-9)
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_quantize_rc(c["Wt"], c["UAt"], c["UBt"], c["alt"], c["bet"])
    assert ei.value.name == "KG_ERR_RANGE"
