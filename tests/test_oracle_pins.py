"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each test pins an oracle function to something other than itself: a library routine
(LAPACK Cholesky/inverse), the literal (mn) x (mn) vectorized algorithm, a closed form,
a special case that reduces to a textbook algorithm, an invariant, or a printed value.
``test_planted_mistakes`` shows that plausible slips in the oracle's loop fail them.
"""
import os

import numpy as np
import pytest

import oracle
from synth_inputs.layers import small_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _factors(m, n, seed, damp=0.01, bits=4, **kw):
    spec, (W, A, B) = small_layer(m, n, seed, bits=bits, **kw)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    UA, Ad = oracle.prepare(A, damp, return_damped=True)
    UB, Bd = oracle.prepare(B, damp, return_damped=True)
    s = oracle.row_scales(W, spec.qmax)
    return dict(W=W, A=A, B=B, Ad=Ad, Bd=Bd, UA=UA, UB=UB, s=s, qmin=spec.qmin, qmax=spec.qmax)


def _parse_golden(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split("=", 1)
        out[k.strip()] = np.array([[float(x) for x in r.split()] for r in v.split(";")])
    return out


# ---------------------------------------------------------------- Kronecker convention
def test_kron_convention_golden():
    g = _parse_golden(os.path.join(GOLDEN, "kron_convention.txt"))
    H = np.kron(g["P"], g["Q"])
    np.testing.assert_array_equal(H, g["H"])
    m = g["Q"].shape[0]
    for j in range(2):
        for i in range(m):
            for jp in range(2):
                for ip in range(m):
                    assert H[j * m + i, jp * m + ip] == g["P"][j, jp] * g["Q"][i, ip]


# ---------------------------------------------------------------- prepare
@pytest.mark.parametrize("n,seed", [(1, 0), (7, 1), (33, 2), (64, 3)])
def test_prepare_matches_lapack(n, seed):
    _, (W, A, B) = small_layer(4, n, seed)
    A = A.numpy()
    U, Ad = oracle.prepare(A, 0.01, return_damped=True)
    Ul = oracle.prepare_lapack(A, 0.01)
    np.testing.assert_allclose(Ad, oracle.damped(A, 0.01), rtol=1e-14, atol=1e-15)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert (np.diag(U) > 0).all()
    np.testing.assert_allclose(U, Ul, rtol=1e-9, atol=1e-9 * np.abs(Ul).max())
    np.testing.assert_allclose(U.T @ U @ Ad, np.eye(n), atol=1e-9)


def test_prepare_kron_factor_identity():
    # kron(U_A, U_B) is the upper Cholesky factor of kron(A_d, B_d)^{-1}
    # ("WaterKron", Section 3: L-hat = L^(A) (x) L^(B))
    f = _factors(5, 4, 11)
    K = np.kron(f["UA"], f["UB"])
    H = np.kron(f["Ad"], f["Bd"])
    Kref = np.linalg.cholesky(np.linalg.inv(H)).T
    np.testing.assert_allclose(K, Kref, rtol=1e-9, atol=1e-12)


def test_prepare_logdet_identity():
    # |A (x) B|^{1/mn} = |A|^{1/n} |B|^{1/m}  ("WaterKron", Section 3), i.e.
    # m logdet A_d + n logdet B_d = -2 sum_{i,j} log(U_A,jj U_B,ii)
    f = _factors(9, 6, 12)
    m, n = 9, 6
    lhs = m * np.linalg.slogdet(f["Ad"])[1] + n * np.linalg.slogdet(f["Bd"])[1]
    uA, uB = np.diag(f["UA"]), np.diag(f["UB"])
    rhs = -2.0 * np.sum(np.log(uB[:, None] * uA[None, :]))
    assert abs(lhs - rhs) < 1e-9 * abs(lhs)


def test_prepare_not_pd():
    A = np.diag([1.0, 2.0, -0.5, 3.0])
    with pytest.raises(oracle.OracleNotPD):
        oracle.prepare(A, 0.0)


def test_row_scales():
    W = np.array([[0.5, -2.0, 1.0], [0.0, 0.0, 0.0], [3.0, 1.0, -1.0]])
    s = oracle.row_scales(W, 7)
    np.testing.assert_array_equal(s, [2.0 / 7, 1.0, 3.0 / 7])


def test_rtn_definition():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((6, 9))
    S = np.full_like(W, 0.3)
    r = oracle.rtn(W, S, -4, 3)
    np.testing.assert_array_equal(r["codes"], np.clip(np.rint(W / 0.3), -4, 3))
    np.testing.assert_array_equal(r["V"], 0.3 * np.clip(np.rint(W / 0.3), -4, 3))


# ---------------------------------------------------------------- naive vs literal
@pytest.mark.parametrize("m,n,seed,bits", [(4, 4, 0, 4), (6, 5, 1, 4), (5, 7, 2, 3), (3, 8, 3, 2), (8, 3, 4, 3)])
def test_naive_equals_literal_vectorized(m, n, seed, bits):
    f = _factors(m, n, seed, bits=bits)
    r = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    lit = oracle.literal_vec(f["W"], f["Ad"], f["Bd"], f["s"], f["qmin"], f["qmax"])
    assert r["n_boundary"] == 0
    np.testing.assert_array_equal(r["codes"], lit["codes"])
    np.testing.assert_allclose(r["V"], lit["V"], rtol=0, atol=0)
    np.testing.assert_allclose(r["E"], lit["E"], rtol=1e-9, atol=1e-12)
    # the literal factor is kron(U_A, U_B) (vector index p = j*m + i)
    np.testing.assert_allclose(lit["K"], np.kron(f["UA"], f["UB"]), rtol=1e-9, atol=1e-12)
    for res in (r, lit):
        c = oracle.certificate(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"],
                               res["codes"], res["V"], res["E"])
        assert c["resid_rel"] < 1e-12 and c["code_mismatch"] == 0 and c["halfstep_violations"] == 0


def test_onesided_equals_literal_with_identity_B():
    f = _factors(4, 6, 21, bits=3)
    m, n = 4, 6
    Bd = np.eye(m)
    lit = oracle.literal_vec(f["W"], f["Ad"], Bd, f["s"], f["qmin"], f["qmax"])
    one = oracle.quantize_onesided(f["W"], f["UA"], np.repeat(f["s"][:, None], n, 1), f["qmin"], f["qmax"])
    np.testing.assert_array_equal(one["codes"], lit["codes"])


# ---------------------------------------------------------------- special cases
def test_identity_factors_reduce_to_rtn():
    f = _factors(12, 10, 31)
    m, n = 12, 10
    r = oracle.quantize_naive(f["W"], np.eye(n), np.eye(m), f["s"], f["qmin"], f["qmax"])
    rt = oracle.rtn(f["W"], np.repeat(f["s"][:, None], n, 1), f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r["codes"], rt["codes"])


def test_diagonal_factors_reduce_to_rtn():
    f = _factors(12, 10, 32)
    m, n = 12, 10
    UA = oracle.prepare(np.diag(np.diag(f["A"])), 0.01)
    UB = oracle.prepare(np.diag(np.diag(f["B"])), 0.01)
    assert np.count_nonzero(np.triu(UA, 1)) == 0
    r = oracle.quantize_naive(f["W"], UA, UB, f["s"], f["qmin"], f["qmax"])
    rt = oracle.rtn(f["W"], np.repeat(f["s"][:, None], n, 1), f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r["codes"], rt["codes"])


def test_identity_B_reduces_to_onesided_gptq():
    # "FastKron", Section 1: with B = I the algorithm recovers standard GPTQ
    f = _factors(24, 40, 41, bits=3)
    m, n = 24, 40
    r = oracle.quantize_naive(f["W"], f["UA"], np.eye(m), f["s"], f["qmin"], f["qmax"])
    one = oracle.quantize_onesided(f["W"], f["UA"], np.repeat(f["s"][:, None], n, 1), f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r["codes"], one["codes"])
    np.testing.assert_allclose(r["E"], one["E"], rtol=1e-9, atol=1e-12)


def test_identity_A_reduces_to_onesided_gptq_of_transpose():
    f = _factors(30, 16, 42, bits=3)
    m, n = 30, 16
    r = oracle.quantize_naive(f["W"], np.eye(n), f["UB"], f["s"], f["qmin"], f["qmax"])
    St = np.repeat(f["s"][None, :], n, 0)           # per-row scales of W = per-column of W^T
    one = oracle.quantize_onesided(f["W"].T, f["UB"], St, f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r["codes"], one["codes"].T)


def test_transpose_symmetry_scalar_scale():
    f = _factors(14, 11, 43, bits=3)
    sig = float(np.abs(f["W"]).max() / f["qmax"])
    s1 = np.full(14, sig)
    s2 = np.full(11, sig)
    r1 = oracle.quantize_naive(f["W"], f["UA"], f["UB"], s1, f["qmin"], f["qmax"])
    r2 = oracle.quantize_naive(f["W"].T, f["UB"], f["UA"], s2, f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r1["codes"], r2["codes"].T)


def test_leading_block_depends_only_on_leading_data():
    # updates reach only entries to the bottom-right ("FastKron", Section 2.3)
    f = _factors(24, 20, 44)
    r = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    mb, nb = 13, 9
    rb = oracle.quantize_naive(f["W"][:mb, :nb], f["UA"][:nb, :nb], f["UB"][:mb, :mb], f["s"][:mb],
                               f["qmin"], f["qmax"])
    np.testing.assert_array_equal(r["codes"][:mb, :nb], rb["codes"])
    np.testing.assert_array_equal(r["E"][:mb, :nb], rb["E"])


# ---------------------------------------------------------------- loss and bounds
def test_loss_identity_and_definition():
    f = _factors(7, 6, 51)
    r = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    lt = oracle.loss(f["W"], r["V"], f["Ad"], f["Bd"])
    # definition: vec(V-W)^T kron(A_d, B_d) vec(V-W), column-major vec
    d = (r["V"] - f["W"]).T.reshape(-1)
    ldef = d @ np.kron(f["Ad"], f["Bd"]) @ d
    assert abs(lt - ldef) < 1e-11 * abs(ldef)
    # the transformed errors are orthonormal coordinates: loss = sum E^2
    assert abs(lt - np.sum(r["E"] ** 2)) < 1e-10 * lt


def test_error_bound_unclipped():
    # each |e_ij| <= s_i / (2 U_B,ii U_A,jj); with unit scales the total is at most
    # tr(A_d) tr(B_d) / 4 (the error bound quoted for BaKron)
    f = _factors(16, 12, 52)
    m, n = 16, 12
    big = 2 ** 30
    s = np.ones(m)
    r = oracle.quantize_naive(f["W"] * 20.0, f["UA"], f["UB"], s, -big, big - 1)
    uA, uB = np.diag(f["UA"]), np.diag(f["UB"])
    lim = (s[:, None] / (2 * uB[:, None] * uA[None, :]))
    assert (np.abs(r["E"]) <= lim * (1 + 1e-12)).all()
    loss = oracle.loss(f["W"] * 20.0, r["V"], f["Ad"], f["Bd"])
    assert loss <= np.sum(lim ** 2) * (1 + 1e-9)
    assert np.sum(lim ** 2) <= 0.25 * np.trace(f["Ad"]) * np.trace(f["Bd"]) * (1 + 1e-12)


def test_certificate_on_oracle_output():
    f = _factors(40, 33, 53, bits=3)
    r = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    c = oracle.certificate(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"], r["codes"], r["V"], r["E"])
    assert c["resid_rel"] < 1e-12 and c["code_mismatch"] == 0 and c["halfstep_violations"] == 0
    cs = oracle.certificate(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"], r["codes"], r["V"], r["E"],
                            rows=[0, 7, 39])
    assert cs["resid_rel"] < 1e-12 and cs["rows"] == 3
    # a corrupted E is caught by the residual
    E2 = r["E"].copy()
    E2[5, 4] += 1e-3
    c2 = oracle.certificate(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"], r["codes"], r["V"], E2)
    assert c2["resid_rel"] > 1e-6


# ---------------------------------------------------------------- parity rule
def test_parity_rule_absorbs_ties_only():
    f = _factors(10, 8, 61)
    W = f["W"].copy()
    s = f["s"].copy()
    W[0, 0] = 0.5 * s[0]              # the first entry sits exactly on a tie
    r = oracle.quantize_naive(W, f["UA"], f["UB"], s, f["qmin"], f["qmax"])
    assert r["boundary"][0, 0]
    forced = np.full(W.shape, oracle.NOT_FORCED, dtype=np.int32)
    forced[0, 0] = int(r["codes"][0, 0]) + 1   # the other side of the tie
    cand = oracle.quantize_naive(W, f["UA"], f["UB"], s, f["qmin"], f["qmax"], forced=forced)["codes"]
    res = oracle.compare_with_oracle(cand, W, f["UA"], f["UB"], s, f["qmin"], f["qmax"])
    assert res["ok"] and len(res["flips"]) == 1
    bad = r["codes"].copy()
    bad[3, 2] += 1
    res2 = oracle.compare_with_oracle(bad, W, f["UA"], f["UB"], s, f["qmin"], f["qmax"])
    assert not res2["ok"] and res2["first"] == (3, 2)


# ---------------------------------------------------------------- planted mistakes
def _naive_py(W, UA, UB, s, qmin, qmax, mutation=None):
    """A pure-Python copy of the oracle's loop with one planted mistake."""
    m, n = W.shape
    Wt = W.copy()
    codes = np.zeros((m, n), dtype=np.int32)
    V = np.zeros((m, n))
    E = np.zeros((m, n))
    for j in range(n):
        for i in range(m):
            x = Wt[i, j]
            c = min(max(np.rint(x / s[i]), qmin), qmax)
            q = s[i] * c
            den = UB[i, i] * UA[j, j] if mutation != "drop_uB_scale" else UA[j, j]
            e = (x - q) / den
            codes[i, j], V[i, j], E[i, j] = c, q, e
            for ip in range(i, m):
                for jp in range(j, n):
                    if ip == i and jp == j:
                        continue
                    if mutation == "skip_same_row" and ip == i:
                        continue
                    b = UB[i, ip] if mutation != "transpose_UB" else UB[ip, i]
                    a = UA[j, jp]
                    sign = -1.0 if mutation != "wrong_sign" else 1.0
                    Wt[ip, jp] += sign * b * e * a
    return codes, V, E


@pytest.mark.parametrize("mutation", ["drop_uB_scale", "skip_same_row", "transpose_UB", "wrong_sign"])
def test_planted_mistakes_fail_a_pin(mutation):
    f = _factors(6, 5, 1, bits=4)
    args = (f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    c0, V0, E0 = _naive_py(*args)
    ref = oracle.quantize_naive(*args)
    np.testing.assert_array_equal(c0, ref["codes"])       # the unmutated copy agrees
    c, V, E = _naive_py(*args, mutation=mutation)
    lit = oracle.literal_vec(f["W"], f["Ad"], f["Bd"], f["s"], f["qmin"], f["qmax"])
    cert = oracle.certificate(*args[:3], f["s"], f["qmin"], f["qmax"], c, V, E)
    caught = (not np.array_equal(c, lit["codes"])) or cert["resid_rel"] > 1e-9 or cert["code_mismatch"] > 0
    assert caught, mutation


def test_generator_leading_block_is_consistent():
    from synth_inputs.layers import LayerSpec, layer_inputs
    spec = LayerSpec(name="t", m=48, n=40, seed=5, n_samples=64, outlier_frac=0.05)
    W, A, B = layer_inputs(spec)
    Wl, Al, Bl = layer_inputs(spec, leading=16)
    assert np.array_equal(W[:16, :16].numpy(), Wl.numpy())
    np.testing.assert_allclose(A[:16, :16].numpy(), Al.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(B[:16, :16].numpy(), Bl.numpy(), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- row- and column-scaled alphabet
# "WaterKron and FlipFlop Hessian", Section 2.1: V = beta alpha^T (.) Z with Z integer and not
# clipped; Section 3: the WaterKron steps alpha_j ~ U_A[j,j], beta_i ~ U_B[i,i].

def _rc_case(m, n, seed, gamma=None, scale_w=1.0):
    f = _factors(m, n, seed)
    W = f["W"] * scale_w
    if gamma is None:
        rng = np.random.default_rng(seed)
        alpha = 0.05 * np.exp(0.5 * rng.standard_normal(n))
        beta = np.exp(0.5 * rng.standard_normal(m))
    else:
        alpha, beta = oracle.waterkron_scales(f["UA"], f["UB"], gamma)
    return f, W, alpha, beta


@pytest.mark.parametrize("m,n,seed,gamma", [(4, 4, 0, None), (6, 5, 1, None), (5, 7, 2, 0.7), (3, 8, 3, 0.2),
                                            (8, 3, 4, 1.5)])
def test_rc_equals_literal_vectorized(m, n, seed, gamma):
    f, W, alpha, beta = _rc_case(m, n, seed, gamma)
    r = oracle.quantize_rc(W, f["UA"], f["UB"], alpha, beta)
    lit = oracle.literal_vec_entry(W, f["Ad"], f["Bd"], beta[:, None] * alpha[None, :])
    assert r["n_boundary"] == 0
    np.testing.assert_array_equal(r["codes"], lit["codes"])
    np.testing.assert_allclose(r["V"], lit["V"], rtol=0, atol=0)
    np.testing.assert_allclose(r["E"], lit["E"], rtol=1e-9, atol=1e-12)
    assert np.abs(r["codes"]).max() > 0


def test_rc_identity_factors_is_entrywise_rounding():
    f, W, alpha, beta = _rc_case(12, 10, 71, scale_w=40.0)
    step = beta[:, None] * alpha[None, :]
    r = oracle.quantize_rc(W, np.eye(10), np.eye(12), alpha, beta)
    np.testing.assert_array_equal(r["codes"], np.rint(W / step).astype(np.int64))
    np.testing.assert_array_equal(r["V"], step * np.rint(W / step))
    # unbounded: codes far outside any clipped grid survive
    assert np.abs(r["codes"]).max() > 127


def test_rc_with_unit_columns_is_the_row_scaled_algorithm():
    # alpha = 1 and beta = s: the row-scaled algorithm on a grid too wide to clip
    f = _factors(14, 11, 72)
    big = 2 ** 30
    r = oracle.quantize_rc(f["W"], f["UA"], f["UB"], np.ones(11), f["s"] * 0.05)
    ref = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"] * 0.05, -big, big - 1)
    np.testing.assert_array_equal(r["codes"], ref["codes"].astype(np.int64))
    np.testing.assert_array_equal(r["V"], ref["V"])
    np.testing.assert_array_equal(r["E"], ref["E"])


def test_waterkron_error_bound_certificate_and_loss():
    gamma = 0.4
    f, W, alpha, beta = _rc_case(20, 16, 73, gamma)
    r = oracle.quantize_rc(W, f["UA"], f["UB"], alpha, beta)
    # with steps gamma U_B[i,i] U_A[j,j] every error lies in [-gamma/2, gamma/2]
    assert np.abs(r["E"]).max() <= 0.5 * gamma * (1 + 1e-12)
    c = oracle.certificate_rc(W, f["UA"], f["UB"], alpha, beta, r["codes"], r["V"], r["E"])
    assert c["resid_rel"] < 1e-12 and c["code_mismatch"] == 0 and c["halfstep_violations"] == 0
    # the proxy loss is sum E^2 for any alphabet (V - W = -U_B^T E U_A)
    lt = oracle.loss(W, r["V"], f["Ad"], f["Bd"])
    assert abs(lt - np.sum(r["E"] ** 2)) < 1e-10 * lt
    # a corrupted code breaks the certificate
    bad = r["codes"].copy()
    bad[3, 5] += 1
    c2 = oracle.certificate_rc(W, f["UA"], f["UB"], alpha, beta, bad, r["V"], r["E"])
    assert c2["code_mismatch"] == 1


def test_waterkron_high_rate_distortion():
    # high rate: the transformed errors are uniform on [-gamma/2, gamma/2], so the mean of E^2
    # is gamma^2 / 12 ("WaterKron and FlipFlop Hessian", Appendix C.2, the limit gamma -> 0)
    gamma = 0.02
    f, W, alpha, beta = _rc_case(64, 64, 74, gamma)
    r = oracle.quantize_rc(W, f["UA"], f["UB"], alpha, beta)
    ratio = np.mean(r["E"] ** 2) / (gamma ** 2 / 12)
    assert abs(ratio - 1.0) < 0.05, ratio
    # halving gamma adds about one bit per entry to the empirical entropy of Z
    alpha2, beta2 = oracle.waterkron_scales(f["UA"], f["UB"], gamma / 2)
    r2 = oracle.quantize_rc(W, f["UA"], f["UB"], alpha2, beta2)
    dh = oracle.code_entropy_bits(r2["codes"]) - oracle.code_entropy_bits(r["codes"])
    assert abs(dh - 1.0) < 0.1, dh


def test_code_entropy_closed_forms():
    assert oracle.code_entropy_bits(np.full((7, 9), -3)) == 0.0
    z = np.tile(np.array([-2, 0, 5, 1000]), 25)
    assert oracle.code_entropy_bits(z) == pytest.approx(2.0, abs=1e-15)
    z = np.array([0] * 300 + [-7] * 100)
    h = -(0.75 * np.log2(0.75) + 0.25 * np.log2(0.25))
    assert oracle.code_entropy_bits(z) == pytest.approx(h, abs=1e-15)
    assert oracle.code_entropy_bits(np.arange(256)) == pytest.approx(8.0, abs=1e-12)


def _rc_py(W, UA, UB, alpha, beta, mutation=None):
    """A pure-Python copy of the scaled-alphabet loop with one planted mistake."""
    m, n = W.shape
    Wt = W.copy()
    codes = np.zeros((m, n), dtype=np.int64)
    V = np.zeros((m, n))
    E = np.zeros((m, n))
    for j in range(n):
        for i in range(m):
            x = Wt[i, j]
            sij = beta[i] * alpha[j] if mutation != "row_step_only" else beta[i]
            z = np.rint(x / sij)
            if mutation == "clip_int8":
                z = min(max(z, -128), 127)
            q = sij * z
            e = (x - q) / (UB[i, i] * UA[j, j])
            if mutation == "error_in_grid_units":
                e = (x - q) / sij
            codes[i, j], V[i, j], E[i, j] = z, q, e
            for ip in range(i, m):
                for jp in range(j, n):
                    if ip == i and jp == j:
                        continue
                    Wt[ip, jp] -= UB[i, ip] * e * UA[j, jp]
    return codes, V, E


@pytest.mark.parametrize("mutation", ["row_step_only", "clip_int8", "error_in_grid_units"])
def test_planted_mistakes_fail_an_rc_pin(mutation):
    f, W, alpha, beta = _rc_case(6, 5, 75)
    W = W * 40.0                       # codes beyond the int8 range
    args = (W, f["UA"], f["UB"], alpha, beta)
    c0, V0, E0 = _rc_py(*args)
    ref = oracle.quantize_rc(*args)
    np.testing.assert_array_equal(c0, ref["codes"])       # the unmutated copy agrees
    c, V, E = _rc_py(*args, mutation=mutation)
    lit = oracle.literal_vec_entry(W, f["Ad"], f["Bd"], beta[:, None] * alpha[None, :])
    cert = oracle.certificate_rc(*args, c, V, E)
    caught = (not np.array_equal(c, lit["codes"])) or cert["resid_rel"] > 1e-9 or cert["code_mismatch"] > 0
    assert caught, mutation


# ---------------------------------------------------------------- the cubic CPU baseline
@pytest.mark.parametrize("m,n,seed,bits", [(6, 5, 1, 4), (40, 33, 2, 3), (127, 129, 3, 3), (200, 70, 4, 2), (1, 90, 5, 4)])
def test_cubic_baseline_equals_the_definition(m, n, seed, bits):
    # the two-chain, anti-diagonal-parallel form reorganises the same sums: equal codes away from
    # rounding ties, E to rounding noise
    f = _factors(m, n, seed, bits=bits)
    r = oracle.quantize_naive(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    c = oracle.quantize_cubic(f["W"], f["UA"], f["UB"], f["s"], f["qmin"], f["qmax"])
    assert r["n_boundary"] == 0
    np.testing.assert_array_equal(c["codes"], r["codes"])
    np.testing.assert_array_equal(c["V"], r["V"])
    np.testing.assert_allclose(c["E"], r["E"], rtol=1e-9, atol=1e-12 * np.abs(r["E"]).max())
    assert oracle.cubic_threads() >= 1
