"""Pins of the Kronecker-factor oracle (oracle/factors.py) against closed forms, a library SVD and
an optimality property (CPU only).

H = E[a a^T (x) b b^T] ("FastKron", Section 3.2; "WaterKron and FlipFlop Hessian", Table 1).
  * A factorial sample design (every pair (a_i, b_j) once) makes H exactly A0 (x) B0 with
    A0 = mean a_i a_i^T, B0 = mean b_j b_j^T; Marginal, one Frobenius and one FlipFlop iteration
    must all return a product equal to H.
  * Frobenius minimises ||H - A (x) B||_F; its fixed point reaches the Van Loan-Pitsianis optimum
    ||R(H)||^2 - sigma_1(R(H))^2 (numpy SVD of the rearranged H).
  * FlipFlop minimises the scale-free mismatch tr(H (A (x) B)^-1) |A (x) B|^(1/mn) / (mn)
    ("WaterKron and FlipFlop Hessian", Sections 4-5): random symmetric perturbations of its fixed
    point never lower it, while they do lower it at the Marginal factors.
"""
import numpy as np
import pytest

from oracle import factors


def _samples(N, n, m, seed, mix=0.7):
    """Correlated a, b with a non-Kronecker joint law (b's scale depends on a)."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((N, n)) @ (np.eye(n) + 0.3 * rng.standard_normal((n, n)))
    b = rng.standard_normal((N, m)) @ (np.eye(m) + 0.3 * rng.standard_normal((m, m)))
    b *= (1.0 + mix * np.abs(a[:, :1]))
    return a, b


def test_hessian_brute_force_is_the_mean_of_kronecker_products():
    a, b = _samples(7, 3, 2, 0)
    H = factors.hessian(a, b)
    assert H.shape == (6, 6)
    ref = sum(np.kron(np.outer(a[i], a[i]), np.outer(b[i], b[i])) for i in range(7)) / 7
    np.testing.assert_allclose(H, ref, rtol=1e-14, atol=0)
    # entry (i1*m + j1, i2*m + j2) = E[a_i1 a_i2 b_j1 b_j2]
    assert H[1 * 2 + 0, 2 * 2 + 1] == pytest.approx(np.mean(a[:, 1] * a[:, 2] * b[:, 0] * b[:, 1]), rel=1e-13)


def test_exact_kronecker_design_is_reproduced_by_all_three():
    rng = np.random.default_rng(1)
    n, m = 4, 3
    ai = rng.standard_normal((5, n))
    bj = rng.standard_normal((6, m))
    a = np.repeat(ai, 6, axis=0)
    b = np.tile(bj, (5, 1))
    H = factors.hessian(a, b)
    A0, B0 = ai.T @ ai / 5, bj.T @ bj / 6
    np.testing.assert_allclose(H, np.kron(A0, B0), rtol=1e-12, atol=1e-14)
    for A, B in (factors.marginal(a, b), factors.frobenius(a, b, 1), factors.flipflop(a, b, 1)):
        np.testing.assert_allclose(np.kron(A, B), H, rtol=1e-10, atol=1e-12)


def test_frobenius_reaches_the_van_loan_pitsianis_optimum():
    n, m = 4, 3
    a, b = _samples(200, n, m, 2)
    H = factors.hessian(a, b)
    R = factors.rearrange(H, n, m)
    s = np.linalg.svd(R, compute_uv=False)
    best = np.sum(s ** 2) - s[0] ** 2
    A, B = factors.frobenius(a, b, 60)
    got = np.sum((H - np.kron(A, B)) ** 2)
    assert got == pytest.approx(best, rel=1e-9)
    Am, Bm = factors.marginal(a, b)
    assert np.sum((H - np.kron(Am, Bm)) ** 2) > got * (1 + 1e-6)
    # the rearrangement is the one that turns a Kronecker product into a rank-one matrix
    np.testing.assert_allclose(factors.rearrange(np.kron(A, B), n, m), np.outer(A.reshape(-1), B.reshape(-1)),
                               rtol=1e-12, atol=1e-14)


def test_flipflop_is_a_local_minimum_of_the_mismatch():
    n, m = 4, 3
    a, b = _samples(300, n, m, 3)
    H = factors.hessian(a, b)
    A, B = factors.flipflop(a, b, 200)
    f0 = factors.mismatch(H, A, B)
    rng = np.random.default_rng(4)
    Ah = np.linalg.cholesky(A)
    Bh = np.linalg.cholesky(B)
    for _ in range(20):
        Sa = rng.standard_normal((n, n)); Sa = 0.5 * (Sa + Sa.T)
        Sb = rng.standard_normal((m, m)); Sb = 0.5 * (Sb + Sb.T)
        eps = 1e-2
        A2 = Ah @ (np.eye(n) + eps * Sa) @ Ah.T
        B2 = Bh @ (np.eye(m) + eps * Sb) @ Bh.T
        assert factors.mismatch(H, A2, B2) >= f0 * (1 - 1e-12)
    # the Marginal factors are not a minimum: FlipFlop lowers the mismatch below theirs
    Am, Bm = factors.marginal(a, b)
    assert factors.mismatch(H, Am, Bm) > f0 * (1 + 1e-6)
    # and the mismatch is scale free
    assert factors.mismatch(H, 3.0 * A, B / 7.0) == pytest.approx(f0, rel=1e-12)


def test_scale_covariance():
    a, b = _samples(100, 5, 4, 5)
    A, B = factors.flipflop(a, b, 3)
    A2, B2 = factors.flipflop(2.0 * a, b, 3)
    np.testing.assert_allclose(A2, 4.0 * A, rtol=1e-12)
    np.testing.assert_allclose(B2, B, rtol=1e-12)
    A, B = factors.frobenius(a, b, 3)
    A3, B3 = factors.frobenius(a, 3.0 * b, 3)
    np.testing.assert_allclose(np.kron(A3, B3), 9.0 * np.kron(A, B), rtol=1e-11)


def test_first_iterations_share_A_and_differ_in_B():
    # from B = I both weight a a^T by b^T b (up to the constant); their B updates differ
    a, b = _samples(50, 4, 3, 6)
    Af, Bf = factors.frobenius(a, b, 1)
    Ap, Bp = factors.flipflop(a, b, 1)
    np.testing.assert_allclose(Af, Ap, rtol=1e-13)
    assert not np.allclose(Bf / np.trace(Bf), Bp / np.trace(Bp))


# ---- planted mistakes: a mutated copy of each estimator must fail one of the pins above ----
# (A slip in the constant of the A update alone is not a mistake: the B update that follows is the
# exact least-squares or flip-flop step for that A, so only the split of scale between the two
# factors moves, which two-sided GPTQ does not see.)

def _mutated(mutation):
    """Copies of marginal / frobenius / flipflop / hessian with one plausible slip planted."""
    def gram(x, w, d):
        return (x.T * w) @ x / d

    def marginal(a, b):
        d = a.shape[0] - 1 if mutation == "marginal_unbiased" else a.shape[0]
        return gram(a, np.ones(a.shape[0]), d), gram(b, np.ones(b.shape[0]), d)

    def frobenius(a, b, iters=1):
        B = np.eye(b.shape[1])
        for _ in range(iters):
            Bw = np.eye(b.shape[1]) if mutation == "frob_drop_B_weight" else B
            w = np.einsum("ki,ij,kj->k", b, Bw, b)
            A = gram(a, w, a.shape[0]) / np.sum(B * B)
            v = np.einsum("ki,ij,kj->k", a, A, a)
            c = np.sqrt(np.sum(A * A)) if mutation == "frob_norm_not_squared" else np.sum(A * A)
            B = gram(b, v, b.shape[0]) / c
        return A, B

    def flipflop(a, b, iters=1):
        n, m = a.shape[1], b.shape[1]
        cA, cB = (n, m) if mutation == "flip_swapped_dims" else (m, n)
        B = np.eye(m)
        for _ in range(iters):
            Bi = B if mutation == "flip_no_inverse" else np.linalg.inv(B)
            A = gram(a, np.einsum("ki,ij,kj->k", b, Bi, b), a.shape[0]) / cA
            v = np.einsum("ki,ij,kj->k", a, np.linalg.inv(A), a)
            B = gram(b, v, b.shape[0]) / cB
        return A, B

    def hessian(a, b):
        H = 0
        for k in range(a.shape[0]):
            pa, pb = np.outer(a[k], a[k]), np.outer(b[k], b[k])
            H = H + (np.kron(pb, pa) if mutation == "kron_order_swapped" else np.kron(pa, pb))
        return H / a.shape[0]

    return marginal, frobenius, flipflop, hessian


def _pins_hold(marginal, frobenius, flipflop, hessian):
    """The checks of the pins above, as one predicate over a set of estimators."""
    a, b = _samples(7, 3, 2, 0)
    H = hessian(a, b)
    if not np.isclose(H[1 * 2 + 0, 2 * 2 + 1], np.mean(a[:, 1] * a[:, 2] * b[:, 0] * b[:, 1]), rtol=1e-12):
        return False
    rng = np.random.default_rng(1)
    ai, bj = rng.standard_normal((5, 4)), rng.standard_normal((6, 3))
    a, b = np.repeat(ai, 6, axis=0), np.tile(bj, (5, 1))
    H = hessian(a, b)
    for A, B in (marginal(a, b), frobenius(a, b, 1), flipflop(a, b, 1)):
        if not np.allclose(np.kron(A, B), H, rtol=1e-9, atol=1e-12):
            return False
    a, b = _samples(200, 4, 3, 2)
    H = hessian(a, b)
    s = np.linalg.svd(factors.rearrange(H, 4, 3), compute_uv=False)
    A, B = frobenius(a, b, 60)
    if not np.isclose(np.sum((H - np.kron(A, B)) ** 2), np.sum(s ** 2) - s[0] ** 2, rtol=1e-8):
        return False
    a, b = _samples(300, 4, 3, 3)
    H = hessian(a, b)
    A, B = flipflop(a, b, 200)
    f0 = factors.mismatch(H, A, B)
    rng = np.random.default_rng(4)
    Ah, Bh = np.linalg.cholesky(A), np.linalg.cholesky(B)
    for _ in range(20):
        Sa = rng.standard_normal((4, 4)); Sa = 0.5 * (Sa + Sa.T)
        Sb = rng.standard_normal((3, 3)); Sb = 0.5 * (Sb + Sb.T)
        A2 = Ah @ (np.eye(4) + 1e-2 * Sa) @ Ah.T
        B2 = Bh @ (np.eye(3) + 1e-2 * Sb) @ Bh.T
        if factors.mismatch(H, A2, B2) < f0 * (1 - 1e-12):
            return False
    return True


def test_unmutated_copy_passes_the_pins():
    assert _pins_hold(*_mutated(None))
    a, b = _samples(40, 4, 3, 9)
    m0, f0, p0, h0 = _mutated(None)
    for mine, ref in ((m0(a, b), factors.marginal(a, b)), (f0(a, b, 3), factors.frobenius(a, b, 3)),
                      (p0(a, b, 3), factors.flipflop(a, b, 3))):
        np.testing.assert_allclose(mine[0], ref[0], rtol=1e-12)
        np.testing.assert_allclose(mine[1], ref[1], rtol=1e-12)
    np.testing.assert_allclose(h0(a, b), factors.hessian(a, b), rtol=1e-12)


@pytest.mark.parametrize("mutation", ["marginal_unbiased", "frob_drop_B_weight", "frob_norm_not_squared",
                                      "flip_no_inverse", "flip_swapped_dims", "kron_order_swapped"])
def test_planted_mistakes_fail_a_factor_pin(mutation):
    with np.errstate(all="ignore"):     # a mutated iteration may run off to inf / nan
        assert not _pins_hold(*_mutated(mutation)), mutation
