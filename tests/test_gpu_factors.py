"""Kronecker factor estimation on the device (kron_gptq_factors) against the oracle
(oracle/factors.py, pinned in tests/test_oracle_factors.py).  Needs a B200.

Both sides get identical fp64 samples (fp32 inputs are promoted by both).  The GPU computes the
same formulas with DGEMMs and the library's Cholesky-based inverse factor; the bar is 1e-9 relative
(Frobenius norm of the difference), far above fp64 rounding and far below any error of method.
"""
import numpy as np
import pytest
import torch

from oracle import factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


def _samples(N, n, m, seed):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((N, n)) @ (np.eye(n) + 0.3 * rng.standard_normal((n, n)) / np.sqrt(n))
    b = rng.standard_normal((N, m)) @ (np.eye(m) + 0.3 * rng.standard_normal((m, m)) / np.sqrt(m))
    b *= (1.0 + 0.7 * np.abs(a[:, :1]))
    return a, b


def _rel(X, Y):
    return np.linalg.norm(X - Y) / np.linalg.norm(Y)


@pytest.mark.parametrize("method,iters", [("marginal", 1), ("frobenius", 1), ("frobenius", 3), ("flipflop", 1),
                                          ("flipflop", 2), ("flipflop", 3)])
@pytest.mark.parametrize("N,n,m", [(300, 48, 40), (1000, 130, 70)])
def test_factors_match_oracle(kg, method, iters, N, n, m):
    a, b = _samples(N, n, m, N + n)
    A, B = kg.kron_gptq_factors(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), method, iters)
    ref = {"marginal": lambda: factors.marginal(a, b), "frobenius": lambda: factors.frobenius(a, b, iters),
           "flipflop": lambda: factors.flipflop(a, b, iters)}[method]()
    A, B = A.cpu().numpy(), B.cpu().numpy()
    assert _rel(A, ref[0]) < 1e-9 and _rel(B, ref[1]) < 1e-9, (_rel(A, ref[0]), _rel(B, ref[1]))
    np.testing.assert_array_equal(A, A.T)
    np.testing.assert_array_equal(B, B.T)


def test_fp32_samples_are_promoted(kg):
    a, b = _samples(500, 64, 32, 7)
    a32, b32 = a.astype(np.float32), b.astype(np.float32)
    A, B = kg.kron_gptq_factors(torch.from_numpy(a32).cuda(), torch.from_numpy(b32).cuda(), "flipflop", 2)
    rA, rB = factors.flipflop(a32.astype(np.float64), b32.astype(np.float64), 2)
    assert _rel(A.cpu().numpy(), rA) < 1e-9 and _rel(B.cpu().numpy(), rB) < 1e-9


def test_exact_kronecker_design(kg):
    rng = np.random.default_rng(8)
    ai, bj = rng.standard_normal((40, 16)), rng.standard_normal((30, 12))
    a, b = np.repeat(ai, 30, axis=0), np.tile(bj, (40, 1))
    A0, B0 = ai.T @ ai / 40, bj.T @ bj / 30
    for method in ("marginal", "frobenius", "flipflop"):
        A, B = kg.kron_gptq_factors(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), method, 1)
        K = np.kron(A.cpu().numpy(), B.cpu().numpy())
        assert _rel(K, np.kron(A0, B0)) < 1e-10, method


def test_feeds_the_solver(kg):
    # the FlipFlop factors of a 256 x 128 layer's samples go straight into prepare and the solve
    a, b = _samples(2000, 128, 256, 9)
    A, B = kg.kron_gptq_factors(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), "flipflop", 2)
    UA, UB, _, _ = kg.kron_gptq_prepare(A, B, 0.01)
    W = torch.randn(256, 128, dtype=torch.float64, device="cuda") / np.sqrt(128)
    s = kg.kron_gptq_row_scales(W, 7)
    codes, V, E = kg.kron_gptq_quantize(W, UA, UB, -8, 7, s, want_E=True)
    assert codes.shape == (256, 128) and torch.isfinite(E).all()


def test_errors(kg):
    a, b = _samples(50, 8, 6, 10)
    at = torch.from_numpy(a).cuda()
    at[3, 2] = float("nan")
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_factors(at, torch.from_numpy(b).cuda(), "marginal")
    assert ei.value.name == "KG_ERR_NONFINITE"
    # an output channel whose gradient is always zero makes B singular (an exactly zero row and
    # column); the second FlipFlop iteration needs B^-1 and reports it instead of returning
    a2, b2 = _samples(60, 8, 6, 11)
    b2[:, 3] = 0.0
    with pytest.raises(kg.KGError) as ei:
        kg.kron_gptq_factors(torch.from_numpy(a2).cuda(), torch.from_numpy(b2).cuda(), "flipflop", 2)
    assert ei.value.name == "KG_ERR_NOT_PD"
