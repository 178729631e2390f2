"""The seeded input recipe (synth_inputs/layers.py), CPU only: the same seed gives the same layer,
and the layers have the stated shapes, grids and distributions."""
import math

import pytest
import torch

from synth_inputs.layers import WORKLOADS, layer_inputs, small_layer, workload


def test_same_seed_same_layer():
    spec = workload("ref128")[0]
    W1, A1, B1 = layer_inputs(spec)
    W2, A2, B2 = layer_inputs(spec)
    assert torch.equal(W1, W2) and torch.equal(A1, A2) and torch.equal(B1, B2)
    _, (W3, _, _) = small_layer(128, 128, seed=1)
    assert not torch.equal(W1, W3)


def test_workload_table():
    assert [(s.m, s.n, s.bits) for s in workload("sq4096")] == [(4096, 4096, 3)]
    assert (workload("sq4096")[0].qmin, workload("sq4096")[0].qmax) == (-4, 3)
    assert (workload("sq4096_2bit")[0].qmin, workload("sq4096_2bit")[0].qmax) == (-2, 1)
    assert (workload("sq4096_4bit")[0].qmin, workload("sq4096_4bit")[0].qmax) == (-8, 7)
    assert (workload("ffn_up")[0].m, workload("ffn_up")[0].n) == (14336, 4096)
    assert (workload("ffn_down")[0].m, workload("ffn_down")[0].n) == (4096, 14336)
    block = workload("block")
    assert [s.name for s in block] == ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]
    assert sum(s.m * s.n for s in block) == 218103808          # 2.18e8 weights
    # layers share a seed only when they are the same layer: the bit-width variants of the 4096^2
    # layer, and the 1024^2 layer with B replaced by I
    by_seed = {}
    for specs in WORKLOADS.values():
        for s in specs:
            by_seed.setdefault(s.seed, set()).add((s.m, s.n, s.n_samples, s.outlier_frac))
    assert all(len(v) == 1 for v in by_seed.values())
    assert len({s.seed for s in block}) == 7


def test_weight_distribution():
    spec = workload("sq1024")[0]
    W, _, _ = layer_inputs(spec, with_factors=False)
    assert W.shape == (1024, 1024) and W.dtype == torch.float64
    big = W.abs() > 5.0 / math.sqrt(spec.n)          # |N(0, 1/n)| beyond 5 sigma: ~6e-7 of entries
    frac = big.double().mean().item()
    # outliers are a Bernoulli(0.01) mask times 10; about 62 % of them exceed the 5-sigma cut
    p, k = spec.outlier_frac, spec.m * spec.n
    expect = p * 0.617
    assert abs(frac - expect) < 6 * math.sqrt(expect * (1 - expect) / k)
    plain = W[~big]
    assert plain.std().item() == pytest.approx(1 / math.sqrt(spec.n), rel=0.05)


def test_factors_are_symmetric_positive_definite():
    spec = workload("ref128")[0]
    _, A, B = layer_inputs(spec)
    for F in (A, B):
        assert F.shape == (128, 128)
        assert torch.equal(F, F.T)
        assert torch.linalg.eigvalsh(F).min().item() > 0
    # input-side channel scales are lognormal(0, 1), output side lognormal(0, 0.5): A is the
    # more anisotropic factor
    ca = torch.linalg.cond(A).item()
    cb = torch.linalg.cond(B).item()
    assert ca > cb


def test_identity_B_workload():
    spec = workload("sq1024_onesided")[0]
    _, _, B = layer_inputs(spec, leading=64)
    assert torch.equal(B, torch.eye(64, dtype=torch.float64))


def test_leading_block_matches_full_layer():
    spec = workload("ref128")[0]
    W, A, B = layer_inputs(spec)
    Wl, Al, Bl = layer_inputs(spec, leading=40)
    assert torch.equal(Wl, W[:40, :40])
    torch.testing.assert_close(Al, A[:40, :40], rtol=1e-12, atol=1e-14)
    torch.testing.assert_close(Bl, B[:40, :40], rtol=1e-12, atol=1e-14)
