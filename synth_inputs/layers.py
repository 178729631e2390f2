"""Seeded synthetic layer generator (W, A, B) and the named workloads.

Recipe, per layer (all draws in float64 from one torch CPU generator, in this order):

* ``W``   : m x n, entries N(0, 1/n); a Bernoulli(``outlier_frac``) mask of entries is
            multiplied by ``outlier_mult`` (10).
* ``Z_A`` : N x n standard normal;  ``M_A`` = diag(s_A) + 0.1 * N(0,1)/sqrt(n), n x n;
  ``s_A`` : lognormal(0, ``sigma_in``) channel scales.  X = Z_A M_A,  A = X^T X / N.
* ``Z_B``, ``M_B``, ``s_B`` : the same for the output side with m and ``sigma_out``;
            G = Z_B M_B,  B = G^T G / N.

A and B are returned undamped; damping is part of the method and happens in
``kron_gptq_prepare`` (and in the oracle's own prepare).  The random draws are made on
the CPU so that they are identical on every machine; the two Gram products may run on
``device`` (a CUDA device for the large layers, where a CPU product takes minutes).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    m: int              # output channels (rows of W)
    n: int              # input channels (columns of W)
    seed: int
    n_samples: int      # N rows of synthetic activations / gradients
    outlier_frac: float
    sigma_in: float = 1.0
    sigma_out: float = 0.5
    bits: int = 3
    identity_B: bool = False   # replace B by I_m (the one-sided special case)

    @property
    def qmin(self) -> int:
        return -(1 << (self.bits - 1))

    @property
    def qmax(self) -> int:
        return (1 << (self.bits - 1)) - 1


def _spec(name, m, n, seed, N, frac, bits, **kw):
    return LayerSpec(name=name, m=m, n=n, seed=seed, n_samples=N, outlier_frac=frac, bits=bits, **kw)


# Named workloads.  Sizes are the Llama-3-8B-class shapes (m = out, n = in).
WORKLOADS: dict[str, list[LayerSpec]] = {
    # small reference layer: the naive oracle finishes in seconds
    "ref128": [_spec("ref128", 128, 128, 0, 512, 0.01, 4)],
    "sq1024": [_spec("sq1024", 1024, 1024, 1000, 2048, 0.01, 3)],
    "sq1024_onesided": [_spec("sq1024_onesided", 1024, 1024, 1000, 2048, 0.01, 3, identity_B=True)],
    # attention q/o projection shape; the headline workload uses the 3-bit grid
    "sq4096": [_spec("sq4096", 4096, 4096, 2000, 4096, 0.005, 3)],
    "sq4096_2bit": [_spec("sq4096_2bit", 4096, 4096, 2000, 4096, 0.005, 2)],
    "sq4096_4bit": [_spec("sq4096_4bit", 4096, 4096, 2000, 4096, 0.005, 4)],
    # FFN shapes: up/gate (m > n) and down (n > m)
    "ffn_up": [_spec("ffn_up", 14336, 4096, 3000, 4096, 0.005, 3)],
    "ffn_down": [_spec("ffn_down", 4096, 14336, 3001, 4096, 0.005, 3)],
    # one decoder block, quantized back to back
    "block": [
        _spec("q_proj", 4096, 4096, 4000, 4096, 0.005, 3),
        _spec("k_proj", 1024, 4096, 4001, 4096, 0.005, 3),
        _spec("v_proj", 1024, 4096, 4002, 4096, 0.005, 3),
        _spec("o_proj", 4096, 4096, 4003, 4096, 0.005, 3),
        _spec("gate_proj", 14336, 4096, 4004, 4096, 0.005, 3),
        _spec("up_proj", 14336, 4096, 4005, 4096, 0.005, 3),
        _spec("down_proj", 4096, 14336, 4006, 4096, 0.005, 3),
    ],
}


def workload(name: str) -> list[LayerSpec]:
    return WORKLOADS[name]


def _gram(gen: torch.Generator, k: int, N: int, sigma: float, device, lead: int | None = None) -> torch.Tensor:
    Z = torch.randn(N, k, generator=gen, dtype=torch.float64)
    Mn = torch.randn(k, k, generator=gen, dtype=torch.float64)
    s = torch.exp(sigma * torch.randn(k, generator=gen, dtype=torch.float64))
    Mm = Mn.mul_(0.1 / math.sqrt(k))
    Mm.diagonal().add_(s)
    if lead is not None:
        Mm = Mm[:, :lead]          # the leading block of X^T X needs only these columns of X
    X = Z.to(device) @ Mm.to(device)
    del Z, Mm
    G = X.T @ X
    G.div_(N)
    return 0.5 * (G + G.T)   # exact symmetry


def layer_inputs(spec: LayerSpec, device="cpu", *, with_factors: bool = True, leading: int | None = None):
    """Return (W, A, B) as float64 tensors on ``device`` (A: n x n, B: m x m).

    ``leading=k`` returns only W[:k,:k], A[:k,:k], B[:k,:k] -- the same values as the full
    layer's leading blocks (same draws), without forming the full Gram products.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(spec.seed))
    W = torch.randn(spec.m, spec.n, generator=gen, dtype=torch.float64) / math.sqrt(spec.n)
    mask = torch.rand(spec.m, spec.n, generator=gen, dtype=torch.float64) < spec.outlier_frac
    W = torch.where(mask, W * 10.0, W)
    if leading is not None:
        W = W[:leading, :leading].contiguous()
    W = W.to(device)
    if not with_factors:
        return W, None, None
    la = None if leading is None else min(leading, spec.n)
    lb = None if leading is None else min(leading, spec.m)
    A = _gram(gen, spec.n, spec.n_samples, spec.sigma_in, device, la)
    if spec.identity_B:
        B = torch.eye(spec.m if lb is None else lb, dtype=torch.float64, device=device)
    else:
        B = _gram(gen, spec.m, spec.n_samples, spec.sigma_out, device, lb)
    return W, A, B


def small_layer(m: int, n: int, seed: int, *, N: int | None = None, outlier_frac: float = 0.01,
                sigma_in: float = 1.0, sigma_out: float = 0.5, bits: int = 4):
    """Ad-hoc small layer (tests, edge cases) with the same recipe."""
    spec = LayerSpec(name=f"small{m}x{n}", m=m, n=n, seed=seed, n_samples=N or max(4 * max(m, n), 16),
                     outlier_frac=outlier_frac, sigma_in=sigma_in, sigma_out=sigma_out, bits=bits)
    return spec, layer_inputs(spec)
