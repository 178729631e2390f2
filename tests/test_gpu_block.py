"""The decoder-block workload on one GPU (needs a B200).

Seven differently shaped layers of a Llama-3-8B-shaped decoder block (m x n = out x in: q and o
4096 x 4096, k and v 1024 x 4096, gate and up 14336 x 4096, down 4096 x 14336), each with its own
seeded W, A and B, quantized in fp32 with a 3-bit grid, all seven in flight at once, one CUDA
stream each.

Checked for every layer:
  * the concurrent solve equals the same layer solved alone on the default stream, bit for bit
    (codes, V and E): solves on different streams share nothing but the GPU;
  * the leading 256 x 256 block of codes agrees with the fp64 oracle on >= 99.5 % of entries -- the
    leading block depends only on the leading data and factor blocks ("FastKron: Efficient
    Quantization with Kronecker-Factored Hessians", Section 2.3), and the fp32 path takes its
    rounding decisions in fp32;
  * the certificate V - W = -U_B^T E U_A and the rounding of W~ = V + E (u_B u_A^T) hold on sampled
    rows.  In fp32 every W~_ij is a sum of up to m + n - 2 updates rounded to fp32, so the relative
    residual is held to the recursive-summation bound (m + n) u with u = 2^-24.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import layer_inputs, workload

pytestmark = pytest.mark.gpu

DAMP = 0.01


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


def test_block_concurrent_streams(kg):
    specs = workload("block")
    assert [(s.m, s.n) for s in specs] == [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096),
                                           (14336, 4096), (14336, 4096), (4096, 14336)]
    layers = []
    for spec in specs:
        W, A, B = layer_inputs(spec, device="cuda")
        _, _, UA32, UB32 = kg.kron_gptq_prepare(A, B, DAMP)
        W32 = W.float().contiguous()
        s32 = kg.kron_gptq_row_scales(W32, spec.qmax)
        layers.append((spec, W32, UA32, UB32, s32))
        del W, A, B

    # each layer alone on the default stream
    alone = []
    for spec, W32, UA32, UB32, s32 in layers:
        codes, V, E = kg.kron_gptq_quantize(W32, UA32, UB32, spec.qmin, spec.qmax, s32, want_E=True)
        alone.append((codes.cpu(), V.cpu(), E.cpu()))

    # all seven in flight at once
    qs = [kg.Quantizer(spec.m, spec.n, torch.float32, "cuda", want_E=True) for spec, *_ in layers]
    streams = [torch.cuda.Stream() for _ in layers]
    torch.cuda.synchronize()
    for q, st, (spec, W32, UA32, UB32, s32) in zip(qs, streams, layers):
        q.run(W32, UA32, UB32, s32, spec.qmin, spec.qmax, stream=st)
    torch.cuda.synchronize()

    for q, st, ref, (spec, W32, UA32, UB32, s32) in zip(qs, streams, alone, layers):
        assert q.status(st) == 0, spec.name
        assert torch.equal(q.codes.cpu(), ref[0]), spec.name
        assert torch.equal(q.V.cpu(), ref[1]), spec.name
        assert torch.equal(q.E.cpu(), ref[2]), spec.name

        W64 = W32.double().cpu().numpy()
        UA64 = UA32.double().cpu().numpy()
        UB64 = UB32.double().cpu().numpy()
        s64 = s32.double().cpu().numpy()
        codes = ref[0].numpy()
        mb, nb = min(256, spec.m), min(256, spec.n)
        o = oracle.quantize_naive(W64[:mb, :nb], UA64[:nb, :nb], UB64[:mb, :mb], s64[:mb], spec.qmin, spec.qmax)
        agree = np.mean(codes[:mb, :nb] == o["codes"])
        assert agree >= 0.995, (spec.name, agree)

        rows = np.unique(np.linspace(0, spec.m - 1, 6).astype(int))
        cert = oracle.certificate(W64, UA64, UB64, s64, spec.qmin, spec.qmax, codes, ref[1].double().numpy(),
                                  ref[2].double().numpy(), rows=rows, tol=1e-4)
        assert cert["resid_rel"] < (spec.m + spec.n) * 2.0 ** -24, (spec.name, cert)
        assert cert["code_mismatch"] <= 1e-3 * len(rows) * spec.n, (spec.name, cert)
