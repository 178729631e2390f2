"""A solve captured into a CUDA graph and replayed (needs a B200).

The recursive solve forks its work from the caller's stream onto four internal streams (the leaves
and three streams of update pieces) and joins them back, all by events, so it can be captured like
any other stream work. Replayed, the graph must compute exactly what a direct call computes on the
same inputs -- the same kernels in the same order on the same data, and no two concurrent pieces
ever write the same tile -- including after the input W has changed in place between capture and
replay.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs.layers import small_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kg():
    from two_sided_gptq_02_b200.build import build
    build()
    import two_sided_gptq_02_b200 as kg
    kg.load_library()
    return kg


@pytest.mark.parametrize("dtype,m,n", [(torch.float32, 768, 640), (torch.float64, 320, 448)])
def test_graph_replay_matches_direct_solve(kg, dtype, m, n):
    spec, (W, A, B) = small_layer(m, n, 23, bits=3)
    npd = np.float64 if dtype == torch.float64 else np.float32
    UA = torch.from_numpy(oracle.prepare_lapack(A.numpy(), 0.01).astype(npd)).cuda()
    UB = torch.from_numpy(oracle.prepare_lapack(B.numpy(), 0.01).astype(npd)).cuda()
    Wd = torch.from_numpy(W.numpy().astype(npd)).cuda()
    sd = kg.kron_gptq_row_scales(Wd, spec.qmax)
    q = kg.Quantizer(m, n, dtype, Wd.device, want_E=True)
    # the first call creates the library's per-thread streams and events and sets kernel attributes:
    # it belongs before any capture
    q.run(Wd, UA, UB, sd, spec.qmin, spec.qmax)
    assert q.status() == 0
    codes_before = q.codes.clone()

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g):
            q.run(Wd, UA, UB, sd, spec.qmin, spec.qmax)
    torch.cuda.synchronize()

    # change W in place (and its scales with it): the replay must read the new values
    gen = torch.Generator(device="cpu").manual_seed(5)
    Wd.copy_(Wd * (1.0 + 0.05 * torch.randn(m, n, generator=gen, dtype=torch.float64).to(dtype).cuda()))
    sd.copy_(kg.kron_gptq_row_scales(Wd, spec.qmax))
    q.codes.fill_(99)
    q.V.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert q.status() == 0
    got = (q.codes.clone(), q.V.clone(), q.E.clone())

    ref_codes, ref_V, ref_E = kg.kron_gptq_quantize(Wd, UA, UB, spec.qmin, spec.qmax, sd, want_E=True)
    assert torch.equal(got[0], ref_codes)
    assert torch.equal(got[1], ref_V)
    assert torch.equal(got[2], ref_E)
    # and the replay solved the new W, not the one present at capture
    assert not torch.equal(got[0], codes_before)
