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


@pytest.mark.parametrize("dtype,m,n", [(torch.float32, 640, 768), (torch.float32, 200, 330),
                                       (torch.float64, 448, 320)])
def test_repeated_calls_replay_the_same_solve(kg, dtype, m, n):
    """kron_gptq_quantize (fp32) captures the second call with the same arguments into a graph and
    replays it from the third on; fp64 always runs directly.  Every call must give what a first call on fresh buffers gives (always run
    directly), with W changed in place between calls, and the launch counters must grow by the same
    amount per call whichever way it ran."""
    spec, (W, A, B) = small_layer(m, n, 29, bits=3)
    npd = np.float64 if dtype == torch.float64 else np.float32
    UA = torch.from_numpy(oracle.prepare_lapack(A.numpy(), 0.01).astype(npd)).cuda()
    UB = torch.from_numpy(oracle.prepare_lapack(B.numpy(), 0.01).astype(npd)).cuda()
    Wd = torch.from_numpy(W.numpy().astype(npd)).cuda()
    sd = kg.kron_gptq_row_scales(Wd, spec.qmax)
    q = kg.Quantizer(m, n, dtype, Wd.device, want_E=True)
    gen = torch.Generator(device="cpu").manual_seed(11)
    per_call = []
    for call in range(4):
        if call >= 2:   # a new W under the same pointer
            Wd.mul_(1.0 + 0.05 * torch.randn(m, n, generator=gen, dtype=torch.float64).to(dtype).cuda())
            sd.copy_(kg.kron_gptq_row_scales(Wd, spec.qmax))
        kg.kron_gptq_profile_read(reset=True)
        q.codes.fill_(99)
        q.run(Wd, UA, UB, sd, spec.qmin, spec.qmax)
        torch.cuda.synchronize()
        counts = kg.kron_gptq_profile_read(reset=True)
        per_call.append(sum(v[0] for v in counts.values()))
        assert q.status() == 0
        fresh = kg.Quantizer(m, n, dtype, Wd.device, want_E=True)   # new buffers: a first call, direct
        fresh.run(Wd, UA, UB, sd, spec.qmin, spec.qmax)
        assert fresh.status() == 0
        assert torch.equal(q.codes, fresh.codes), f"call {call}"
        assert torch.equal(q.V, fresh.V), f"call {call}"
        assert torch.equal(q.E, fresh.E), f"call {call}"
    assert len(set(per_call)) == 1 and per_call[0] > 0, per_call


def test_repeated_rc_calls_replay_the_same_solve(kg):
    """The scaled-alphabet call (kron_gptq_quantize_rc) is replayed the same way: every call equals
    a first call on fresh buffers, with W changed in place between calls."""
    m, n = 384, 512
    spec, (W, A, B) = small_layer(m, n, 31, bits=3)
    UA = torch.from_numpy(oracle.prepare_lapack(A.numpy(), 0.01).astype(np.float32)).cuda()
    UB = torch.from_numpy(oracle.prepare_lapack(B.numpy(), 0.01).astype(np.float32)).cuda()
    Wd = torch.from_numpy(W.numpy().astype(np.float32)).cuda()
    alpha, beta = kg.kron_gptq_waterkron_scales(UA, UB, 0.05)
    q = kg.RcQuantizer(m, n, torch.float32, Wd.device, want_E=True)
    gen = torch.Generator(device="cpu").manual_seed(13)
    for call in range(4):
        if call >= 2:
            Wd.mul_(1.0 + 0.05 * torch.randn(m, n, generator=gen).cuda())
        q.Z.fill_(12345)
        q.run(Wd, UA, UB, alpha, beta)
        assert q.status() == 0
        fresh = kg.RcQuantizer(m, n, torch.float32, Wd.device, want_E=True)
        fresh.run(Wd, UA, UB, alpha, beta)
        assert fresh.status() == 0
        assert torch.equal(q.Z, fresh.Z), f"call {call}"
        assert torch.equal(q.V, fresh.V), f"call {call}"
        assert torch.equal(q.E, fresh.E), f"call {call}"
