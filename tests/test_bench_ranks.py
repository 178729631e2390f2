"""The bench's multi-GPU host path, run as two `gloo` ranks on host cores (no GPU).

On N GPUs the bench runs one process per GPU; the solve does not shard, so each rank quantizes a
layer of its own and the ranks exchange nothing but two barriers and one max-reduction of their
device times. These tests drive that same plumbing (`bench.Replicas`) with the gloo backend:

  * every rank gets its own seed, rank 0's layer is the single-GPU layer, and each rank's result
    depends only on its own seed (a rank's two-sided GPTQ codes, computed by the oracle on a small
    leading block, equal those of a one-process run of that seed);
  * the job time is the slowest rank's, on every rank, and the job throughput counts the units of
    all ranks;
  * a rank that leaves before the reduction makes the other rank's collective end with an error
    instead of waiting for ever;
  * the reference arm runs on rank 0 only; the other ranks return without work.
"""
import argparse
import json
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LEAD = 16


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _leading_codes(spec):
    """Oracle codes of the leading LEAD x LEAD block of `spec`'s layer (its own leading factors)."""
    import oracle
    from synth_inputs.layers import layer_inputs
    W, A, B = layer_inputs(spec, leading=LEAD)
    W, A, B = W.numpy(), A.numpy(), B.numpy()
    UA, UB = oracle.prepare(A, 0.01), oracle.prepare(B, 0.01)
    s = oracle.row_scales(W, spec.qmax)
    return oracle.quantize_naive(W, UA, UB, s, spec.qmin, spec.qmax)["codes"].astype(int).tolist()


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _rank_main(rank, world, port, out_dir):
    _env(rank, world, port)
    import torch

    import bench
    from synth_inputs.layers import workload

    r = bench.Replicas(rank, world, "gloo", torch.device("cpu"), timeout_s=60)
    spec = r.replica_spec(workload("sq4096")[0])
    codes = _leading_codes(spec)
    r.barrier()
    ms = 10.0 + 5.0 * rank                      # this rank's (fake) device time
    ms_max = r.max_over_ranks(ms)
    units = 3 * spec.m * spec.n                 # three solves of this rank's layer
    value = r.job_throughput(units, ms_max / 1e3)
    r.barrier()
    r.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"seed": spec.seed, "m": spec.m, "n": spec.n, "ms_max": ms_max, "value": value,
                   "units": units, "codes": codes}, f)


def _leaver_main(rank, world, port, out_dir):
    """Rank 1 leaves after the first barrier; rank 0's reduction must then fail, not hang."""
    _env(rank, world, port)
    import torch

    import bench

    r = bench.Replicas(rank, world, "gloo", torch.device("cpu"), timeout_s=15)
    r.barrier()
    if rank == 1:
        os._exit(0)                             # leaves between steps, nothing in flight
    outcome = "returned"
    try:
        r.max_over_ranks(1.0)
    except Exception as e:                      # the collective ends with an error
        outcome = "error: " + type(e).__name__
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"outcome": outcome}, f)
    os._exit(0)


def _spawn(target, world, tmp_path, timeout=180):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
        p.join()
    assert not alive, "a rank did not finish"
    return [p.exitcode for p in procs]


def test_two_replicas_gloo(tmp_path):
    codes = _spawn(_rank_main, 2, tmp_path)
    assert codes == [0, 0]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]

    from synth_inputs.layers import LayerSpec, workload
    base = workload("sq4096")[0]
    # own seed per rank; rank 0 solves the single-GPU layer
    assert res[0]["seed"] == base.seed
    assert res[1]["seed"] != res[0]["seed"]
    assert all((x["m"], x["n"]) == (base.m, base.n) for x in res)
    # each rank's result is that of a one-process run of its own seed
    for x in res:
        alone = _leading_codes(LayerSpec(**{**base.__dict__, "seed": x["seed"]}))
        assert x["codes"] == alone
    assert res[0]["codes"] != res[1]["codes"]
    # job time = the slowest rank's, seen by every rank; throughput counts both ranks' units
    assert res[0]["ms_max"] == res[1]["ms_max"] == 15.0
    for x in res:
        assert x["value"] == pytest.approx(2 * x["units"] / 0.015, rel=1e-12)


def test_rank_leaving_ends_the_collective_with_an_error(tmp_path):
    codes = _spawn(_leaver_main, 2, tmp_path, timeout=120)
    assert codes == [0, 0]
    out = json.load(open(tmp_path / "rank0.json"))
    assert out["outcome"].startswith("error"), out


def test_single_rank_needs_no_process_group():
    import torch

    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    r = bench.Replicas(0, 1, "gloo", torch.device("cpu"))
    assert not dist.is_initialized()
    r.barrier()
    assert r.max_over_ranks(7.5) == 7.5
    assert r.job_throughput(100, 0.5) == 200
    r.close()


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    args = argparse.Namespace(workload="sq4096", steps=1, warmup=0, damp=0.01)
    assert bench.run_reference(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
