#!/usr/bin/env python
"""Two-sided GPTQ throughput on B200: weights/s and ms per layer, with roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload sq4096] [--dtype f32|f64]
    python bench.py --impl reference ...      # the CPU oracle on host cores (bounded sample)

One step = one kron_gptq_quantize solve (all sweep + update kernels) of one synthetic layer
whose inputs (W, U_A, U_B, scales) are already resident in HBM.  Factor preparation is
untimed, as in the pages' timings of the core solve.  With N GPUs (torchrun, one process per
GPU) each rank solves its own independently seeded layer: the solve does not shard, so the
ranks are replicas and `value` is the total weights/s over all ranks (weak scaling).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

# Every recursive solve runs on four internal streams (its leaves and three streams of update pieces);
# with the default eight hardware connections, streams of concurrent solves share queues and
# serialise.  This must be set before the process creates its CUDA context; a value in the
# environment wins.
os.environ.setdefault("CUDA_DEVICE_MAX_CONNECTIONS", "32")

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

HERE = os.path.dirname(os.path.abspath(__file__))
METRIC = "two-sided GPTQ weights/s & ms/layer (4096x4096, 3-bit) + % of roofline"
TILE = 64
# B200: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz (max SM clock)
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FP64_ALU_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
TF32_OVER_BF16_NOMINAL = 1.1 / 2.25


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sq4096")
    ap.add_argument("--dtype", choices=["f32", "f64"], default="f32")
    ap.add_argument("--damp", type=float, default=0.01)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-block", action="store_true")
    ap.add_argument("--no-waterkron", action="store_true")
    ap.add_argument("--no-onesided", action="store_true")
    ap.add_argument("--no-factors", action="store_true")
    ap.add_argument("--no-antidiagonal", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (fp64 4096x4096, fp32 14336x4096 and 4096x14336)")
    ap.add_argument("--gamma", type=float, default=0.02, help="WaterKron step knob for the scaled-alphabet line")
    return ap.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "MEASURED_PEAKS.json"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="kg_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---------------------------------------------------------------------------------------------- helpers
def _adjacent_pairs(Mt, Nt):
    """(source, target) tile pairs of the near field: a tile and its right neighbour in the row
    chain, a tile and the one below it in the column chain."""
    return Mt * (Nt - 1) + Nt * (Mt - 1)


def _push_flops(m, n, near_in_leaf=False):
    """FLOPs the trailing-update kernels perform per solve: each (source tile, target tile)
    pair of the row chain and of the column chain is one 64^3 multiply-add block.  With
    near_in_leaf (the fp32 path) the adjacent pairs are the leaves' work instead."""
    Mt, Nt = math.ceil(m / TILE), math.ceil(n / TILE)
    pairs = Mt * Nt * (Nt - 1) // 2 + Nt * Mt * (Mt - 1) // 2
    if near_in_leaf:
        pairs -= _adjacent_pairs(Mt, Nt)
    return 2.0 * TILE ** 3 * pairs


def _leaf_flops(m, n, near_in_leaf=False):
    """FLOPs of the in-tile sweeps per solve: per 64x64 tile the two in-tile chains
    (sum over entries of j resp. i multiply-adds, 64 * 2016 each) and the fold of the external
    row chain through the triangular U_B block (64 * 2080 multiply-adds); with near_in_leaf (the
    fp32 leaf) also the near field, one 64^3 multiply-add block per adjacent tile pair."""
    Mt, Nt = math.ceil(m / TILE), math.ceil(n / TILE)
    per_tile = 2 * (TILE * (TILE * (TILE - 1) // 2)) + TILE * (TILE * (TILE + 1) // 2)
    near = 2.0 * TILE ** 3 * _adjacent_pairs(Mt, Nt) if near_in_leaf else 0.0
    return 2.0 * per_tile * Mt * Nt + near


def _block_seconds(kg, torch, damp, reps=3):
    """The decoder-block workload: seven layers (q, k, v, o, gate, up, down), fp32, 3-bit,
    quantized back to back -- once on one stream, once all seven in flight on one stream each.
    Inputs are resident on the device; returns seconds per block (median of reps)."""
    from synth_inputs.layers import layer_inputs, workload
    specs = workload("block")
    layers = []
    for spec in specs:
        W, A, B = layer_inputs(spec, device="cuda")
        _, _, UA32, UB32 = kg.kron_gptq_prepare(A, B, damp)
        W32 = W.float().contiguous()
        s32 = kg.kron_gptq_row_scales(W32, spec.qmax)
        del W, A, B
        layers.append((spec, W32, UA32, UB32, s32, kg.Quantizer(spec.m, spec.n, torch.float32, "cuda")))
    streams = [torch.cuda.Stream() for _ in layers]
    main = torch.cuda.current_stream()

    def one(concurrent):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(main)
        for st, (spec, W32, UA32, UB32, s32, q) in zip(streams, layers):
            st_use = st if concurrent else main
            if concurrent:
                st.wait_event(e0)
            q.run(W32, UA32, UB32, s32, spec.qmin, spec.qmax, stream=st_use)
        if concurrent:
            for st in streams:
                main.wait_stream(st)
        e1.record(main)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3

    one(False)
    one(True)
    seq = statistics.median(one(False) for _ in range(reps))
    con = statistics.median(one(True) for _ in range(reps))
    for spec, *_, q in layers:
        if q.status() != 0:
            raise RuntimeError(f"block layer {spec.name}: status {q.status()}")
    weights = sum(spec.m * spec.n for spec, *_ in layers)
    return {"layers": [f"{spec.name} {spec.m}x{spec.n}" for spec, *_ in layers], "weights": weights,
            "dtype": "f32", "bits": 3, "seconds_per_block_one_stream": seq,
            "seconds_per_block_seven_streams": con, "weights_per_s_seven_streams": weights / con, "reps": reps,
            "note": "inputs on the device; each layer its own seeded W, A, B (N=4096 rows); median of reps"}


def _waterkron(kg, torch, spec, Wd, UAd, UBd, gamma, steps, solve_ms, roofline_ms):
    """The same layer on the WaterKron alphabet (row and column steps, unclipped int32 codes):
    device time per solve with inputs resident, the rate (entropy of Z) and the distortion against
    the high-rate value gamma^2 / 12 per entry."""
    stream = torch.cuda.current_stream()
    alpha, beta = kg.kron_gptq_waterkron_scales(UAd, UBd, gamma)
    q = kg.RcQuantizer(spec.m, spec.n, Wd.dtype, Wd.device, want_E=True)
    for _ in range(2):
        q.run(Wd, UAd, UBd, alpha, beta)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        q.run(Wd, UAd, UBd, alpha, beta)
    e1.record(stream)
    torch.cuda.synchronize()
    st = q.status()
    if st != 0:
        raise kg.KGError(st, "waterkron solve")
    ms = e0.elapsed_time(e1) / steps
    bits = kg.kron_gptq_code_entropy(q.Z)
    mse = float((q.E.double() ** 2).mean().item())
    return {"gamma": gamma, "ms_per_solve": ms, "weights_per_s": spec.m * spec.n / (ms / 1e3),
            "overhead_vs_row_scaled": ms / solve_ms - 1.0,
            "solve_roofline_frac": roofline_ms / ms,
            "entropy_bits_per_weight": bits, "max_abs_code": int(q.Z.abs().max().item()),
            "mean_E2_over_gamma2_12": mse / (gamma ** 2 / 12.0), "steps": steps,
            "note": "kron_gptq_quantize_rc with kron_gptq_waterkron_scales on the same layer and dtype; "
                    "inputs resident; the step rescaling and the V, E rescaling are inside the time"}


def _onesided(kg, torch, spec, Wd, UAd, sd, steps, solve_ms):
    """One-sided GPTQ (B = I, recursively batched updates) of the same layer, dtype and grid:
    device time per solve with inputs resident, and the two-sided / one-sided time ratio."""
    stream = torch.cuda.current_stream()
    q = kg.OnesidedQuantizer(spec.m, spec.n, Wd.dtype, Wd.device)
    for _ in range(2):
        q.run(Wd, UAd, sd, spec.qmin, spec.qmax)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        q.run(Wd, UAd, sd, spec.qmin, spec.qmax)
    e1.record(stream)
    torch.cuda.synchronize()
    st = q.status()
    if st != 0:
        raise kg.KGError(st, "one-sided solve")
    ms = e0.elapsed_time(e1) / steps
    # one pass with events around every launch: the leaves against the GEMM updates
    kg.kron_gptq_profile_read(reset=True)
    kg.kron_gptq_profile_enable(True)
    q.run(Wd, UAd, sd, spec.qmin, spec.qmax)
    torch.cuda.synchronize()
    kg.kron_gptq_profile_enable(False)
    prof = kg.kron_gptq_profile_read(reset=True)
    m, n = spec.m, spec.n
    return {"ms_per_solve": ms, "weights_per_s": m * n / (ms / 1e3), "two_sided_over_one_sided": solve_ms / ms,
            "leaf_ms": prof["leaf"][1], "leaf_launches": prof["leaf"][0], "gemm_ms": prof["push"][1],
            "gemm_launches": prof["push"][0],
            "gemm_flops": float(m) * n * n, "steps": steps,
            "note": "kron_gptq_quantize_onesided (64-column leaves + the library's own tensor-core GEMM updates: "
                    "tcgen05 3xTF32 in fp32, FP64 mma in fp64) on the same W, U_A, scales and grid; inputs resident"}


def _factors(kg, torch, spec, fp64_peak, reps=3, iters=2, N=4096):
    """FlipFlop Kronecker factors (iters alternating updates) of the layer's size from N seeded
    synthetic samples a (N x n), b (N x m), on the device in fp64.  Counted work: the DGEMMs
    (per side and iteration one N k^2 GEMM for the weights and one for the weighted Gram)."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(int(spec.seed) + 17)
    a = torch.randn(N, spec.n, generator=gen, device="cuda", dtype=torch.float64)
    b = torch.randn(N, spec.m, generator=gen, device="cuda", dtype=torch.float64)
    b *= 1.0 + 0.5 * a[:, :1].abs()
    kg.kron_gptq_factors(a, b, "flipflop", iters)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kg.kron_gptq_factors(a, b, "flipflop", iters, check=False)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    gemm_flops = iters * 2 * (2.0 * N * spec.n ** 2 + 2.0 * N * spec.m ** 2)
    return {"method": "flipflop", "iters": iters, "samples": N, "n": spec.n, "m": spec.m, "ms": ms,
            "gemm_tflops": gemm_flops / (ms / 1e3) / 1e12, "fp64_peak_tflops": fp64_peak,
            "gemm_frac": gemm_flops / (ms / 1e3) / 1e12 / fp64_peak,
            "note": "kron_gptq_factors; includes the Cholesky-based inverse factors (kron_gptq_prepare) of every "
                    "iterate, which gemm_tflops does not count; seeded synthetic samples; median of reps"}


def _antidiagonal(kg, torch, spec, W, UA, UB, reps=3):
    """The non-recursive anti-diagonal baseline (fp64, quartic) against the recursive fp64 solve on
    the same layer: device time of each (the baseline once, the recursive solve median of reps)."""
    stream = torch.cuda.current_stream()
    W64 = W.double().contiguous()
    s = kg.kron_gptq_row_scales(W64, spec.qmax)
    q = kg.Quantizer(spec.m, spec.n, torch.float64, W.device)
    q.run(W64, UA, UB, s, spec.qmin, spec.qmax)
    torch.cuda.synchronize()

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    fk = statistics.median(timed(lambda: q.run(W64, UA, UB, s, spec.qmin, spec.qmax)) for _ in range(reps))
    kg.kron_gptq_quantize_antidiagonal(W64, UA, UB, spec.qmin, spec.qmax, s, check=True)   # warm-up
    anti = timed(lambda: kg.kron_gptq_quantize_antidiagonal(W64, UA, UB, spec.qmin, spec.qmax, s, check=False))
    m, n = spec.m, spec.n
    steps = (m + 63) // 64 + (n + 63) // 64 - 1
    return {"dtype": "f64", "fastkron_ms": fk, "antidiagonal_ms": anti, "antidiagonal_over_fastkron": anti / fk,
            "antidiagonal_dense_flops": float(steps - 1) * 2.0 * m * n * (m + n),
            "note": "kron_gptq_quantize_antidiagonal (leaf per tile anti-diagonal + two dense DGEMMs over the "
                    "whole matrix) vs kron_gptq_quantize, fp64, same layer; inputs resident"}


def _prepare_flops(n, m):
    """FLOPs of kron_gptq_prepare per factor pair: a Cholesky (k^3/3) and a triangular inverse
    (k^3/3) of each k x k factor; the damping, the output copies and the fp32 rounding are O(k^2)."""
    return 2.0 / 3.0 * (float(n) ** 3 + float(m) ** 3)


def _time_prepare(kg, torch, A, B, damp, fp64_peak, reps=3):
    """kron_gptq_prepare (damping, reversed Cholesky and triangular inverse of A and B, fp64, with
    the fp32 copies the fp32 solve uses): device time, median of reps (CUDA events on the stream)."""
    stream = torch.cuda.current_stream()
    kg.kron_gptq_prepare(A, B, damp)   # warm-up, checked
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kg.kron_gptq_prepare(A, B, damp, check=False)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    fl = _prepare_flops(A.shape[0], B.shape[0])
    return {"ms": ms, "n": int(A.shape[0]), "m": int(B.shape[0]), "flops": fl, "tflops": fl / (ms / 1e3) / 1e12,
            "fp64_peak_tflops": fp64_peak, "frac_of_fp64": fl / (ms / 1e3) / 1e12 / fp64_peak,
            "note": "kron_gptq_prepare(A, B, damp) with fp32 copies, inputs resident; FLOPs 2/3 (n^3 + m^3) "
                    "(Cholesky and triangular inverse of each factor); fraction of the cuBLAS DGEMM rate "
                    "measured in this run; median of reps"}


def _config_line(kg, torch, name, dtype, damp, steps, fp64_peak, tf32_peak, hbm, cubic):
    """One more workload of the pages' shapes: the solve (device time with inputs resident, median
    over steps), its solve-roofline fraction, kron_gptq_prepare of its factors, and (cubic) the
    cubic CPU baseline on the full layer."""
    from synth_inputs.layers import layer_inputs, workload
    spec = workload(name)[0]
    dt = torch.float32 if dtype == "f32" else torch.float64
    W, A, B = layer_inputs(spec, device="cuda")
    prep = _time_prepare(kg, torch, A, B, damp, fp64_peak)
    UA, UB, UA32, UB32 = kg.kron_gptq_prepare(A, B, damp)
    del A, B
    Wd, UAd, UBd = (W.float().contiguous(), UA32, UB32) if dt == torch.float32 else (W, UA, UB)
    sd = kg.kron_gptq_row_scales(Wd, spec.qmax)
    q = kg.Quantizer(spec.m, spec.n, dt, Wd.device)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        q.run(Wd, UAd, UBd, sd, spec.qmin, spec.qmax)
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        q.run(Wd, UAd, UBd, sd, spec.qmin, spec.qmax)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    st = q.status()
    if st != 0:
        raise kg.KGError(st, f"{name} solve")
    ms = statistics.median(times)
    m, n = spec.m, spec.n
    es = 4 if dt == torch.float32 else 8
    p_tensor = tf32_peak / 3.0 if dt == torch.float32 else fp64_peak
    t_roof = max(2.0 * m * n * (m + n) / (p_tensor * 1e12), (es * (2 * m * n + n * n + m * m + m) + m * n) / (hbm * 1e9))
    out = {"workload": f"{name}: {m}x{n} (out x in), {spec.bits}-bit", "dtype": dtype, "ms_per_solve": ms,
           "weights_per_s": m * n / (ms / 1e3), "solve_roofline_ms": t_roof * 1e3,
           "solve_roofline_frac": t_roof * 1e3 / ms, "p_tensor_tflops": p_tensor, "prepare": prep,
           "prepare_plus_solve_ms": prep["ms"] + ms, "steps": steps,
           "note": "inputs resident; CUDA events around each solve, median; roofline as the headline's "
                   "(TF32/3 for fp32, DGEMM for fp64, measured in this run)"}
    if cubic:
        out["cpu_cubic"] = _cpu_cubic(spec, W, UA, UB)
    del q, Wd, UAd, UBd, W, UA, UB, UA32, UB32
    torch.cuda.empty_cache()
    return out


def _host():
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def _cpu_cubic(spec, W, UA, UB):
    """The cubic CPU baseline (oracle.quantize_cubic: the two-chain form entry by entry, OpenMP over
    each anti-diagonal's entries, all host cores) on the full layer, fp64."""
    import oracle
    Wn = W.double().cpu().numpy()
    UAn, UBn = UA.double().cpu().numpy(), UB.double().cpu().numpy()
    s = oracle.row_scales(Wn, spec.qmax)
    t0 = time.perf_counter()
    oracle.quantize_cubic(Wn, UAn, UBn, s, spec.qmin, spec.qmax)
    t = time.perf_counter() - t0
    return {"value": spec.m * spec.n / t, "unit": "weights/s", "seconds": t, "cores": oracle.cubic_threads(),
            "kind": "cubic two-chain CPU baseline (oracle.quantize_cubic)", "sample": f"the full {spec.m}x{spec.n} layer"}


def _traffic(kernel: str, units_per_launch: float):
    """DRAM bytes per launch of `kernel` from the committed ncu record (profiles/traffic.json):
    bytes per unit of work (a tile for the leaves) x the units one launch processes on average.
    None when there is no record or the kernel's source has changed since it was captured."""
    import hashlib
    path = os.path.join(HERE, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    src = os.path.join(HERE, rec["source"])
    try:
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
                return None
    except OSError:
        return None
    return rec["dram_bytes_per_unit"] * units_per_launch


def _measure_dgemm_tflops(torch, dev, dtype=None):
    """Burst rate of one 8192^3 cuBLAS GEMM (best of 5): fp64 by default; fp32 with TF32 allowed
    when dtype is torch.float32 (the TF32 tensor-core peak)."""
    n = 8192
    dtype = dtype or torch.float64
    a = torch.randn(n, n, dtype=dtype, device=dev)
    b = torch.randn(n, n, dtype=dtype, device=dev)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = dtype == torch.float32
    for _ in range(2):
        a @ b
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        a @ b
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) / 1e3)
    torch.backends.cuda.matmul.allow_tf32 = prev
    del a, b
    return 2.0 * n ** 3 / best / 1e12


def _cpu_baseline(spec, W, A, B, damp, budget_s=12.0):
    """The naive oracle (single thread, plain C) on the leading block of the same layer."""
    import numpy as np

    import oracle
    k = 320
    mb, nb = min(k, spec.m), min(k, spec.n)
    Wb = W[:mb, :nb].cpu().double().numpy()
    UA = oracle.prepare(A[:nb, :nb].cpu().double().numpy(), damp)
    UB = oracle.prepare(B[:mb, :mb].cpu().double().numpy(), damp)
    s = oracle.row_scales(Wb, spec.qmax)
    times = []
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle.quantize_naive(Wb, UA, UB, s, spec.qmin, spec.qmax)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > budget_s or len(times) >= 8:
            break
    t = statistics.median(times)
    return {"value": mb * nb / t, "unit": "weights/s", "cores": 1, "kind": "oracle",
            "sample": f"leading {mb}x{nb} block of {spec.name} (its own leading blocks of A, B), naive "
                      f"O(m^2 n^2) oracle, median of {len(times)} runs of {t:.2f} s; the full "
                      f"{spec.m}x{spec.n} layer scales by (mn)^2 (extrapolated {t * (spec.m * spec.n / (mb * nb)) ** 2:.3g} s)"}


# ---------------------------------------------------------------------------------------------- ranks
class Replicas:
    """The multi-GPU plumbing of the bench: one process per GPU, each an independent replica.

    The solve does not shard (every layer is one sequential recursion over its anti-diagonals), so
    each rank solves its own seeded layer and no data crosses between ranks. The only collectives
    are the barriers around the timed region and one max-reduction of each rank's device time, so
    that the job's time is that of its slowest rank. `backend` is "nccl" on GPUs and "gloo" for the
    same logic on host cores.
    """

    SEED_STRIDE = 7919

    def __init__(self, rank: int, world: int, backend: str = "nccl", device=None, timeout_s: float = 180.0):
        import torch
        import torch.distributed as dist
        self.rank, self.world, self.backend = rank, world, backend
        self.device = device if device is not None else torch.device("cpu")
        self._dist = dist
        if world > 1 and not dist.is_initialized():
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self) -> None:
        if self.world == 1:
            return
        if self.backend == "nccl":
            self._dist.barrier(device_ids=[self.device.index])
        else:
            self._dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def replica_spec(self, base):
        """This rank's layer: the workload's shape with a seed of its own."""
        from synth_inputs.layers import LayerSpec
        return LayerSpec(**{**base.__dict__, "seed": base.seed + self.SEED_STRIDE * self.rank})

    def job_throughput(self, units_per_rank: float, seconds_max: float) -> float:
        """Whole-job units/s: every rank's units over the slowest rank's time."""
        return self.world * units_per_rank / seconds_max

    def close(self) -> None:
        if self.world > 1 and self._dist.is_initialized():
            self._dist.destroy_process_group()


# ---------------------------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import torch  # noqa: F401

    from synth_inputs.layers import layer_inputs, workload
    spec = workload(args.workload)[0]
    W, A, B = layer_inputs(spec, device="cpu", leading=320)
    import oracle
    oracle.build()
    for _ in range(args.warmup):
        _cpu_baseline(spec, W, A, B, args.damp, budget_s=0.0)
    t0 = time.perf_counter()
    vals = []
    for _ in range(args.steps):
        vals.append(_cpu_baseline(spec, W, A, B, args.damp, budget_s=0.0))
    el = time.perf_counter() - t0
    v = statistics.median(x["value"] for x in vals)
    line = {"metric": METRIC, "value": v, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "m": spec.m, "n": spec.n, "bits": spec.bits,
                       "sample": vals[0]["sample"]},
            "cpu_baseline": {"value": v, "unit": "weights/s", "cores": 1, "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "host": _host()}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch

    import two_sided_gptq_02_b200 as kg
    from synth_inputs.layers import layer_inputs, workload

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ranks = Replicas(rank, world, "nccl", dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    spec = ranks.replica_spec(workload(args.workload)[0])
    dt = torch.float32 if args.dtype == "f32" else torch.float64
    W, A, B = layer_inputs(spec, device=dev)
    UA, UB, UA32, UB32 = kg.kron_gptq_prepare(A, B, args.damp)
    if dt == torch.float32:
        Wd, UAd, UBd = W.float().contiguous(), UA32, UB32
    else:
        Wd, UAd, UBd = W, UA, UB
    sd = kg.kron_gptq_row_scales(Wd, spec.qmax)
    q = kg.Quantizer(spec.m, spec.n, dt, dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        q.run(Wd, UAd, UBd, sd, spec.qmin, spec.qmax)
    st = q.status()
    if st != 0:
        raise kg.KGError(st, "warm-up solve")

    # ---- timed region (device time, CUDA events on the launching stream)
    kg.kron_gptq_profile_read(reset=True)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
    with ClockSampler(gpu_id) as clk:
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            q.run(Wd, UAd, UBd, sd, spec.qmin, spec.qmax)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = e0.elapsed_time(e1)
    counts = kg.kron_gptq_profile_read(reset=True)
    gpu_launches = sum(v[0] for v in counts.values())
    st = q.status()
    if st != 0:
        raise kg.KGError(st, "timed solve")
    ms_max = max_over_ranks(ms)
    clocks = clk.summary()
    weights = spec.m * spec.n
    value = ranks.job_throughput(args.steps * weights, ms_max / 1e3)
    ms_per_step = ms_max / args.steps

    # ---- per-kernel durations (separate pass with event timing of every launch)
    kg.kron_gptq_profile_enable(True)
    nprof = 3
    for _ in range(nprof):
        q.run(Wd, UAd, UBd, sd, spec.qmin, spec.qmax)
    torch.cuda.synchronize()
    prof = kg.kron_gptq_profile_read(reset=True)
    kg.kron_gptq_profile_enable(False)

    peaks, peak_src = _peaks()
    hbm = float(peaks["hbm_gbs"])
    fp64_peak = _measure_dgemm_tflops(torch, dev)
    tf32_derived = float(peaks["bf16_tflops"]) * TF32_OVER_BF16_NOMINAL
    tf32_peak = _measure_dgemm_tflops(torch, dev, torch.float32)
    es = 4 if dt == torch.float32 else 8
    m, n = spec.m, spec.n
    graded_flops = 2.0 * m * n * (m + n)
    bytes_compulsory = es * (2 * m * n + n * n + m * m + m) + m * n
    if dt == torch.float32:
        p_tensor, p_name = tf32_peak / 3.0, "TF32/3 (3xTF32): cuBLAS fp32 GEMM with TF32, 8192^3, measured in this run / 3"
    else:
        p_tensor, p_name = fp64_peak, "FP64: cuBLAS DGEMM 8192^3 measured in this run (burst)"
    t_roof = max(graded_flops / (p_tensor * 1e12), bytes_compulsory / (hbm * 1e9))
    solve = {"roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_per_step, "graded_flops": graded_flops,
             "triangular_flops": graded_flops / 2, "p_tensor_tflops": p_tensor, "p_tensor": p_name,
             "compulsory_bytes": bytes_compulsory}
    if dt == torch.float32:
        solve["frac_of_raw_tf32"] = graded_flops / (tf32_peak * 1e12) * 1e3 / ms_per_step

    # per-kernel rooflines from the profiled pass: the trailing update (a contraction on the
    # tensor cores) and the in-tile sweep (latency-bound; reported against the ALU peak of its
    # dtype, derived from unit counts); the one with the larger share of the solve is `roofline`
    pl, pms = prof["push"]
    ll, lms = prof["leaf"]
    il, ims = prof["init"]
    push_avg_s = pms / pl / 1e3
    near_in_leaf = dt == torch.float32   # the fp32 leaf computes the near field itself
    push_achieved = _push_flops(m, n, near_in_leaf) / (pl / nprof) / push_avg_s / 1e12
    leaf_avg_s = lms / ll / 1e3
    leaf_achieved = _leaf_flops(m, n, near_in_leaf) / (ll / nprof) / leaf_avg_s / 1e12
    if dt == torch.float32:
        push_rl = {"bound": "tensor", "achieved": push_achieved, "peak": tf32_peak / 3.0, "unit": "TFLOP/s",
                   "frac": push_achieved / (tf32_peak / 3.0), "traffic": None, "kernel": "k_push_tc32",
                   "peak_source": "3xTF32: cuBLAS fp32 GEMM with TF32 allowed, 8192^3, measured in this run / 3",
                   "frac_of_raw_tf32": 3.0 * push_achieved / tf32_peak}
        leaf_rl = {"bound": "alu", "achieved": leaf_achieved, "peak": FP32_SIMT_PEAK_TFLOPS, "unit": "TFLOP/s",
                   "frac": leaf_achieved / FP32_SIMT_PEAK_TFLOPS, "traffic": None, "kernel": "k_leaf_ws",
                   "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"}
    else:
        push_rl = {"bound": "tensor", "achieved": push_achieved, "peak": fp64_peak, "unit": "TFLOP/s",
                   "frac": push_achieved / fp64_peak, "traffic": None, "kernel": "k_push_f64",
                   "peak_source": "cuBLAS DGEMM 8192^3 measured in this run"}
        leaf_rl = {"bound": "alu", "achieved": leaf_achieved, "peak": FP64_ALU_PEAK_TFLOPS, "unit": "TFLOP/s",
                   "frac": leaf_achieved / FP64_ALU_PEAK_TFLOPS, "traffic": None, "kernel": "k_leaf",
                   "peak_source": "148 SMs x 64 FP64 lanes x 2 x 1.965 GHz"}
    for r_, ms_ in ((push_rl, pms), (leaf_rl, lms)):
        r_["ms_per_solve"] = ms_ / nprof
    Mt_, Nt_ = math.ceil(m / TILE), math.ceil(n / TILE)
    leaf_rl["traffic"] = _traffic(leaf_rl["kernel"], Mt_ * Nt_ / (ll / nprof))
    leaf_rl["traffic_unit"] = "DRAM bytes per launch (ncu record x tiles per launch)"
    rl, rl_other = (push_rl, leaf_rl) if pms >= lms else (leaf_rl, push_rl)
    breakdown = {"push_ms_per_solve": pms / nprof, "leaf_ms_per_solve": lms / nprof, "init_ms_per_solve": ims / nprof,
                 "push_launches_per_solve": pl // nprof, "leaf_launches_per_solve": ll // nprof,
                 "note": "separate pass with CUDA events around every launch"}
    # latency floor: one dependent entry step t_step (a leaf's time over its 2*64-1 steps, set-up
    # included), the entry-level chain (m + n - 1) t_step, and the tile-level chain the schedule
    # runs (every leaf is on the critical path)
    leaf_launch_ms = (lms / nprof) / max(1, ll // nprof)
    t_step_us = leaf_launch_ms * 1e3 / (2 * TILE - 1)
    latency = {"t_step_us": t_step_us, "entry_chain_ms": (m + n - 1) * t_step_us / 1e3,
               "tile_chain_ms": (ll // nprof) * leaf_launch_ms, "ms_per_step": ms_per_step,
               "critical_updates_ms": max(0.0, ms_per_step - (ll // nprof) * leaf_launch_ms),
               "note": "entry_chain_ms: (m+n-1) dependent steps at the leaf's measured step time, the floor of "
                       "a schedule that overlaps consecutive tile anti-diagonals; tile_chain_ms: the leaves "
                       "alone; the rest of ms_per_step is the critical-stream update work"}

    # ---- end to end: host buffers through the same public call
    e2e = None
    if not args.no_e2e:
        # A user pipeline with host buffers through the public call: every step copies its inputs
        # (W, U_A, U_B, scales) host -> device from pinned memory, solves, and copies its codes
        # device -> host; step k+1's inputs travel while step k solves (two device input sets, one
        # stream per copy direction), and step k's codes travel while step k+1 solves.
        hW = Wd.cpu().pin_memory()
        hUA, hUB, hs = UAd.cpu().pin_memory(), UBd.cpu().pin_memory(), sd.cpu().pin_memory()
        nb = 2
        bufs = [(torch.empty_like(Wd), torch.empty_like(UAd), torch.empty_like(UBd), torch.empty_like(sd))
                for _ in range(nb)]
        qs = [kg.Quantizer(m, n, dt, dev) for _ in range(nb)]
        hcodes = [torch.empty(m, n, dtype=torch.int8).pin_memory() for _ in range(nb)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]      # inputs of set b on the device
        ev_used = [torch.cuda.Event() for _ in range(nb)]    # solve on set b finished (inputs free)
        ev_out = [torch.cuda.Event() for _ in range(nb)]     # codes of set b on the host
        for b in range(nb):
            ev_used[b].record(stream)
            ev_out[b].record(stream)
        ke = max(2, min(args.steps, 6))

        def e2e_step(k):
            b = k % nb
            dW_, dUA_, dUB_, ds_ = bufs[b]
            h2d.wait_event(ev_used[b])
            with torch.cuda.stream(h2d):
                dW_.copy_(hW, non_blocking=True)
                dUA_.copy_(hUA, non_blocking=True)
                dUB_.copy_(hUB, non_blocking=True)
                ds_.copy_(hs, non_blocking=True)
            ev_in[b].record(h2d)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])          # set b's previous codes have left the device
            qs[b].run(dW_, dUA_, dUB_, ds_, spec.qmin, spec.qmax, stream=stream)
            ev_used[b].record(stream)
            d2h.wait_event(ev_used[b])
            with torch.cuda.stream(d2h):
                hcodes[b].copy_(qs[b].codes, non_blocking=True)
            ev_out[b].record(d2h)

        # warm-up: twice per input set, so that the library's capture of each set's solve into a CUDA
        # graph (on the second call with the same arguments) happens before the timed region
        for k in range(2 * nb):
            e2e_step(k)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        h2d.wait_event(f0)
        for k in range(ke):
            e2e_step(k)
        for b in range(nb):
            stream.wait_event(ev_out[b])
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        for q_ in qs:
            if q_.status() != 0:
                raise RuntimeError(f"e2e solve status {q_.status()}")
        t_e2e = max_over_ranks(f0.elapsed_time(f1))
        e2e = {"value": ranks.job_throughput(ke * weights, t_e2e / 1e3), "unit": "weights/s",
               "h2d_bytes_per_step": int(hW.numel() * es + hUA.numel() * es + hUB.numel() * es + hs.numel() * es),
               "d2h_bytes_per_step": int(m * n), "ms_per_step": t_e2e / ke, "steps": ke,
               "note": "pipelined: step k+1's host-to-device copies overlap step k's solve; every step's "
                       "copies are inside the timed region"}

    block = None
    if rank == 0 and world == 1 and not args.no_block:
        block = _block_seconds(kg, torch, args.damp)

    waterkron = None
    if rank == 0 and world == 1 and not args.no_waterkron:
        waterkron = _waterkron(kg, torch, spec, Wd, UAd, UBd, args.gamma, max(3, min(args.steps, 10)), ms_per_step,
                               solve["roofline_ms"])

    onesided = None
    if rank == 0 and world == 1 and not args.no_onesided:
        onesided = _onesided(kg, torch, spec, Wd, UAd, sd, max(3, min(args.steps, 10)), ms_per_step)

    fac = None
    if rank == 0 and world == 1 and not args.no_factors:
        fac = _factors(kg, torch, spec, fp64_peak)

    anti = None
    if rank == 0 and world == 1 and not args.no_antidiagonal:
        anti = _antidiagonal(kg, torch, spec, W, UA, UB)

    cpu = None
    cubic = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _cpu_baseline(spec, W, A, B, args.damp)
        cubic = _cpu_cubic(spec, W, UA, UB)

    prep = None
    configs = None
    if rank == 0 and world == 1:
        prep = _time_prepare(kg, torch, A, B, args.damp, fp64_peak)
        prep["prepare_plus_solve_ms"] = prep["ms"] + ms_per_step
        if not args.no_configs:
            del W, A, B, UA, UB
            torch.cuda.empty_cache()
            other = [("sq4096", "f64"), ("ffn_up", "f32"), ("ffn_down", "f32")]
            if args.workload != "sq4096" or args.dtype != "f32":
                other = [("sq4096", "f32")] + [c for c in other if c != (args.workload, args.dtype)]
            configs = [_config_line(kg, torch, nm, dt_, args.damp, max(3, min(args.steps, 10)), fp64_peak, tf32_peak,
                                    hbm, cubic=not args.no_cpu_baseline and nm != "sq4096")
                       for nm, dt_ in other if (nm, dt_) != (args.workload, args.dtype)]

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
                "config": {"workload": f"{args.workload}: {m}x{n} (out x in), {spec.bits}-bit grid "
                                       f"[{spec.qmin},{spec.qmax}], per-row scale, damp {args.damp}",
                           "m": m, "n": n, "bits": spec.bits, "solve_dtype": args.dtype,
                           "parallelism": f"replicas x{world} (independent layers, no collective)",
                           "l2": "inputs larger than L2 (W, U_A, U_B and a 3-buffer workspace: "
                                 f"{(bytes_compulsory + 3 * m * n * es) / 1e6:.0f} MB)"},
                "roofline": rl, "roofline_other": rl_other, "solve_roofline": solve, "kernel_breakdown": breakdown,
                "latency_floor": latency,
                "clocks": clocks, "gpu_launches": int(gpu_launches), "e2e": e2e, "cpu_baseline": cpu,
                "block": block, "waterkron": waterkron, "onesided": onesided, "factors": fac,
                "antidiagonal": anti, "cpu_cubic": cubic, "prepare": prep, "configs": configs, "host": _host(),
                "peaks": {"hbm_gbs": hbm, "fp64_tflops_measured": fp64_peak, "tf32_tflops_measured": tf32_peak,
                          "tf32_tflops_derived": tf32_derived,
                          "source": peak_src}}
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def main():
    args = _args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
