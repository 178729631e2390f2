"""A bounded device wait that runs out (needs a B200).

Every inter-warp wait in the fp32 leaf is bounded in time; when one runs out the leaf records
KG_ERR_TIMEOUT in the call's status word and returns, and the CUDA context stays usable.  The test
build KG_TEST_HANDOFF_FAULT (a library of its own, built here) has a device switch that makes the
helpers of one row withhold one arrival in the first leaf's hand-off ring, so that the rounding
warp's wait on that slot runs out (its limit is ~2 ms in that build).  Nothing faults or traps.

A child process loads the test library and checks, on one context: a normal solve succeeds; with
the switch on the solve returns KG_ERR_TIMEOUT, well within a second; with the switch off again the
next solve succeeds and gives the same codes as the first.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import ctypes, json, time
import numpy as np, torch
import two_sided_gptq_02_b200 as kg
from synth_inputs.layers import small_layer
import oracle
lib = kg.load_library()
spec, (W, A, B) = small_layer(192, 192, 21, bits=3)
UA = oracle.prepare_lapack(A.numpy(), 0.01); UB = oracle.prepare_lapack(B.numpy(), 0.01)
Wt = W.float().cuda(); UAt = torch.from_numpy(UA.astype(np.float32)).cuda(); UBt = torch.from_numpy(UB.astype(np.float32)).cuda()
s = kg.kron_gptq_row_scales(Wt, spec.qmax)
q = kg.Quantizer(192, 192, torch.float32, "cuda")
def solve():
    t0 = time.perf_counter()
    q.run(Wt, UAt, UBt, s, spec.qmin, spec.qmax)
    st = q.status()
    return st, time.perf_counter() - t0, q.codes.clone()
out = {}
out["first"], _, c0 = solve()
assert lib.kron_gptq_debug_handoff_fault(1) == 0
out["faulted"], out["faulted_s"], _ = solve()
assert lib.kron_gptq_debug_handoff_fault(0) == 0
out["after"], _, c1 = solve()
out["same_codes"] = bool(torch.equal(c0, c1))
print("RESULT " + json.dumps(out))
'''


def test_leaf_wait_times_out_and_context_stays_usable(tmp_path):
    lib = tmp_path / "libkrongptq_fault.so"
    r = subprocess.run([sys.executable, "-m", "two_sided_gptq_02_b200.build", "--define", "KG_TEST_HANDOFF_FAULT",
                        "--out", str(lib)], cwd=ROOT, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-3000:]
    env = dict(os.environ, KRON_GPTQ_LIB=str(lib), PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-3000:])
    res = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1][7:])
    assert res["first"] == 0, res
    assert res["faulted"] == -7, res          # KG_ERR_TIMEOUT
    assert res["faulted_s"] < 1.0, res
    assert res["after"] == 0 and res["same_codes"], res
