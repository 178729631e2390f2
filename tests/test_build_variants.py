"""The test build with a withheld leaf hand-off (KG_TEST_HANDOFF_FAULT, used by
tests/test_gpu_timeout.py to make a bounded device wait run out) must keep compiling for sm_100a
without register spills, must leave the default translation unit untouched, and must build into a
library of its own.  CPU only: nvcc cross-compiles; nothing runs."""
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "two_sided_gptq_02_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]

pytestmark = pytest.mark.skipif(not shutil.which(NVCC), reason="nvcc not found")


def test_handoff_fault_variant_compiles_without_spills(tmp_path):
    out = subprocess.run([NVCC, *FLAGS, "-DKG_TEST_HANDOFF_FAULT", "-Xptxas", "-v", "-c",
                          os.path.join(CSRC, "kg_quantize.cu"), "-o", str(tmp_path / "kq.o")],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    log = out.stderr.splitlines()
    at = [k for k, line in enumerate(log) if "Compiling entry function" in line and "k_leaf_ws" in line]
    assert len(at) == 1, "the fp32 leaf is compiled once"
    info = " ".join(log[at[0] + 1: at[0] + 4])
    assert re.search(r"0 bytes spill stores, 0 bytes spill loads", info), info


def test_default_build_does_not_contain_the_test_hook():
    out = subprocess.run([NVCC, *FLAGS, "-E", os.path.join(CSRC, "kg_quantize.cu")], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "g_test_handoff_fault" not in out.stdout and "kron_gptq_debug_handoff_fault" not in out.stdout


def test_variant_library_builds_apart_and_loads(tmp_path):
    """build.py --define/--out: a variant library of its own, loadable on the host, exporting the
    test switch, while the default library keeps its own objects and does not export it."""
    import ctypes
    out = tmp_path / "libkrongptq_fault.so"
    r = subprocess.run([sys.executable, "-m", "two_sided_gptq_02_b200.build", "--define", "KG_TEST_HANDOFF_FAULT",
                        "--out", str(out)], cwd=ROOT, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-3000:]
    assert out.exists() and (tmp_path / "libkrongptq_fault_objs" / "flags.txt").read_text().endswith(
        "-DKG_TEST_HANDOFF_FAULT")
    lib = ctypes.CDLL(str(out))
    assert lib.kron_gptq_version() > 0
    assert hasattr(lib, "kron_gptq_debug_handoff_fault")
    default = ctypes.CDLL(os.path.join(ROOT, "two_sided_gptq_02_b200", "libkrongptq.so"))
    assert not hasattr(default, "kron_gptq_debug_handoff_fault")
