"""The optional build of the fp32 solve with paired tile anti-diagonals (kg_leaf_pair.cuh, switched
on by KG_EXPERIMENTAL_PAIR, with KG_PAIR_TIMELINE for its per-CTA timestamps) must keep compiling
for sm_100a without register spills, and must leave the default translation unit untouched.
CPU only: nvcc cross-compiles; nothing runs."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "two_sided_gptq_02_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]

pytestmark = pytest.mark.skipif(not shutil.which(NVCC), reason="nvcc not found")


@pytest.mark.parametrize("defines", [["-DKG_EXPERIMENTAL_PAIR"], ["-DKG_EXPERIMENTAL_PAIR", "-DKG_PAIR_TIMELINE"]])
def test_paired_leaf_variant_compiles_without_spills(tmp_path, defines):
    out = subprocess.run([NVCC, *FLAGS, *defines, "-Xptxas", "-v", "-c", os.path.join(CSRC, "kg_quantize.cu"),
                          "-o", str(tmp_path / "kq.o")], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    log = out.stderr.splitlines()
    at = [k for k, line in enumerate(log) if "Compiling entry function" in line and "k_leaf_pair" in line]
    assert len(at) == 1, "the paired leaf kernel is compiled once"
    info = " ".join(log[at[0] + 1: at[0] + 4])
    assert re.search(r"0 bytes spill stores, 0 bytes spill loads", info), info
    regs = int(re.search(r"Used (\d+) registers", info).group(1))
    assert regs * 608 <= 65536, regs        # one CTA of 608 threads fits the register file


def test_default_build_does_not_contain_the_paired_leaf(tmp_path):
    out = subprocess.run([NVCC, *FLAGS, "-E", os.path.join(CSRC, "kg_quantize.cu")], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "k_leaf_pair" not in out.stdout and "kron_gptq_debug_pair_timeline" not in out.stdout


def test_variant_library_builds_apart_and_loads(tmp_path):
    """build.py --define/--out: a variant library of its own, loadable on the host, exporting the
    timeline reader, while the default library keeps its own objects."""
    import ctypes
    import subprocess
    import sys
    out = tmp_path / "libkrongptq_pair.so"
    r = subprocess.run([sys.executable, "-m", "two_sided_gptq_02_b200.build", "--define", "KG_EXPERIMENTAL_PAIR",
                        "--define", "KG_PAIR_TIMELINE", "--out", str(out)], cwd=ROOT, capture_output=True,
                       text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-3000:]
    assert out.exists() and (tmp_path / "libkrongptq_pair_objs" / "flags.txt").read_text().endswith(
        "-DKG_EXPERIMENTAL_PAIR -DKG_PAIR_TIMELINE")
    lib = ctypes.CDLL(str(out))
    assert lib.kron_gptq_version() > 0
    assert hasattr(lib, "kron_gptq_debug_pair_timeline")
    default = ctypes.CDLL(os.path.join(ROOT, "two_sided_gptq_02_b200", "libkrongptq.so"))
    assert not hasattr(default, "kron_gptq_debug_pair_timeline")
