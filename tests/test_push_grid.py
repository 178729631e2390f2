"""Launch shapes of the fp32 trailing update (kg_push_tc.cuh: push_variant, push_grid, push_cta).

The update kernel finds its tiles with push_cta, a host-and-device function, from the grid that
push_grid gives its launch.  tests/push_cta_check.cu compiles those same functions for the host and
enumerates every CTA of every update piece of the solve's schedule (kron_gptq_schedule_plan) on
several tile grids, square, tall, wide and ragged.  Per piece it checks that each target tile of the
band is written by exactly one CTA (at most one where the tile has no source in the piece: two
read-modify-writes of one tile in one launch would race), and that the CTA's K range covers the
tile's own.  CPU only: nvcc builds a host program; no kernel runs.
"""
import os
import shutil
import subprocess

import pytest

import two_sided_gptq_02_b200 as kg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "two_sided_gptq_02_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

pytestmark = pytest.mark.skipif(not shutil.which(NVCC), reason="nvcc not found")

# tile grids (Mt x Nt, 64-row tiles): the 4096^2 layer, the 14336 x 4096 and 4096 x 14336 FFN
# layers, k/v projections, and ragged small cases with one or a few tiles on a side
SHAPES = [(64, 64), (224, 64), (64, 224), (16, 64), (64, 16), (1, 1), (1, 6), (6, 1), (2, 3), (3, 2),
          (5, 7), (7, 4), (3, 11), (13, 13), (33, 2), (2, 33), (9, 40)]


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = tmp_path_factory.mktemp("pushgrid") / "push_cta_check"
    out = subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                          "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                          os.path.join(ROOT, "tests", "push_cta_check.cu"), "-o", str(exe)],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    return str(exe)


def _run(exe, pieces, *args):
    text = "".join(f"{d0} {mid} {t0} {d1} {mt} {nt}\n" for d0, mid, t0, d1, mt, nt in pieces)
    out = subprocess.run([exe, *args], input=text, capture_output=True, text=True, timeout=600)
    return out.returncode, out.stdout.strip()


@pytest.mark.parametrize("mt,nt", SHAPES)
def test_every_target_tile_written_once(checker, mt, nt):
    ndiag = mt + nt - 1
    pieces = [(d0, mid, t0, d1, mt, nt) for d0, mid, t0, d1, _ in kg.kron_gptq_schedule_plan(ndiag)]
    # and the unsplit pushes of the recursion, push(D0 | mid | D1), each as one launch
    def split(d0, d1):
        if d1 - d0 < 2:
            return
        mid = (d0 + d1) // 2
        split(d0, mid)
        pieces.append((d0, mid, mid, d1, mt, nt))
        split(mid, d1)
    split(0, ndiag)
    rc, msg = _run(checker, pieces)
    assert rc == 0 and msg.startswith("ok"), msg
    assert int(msg.split()[1]) == len(pieces)


@pytest.mark.parametrize("piece", [(0, 31, 63, 127, 64, 64), (0, 71, 143, 287, 224, 64), (60, 63, 63, 64, 64, 64),
                                   (2, 4, 4, 6, 3, 3)])
def test_check_fails_without_a_row_of_ctas(checker, piece):
    # the same pieces pass in full, and fail once the CTAs of one grid row are left out
    assert _run(checker, [piece])[0] == 0
    rc, msg = _run(checker, [piece], "--skip-first-row")
    assert rc == 1 and "written 0 times" in msg, msg
