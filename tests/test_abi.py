"""The C-ABI library loads and exports every symbol include/*.h declares (CPU only: no
compute calls, only host-side argument validation that returns before any CUDA call)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"KG_API\s+[\w\s\*]+?\b(kron_gptq_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from two_sided_gptq_02_b200.build import build
    build()
    from two_sided_gptq_02_b200 import load_library
    return load_library()


def test_header_declares_the_api():
    names = _declared()
    for required in ("kron_gptq_prepare", "kron_gptq_quantize", "kron_gptq_loss"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    path = lib._name
    raw = ctypes.CDLL(path)
    missing = [n for n in _declared() if not hasattr(raw, n)]
    assert not missing, missing


def test_library_exports_only_declared_entry_points(lib):
    """No undeclared kron_gptq_* symbol (a debug entry point of a variant build) in the default
    library."""
    import shutil
    import subprocess
    if not shutil.which("nm"):
        pytest.skip("nm not found")
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True, check=True)
    exported = {ln.split()[-1] for ln in out.stdout.splitlines() if ln.split() and ln.split()[-1].startswith("kron_gptq_")}
    assert exported == set(_declared()), sorted(exported ^ set(_declared()))


def test_version_and_status_strings(lib):
    assert lib.kron_gptq_version() >= 10000
    for code in range(0, -9, -1):
        s = lib.kron_gptq_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.kron_gptq_status_string(-99).decode() == "unknown status"


def test_workspace_sizes(lib):
    s32 = lib.kron_gptq_quantize_workspace_size(4096, 4096, 1)
    s64 = lib.kron_gptq_quantize_workspace_size(4096, 4096, 2)
    assert s32 >= 3 * 4096 * 4096 * 4 and s64 >= 3 * 4096 * 4096 * 8
    # ragged shapes need room for the identity-padded factors
    assert lib.kron_gptq_quantize_workspace_size(100, 70, 2) >= 3 * 128 * 128 * 8 + 128 * 128 * 8 + 128 * 128 * 8
    assert lib.kron_gptq_quantize_workspace_size(0, 5, 1) == 256
    assert lib.kron_gptq_quantize_workspace_size(5, 5, 7) == 0
    assert lib.kron_gptq_prepare_workspace_size(100) >= 2 * 128 * 128 * 8
    assert lib.kron_gptq_loss_workspace_size(100, 100) >= 256


def test_host_side_argument_errors(lib):
    from two_sided_gptq_02_b200._lib import _Grid
    P = ctypes.c_void_p
    fake = P(256 * 1000)          # never dereferenced: validation fails first
    g = _Grid(-4, 3, fake)
    # unsupported dtype
    assert lib.kron_gptq_quantize(fake, 8, 8, 7, fake, fake, g, fake, fake, None, fake, 1 << 20, None) == -2
    # negative size
    assert lib.kron_gptq_quantize(fake, -1, 8, 1, fake, fake, g, fake, fake, None, fake, 1 << 20, None) == -1
    # unaligned / null workspace
    assert lib.kron_gptq_quantize(fake, 8, 8, 1, fake, fake, g, fake, fake, None, P(257), 1 << 20, None) == -1
    assert lib.kron_gptq_quantize(fake, 8, 8, 1, fake, fake, g, fake, fake, None, None, 1 << 20, None) == -1
    # grid must straddle zero inside int8
    assert lib.kron_gptq_quantize(fake, 8, 8, 1, fake, fake, _Grid(0, 3, fake), fake, fake, None, fake, 1 << 20,
                                  None) == -2
    assert lib.kron_gptq_quantize(fake, 8, 8, 1, fake, fake, _Grid(-4, 200, fake), fake, fake, None, fake, 1 << 20,
                                  None) == -2
    # null operand
    assert lib.kron_gptq_quantize(None, 8, 8, 1, fake, fake, g, fake, fake, None, fake, 1 << 20, None) == -1
    # workspace too small
    assert lib.kron_gptq_quantize(fake, 64, 64, 1, fake, fake, g, fake, fake, None, fake, 1024, None) == -4
    # prepare: bad damping, missing output, small workspace
    assert lib.kron_gptq_prepare(fake, 8, None, 0, 2, -1.0, fake, None, None, None, fake, 1 << 20, None) == -1
    assert lib.kron_gptq_prepare(fake, 8, None, 0, 2, 0.01, None, None, None, None, fake, 1 << 20, None) == -1
    assert lib.kron_gptq_prepare(fake, 64, None, 0, 2, 0.01, fake, None, None, None, fake, 1024, None) == -4
    assert lib.kron_gptq_prepare(fake, 8, None, 0, 9, 0.01, fake, None, None, None, fake, 1 << 20, None) == -2
    # loss
    assert lib.kron_gptq_loss(fake, fake, 0, 4, 1, fake, fake, 1, 0.0, fake, fake, 1 << 20, None) == -1
    assert lib.kron_gptq_loss(fake, fake, 4, 4, 1, fake, fake, 1, 0.0, fake, fake, 8, None) == -4
    assert lib.kron_gptq_row_scales(fake, 4, 4, 1, 0, fake, None) == -1
    assert lib.kron_gptq_sync_status(None, None) == -1


def test_host_side_argument_errors_of_the_next_rows(lib):
    from two_sided_gptq_02_b200._lib import _Grid
    P = ctypes.c_void_p
    fake = P(256 * 1000)
    big = 1 << 40
    g = _Grid(-4, 3, fake)
    # scaled alphabet: dtype, sizes, workspace alignment, null steps, small workspace
    rc = lib.kron_gptq_quantize_rc
    assert rc(fake, 8, 8, 5, fake, fake, fake, fake, fake, fake, None, fake, big, None) == -2
    assert rc(fake, -1, 8, 1, fake, fake, fake, fake, fake, fake, None, fake, big, None) == -1
    assert rc(fake, 8, 8, 1, fake, fake, fake, fake, fake, fake, None, P(300), big, None) == -1
    assert rc(fake, 8, 8, 1, fake, fake, None, fake, fake, fake, None, fake, big, None) == -1
    assert rc(fake, 64, 64, 1, fake, fake, fake, fake, fake, fake, None, fake, 4096, None) == -4
    assert lib.kron_gptq_quantize_rc_workspace_size(64, 64, 1) > lib.kron_gptq_quantize_workspace_size(64, 64, 1)
    assert lib.kron_gptq_waterkron_scales(fake, 8, fake, 8, 1, -1.0, fake, fake, None) == -1
    assert lib.kron_gptq_waterkron_scales(fake, 8, fake, 8, 1, float("nan"), fake, fake, None) == -1
    assert lib.kron_gptq_waterkron_scales(fake, 8, fake, 8, 3, 0.1, fake, fake, None) == -2
    # entropy: count, output, workspace, the 32-bit counters
    ent = lib.kron_gptq_code_entropy
    assert ent(fake, -1, fake, fake, big, None) == -1
    assert ent(fake, 10, None, fake, big, None) == -1
    assert ent(fake, 10, fake, P(7), big, None) == -1
    assert ent(fake, 10, fake, fake, 16, None) == -4
    assert ent(fake, 1 << 32, fake, fake, big, None) == -2
    assert lib.kron_gptq_code_entropy_workspace_size(1000) >= 256 + 4000
    # one-sided: grid, misaligned U_A, small workspace
    os_ = lib.kron_gptq_quantize_onesided
    assert os_(fake, 8, 8, 1, fake, _Grid(-4, 300, fake), fake, fake, None, fake, big, None) == -2
    assert os_(fake, 8, 8, 1, P(256 * 1000 + 4), g, fake, fake, None, fake, big, None) == -1
    assert os_(fake, 64, 64, 1, fake, g, fake, fake, None, fake, 4096, None) == -4
    # factors: method, sizes, iterations, workspace
    fac = lib.kron_gptq_factors
    assert fac(fake, fake, 10, 4, 4, 2, 7, 1, fake, fake, fake, big, None) == -2
    assert fac(fake, fake, 0, 4, 4, 2, 2, 1, fake, fake, fake, big, None) == -1
    assert fac(fake, fake, 10, 4, 4, 2, 2, 0, fake, fake, fake, big, None) == -1
    assert fac(fake, fake, 10, 4, 4, 2, 2, 1, fake, fake, fake, 1024, None) == -4
    assert lib.kron_gptq_factors_workspace_size(0, 4, 4) == 0
    # anti-diagonal baseline: grid, sizes, workspace
    an = lib.kron_gptq_quantize_antidiagonal
    assert an(fake, 8, 8, fake, fake, _Grid(1, 3, fake), fake, fake, None, fake, big, None) == -2
    assert an(fake, 1 << 18, 8, fake, fake, g, fake, fake, None, fake, big, None) == -2
    assert an(fake, 64, 64, fake, fake, g, fake, fake, None, fake, 4096, None) == -4


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import two_sided_gptq_02_b200._lib as L
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "lib_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        L.load_library()
