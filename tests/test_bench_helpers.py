"""Host-side arithmetic of bench.py (CPU only): the algorithmic FLOP counts behind the roofline
fractions, the gate that drops a DRAM-traffic record once its kernel source has changed, and the
parser of the clock samples taken during the timed region."""
import hashlib
import json
import math

import pytest

import bench


def _tile_pairs_brute(Mt, Nt):
    """(source, target) tile pairs of the two chains, enumerated: the row chain sends tile (I, J')
    to every (I, J) with J' < J, the column chain tile (I', J) to every (I, J) with I' < I."""
    row = sum(1 for I in range(Mt) for J in range(Nt) for Jp in range(J))
    col = sum(1 for I in range(Mt) for J in range(Nt) for Ip in range(I))
    return row + col


@pytest.mark.parametrize("m,n", [(64, 64), (128, 320), (1000, 130), (4096, 4096), (14336, 4096)])
def test_push_flops_count_every_tile_pair_once(m, n):
    Mt, Nt = math.ceil(m / 64), math.ceil(n / 64)
    assert bench._push_flops(m, n) == 2.0 * 64 ** 3 * _tile_pairs_brute(Mt, Nt)


def test_push_flops_approach_mn_m_plus_n():
    # the two chains of the two-sided update: about mn(m+n) FLOP (one multiply-add per pair of
    # entries in one row or one column, each counted as 2 FLOP)
    m = n = 4096
    assert bench._push_flops(m, n) == pytest.approx(m * n * (m + n) * (1 - 64 / 4096), rel=1e-12)


@pytest.mark.parametrize("m,n", [(64, 64), (128, 320), (1000, 130), (4096, 4096), (14336, 4096)])
def test_near_field_moves_between_update_and_leaf(m, n):
    # the fp32 leaf computes the adjacent-tile pairs itself: the total is conserved and the moved part
    # is one 64^3 block per (tile, right neighbour) and (tile, lower neighbour) pair, enumerated
    Mt, Nt = math.ceil(m / 64), math.ceil(n / 64)
    adj = sum(1 for I in range(Mt) for J in range(1, Nt)) + sum(1 for I in range(1, Mt) for J in range(Nt))
    moved = bench._push_flops(m, n) - bench._push_flops(m, n, near_in_leaf=True)
    assert moved == 2.0 * 64 ** 3 * adj
    assert bench._leaf_flops(m, n, near_in_leaf=True) - bench._leaf_flops(m, n) == moved


def test_leaf_flops_per_tile_by_enumeration():
    T = 64
    row_chain = sum(j for i in range(T) for j in range(T))            # r_ij = sum_{k<j}
    col_chain = sum(i for i in range(T) for j in range(T))            # c_ij = sum_{k<i}
    fold = sum(i + 1 for i in range(T) for j in range(T))             # (U_B^T R)_ij = sum_{k<=i}
    assert 2 * (row_chain + col_chain + fold) == 782336
    assert bench._leaf_flops(64, 64) == 782336
    assert bench._leaf_flops(4096, 4096) == 782336 * 64 * 64
    assert bench._leaf_flops(65, 1) == 782336 * 2          # ragged edges count as whole tiles


def test_traffic_record_is_dropped_when_the_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cuh"
    src.write_bytes(b"// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"k": {"dram_bytes_per_unit": 1000.0, "source": "kernel.cuh",
                 "source_sha256": hashlib.sha256(b"// kernel v1\n").hexdigest()}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    assert bench._traffic("k", 64) == 64000.0
    assert bench._traffic("other", 64) is None
    src.write_bytes(b"// kernel v2\n")
    assert bench._traffic("k", 64) is None


def test_committed_traffic_records_name_existing_sources():
    with open(bench.HERE + "/profiles/traffic.json") as f:
        recs = json.load(f)
    for name, rec in recs.items():
        assert rec["dram_bytes_per_unit"] > 0 and rec["unit"] == "tile", name
        assert rec["captured_bytes"] == pytest.approx(rec["dram_bytes_per_unit"] * rec["captured_tiles"]), name
        with open(bench.HERE + "/" + rec["source"], "rb"):
            pass


def test_clock_summary_parses_samples_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 300.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 650.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 10.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")
    s = bench.ClockSampler("0")
    s.path = str(path)
    out = s.summary()
    assert out["samples"] == 4
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == 990.5


def test_clock_summary_without_samples(tmp_path):
    s = bench.ClockSampler("0")
    s.path = str(tmp_path / "missing.csv")
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}


def test_prepare_flops_count_cholesky_and_inverse():
    # a Cholesky of a k x k matrix costs sum_j (k - j - 1)(k - j) ~ k^3/3 FLOP, the triangular
    # inverse as much again; the bench counts 2/3 k^3 per factor
    k = 4096
    chol = sum(2 * (k - j - 1) * (k - j) // 2 + (k - j - 1) for j in range(k))
    assert chol == pytest.approx(k ** 3 / 3, rel=1e-3)
    assert bench._prepare_flops(k, k) == pytest.approx(2 * 2 * k ** 3 / 3, rel=1e-12)
    assert bench._prepare_flops(4096, 14336) == pytest.approx(2 / 3 * (4096 ** 3 + 14336 ** 3), rel=1e-12)
