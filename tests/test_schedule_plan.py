"""The solve's update schedule, read through kron_gptq_schedule_plan (host only, CPU).

The recursion of "FastKron" (Section 2.5) assigns every pair (source diagonal s, target diagonal t),
s < t, of tile anti-diagonals to exactly one update; the solve cuts those updates into pieces by when
they are needed and issues them on three streams.  What must hold for any cut:
  * every pair s < t is carried by exactly one piece (each error reaches each later tile once);
  * a piece starts only after the leaves of all its sources, and it is issued after those leaves;
  * every piece that targets diagonal t, except the near piece (t-1 -> t) on the critical stream,
    is free at least one leaf before leaf t, and is issued before the near piece of t;
  * pieces due within a few leaves (urgent, soon) span at most four source diagonals.
"""
import numpy as np
import pytest

import two_sided_gptq_02_b200 as kg

CRIT, URGENT, SOON, BACK = 0, 1, 2, 3


def _plan(ndiag):
    plan = kg.kron_gptq_schedule_plan(ndiag)
    assert all(len(p) == 5 for p in plan)
    return plan


@pytest.mark.parametrize("ndiag", [1, 2, 3, 4, 5, 7, 8, 9, 16, 31, 64, 100, 127, 287])
def test_pieces_cover_every_pair_once(ndiag):
    cover = np.zeros((ndiag, ndiag), dtype=np.int64)
    for s0, s1, t0, t1, st in _plan(ndiag):
        assert 0 <= s0 < s1 <= t0 < t1 <= ndiag, (s0, s1, t0, t1)
        assert st in (CRIT, URGENT, SOON, BACK)
        cover[s0:s1, t0:t1] += 1
    want = np.triu(np.ones((ndiag, ndiag), dtype=np.int64), 1)
    assert np.array_equal(cover, want)


@pytest.mark.parametrize("ndiag", [2, 5, 16, 63, 127, 287])
def test_issue_order_respects_leaves(ndiag):
    plan = _plan(ndiag)
    near_seen = 0          # near pieces issued so far: the leaf of diagonal near_seen - 1 is issued
    near_pos = {}
    for k, (s0, s1, t0, t1, st) in enumerate(plan):
        if st == CRIT:
            assert (s0, s1, t1) == (t0 - 1, t0, t0 + 1), "the critical stream carries only near pieces"
            assert t0 == near_seen + 1, "one near piece per leaf, in order"
            near_seen += 1
            near_pos[t0] = k
            continue
        # issued right after the leaf of its last source (leaf L follows the near piece of L)
        assert near_seen == s1 - 1, (k, plan[k], near_seen)
        # free at least one leaf before its first target's leaf
        assert s1 <= t0 - 1, plan[k]
        if st in (URGENT, SOON):
            assert s1 - s0 <= 4, plan[k]
    assert near_seen == ndiag - 1
    for k, (s0, s1, t0, t1, st) in enumerate(plan):
        if st != CRIT:
            assert all(k < near_pos[t] for t in range(t0, t1)), "every piece into t precedes t's near piece"


def test_top_update_of_4096_square_is_split():
    # 127 tile diagonals: the top update (sources [0, 63), targets [63, 127)) leaves the critical
    # stream only its near piece; its older sources go to the background stream in halves
    plan = _plan(127)
    into63 = [p for p in plan if p[2] <= 63 < p[3]]
    assert (62, 63, 63, 64, CRIT) in into63
    assert sum(p[1] - p[0] for p in into63) == 63
    assert max(p[1] - p[0] for p in into63 if p[4] != BACK) <= 4
    assert all(p[3] == 127 for p in into63 if p[4] == BACK)


def test_bad_arguments():
    L = kg.load_library()
    assert L.kron_gptq_schedule_plan(0, None, 0) == -1
    assert L.kron_gptq_schedule_plan(5, None, -1) == -1
    assert L.kron_gptq_schedule_plan(1, None, 0) == 0
