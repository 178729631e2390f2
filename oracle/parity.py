"""Code-level comparison of a candidate solver with the oracle.  TEST INFRASTRUCTURE.

The four FastKron variants are equivalent in exact arithmetic with a fixed tie-break
("FastKron", Section 2.5, equivalence theorem); in floating point a different
summation order can move a pre-rounding value across a rounding tie, and such a flip
changes every later entry to the bottom-right ("FastKron", Section 2.3).  The rule used
here: walk the mismatches in anti-diagonal order; the earliest one has no mismatching
entry to its top-left, so its pre-rounding value differs from the oracle's only by
rounding noise.  If the oracle saw that entry within ``tol`` grid steps of a half-integer,
the candidate's decision is forced into the oracle (counted as a boundary flip) and the
oracle is rerun; any other mismatch is a failure.
"""
from __future__ import annotations

import numpy as np

from . import NOT_FORCED, quantize_naive


def compare_with_oracle(codes, W, UA, UB, s, qmin: int, qmax: int, *, tol: float = 1e-9,
                        max_flips: int = 64):
    codes = np.asarray(codes).astype(np.int32)
    m, n = codes.shape
    forced = np.full((m, n), NOT_FORCED, dtype=np.int32)
    flips = []
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    while True:
        r = quantize_naive(W, UA, UB, s, qmin, qmax, forced=forced, tol=tol)
        diff = r["codes"] != codes
        if not diff.any():
            return dict(ok=True, flips=flips, oracle=r, mismatches=0)
        d = np.where(diff, ii + jj, np.iinfo(np.int64).max)
        dmin = d.min()
        first = np.argwhere(d == dmin)
        bad = [(int(i), int(j)) for i, j in first if not r["boundary"][i, j]]
        if bad or len(flips) + len(first) > max_flips:
            i, j = bad[0] if bad else tuple(first[0])
            return dict(ok=False, flips=flips, oracle=r, mismatches=int(diff.sum()),
                        first=(int(i), int(j)), t=float(r["t"][i, j]),
                        oracle_code=int(r["codes"][i, j]), candidate_code=int(codes[i, j]))
        for i, j in first:
            forced[i, j] = codes[i, j]
            flips.append((int(i), int(j), float(r["t"][i, j])))


def compare_with_oracle_rc(codes, W, UA, UB, alpha, beta, *, tol: float = 1e-9, max_flips: int = 64):
    """The same rule for the row- and column-scaled alphabet (oracle ``quantize_rc``)."""
    from . import NOT_FORCED_64, quantize_rc
    codes = np.asarray(codes).astype(np.int64)
    m, n = codes.shape
    forced = np.full((m, n), NOT_FORCED_64, dtype=np.int64)
    flips = []
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    while True:
        r = quantize_rc(W, UA, UB, alpha, beta, forced=forced, tol=tol)
        diff = r["codes"] != codes
        if not diff.any():
            return dict(ok=True, flips=flips, oracle=r, mismatches=0)
        d = np.where(diff, ii + jj, np.iinfo(np.int64).max)
        dmin = d.min()
        first = np.argwhere(d == dmin)
        bad = [(int(i), int(j)) for i, j in first if not r["boundary"][i, j]]
        if bad or len(flips) + len(first) > max_flips:
            i, j = bad[0] if bad else tuple(first[0])
            return dict(ok=False, flips=flips, oracle=r, mismatches=int(diff.sum()),
                        first=(int(i), int(j)), t=float(r["t"][i, j]),
                        oracle_code=int(r["codes"][i, j]), candidate_code=int(codes[i, j]))
        for i, j in first:
            forced[i, j] = codes[i, j]
            flips.append((int(i), int(j), float(r["t"][i, j])))
