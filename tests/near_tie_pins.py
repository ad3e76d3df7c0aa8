"""Pins for the two near-tie helpers of the oracle (``topk_gap`` and
``inner_gap`` in oracle/oracle.py).

These helpers decide which tokens the parity tests leave out of the
bit-exact expert-id check (a k-th / (k+1)-th probability gap below the tie
threshold) and which tokens they compare as sets (a near tie between two
selected slots).  They are pinned here to hand-built probability rows whose
gaps are dyadic rationals, so every expected value is exact in binary
floating point and is written out below by hand, not computed by a sort.

``check_near_tie_helpers(topk_gap, inner_gap)`` raises AssertionError on any
mismatch; test_near_tie_pins.py runs it on the real helpers and on copies of
them with a planted mistake.
"""
from __future__ import annotations

import numpy as np

INF = np.inf

# One row per case: (probabilities, k, expected topk_gap, expected inner_gap).
# Ordered descending, row A is 3/8, 1/4, 7/32, 1/8, 1/32, 0.
ROW_A = [1 / 32, 3 / 8, 1 / 8, 1 / 4, 7 / 32, 0.0]        # unsorted on purpose
CASES = [
    (ROW_A, 1, 3 / 8 - 1 / 4, INF),            # k = 1: no pair inside the top k
    (ROW_A, 2, 1 / 4 - 7 / 32, 3 / 8 - 1 / 4),
    (ROW_A, 3, 7 / 32 - 1 / 8, 1 / 32),        # inner: min(1/8, 1/32)
    (ROW_A, 5, 1 / 32, 1 / 32),                # boundary 1/32 - 0; inner min(1/8, 1/32, 3/32, 3/32)
    (ROW_A, 6, INF, 1 / 32),                   # k = E: nothing outside the top k
    # a tie inside the top k: inner gap exactly zero, boundary gap 1/8
    ([1 / 4, 1 / 8, 1 / 4, 1 / 8, 1 / 4], 3, 1 / 8, 0.0),
    # an exact tie at the boundary: p_(k) = p_(k+1)
    ([1 / 8, 1 / 2, 1 / 8, 1 / 4], 3, 0.0, 1 / 8),
    # a boundary gap of exactly 2^-20 (just under 1e-6) and of 2^-19 (just over)
    ([1 / 2, 1 / 4 - 2.0 ** -20, 1 / 4, 0.0], 2, 2.0 ** -20, 1 / 4),
    ([1 / 4 - 2.0 ** -19, 1 / 2, 0.0, 1 / 4], 2, 2.0 ** -19, 1 / 4),
    # the largest value last, equal values spread out: order must not matter
    ([0.0, 1 / 16, 1 / 16, 1 / 8, 3 / 4], 4, 1 / 16, 0.0),
]

# The parity tests' threshold: a boundary gap below it leaves the token out.
TIE_EPS = 1e-6


def check_near_tie_helpers(topk_gap, inner_gap):
    for probs, k, want_top, want_inner in CASES:
        p = np.array([probs], dtype=np.float64)
        got_top = topk_gap(p, k)
        got_inner = inner_gap(p, k)
        assert got_top.shape == (1,) and got_inner.shape == (1,), "one value per token"
        assert got_top[0] == want_top, ("topk_gap", probs, k, got_top[0], want_top)
        assert got_inner[0] == want_inner, ("inner_gap", probs, k, got_inner[0], want_inner)
    # several tokens at once: each row on its own, in its own place
    rows = np.array([ROW_A, ROW_A[::-1], [1 / 6] * 6], dtype=np.float64)
    got = topk_gap(rows, 3)
    assert got[0] == 7 / 32 - 1 / 8 and got[1] == 7 / 32 - 1 / 8 and got[2] == 0.0, ("rows", got)
    got = inner_gap(rows, 3)
    assert got[0] == 1 / 32 and got[1] == 1 / 32 and got[2] == 0.0, ("rows", got)
    # the 2^-20 boundary gap is a near tie, the 2^-19 one is not
    near = topk_gap(np.array([CASES[7][0], CASES[8][0]]), 2) < TIE_EPS
    assert near.tolist() == [True, False], ("threshold", near)
