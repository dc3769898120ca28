"""The benchmark's algorithmic bytes (the roofline numerator) against the plane rule.

A verification call at loop r must read every (key, plane) pair that some query of the block
selects; bench.verify_bytes counts T + B + dual rows per (sequence, kv head).  Here the pairs
are enumerated one by one with the oracle's plane rule and counted.
"""
import itertools

import pytest

import bench
from oracle import ripe_oracle as orc


def _needed_pairs(T, B, r, R, W, mode):
    return {(t, orc.plane_of(T + j, t, r, R, T, W, mode)) for j in range(B) for t in range(T + j + 1)}


@pytest.mark.parametrize("T,W,B,R", [(0, 4, 3, 4), (5, 9, 4, 4), (20, 4, 6, 4), (40, 16, 8, 6), (33, 0, 5, 3),
                                     (70, 200, 8, 4), (64, 63, 1, 2)])
def test_verify_bytes_count_each_needed_pair_once(T, W, B, R):
    cfg = dict(N=1, kvH=1, d=1, Hq=1, B=B, R=R, W=W)
    for r, mode in itertools.product(range(R), (orc.QUERY_RELATIVE, orc.CACHE_RELATIVE)):
        pairs = len(_needed_pairs(T, B, r, R, W, mode))
        rows = T + B + bench.dual_keys(T, W, B, R, r, mode)
        assert rows == pairs, (r, mode)
        if mode == orc.QUERY_RELATIVE:
            # bytes: 4 per row (K + V, bf16, d = 1) plus the queries and outputs
            assert bench.verify_bytes(cfg, [T], r) == 4 * pairs + 4 * B


@pytest.mark.parametrize("T,W,j,sink,window", [(300, 16, 3, 4, 40), (900, 32, 5, 100, 10), (77, 32, 2, 100, 10),
                                                (500, 0, 2, 1, 0), (300, 64, 4, 0, 1000)])
def test_windowed_draft_bytes_cover_the_attended_keys(T, W, j, sink, window):
    """The plan of a windowed draft reads every attended (key, plane) pair, and beyond them at most
    the window ring's rows [T - W, p] outside the draft window (W + j rows) and the dual rows."""
    R, r = 4, 0
    cfg = dict(N=1, kvH=1, d=1, Hq=1, R=R)
    p = T + j
    attended = [t for t in range(p + 1) if t < sink or t >= p - window]
    read_rows = (bench.draft_window_bytes(cfg, [T], r, j, W, sink, window) - 4) // 4
    assert len(attended) <= read_rows <= len(attended) + W + j + bench.dual_keys(T, W, j + 1, R, r)
