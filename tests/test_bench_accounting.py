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


def test_fixed_memory_batch_fit():
    """The largest batch whose key/value regions fit a budget: floor(budget / bytes per sequence),
    capped at the library's batch limit."""
    assert bench.fit_batch(3.18e9, 20e9) == 6
    assert bench.fit_batch(289e6, 20e9) == 69
    assert bench.fit_batch(121e6, 20e9) == 165
    assert bench.fit_batch(10, 1e9) == 1024                    # capped
    assert bench.fit_batch(21e9, 20e9) == 0                    # one sequence does not fit
    with pytest.raises(ValueError):
        bench.fit_batch(0, 1e9)


def test_two_point_cost_model_recovers_a_line():
    """t(N) = a + b N through two measured points gives back a and b exactly for a linear cost, and
    predicts the third point."""
    a, b = 0.8, 0.57
    t = lambda n: a + b * n
    fa, fb = bench.two_point_cost_model(t(1), t(138), 138)
    assert abs(fa - a) < 1e-12 and abs(fb - b) < 1e-12
    assert abs(fa + fb * 40 - t(40)) < 1e-12
    assert bench.two_point_cost_model(2.0, 2.0, 1) == (2.0, 0.0)


def test_l2_note_classifies_working_sets():
    l2 = 126 * 2 ** 20
    assert "both stream from HBM" in bench.l2_note(1.07e9, 4.5e9, l2)        # long-context call
    assert "partly served" in bench.l2_note(22e6, 300e6, l2)                  # Huginn call, step > L2
    assert "largely from L2" in bench.l2_note(1e6, 50e6, l2)                  # tiny
    # the step's distinct bytes: deepest region once per layer plus every loop's window ring
    cfg = dict(N=1, kvH=55, d=96, R=32, B=8)
    row = 4 * 55 * 96
    assert bench.step_distinct_bytes(cfg, 1024, 64, 4) == 4 * row * (960 + 32 * 72)


def test_captured_traffic_stands_only_for_the_sources_it_hashes(tmp_path, monkeypatch):
    """A committed ncu capture is used while the kernel's sources hash to the recorded digest and is
    scaled by algorithmic bytes to the timed launch; once the sources change the bench reports no
    traffic rather than a stale figure."""
    f = tmp_path / "ripe_verify_traffic.txt"
    f.write_text("# header\n"
                 f"ripe_verify_kernel.sources_sha256 = {bench.sources_digest('ripe_verify_kernel')}\n"
                 "long_gqa.ripe_verify_kernel.bytes_per_launch = 1010\n"
                 "long_gqa.ripe_verify_kernel.T = 32768\n"
                 "long_gqa.ripe_verify_kernel.algorithmic_bytes = 1000\n")
    real_join = bench.os.path.join
    monkeypatch.setattr(bench.os.path, "join",
                        lambda *p: str(f) if p[-1] == "ripe_verify_traffic.txt" else real_join(*p))
    k = "ripe_verify_kernel"
    assert bench.captured_traffic("long_gqa", k) == {"bytes_per_launch": 1010.0, "T": 32768,
                                                     "algorithmic_bytes": 1000.0}
    assert bench.traffic_for("long_gqa", 2000, k) == 2020.0           # scaled by algorithmic bytes
    assert bench.captured_traffic("huginn", k) is None                 # no capture of that workload
    monkeypatch.setattr(bench, "sources_digest", lambda kernel="ripe_verify_kernel": "0" * 64)
    assert bench.captured_traffic("long_gqa", k) is None               # the sources changed
    assert bench.traffic_for("long_gqa", 2000, k) is None
    assert bench.traffic_basis("long_gqa", k).startswith("no ncu capture")


def test_sources_digest_ignores_comments_only():
    """Comment and blank-line edits keep a capture valid; a change of code does not."""
    code = "int f(int a) {\n  return a + 1;  // one more\n}\n"
    assert bench._code_only(code) == bench._code_only("/* doc */\nint f(int a) {\n\n  return a + 1;\n}\n")
    assert bench._code_only(code) != bench._code_only(code.replace("a + 1", "a + 2"))
