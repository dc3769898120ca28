"""The verify kernels' tile plan against the oracle's plane rule, on the host.

The kernels read a (sequence, kv head)'s keys as a list of tiles (deepest-plane region, the window
ring at each loop of the call, the window keys older than W at the deepest plane).  The plan
(seq_geom / tile_at in csrc/ripe_common.cuh) is host-callable: tests/tile_plan_dump.cu prints it
with the plan set up as the launch code sets it up.  Here the (key, plane) pairs it reads are
compared with the pairs the queries of the block select under the RIPE rule (oracle.plane_of):
  * a single-loop verification reads exactly the needed pairs, each once;
  * a wavefront call (block positions at different loops) reads every needed pair, and otherwise
    only the ring of each of its loops over the window and the block (the masks drop keys that no
    row at that loop sees); a pair is read twice only at the deepest plane, when the call includes
    the deepest loop (its ring tiles and the older window keys then cover the same rows; the masks
    give each query one of them);
  * a draft step (one query at block position j, optionally restricted to an attention sink and a
    sliding window) reads every pair its query selects; of the deepest-plane region it reads
    exactly the selected rows (a windowed draft skips the rows between the sink and the window),
    and beyond that only the ring at its loop and the older window keys at the deepest plane;
  * every tile is one box of consecutive rows: deepest-plane rows at row t, ring rows at slot
    t mod S, never across the ring's wrap, never past the committed positions and the block.
"""
import collections
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import ripe_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KDEEP, KRING, KDUAL = 0, 1, 2


@pytest.fixture(scope="module")
def dump(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    exe = str(tmp_path_factory.mktemp("plan") / "tile_plan_dump")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "self_speculative_decode_b200", "csrc"),
                    "-o", exe, os.path.join(ROOT, "tests", "tile_plan_dump.cu")],
                   check=True, capture_output=True, timeout=600)

    def run(cases):
        lines = [" ".join(str(x) for x in c) if c[0] == "D" else
                 " ".join(str(x) for x in ("V", *c[:7], len(c[7]), *c[7])) for c in cases]
        text = "\n".join(lines) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True, timeout=120).stdout
        plans, cur = [], []
        for line in out.splitlines():
            f = line.split()
            if f[0] == "E":
                assert int(f[1]) == len(cur)
                plans.append(cur)
                cur = []
            else:
                cur.append(tuple(int(x) for x in f))
        assert len(plans) == len(cases)
        return plans
    return run


def _geometry(W, max_T, max_B):
    Wc = min(W, max_T)
    return Wc, min(Wc + max_B, max_T)


def _needed(T, B, R, W, mode, loop_of_j):
    return {(t, orc.plane_of(T + j, t, loop_of_j[j], R, T, W, mode))
            for j in range(B) for t in range(T + j + 1)}


def _read(T, B, W, S, tiles):
    D = max(0, T - W)
    pairs = collections.Counter()
    for kind, t0, cnt, y, plane in tiles:
        assert cnt >= 1 and cnt <= 64
        if kind == KDEEP:
            assert y == t0 and t0 + cnt <= D
        else:
            assert kind in (KRING, KDUAL)
            assert t0 >= D and y == t0 % S and y + cnt <= S       # one box, no wrap inside
            assert t0 + cnt <= (T if kind == KDUAL else T + B)
        for t in range(t0, t0 + cnt):
            pairs[(t, plane)] += 1
    return pairs


def _cases(rng, n, waves):
    out = []
    for _ in range(n):
        R = int(rng.choice([1, 2, 5, 32]))
        B = int(rng.integers(1, 17))
        T = int(rng.choice([0, 1, 7, 63, 64, 65, 130, int(rng.integers(0, 400))]))
        W = int(rng.choice([0, 1, 3, 8, 64, 65, 250, 5000]))
        max_B = B + int(rng.integers(0, 4))
        max_T = max(T + B + int(rng.choice([0, 1, 9, 200])), max_B)
        mode = int(rng.integers(0, 2))
        if waves:
            loops = [int(x) for x in rng.integers(0, R, size=min(B, 4))]
        else:
            loops = [int(rng.integers(0, R))]
        out.append((T, W, B, R, max_T, max_B, mode, loops))
    return out


def test_single_loop_plan_reads_each_needed_pair_once(dump):
    rng = np.random.default_rng(11)
    cases = _cases(rng, 400, waves=False)
    # boxes shorter than 64 rows (small capacities) and the ring's wrap at every offset
    cases += [(T, 3, 4, 4, 13, 4, 0, [1]) for T in range(0, 10)]
    cases += [(T, 70, 8, 6, 400, 8, m, [r]) for T in (0, 69, 70, 71, 140, 300) for m in (0, 1) for r in (0, 5)]
    for case, tiles in zip(cases, dump(cases)):
        T, W, B, R, max_T, max_B, mode, loops = case
        Wc, S = _geometry(W, max_T, max_B)
        got = _read(T, B, Wc, S, tiles)
        need = _needed(T, B, R, Wc, mode, [loops[0]] * B)
        assert set(got) == need, case
        assert max(got.values(), default=1) == 1, case


def test_wavefront_plan_covers_every_row_at_its_loop(dump):
    rng = np.random.default_rng(12)
    cases = _cases(rng, 300, waves=True)
    for case, tiles in zip(cases, dump(cases)):
        T, W, B, R, max_T, max_B, mode, loops = case
        Wc, S = _geometry(W, max_T, max_B)
        got = _read(T, B, Wc, S, tiles)
        loop_of_j = [loops[j % len(loops)] for j in range(B)]
        need = _needed(T, B, R, Wc, mode, loop_of_j)
        assert need <= set(got), case
        # beyond the needed pairs the call reads only what its design reads: the ring of each of
        # its loops over the window and the whole block (keys after that loop's last row are
        # masked), and the deepest plane of the window; a pair read twice is a deepest-plane
        # window row read by both the deepest loop's ring tiles and the older-window-key tiles
        D = max(0, T - Wc)
        allowed = {(t, r) for r in set(loop_of_j) for t in range(D, T + B)} | {(t, R - 1) for t in range(T)}
        assert set(got) - need <= allowed, case
        for (t, plane), k in got.items():
            if k > 1:
                assert k == 2 and plane == R - 1 and R - 1 in loop_of_j and t < T, (case, t)


def test_draft_step_plans(dump):
    rng = np.random.default_rng(13)
    cases = []
    for _ in range(400):
        R = int(rng.choice([1, 2, 5, 32]))
        T = int(rng.choice([0, 1, 5, 64, 65, 200, int(rng.integers(0, 600))]))
        W = int(rng.choice([0, 1, 4, 8, 64, 300, 5000]))
        max_B = int(rng.integers(1, 17))
        j = int(rng.integers(0, max_B))
        max_T = T + max_B + int(rng.choice([0, 3, 100]))
        window = int(rng.choice([-1, 0, 1, 7, 64, 100, 1000]))
        sink = int(rng.choice([0, 1, 4, 70])) if window >= 0 else 0
        cases.append(("D", T, W, R, max_T, max_B, int(rng.integers(0, 2)), int(rng.integers(0, R)), j, sink, window))
    for case, tiles in zip(cases, dump(cases)):
        _, T, W, R, max_T, max_B, mode, r, j, sink, window = case
        Wc, S = _geometry(W, max_T, max_B)
        got = _read(T, j + 1, Wc, S, tiles)
        p = T + j
        keep = [t for t in range(p + 1) if window < 0 or t < sink or t >= p - window]
        need = {(t, orc.plane_of(p, t, r, R, T, Wc, mode)) for t in keep}
        assert need <= set(got), case
        D = max(0, T - Wc)
        assert {(t, pl) for (t, pl) in got if t < D} == {(t, pl) for (t, pl) in need if t < D}, case
        allowed = {(t, r) for t in range(D, p + 1)} | {(t, R - 1) for t in range(D, T)}
        assert set(got) - need <= allowed, case
