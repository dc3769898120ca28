"""Pins for the CPU oracle, checked against what the pages and the mathematics fix.

Each test compares the oracle with something other than itself: the worked
memory figure printed in the RIPE abstract, closed forms, textbook attention
computed by a library routine (torch scaled_dot_product_attention in fp64),
an independent brute-force formulation, and the block-independence property
the abstract states.  Runs on CPU only.
"""
import os

import numpy as np
import pytest
import torch

from oracle import ripe_oracle as orc
from self_speculative_decode_b200.synth import PlaneSource, block_from_planes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(bits):
    # local widening of bf16 bits, independent of the oracle's helper
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def _cache(N, kvH, g, d, R, W, T, B, rho=0.88, seed=0, mode=orc.QUERY_RELATIVE, independent=False):
    src = PlaneSource(N, kvH, d, R, T + B, rho, seed, independent=independent)
    PK = [src.plane(r, "K") for r in range(R)]
    PV = [src.plane(r, "V") for r in range(R)]
    c = orc.OracleCache(N, 1, kvH, d, R, W, T + B, mode)
    for pl in range(R):
        c.load_prefix(0, pl, [T] * N, PK[pl], PV[pl])
    for r in range(R):
        c.append(0, r, block_from_planes(PK[r], T, B), block_from_planes(PV[r], T, B))
    return c, PK, PV, src


def _sdpa(q, K, V, T, B, g, scale):
    """Textbook causal attention of block queries over keys [0, T+B) (torch, fp64)."""
    Hq = q.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2).unsqueeze(0)               # [1, Hq, B, d]
    kt = torch.from_numpy(K).repeat_interleave(g, dim=0).unsqueeze(0)   # [1, Hq, T+B, d]
    vt = torch.from_numpy(V).repeat_interleave(g, dim=0).unsqueeze(0)
    j = torch.arange(B)[:, None]
    t = torch.arange(T + B)[None, :]
    mask = t <= T + j
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    assert o.shape == (1, Hq, B, q.shape[2])
    return o[0].permute(1, 0, 2).numpy()


# ---------------------------------------------------------------- P1: memory
def test_memory_fraction_matches_printed_worked_example():
    vals = {}
    with open(os.path.join(GOLDEN, "huginn_memory_fraction.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.strip().split("=")
                vals[k] = float(v)
    frac, stored = orc.memory_fraction(int(vals["T"]), int(vals["W"]), int(vals["R"]),
                                       int(vals["recurrent_layers"]), int(vals["other_layers"]))
    assert round(100 * frac, 1) == vals["printed_percent"]
    # dropping the window planes (or counting W-1 of them) misses the printed figure
    frac_short, _ = orc.memory_fraction(int(vals["T"]), int(vals["W"]) - 1, int(vals["R"]), 4, 4)
    assert round(100 * frac_short, 1) != vals["printed_percent"]


@pytest.mark.parametrize("T,W,R", [(1, 0, 3), (10, 3, 4), (7, 20, 5), (40, 8, 1), (33, 33, 2)])
def test_stored_count_closed_form(T, W, R):
    """Deepest plane everywhere + all R planes in the last W positions: T + min(W, T) * (R - 1)."""
    frac, stored = orc.memory_fraction(T, W, R)
    assert stored == T + min(W, T) * (R - 1)
    assert abs(frac - (T + min(W, T) * (R - 1)) / (R * T)) < 1e-15


def test_stored_count_independent_of_block_history():
    rng = np.random.default_rng(5)
    R, W = 4, 6
    c = orc.OracleCache(N=2, L=2, kvH=1, d=2, R=R, W=W, max_T=200)
    for _ in range(40):
        B = int(rng.integers(1, 7))
        blk = np.ones((2, B, 1, 2), dtype=np.uint16)
        for layer in range(2):
            for r in range(R):
                c.append(layer, r, blk, blk)
        c.commit(rng.integers(0, B + 1, size=2))
        for n in range(2):
            T = int(c.T[n])
            for layer in range(2):
                assert c.stored_position_planes(layer, n) == T + min(W, T) * (R - 1)


# ---------------------------------------------------------------- P2 / P3 / P4
@pytest.mark.parametrize("r", [0, 2, 3])
def test_full_cache_is_textbook_attention_on_plane_r(r):
    N, kvH, g, d, R, T, B = 1, 2, 2, 16, 4, 37, 5
    c, PK, PV, src = _cache(N, kvH, g, d, R, W=T + B, T=T, B=B, seed=1)
    q = src.queries(r, B, kvH * g)
    out, _ = c.verify(0, r, q, g, scale=0.7)
    ref = _sdpa(_f64(q[0]), _f64(PK[r][0]), _f64(PV[r][0]), T, B, g, 0.7)
    assert np.abs(out[0] - ref).max() < 1e-12


@pytest.mark.parametrize("r", [0, 1, 3])
def test_window_zero_is_deepest_plane_prefix(r):
    N, kvH, g, d, R, T, B = 1, 1, 3, 8, 4, 29, 6
    c, PK, PV, src = _cache(N, kvH, g, d, R, W=0, T=T, B=B, seed=2)
    q = src.queries(r, B, kvH * g)
    out, _ = c.verify(0, r, q, g)
    K = np.concatenate([_f64(PK[R - 1][0])[:, :T], _f64(PK[r][0])[:, T:]], axis=1)
    V = np.concatenate([_f64(PV[R - 1][0])[:, :T], _f64(PV[r][0])[:, T:]], axis=1)
    ref = _sdpa(_f64(q[0]), K, V, T, B, g, 1.0)
    assert np.abs(out[0] - ref).max() < 1e-12


@pytest.mark.parametrize("W", [0, 3, 100])
def test_single_loop_is_ordinary_attention(W):
    N, kvH, g, d, T, B = 1, 2, 1, 8, 21, 4
    c, PK, PV, src = _cache(N, kvH, g, d, R=1, W=W, T=T, B=B, seed=3)
    q = src.queries(0, B, kvH * g)
    out, _ = c.verify(0, 0, q, g)
    ref = _sdpa(_f64(q[0]), _f64(PK[0][0]), _f64(PV[0][0]), T, B, g, 1.0)
    assert np.abs(out[0] - ref).max() < 1e-12


# ---------------------------------------------------------------- P5
def test_softmax_weights_sum_to_one():
    N, kvH, g, d, R, W, T, B = 1, 1, 1, 8, 4, 5, 30, 4
    c, PK, PV, src = _cache(N, kvH, g, d, R, W, T, B, seed=4)
    Kr, Vr, Kl, Vl, _ = c.verify_inputs(0, 1)
    q = orc.bf16_to_f64(src.queries(1, B, 1))
    for j in range(B):
        for scale in (1.0, 8.0):
            w = orc.weights(T, j, 1, R, W, Kr[0, 0], Kl[0, 0], q[0, j, 0], scale)
            assert abs(w.sum() - 1.0) < 1e-12 and (w >= 0).all()
    # with every value equal to one the output is exactly the weight sum
    ones = np.ones_like(Vr)
    out, _ = orc.verify(c.T, B, 1, R, W, g, Kr, np.where(np.isnan(Vr), np.nan, ones),
                        Kl, np.where(np.isnan(Vl), np.nan, ones), q)
    assert np.abs(out - 1.0).max() < 1e-12



def test_zero_scale_is_the_mean_of_the_visible_values():
    """Scale 0 makes every logit 0: the weights are uniform over keys 0..p, so the output is the
    plain mean of the values there and the log-sum-exp is ln(p + 1), whichever planes the rule
    picks when every stored plane of a position holds the same value."""
    N, kvH, g, d, R, W, T, B = 2, 2, 2, 8, 4, 5, 30, 4
    c, PK, PV, src = _cache(N, kvH, g, d, R, W, T, B, seed=7, independent=True)
    q = orc.bf16_to_f64(src.queries(1, B, kvH * g))
    for r in (0, 1, R - 1):
        Kr, Vr, Kl, Vl, _ = c.verify_inputs(0, r)
        X = np.random.default_rng(3).standard_normal(Vr.shape)
        out, lse = orc.verify(c.T, B, r, R, W, g, Kr, np.where(np.isnan(Vr), np.nan, X),
                              Kl, np.where(np.isnan(Vl), np.nan, X), q, scale=0.0)
        for n in range(N):
            for j in range(B):
                p = int(c.T[n]) + j
                for h in range(kvH * g):
                    assert np.abs(out[n, j, h] - X[n, h // g, :p + 1].mean(axis=0)).max() < 1e-12
                    assert abs(lse[n, j, h] - np.log(p + 1)) < 1e-12


def test_negative_scale_is_attention_with_negated_queries():
    """softmax(-s <q, k>) = softmax(s <-q, k>): the full cache at scale -0.7 is textbook causal
    attention (torch SDPA, fp64) of the negated queries at scale 0.7."""
    N, kvH, g, d, R, T, B = 1, 2, 2, 16, 4, 37, 5
    c, PK, PV, src = _cache(N, kvH, g, d, R, W=T + B, T=T, B=B, seed=2)
    for r in (0, 3):
        q = src.queries(r, B, kvH * g)
        out, _ = c.verify(0, r, q, g, scale=-0.7)
        ref = _sdpa(-_f64(q[0]), _f64(PK[r][0]), _f64(PV[r][0]), T, B, g, 0.7)
        assert np.abs(out[0] - ref).max() < 1e-12

def test_softmax_weights_match_independent_formulations():
    """oracle.weights against two formulations that share none of its code.

    (1) brute_verify with one-hot values (the value of key t is e_t on every plane, d >= T + B):
    its output row for query j is exactly that query's weight vector, computed from brute_verify's
    own full-depth key sets and its own softmax.  (2) torch.softmax over logits built here from the
    tagged planes, the plane of key t being r for the block and the window and R-1 otherwise.
    Independent key planes and scale 8 make a wrong plane, a dropped scale or a shifted window an
    O(1) difference; the last lines check that such mistakes would indeed be seen."""
    import torch
    R, W, T, B = 4, 5, 30, 4
    d = T + B + 2
    rng = np.random.default_rng(11)
    Kp = rng.standard_normal((R, 1, T + B, d))
    Vp = np.broadcast_to(np.eye(T + B, d)[None, None], (R, 1, T + B, d)).copy()
    q = rng.standard_normal((B, 1, d)) / np.sqrt(d)
    for r in range(R):
        for scale in (1.0, 8.0):
            ob, _ = orc.brute_verify(Kp, Vp, T, B, r, W, 1, q, scale)
            for j in range(B):
                p = T + j
                w = orc.weights(T, j, r, R, W, Kp[r, 0], Kp[R - 1, 0], q[j, 0], scale)
                assert np.abs(w - ob[j, 0, :p + 1]).max() < 1e-12
                assert np.abs(ob[j, 0, p + 1:]).max() == 0.0
                Ksel = np.stack([Kp[r, 0, t] if (t >= T or t >= p - W) else Kp[R - 1, 0, t] for t in range(p + 1)])
                ref = torch.softmax(scale * torch.from_numpy(Ksel @ q[j, 0]), dim=0).numpy()
                assert np.abs(w - ref).max() < 1e-12
                if r < R - 1 and scale == 1.0:   # every key at the deepest plane instead
                    wrong_plane = orc.weights(T, j, R - 1, R, W, Kp[R - 1, 0], Kp[R - 1, 0], q[j, 0], scale)
                    assert np.abs(wrong_plane - ref).sum() > 0.05
                if scale != 1.0:
                    no_scale = torch.softmax(torch.from_numpy(Ksel @ q[j, 0]), dim=0).numpy()
                    assert np.abs(w - no_scale).sum() > 0.05


# ---------------------------------------------------------------- plane counts (closed form)
def _count_closed_form(T, j, r, R, W, mode):
    """Keys read at plane r by query p = T + j: [min(T, max(0, p - W)), p] (query window) or
    [max(0, T - W), p] (cache window); the rest read plane R - 1."""
    p = T + j
    lo = min(T, max(0, p - W)) if mode == orc.QUERY_RELATIVE else max(0, T - W)
    return p - lo + 1


@pytest.mark.parametrize("mode", [orc.QUERY_RELATIVE, orc.CACHE_RELATIVE])
@pytest.mark.parametrize("T,W,B,r", [(20, 4, 6, 1), (20, 0, 3, 0), (5, 9, 4, 2), (30, 6, 6, 3)])
def test_plane_usage_counts(mode, T, W, B, r):
    """Zero keys give uniform weights; one-hot values per plane reveal which planes were read."""
    R, d = 4, 8
    L = T + B
    Kz = np.zeros((1, 1, L, d))
    onehot = lambda pl: np.broadcast_to(np.eye(d)[pl], (1, 1, L, d)).copy()
    out, _ = orc.verify([T], B, r, R, W, 1, Kz, onehot(r), Kz, onehot(R - 1), np.zeros((1, B, 1, d)),
                        mode=mode)
    for j in range(B):
        p = T + j
        n_r = _count_closed_form(T, j, r, R, W, mode)
        if r == R - 1:
            assert abs(out[0, j, 0, R - 1] - 1.0) < 1e-12
        else:
            assert abs(out[0, j, 0, r] * (p + 1) - n_r) < 1e-9
            assert abs(out[0, j, 0, R - 1] * (p + 1) - (p + 1 - n_r)) < 1e-9


def test_absent_plane_is_detected():
    """Planes that RIPE does not store are NaN; asking for a wider window must fail loudly."""
    N, kvH, g, d, R, W, T, B = 1, 1, 1, 8, 4, 3, 20, 2
    c, PK, PV, src = _cache(N, kvH, g, d, R, W, T, B, seed=6)
    Kr, Vr, Kl, Vl, _ = c.verify_inputs(0, 0)
    q = orc.bf16_to_f64(src.queries(0, B, 1))
    orc.verify(c.T, B, 0, R, W, g, Kr, Vr, Kl, Vl, q)          # the cache's own window: fine
    with pytest.raises(RuntimeError):
        orc.verify(c.T, B, 0, R, W + 2, g, Kr, Vr, Kl, Vl, q)  # reads plane 0 outside the window


# ---------------------------------------------------------------- P7 brute force
@pytest.mark.parametrize("mode", [orc.QUERY_RELATIVE, orc.CACHE_RELATIVE])
@pytest.mark.parametrize("T,W,B,r,g", [(12, 3, 4, 0, 2), (12, 0, 4, 2, 1), (6, 10, 3, 1, 3),
                                       (15, 5, 6, 3, 1), (9, 1, 5, 1, 2)])
def test_brute_force_twin(mode, T, W, B, r, g):
    N, kvH, d, R = 1, 2, 8, 4
    c, PK, PV, src = _cache(N, kvH, g, d, R, W, T, B, seed=7, mode=mode, independent=True)
    q = src.queries(r, B, kvH * g)
    out, lse = c.verify(0, r, q, g, scale=1.3)
    Kall = np.stack([_f64(PK[pl][0]) for pl in range(R)])
    Vall = np.stack([_f64(PV[pl][0]) for pl in range(R)])
    bo, bl = orc.brute_verify(Kall, Vall, T, B, r, W, g, _f64(q[0]), 1.3, mode)
    assert np.abs(out[0] - bo).max() < 1e-12
    assert np.abs(lse[0] - bl).max() < 1e-12
    # planted mistake: an off-by-one window in the twin is visible at this size
    if 0 < W < T and r != R - 1:
        bo2, _ = orc.brute_verify(Kall, Vall, T, B, r, W + 1, g, _f64(q[0]), 1.3, mode)
        assert np.abs(out[0] - bo2).max() > 1e-6


# ---------------------------------------------------------------- P6 block independence
def _decode(W, splits, mode, R=4, T0=10, S=12, kvH=1, g=2, d=8, seed=11):
    """Verify positions T0..T0+S-1 in the given block split, committing every position.

    Returns {(position, r): output row [Hq][d]} from the oracle state machine.
    """
    src = PlaneSource(1, kvH, d, R, T0 + S, 0.88, seed, independent=True)
    PK = [src.plane(r, "K") for r in range(R)]
    PV = [src.plane(r, "V") for r in range(R)]
    qsrc = PlaneSource(1, kvH * g, d, R, T0 + S, 0.88, seed + 1000)
    Q = [qsrc.plane(r, "K") for r in range(R)]           # per-position queries [1][Hq][pos][d]
    c = orc.OracleCache(1, 1, kvH, d, R, W, T0 + S, mode)
    for pl in range(R):
        c.load_prefix(0, pl, [T0], PK[pl], PV[pl])
    res = {}
    t = T0
    for B in splits:
        for r in range(R):
            c.append(0, r, block_from_planes(PK[r], t, B), block_from_planes(PV[r], t, B))
        for r in range(R):
            q = np.ascontiguousarray(Q[r][:, :, t:t + B].transpose(0, 2, 1, 3))
            out, _ = c.verify(0, r, q, g)
            for j in range(B):
                res[(t + j, r)] = out[0, j]
        c.commit([B])
        t += B
    assert t == T0 + 12
    return res


def _max_diff(a, b):
    return max(np.abs(a[k] - b[k]).max() for k in a)


@pytest.mark.parametrize("W", [4, 5, 9])
def test_block_independence_when_window_covers_block(W):
    B = 4
    rng = np.random.default_rng(W)
    ref = _decode(W, [1] * 12, orc.QUERY_RELATIVE)               # position by position
    batched = _decode(W, [B] * 3, orc.QUERY_RELATIVE)            # blocks of B
    splits = []
    while sum(splits) < 12:
        splits.append(int(min(rng.integers(1, W + 2), 12 - sum(splits))))
    rand = _decode(W, splits, orc.QUERY_RELATIVE)                # random blocks of <= W+1
    assert _max_diff(ref, batched) < 1e-12
    assert _max_diff(ref, rand) < 1e-12


def test_block_dependence_negative_controls():
    # window shorter than the block: the batched result differs from the sequential one
    assert _max_diff(_decode(1, [1] * 12, 0), _decode(1, [4] * 3, 0)) > 1e-3
    # window measured from the cache end: differs even with W >= B
    assert _max_diff(_decode(5, [1] * 12, orc.CACHE_RELATIVE),
                     _decode(5, [4] * 3, orc.CACHE_RELATIVE)) > 1e-3


# ---------------------------------------------------------------- state machine
def test_rollback_discards_rejected_positions_and_evicts():
    R, W = 3, 2
    c = orc.OracleCache(N=1, L=1, kvH=1, d=1, R=R, W=W, max_T=20)
    blk = lambda v, B: np.full((1, B, 1, 1), v, dtype=np.uint16)
    for r in range(R):
        c.append(0, r, blk(10 + r, 4), blk(20 + r, 4))
    c.commit([3])                  # positions 0..2 kept, 3 discarded
    assert int(c.T[0]) == 3
    assert not c.present[0, :, 0, 3].any()
    # window W=2 -> position 0 keeps only the deepest plane, 1 and 2 keep all
    assert c.present[0, :, 0, 0].tolist() == [False, False, True]
    assert c.present[0, :, 0, 1:3].all()
    assert c.values(0, R - 1, "K")[0, 0, 0, 0] == 10 + R - 1
    with pytest.raises(ValueError):
        for r in range(R):
            c.append(0, r, blk(1, 2), blk(1, 2))
        c.commit([3])              # more than the block length


# ---------------------------------------------------------------- loop per position (wavefront)
def test_wave_rows_match_the_brute_force_at_each_rows_loop():
    """Each block position evaluated at its own loop equals the independent brute-force
    formulation run at that loop, row by row (a diagonal wave: older positions deeper)."""
    N, kvH, g, d, R, W, T, B = 1, 2, 2, 8, 6, 3, 20, 5
    c, PK, PV, src = _cache(N, kvH, g, d, R, W, T, B, seed=13, independent=True)
    loops = [5, 4, 2, 1, 0]
    q = src.queries(0, B, kvH * g)
    out, lse = orc.verify_wave(c, 0, loops, q, g, 1.1)
    Kall = np.stack([_f64(PK[pl][0]) for pl in range(R)])
    Vall = np.stack([_f64(PV[pl][0]) for pl in range(R)])
    for j, r in enumerate(loops):
        bo, bl = orc.brute_verify(Kall, Vall, T, B, r, W, g, _f64(q[0]), 1.1)
        assert np.abs(out[0, j] - bo[j]).max() < 1e-12
        assert np.abs(lse[0, j] - bl[j]).max() < 1e-12
    # a single loop for every position is the ordinary verification
    o1, _ = orc.verify_wave(c, 0, [3] * B, q, g)
    o2, _ = c.verify(0, 3, q, g)
    assert np.array_equal(o1, o2)


# ---------------------------------------------------------------- draft phase
def _prefix_cache(N, kvH, g, d, R, W, T, B, seed, max_extra=0):
    src = PlaneSource(N, kvH, d, R, T + B + max_extra, 0.88, seed, independent=True)
    PK = [src.plane(r, "K") for r in range(R)]
    PV = [src.plane(r, "V") for r in range(R)]
    c = orc.OracleCache(N, 1, kvH, d, R, W, T + B + max_extra)
    for pl in range(R):
        c.load_prefix(0, pl, [T] * N, PK[pl], PV[pl])
    return c, PK, PV, src


@pytest.mark.parametrize("T,W,B,r,g", [(20, 3, 5, 0, 2), (20, 0, 4, 1, 1), (6, 10, 4, 2, 3), (15, 5, 6, 4, 1),
                                       (0, 3, 4, 0, 1), (1, 0, 3, 2, 2)])
def test_draft_steps_match_the_brute_force(T, W, B, r, g):
    """Draft step j (one query at p = T + j, the drafts 0..j at plane r) equals row j of the
    independent brute-force formulation over the same planes; the drafted rows then verified
    as a block give the same rows."""
    N, kvH, d, R = 1, 2, 8, 5
    c, PK, PV, src = _prefix_cache(N, kvH, g, d, R, W, T, B, seed=17)
    Kall = np.stack([_f64(PK[pl][0]) for pl in range(R)])
    Vall = np.stack([_f64(PV[pl][0]) for pl in range(R)])
    kb, vb = block_from_planes(PK[r], T, B), block_from_planes(PV[r], T, B)
    q = src.queries(r, B, kvH * g)
    drafts = []
    for j in range(B):
        out, lse = c.draft(0, r, j, kb[:, j:j + 1], vb[:, j:j + 1], q[:, j:j + 1], g, 1.2)
        bo, bl = orc.brute_verify(Kall, Vall, T, j + 1, r, W, g, _f64(q[0, : j + 1]), 1.2)
        assert np.abs(out[0, 0] - bo[j]).max() < 1e-12
        assert np.abs(lse[0, 0] - bl[j]).max() < 1e-12
        if 0 < W < T and j >= 1 and r != R - 1:
            # planted mistake: the window measured from the cache end instead of the query
            bc, _ = orc.brute_verify(Kall, Vall, T, j + 1, r, W, g, _f64(q[0, : j + 1]), 1.2, orc.CACHE_RELATIVE)
            assert np.abs(out[0, 0] - bc[j]).max() > 1e-6
        drafts.append(out[0, 0])
    for pl in range(R):
        c.append(0, pl, block_from_planes(PK[pl], T, B), block_from_planes(PV[pl], T, B))
    vo, _ = c.verify(0, r, q, g, 1.2)
    for j in range(B):
        assert np.abs(vo[0, j] - drafts[j]).max() < 1e-12


def test_draft_state_rules():
    """Drafts are written in order per plane; redrafting makes later drafts stale; a
    verification block ends the draft phase; commit discards drafts past the block."""
    N, kvH, g, d, R, W, T, B = 1, 1, 1, 4, 3, 2, 8, 4
    c, PK, PV, src = _prefix_cache(N, kvH, g, d, R, W, T, B, seed=19, max_extra=2)
    kb, vb = block_from_planes(PK[0], T, B + 2), block_from_planes(PV[0], T, B + 2)
    q = src.queries(0, B + 2, kvH * g)
    step = lambda j: c.draft(0, 0, j, kb[:, j:j + 1], vb[:, j:j + 1], q[:, j:j + 1], g)
    with pytest.raises(RuntimeError):
        step(1)                                    # position 0 not drafted yet
    for j in range(B + 2):
        step(j)
    assert c.present[0, 0, 0, T:T + B + 2].all()
    step(2)                                        # redraft: positions 3.. of plane 0 are stale
    assert c.present[0, 0, 0, T:T + 3].all() and not c.present[0, 0, 0, T + 3:].any()
    with pytest.raises(RuntimeError):
        step(4)
    with pytest.raises(RuntimeError):
        c.load_prefix(0, 0, [T], PK[0], PV[0])     # a draft is in flight
    step(3)
    step(4)
    for pl in range(R):
        c.append(0, pl, block_from_planes(PK[pl], T, 2), block_from_planes(PV[pl], T, 2))
    with pytest.raises(RuntimeError):
        step(0)                                    # the verification block ended the draft phase
    c.commit([1])
    assert int(c.T[0]) == T + 1
    assert not c.present[0, :, 0, T + 1:].any()    # rejected block rows and drafts past the block
    assert c.drafted.sum() == 0


# ---------------------------------------------------------------- windowed draft attention
def test_windowed_draft_without_restriction_is_the_draft():
    """sink = 0 and a window reaching position 0: every key is attended, as in the draft."""
    N, kvH, g, d, R, W, T, B = 2, 2, 2, 8, 4, 5, 30, 4
    c, PK, PV, src = _prefix_cache(N, kvH, g, d, R, W, T, B, seed=29)
    kb, vb = block_from_planes(PK[1], T, B), block_from_planes(PV[1], T, B)
    q = src.queries(1, B, kvH * g)
    for j in range(B):
        a, la = c.draft(0, 1, j, kb[:, j:j + 1], vb[:, j:j + 1], q[:, j:j + 1], g, 1.1)
        b, lb = c.draft(0, 1, j, kb[:, j:j + 1], vb[:, j:j + 1], q[:, j:j + 1], g, 1.1, sink=0, window=T + j)
        assert np.abs(a - b).max() < 1e-12 and np.abs(la - lb).max() < 1e-12


@pytest.mark.parametrize("window", [0, 1, 3, 5])
def test_windowed_draft_inside_the_ripe_window_is_sdpa_on_plane_r(window):
    """No sink and a draft window no longer than the RIPE window: every attended key reads plane
    r, so the result is textbook attention over keys [p - window, p] of plane r (torch SDPA)."""
    N, kvH, g, d, R, W, T, B = 1, 2, 2, 8, 4, 5, 30, 3
    r = 1
    c, PK, PV, src = _prefix_cache(N, kvH, g, d, R, W, T, B, seed=31)
    kb, vb = block_from_planes(PK[r], T, B), block_from_planes(PV[r], T, B)
    q = src.queries(r, B, kvH * g)
    for j in range(B):
        out, _ = c.draft(0, r, j, kb[:, j:j + 1], vb[:, j:j + 1], q[:, j:j + 1], g, 1.0, sink=0, window=window)
        p = T + j
        K = _f64(PK[r][0, :, p - window:p + 1])          # [kvH][window+1][d], plane r
        V = _f64(PV[r][0, :, p - window:p + 1])
        qt = torch.from_numpy(_f64(q[0, j]))[:, None, :]  # [Hq][1][d]
        kt = torch.from_numpy(K).repeat_interleave(g, dim=0)
        vt = torch.from_numpy(V).repeat_interleave(g, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=1.0)[:, 0].numpy()
        assert np.abs(out[0, 0] - ref).max() < 1e-12


def test_windowed_draft_ignores_keys_between_sink_and_window():
    """Keys between the sink and the window do not enter the result; sink and window keys do."""
    N, kvH, g, d, R, W, T, B = 1, 1, 1, 8, 3, 4, 40, 2
    c, PK, PV, src = _prefix_cache(N, kvH, g, d, R, W, T, B, seed=37)
    kb, vb = block_from_planes(PK[0], T, B), block_from_planes(PV[0], T, B)
    q = src.queries(0, B, 1)
    sink, window = 3, 6
    base, _ = c.draft(0, 0, 0, kb[:, :1], vb[:, :1], q[:, :1], g, 1.0, sink=sink, window=window)
    for t, inside in ((10, False), (25, False), (1, True), (T - 2, True)):
        plane = R - 1 if t < T - W else 0
        saved = c.values(0, plane, "V")[0, 0, t].copy()
        bumped = (_f64(saved) + 3.0).astype(np.float32).view(np.uint32) >> np.uint32(16)
        c.values(0, plane, "V")[0, 0, t] = bumped.astype(np.uint16)   # that value + 3
        moved, _ = c.draft(0, 0, 0, kb[:, :1], vb[:, :1], q[:, :1], g, 1.0, sink=sink, window=window)
        c.values(0, plane, "V")[0, 0, t] = saved
        assert (np.abs(moved - base).max() > 1e-6) == inside, t
