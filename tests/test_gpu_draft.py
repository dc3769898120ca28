"""GPU parity of ripe_draft_attn (the draft phase: one block position at a shallow loop)
against the CPU oracle, element by element, and against the verification of the same block.

Draft-then-verify builds the draft block one position at a time at a few loops, then checks
it at every loop.  Each draft step writes plane r of position T + j and attends with the
verification rule for the query p = T + j.  Shapes: several 64-key tiles and a ragged tail,
T < W and T = 0, ring wrap-around, GQA groups, the deepest loop, and the Huginn-shaped cache.
"""
import numpy as np
import pytest
import torch

from harness import Case, assert_same_result, check_close, check_lse
from self_speculative_decode_b200.ripe import RipeError

pytestmark = pytest.mark.gpu


def _rows(x, j):
    return np.ascontiguousarray(x[:, j:j + 1]) if isinstance(x, np.ndarray) else x[:, j:j + 1].contiguous()


def _draft_phase(c, layer, loops, J, scale=1.0):
    """Draft positions 0..J-1 at every loop of ``loops`` on both sides (position-major, as a
    decoder drafts); returns {(j, r): gpu out [N][1][Hq][d]}."""
    idx_n = torch.tensor(c.oseq, device=c.device)
    idx_h = torch.tensor(c.oheads, device=c.device)
    outs = {}
    for j in range(J):
        for r in loops:
            kb, vb = c.blocks[(layer, r)]
            k1, v1 = _rows(kb, j), _rows(vb, j)
            q = c.src[layer].queries(r, c.B, c.Hq, 0)
            q1 = _rows(q, j)
            lse = torch.empty((c.N, 1, c.Hq), dtype=torch.float32, device=c.device)
            out = c.gpu.draft_attn(layer, r, j, c._dev(k1), c._dev(v1), c._dev(q1), lse=lse, scale=scale)
            ro, rl = c.orc.draft(layer, r, j, c._sub_block(k1), c._sub_block(v1),
                                 np.ascontiguousarray(c._host(q1)[c.oseq][:, :, c.oheads]), c.g, scale)
            check_close(out.index_select(0, idx_n).index_select(2, idx_h), ro, f"draft j={j} loop {r}")
            check_lse(lse.index_select(0, idx_n).index_select(2, idx_h), rl)
            outs[(j, r)] = out.clone()
    return outs


def _then_verify(c, layer, loops, outs, J):
    """Append the block (the same rows) and verify: row j equals draft step j."""
    c.append_blocks()
    for r in loops:
        qd, _ = c.queries(layer, r, 0)
        v = c.gpu.verify_attn(layer, r, qd)
        for j in range(J):
            assert_same_result(v[:, j:j + 1], outs[(j, r)], f"verify row {j} vs draft, loop {r}")


@pytest.mark.parametrize("kw", [
    dict(N=3, Hq=8, kvH=4, d=128, R=6, T=[300, 40, 7], W=16, B=8),     # GQA 2, T < W, ring wrap
    dict(N=2, Hq=3, kvH=3, d=96, R=4, T=[0, 129], W=5, B=6),           # empty prefix, ragged tail
    dict(N=2, Hq=4, kvH=1, d=64, R=3, T=[70, 64], W=0, B=4),           # deepest-only layout, g = 4
    dict(N=1, Hq=2, kvH=2, d=64, R=3, T=[200], W=10 ** 6, B=5),       # full cache
    dict(N=2, Hq=60, kvH=30, d=96, R=4, T=[500, 500], W=16, B=8),      # two CTAs per head (cluster pairs)
])
def test_draft_phase_parity(kw, cuda_device):
    c = Case(L=1, seed=21, independent=True, append_block=False, **kw)
    loops = [0, 1, kw["R"] - 1]
    outs = _draft_phase(c, 0, loops, kw["B"])
    _then_verify(c, 0, loops, outs, kw["B"])
    c.close()


def test_draft_phase_huginn_shape(cuda_device):
    """55 MHA heads x 96, R=32, T=1024, W=64: drafts of 8 positions at loops 0..3, sampled heads."""
    loops = [0, 1, 2, 3]
    c = Case(N=1, L=1, Hq=55, kvH=55, d=96, R=32, T=1024, W=64, B=8, rho=0.88, seed=23, backend="torch",
             oracle_kvh=[0, 13, 54], oracle_planes=set(loops + [31]), append_block=False)
    outs = _draft_phase(c, 0, loops, 8)
    _then_verify(c, 0, loops, outs, 8)
    c.close()


def test_draft_redraft_and_state_errors(cuda_device):
    """Redrafting position j replaces its row; out-of-order drafts, drafts inside a
    verification block and a prefix load during the draft phase are refused."""
    c = Case(N=2, L=1, Hq=2, kvH=2, d=64, R=3, T=[90, 33], W=8, B=4, seed=25, independent=True,
             append_block=False)
    kb, vb = c.blocks[(0, 0)]
    q = c.src[0].queries(0, c.B, c.Hq, 0)
    step = lambda j, k=kb, v=vb: c.gpu.draft_attn(0, 0, j, c._dev(_rows(k, j)), c._dev(_rows(v, j)),
                                                  c._dev(_rows(q, j)))
    with pytest.raises(RipeError):
        step(1)
    step(0)
    step(1)
    step(2)
    # redraft position 1 with other values: position 2 becomes stale, so 3 is refused
    kb2, vb2 = c.blocks[(0, 1)]
    out = step(1, kb2, vb2)
    ro, _ = c.orc.draft(0, 0, 0, c._sub_block(_rows(kb, 0)), c._sub_block(_rows(vb, 0)),
                        np.ascontiguousarray(c._host(_rows(q, 0))), c.g)
    ro, _ = c.orc.draft(0, 0, 1, c._sub_block(_rows(kb2, 1)), c._sub_block(_rows(vb2, 1)),
                        np.ascontiguousarray(c._host(_rows(q, 1))), c.g)
    check_close(out, ro, "redraft")
    with pytest.raises(RipeError):
        step(3)
    with pytest.raises(RipeError):
        c.gpu.load_prefix(0, 0, c.T, torch.zeros((2, 2, 100, 64), dtype=torch.bfloat16, device=c.device),
                          torch.zeros((2, 2, 100, 64), dtype=torch.bfloat16, device=c.device))
    c.append_blocks()
    with pytest.raises(RipeError):
        step(0)
    c.gpu.commit([2, 1])
    c.orc.commit([2, 1])
    assert c.gpu.sync_lengths() == [92, 34]
    step(0)                      # a new draft phase after the commit
    c.close()


@pytest.mark.parametrize("kw,sink,window", [
    (dict(N=2, Hq=4, kvH=2, d=128, R=4, T=[700, 300], W=16, B=6), 4, 40),      # window reaches the deep region
    (dict(N=2, Hq=3, kvH=3, d=96, R=3, T=[900, 77], W=32, B=8), 100, 10),      # two sink tiles; sink covers seq 1
    (dict(N=1, Hq=2, kvH=2, d=64, R=3, T=[500], W=0, B=4), 1, 0),              # deepest only: sink + the query
    (dict(N=2, Hq=60, kvH=30, d=96, R=4, T=[600, 600], W=16, B=8), 4, 200),    # two CTAs per head
    (dict(N=1, Hq=2, kvH=2, d=64, R=3, T=[300], W=10 ** 6, B=5), 8, 64),       # full cache
])
def test_windowed_draft_parity(kw, sink, window, cuda_device):
    """Windowed draft attention (attention sink + sliding window on the draft only) against the
    oracle; with a window reaching position 0 it equals the plain draft step."""
    c = Case(L=1, seed=43, independent=True, append_block=False, **kw)
    idx_n = torch.tensor(c.oseq, device=c.device)
    idx_h = torch.tensor(c.oheads, device=c.device)
    loops = [0, kw["R"] - 1]
    for j in range(kw["B"]):
        for r in loops:
            kb, vb = c.blocks[(0, r)]
            k1, v1 = _rows(kb, j), _rows(vb, j)
            q1 = _rows(c.src[0].queries(r, c.B, c.Hq, 0), j)
            lse = torch.empty((c.N, 1, c.Hq), dtype=torch.float32, device=c.device)
            out = c.gpu.draft_attn(0, r, j, c._dev(k1), c._dev(v1), c._dev(q1), lse=lse, sink=sink, window=window)
            ro, rl = c.orc.draft(0, r, j, c._sub_block(k1), c._sub_block(v1),
                                 np.ascontiguousarray(c._host(q1)[c.oseq][:, :, c.oheads]), c.g,
                                 sink=sink, window=window)
            check_close(out.index_select(0, idx_n).index_select(2, idx_h), ro, f"windowed draft j={j} loop {r}")
            check_lse(lse.index_select(0, idx_n).index_select(2, idx_h), rl)
            if j == 0:
                full = c.gpu.draft_attn(0, r, j, c._dev(k1), c._dev(v1), c._dev(q1), sink=0, window=1 << 20)
                plain = c.gpu.draft_attn(0, r, j, c._dev(k1), c._dev(v1), c._dev(q1))
                assert torch.equal(full, plain)
    c.close()
