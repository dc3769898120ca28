"""GPU parity at the workloads' full sizes, on outputs the oracle computes one by one.

* window/block sweep: 55 MHA heads x 96, R=32, T=4096, batch 4, rho 0.81,
  W in {0, 8, 64, 256, 4096} x B in {4, 8, 16}; sampled (sequence, kv head) pairs checked
  against the oracle, and block-split independence checked on the GPU for every W >= B-1;
* long-context GQA: 32 q / 8 kv heads x 128, R=32, T=32768, W=64, B=8, batch 8, rho 0.85
  (one layer of four), RIPE and full-cache layouts; and the same with 64 q heads (64 query rows
  per kv head);
* streaming decode: 16 sequences, Huginn heads, R=32, W=64, B=8, accepted lengths drawn
  U{0..8} per step, fresh drafts every step, from T0=512 and from ragged lengths near 4000
  (where 1000 steps end): verify parity on sampled steps, loops, sequences and heads, and the
  exported cache state bit-exact against the oracle's;
* edge shapes: B=1 (draft-phase decode), R=1, 64 query rows per kv head.
"""
import numpy as np
import pytest
import torch

from harness import Case, assert_same_result, check_close, check_lse, dev_to_bits
from oracle import ripe_oracle as orc
from self_speculative_decode_b200.ripe import RipeCache
from self_speculative_decode_b200.synth import PlaneSource, acceptance_draws

pytestmark = pytest.mark.gpu

SWEEP_W = [0, 8, 64, 256, 4096]
SWEEP_B = [4, 8, 16]


@pytest.mark.parametrize("B", SWEEP_B)
@pytest.mark.parametrize("W", SWEEP_W)
def test_window_block_sweep_sampled(W, B, cuda_device):
    loops = [0, 15, 31]
    c = Case(N=4, L=1, Hq=55, kvH=55, d=96, R=32, T=4096, W=W, B=B, rho=0.81, seed=100 + W + B,
             backend="torch", oracle_seqs=[0, 3], oracle_kvh=[0, 27, 54], oracle_planes=set(loops))
    for r in loops:
        c.check(0, r)
    c.close()


@pytest.mark.parametrize("W,B", [(w, b) for w in SWEEP_W for b in SWEEP_B if w >= b - 1])
def test_window_block_sweep_block_independence(W, B, cuda_device):
    """Two blocks of B vs 2B blocks of 1 over the same positions give the same outputs (W >= B-1).

    Both decodes are also checked against the oracle at every position on sampled heads."""
    N, kvH, d, R, T0 = 4, 55, 96, 32, 4096
    S = 2 * B
    loops = [0, 30, 31]
    seqs, heads = [0, 2], [0, 31]
    src = PlaneSource(N, kvH, d, R, T0 + S, 0.81, 7, backend="torch", device=cuda_device)
    qsrc = PlaneSource(N, kvH, d, R, T0 + S, 0.81, 8, backend="torch", device=cuda_device)
    caches = {blk: RipeCache(N, 1, kvH, kvH, d, R, W, T0 + S, blk) for blk in (B, 1)}
    oracles = {blk: orc.OracleCache(len(seqs), 1, len(heads), d, R, W, T0 + S, value_planes=set(loops))
               for blk in (B, 1)}
    sub = lambda x: np.ascontiguousarray(dev_to_bits(x)[seqs][:, heads])
    subb = lambda x: np.ascontiguousarray(dev_to_bits(x)[seqs][:, :, heads])
    tail = []                                    # planes of positions [T0, T0 + S), block layout
    for pl in range(R):
        k, v = src.plane(pl, "K"), src.plane(pl, "V")
        for cache in caches.values():
            cache.load_prefix(0, pl, [T0] * N, k, v)
        for oc in oracles.values():
            keep = pl in loops
            oc.load_prefix(0, pl, [T0] * len(seqs), sub(k) if keep else None, sub(v) if keep else None)
        tail.append((k[:, :, T0:].permute(0, 2, 1, 3).contiguous(), v[:, :, T0:].permute(0, 2, 1, 3).contiguous()))
        del k, v
    src.release()
    Q = {r: qsrc.plane(r, "K")[:, :, T0:].permute(0, 2, 1, 3).contiguous() for r in loops}
    nsel, hsel = torch.tensor(seqs, device=cuda_device), torch.tensor(heads, device=cuda_device)

    def decode(block):
        cache, oc = caches[block], oracles[block]
        outs = {}
        for t in range(0, S, block):
            for pl in range(R):
                kb, vb = tail[pl][0][:, t:t + block].contiguous(), tail[pl][1][:, t:t + block].contiguous()
                cache.append_block(0, pl, kb, vb)
                if pl in loops:
                    oc.append(0, pl, subb(kb), subb(vb))
                else:
                    oc.append(0, pl, None, None, B=block)
            for r in loops:
                q = Q[r][:, t:t + block].contiguous()
                lse = torch.empty((N, block, kvH), dtype=torch.float32, device=cuda_device)
                out = cache.verify_attn(0, r, q, lse=lse)
                ro, rl = oc.verify(0, r, subb(q), 1)
                check_close(out.index_select(0, nsel).index_select(2, hsel), ro, f"block {block} pos {t} loop {r}")
                check_lse(lse.index_select(0, nsel).index_select(2, hsel), rl)
                for j in range(block):
                    outs[(t + j, r)] = out[:, j].clone()
            cache.commit([block] * N)
            oc.commit([block] * len(seqs))
        assert cache.device_error() == 0
        cache.close()
        return outs

    a, b = decode(B), decode(1)
    for key in a:
        assert_same_result(a[key], b[key], f"position {key[0]} loop {key[1]}")


@pytest.mark.parametrize("layout", ["ripe", "full"])
def test_long_context_gqa_sampled(layout, cuda_device):
    loops = [0, 17, 31] if layout == "ripe" else [0, 31]
    c = Case(N=8, L=1, Hq=32, kvH=8, d=128, R=32, T=32768, W=64 if layout == "ripe" else 10 ** 6, B=8,
             rho=0.85, seed=5, backend="torch", oracle_seqs=[0, 7], oracle_kvh=[0, 5],
             oracle_planes=set(loops))
    for r in loops:
        c.check(0, r)
    c.close()


def test_long_context_64_rows_sampled(cuda_device):
    """64 query rows per kv head (GQA 8, block 8), head_dim 128, 32K keys (tests/test_gpu_consumers.py
    reruns it on each consumer)."""
    c = Case(N=8, L=1, Hq=64, kvH=8, d=128, R=4, T=32768, W=64, B=8, rho=0.85, seed=9, backend="torch",
             oracle_seqs=[0, 7], oracle_kvh=[0, 5], oracle_planes={0, 3})
    for r in (0, 3):
        c.check(0, r)
    c.close()


def _streaming(T0, steps, seed, device):
    """16 sequences, Huginn heads, R=32, W=64, B=8 from committed lengths T0 (one per sequence):
    fresh block planes every step, accepted lengths U{0..8}; verify parity on sampled steps, loops,
    sequences and heads, then the exported cache state bit for bit."""
    N, kvH, d, R, W, B = 16, 55, 96, 32, 64, 8
    loops_checked = [0, 31]
    seqs, heads = [0, 5, 15], [0, 54]
    acc = acceptance_draws(seed, steps, N, B)
    max_T = max(T0) + B * (steps + 1)
    src = PlaneSource(N, kvH, d, R, max(T0), 0.88, seed, backend="torch", device=device)
    gpu = RipeCache(N, 1, kvH, kvH, d, R, W, max_T, B)
    oc = orc.OracleCache(len(seqs), 1, len(heads), d, R, W, max_T, value_planes=set(loops_checked))
    sub = lambda x: np.ascontiguousarray(dev_to_bits(x)[seqs][:, heads])
    subb = lambda x: np.ascontiguousarray(dev_to_bits(x)[seqs][:, :, heads])
    To = [T0[n] for n in seqs]
    for pl in range(R):
        k, v = src.plane(pl, "K"), src.plane(pl, "V")
        gpu.load_prefix(0, pl, T0, k, v)
        keep = pl in loops_checked
        oc.load_prefix(0, pl, To, sub(k) if keep else None, sub(v) if keep else None)
        del k, v
    src.release()
    hsel = torch.tensor(heads, device=device)
    nsel = torch.tensor(seqs, device=device)
    for step in range(steps):
        for pl in range(R):
            kb, vb = src.block(step, pl, B, "K"), src.block(step, pl, B, "V")
            gpu.append_block(0, pl, kb, vb)
            if pl in loops_checked:
                oc.append(0, pl, subb(kb), subb(vb))
            else:
                oc.append(0, pl, None, None, B=B)
        for r in range(R):
            q = src.queries(r, B, kvH, step)
            lse = torch.empty((N, B, kvH), dtype=torch.float32, device=device)
            out = gpu.verify_attn(0, r, q, lse=lse)
            if r in loops_checked and step in (0, steps // 2, steps - 1):
                ro, rl = oc.verify(0, r, subb(q), 1)
                check_close(out.index_select(0, nsel).index_select(2, hsel), ro, f"step {step} loop {r}")
                check_lse(lse.index_select(0, nsel).index_select(2, hsel), rl)
        gpu.commit(acc[step])
        oc.commit(acc[step][seqs])
    T = gpu.sync_lengths()
    assert T == [T0[n] + int(x) for n, x in enumerate(acc.sum(0))]
    assert len(set(T)) > 1                       # ragged lengths
    for i, n in enumerate(seqs):                 # exported state of the sampled sequences, bit for bit
        k, v, present = gpu.export(n, 0)
        pres = oc.present[0, :, i, : T[n]]
        np.testing.assert_array_equal(present.cpu().numpy().astype(bool), pres)
        kb, vbits = dev_to_bits(k), dev_to_bits(v)
        for pl in loops_checked:
            m = pres[pl][None, :, None]
            for which, bits in (("K", kb), ("V", vbits)):
                ok = oc.values(0, pl, which)[i, :, : T[n]]
                np.testing.assert_array_equal(np.where(m, bits[pl][heads], 0), np.where(m, ok, 0))
    assert gpu.device_error() == 0
    gpu.close()


def test_streaming_decode_with_maintenance(cuda_device):
    """The streaming workload from its start: every sequence at T0 = 512."""
    _streaming([512] * 16, 24, 3, cuda_device)


def test_streaming_decode_late_lengths(cuda_device):
    """The streaming workload near where it ends (about 4000 committed positions after 1000 steps
    of U{0..8} accepted lengths): ragged starting lengths 3900..4400, 24 more steps."""
    rng = np.random.default_rng(17)
    T0 = [int(x) for x in rng.integers(3900, 4401, size=16)]
    _streaming(T0, 24, 17, cuda_device)


@pytest.mark.parametrize("kw", [
    dict(N=3, L=1, Hq=8, kvH=2, d=128, R=6, T=[900, 33, 2], W=64, B=1),      # draft-phase decode shape
    dict(N=2, L=1, Hq=4, kvH=4, d=96, R=1, T=[500, 77], W=16, B=8),          # one loop: ordinary attention
    dict(N=2, L=1, Hq=64, kvH=8, d=128, R=3, T=[700, 64], W=20, B=8),        # 64 query rows per kv head
    dict(N=1, L=1, Hq=2, kvH=1, d=64, R=2, T=[63], W=63, B=1),               # a single key tile, W = T
    dict(N=1024, L=1, Hq=2, kvH=1, d=64, R=2, T=[(37 * n) % 97 for n in range(1024)], W=8, B=2),
    # the largest batch a cache takes, ragged lengths 0..96
])
def test_edge_shapes(kw, cuda_device):
    c = Case(**kw, seed=9, independent=True)
    for r in range(kw["R"]):
        c.check(0, r)
    c.close()
