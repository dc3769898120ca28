"""GPU parity of ripe_verify_attn against the CPU oracle (element by element).

Tolerance: max abs <= 2e-2 and relative L2 <= 5e-3 on the bf16 output (bf16 inputs,
fp32 accumulation); lse within 1e-3 (harness.LSE_ABS).  Sizes span several 64-key tiles, ragged tails,
ring wrap-around, splits of one (sequence, kv head) over many CTAs, and the three
layouts: full cache (W >= max_T), RIPE, deepest plane only (W = 0).
"""
import numpy as np
import pytest
import torch

from harness import Case, assert_same_result, check_close

pytestmark = pytest.mark.gpu

LAYOUTS = {"full": 10 ** 6, "ripe": 16, "deepest": 0}


@pytest.mark.parametrize("layout", ["full", "ripe", "deepest"])
def test_tiny_config_every_loop(layout, cuda_device):
    """1 layer, 2 heads, d=64, R=4, T=128, W=16, B=4, batch 1, rho 0.88, seed 0."""
    c = Case(N=1, L=1, Hq=2, kvH=2, d=64, R=4, T=128, W=LAYOUTS[layout], B=4, rho=0.88, seed=0)
    for r in range(4):
        c.check(0, r)
    c.close()


def test_tiny_config_cache_relative_window(cuda_device):
    c = Case(N=1, L=1, Hq=2, kvH=2, d=64, R=4, T=128, W=16, B=4, rho=0.88, seed=0, mode=1)
    for r in range(4):
        c.check(0, r)
    c.close()


@pytest.mark.parametrize("d,g,B,W", [(96, 2, 6, 5), (64, 1, 16, 3), (128, 4, 8, 9), (128, 4, 16, 40),
                                     (96, 1, 8, 0), (64, 3, 5, 70)])
def test_ragged_tagged_planes(d, g, B, W, cuda_device):
    """Independent planes: any wrong plane choice moves the output by O(1)."""
    kvH = 3
    T = [0, 1, 37, 200, 129]
    c = Case(N=5, L=2, Hq=kvH * g, kvH=kvH, d=d, R=5, T=T, W=W, B=B, seed=3, independent=True,
             max_T=max(T) + B + 11)
    for layer in range(2):
        for r in range(5):
            c.check(layer, r)
    c.close()


@pytest.mark.parametrize("d,g,B", [(64, 1, 8), (128, 4, 8), (128, 4, 16), (96, 2, 12)])
def test_long_pair_split_over_many_ctas(d, g, B, cuda_device):
    """One sequence and one kv head over thousands of keys: the merge of many partials."""
    c = Case(N=1, L=1, Hq=g, kvH=1, d=d, R=3, T=5000, W=64, B=B, seed=4, independent=True)
    for r in range(3):
        c.check(0, r)
    c.close()


def test_large_logit_scale(cuda_device):
    """scale 8 gives logits of std ~8: the online softmax max handling matters."""
    c = Case(N=2, L=1, Hq=4, kvH=2, d=64, R=3, T=[300, 77], W=20, B=8, seed=5)
    for r in range(3):
        c.check(0, r, scale=8.0)
    c.close()



@pytest.mark.parametrize("g,B", [(1, 8), (4, 8)])
def test_degenerate_logit_scales(g, B, cuda_device):
    """Scale 0 (uniform weights over the visible keys: every tile's logits tie) and negative scales
    (the largest logit comes from the smallest score), on 8 and 32 query rows per kv head."""
    c = Case(N=2, L=1, Hq=2 * g, kvH=2, d=128, R=3, T=[300, 77], W=20, B=B, seed=6, independent=True)
    for r in range(3):
        for scale in (0.0, -1.0, -8.0):
            c.check(0, r, scale=scale)
    c.close()


@pytest.mark.parametrize("layout", ["full", "ripe", "deepest"])
def test_huginn_shape(layout, cuda_device):
    """4 recurrent layers, 55 MHA heads x 96, R=32, T=1024, W=64, B=8, batch 1, rho 0.88."""
    loops = [0, 1, 17, 30, 31]
    c = Case(N=1, L=4, Hq=55, kvH=55, d=96, R=32, T=1024, W=LAYOUTS[layout] if layout != "ripe" else 64,
             B=8, rho=0.88, seed=1, backend="torch", oracle_planes=set(loops + [31]))
    for layer in range(4):
        for r in loops:
            c.check(layer, r)
    c.close()


def test_block_split_independence_on_gpu(cuda_device):
    """W >= B: verifying 16 positions as 2 blocks of 8 or 16 blocks of 1 gives the same outputs."""
    from self_speculative_decode_b200.ripe import RipeCache
    from self_speculative_decode_b200.synth import PlaneSource

    N, kvH, g, d, R, W, T0, S = 2, 3, 2, 96, 4, 8, 700, 16
    dev = torch.device("cuda")
    src = PlaneSource(N, kvH, d, R, T0 + S, 0.81, 9, backend="torch", device=dev)
    P = [(src.plane(r, "K"), src.plane(r, "V")) for r in range(R)]
    qsrc = PlaneSource(N, kvH * g, d, R, T0 + S, 0.81, 10, backend="torch", device=dev)
    Q = [qsrc.plane(r, "K") for r in range(R)]   # per-position queries [N][Hq][pos][d]

    def decode(block):
        c = RipeCache(N, 1, kvH * g, kvH, d, R, W, T0 + S, block)
        for r in range(R):
            c.load_prefix(0, r, [T0] * N, P[r][0], P[r][1])
        outs = {}
        for t in range(T0, T0 + S, block):
            for r in range(R):
                c.append_block(0, r, P[r][0][:, :, t:t + block].permute(0, 2, 1, 3).contiguous(),
                               P[r][1][:, :, t:t + block].permute(0, 2, 1, 3).contiguous())
            for r in range(R):
                q = Q[r][:, :, t:t + block].permute(0, 2, 1, 3).contiguous()
                out = c.verify_attn(0, r, q)
                for j in range(block):
                    outs[(t + j, r)] = out[:, j].clone()
            c.commit([block] * N)
        assert c.device_error() == 0
        c.close()
        return outs

    a, b = decode(8), decode(1)
    # same keys and planes: both splits are within the parity tolerance of the exact value
    for key in a:
        assert_same_result(a[key], b[key], f"position {key[0]} loop {key[1]}")


@pytest.mark.parametrize("kw", [
    dict(N=2, Hq=30, kvH=30, d=96, R=4, T=[700, 700], W=64, B=8),            # 60 heads, two sequences
    dict(N=3, Hq=48, kvH=24, d=128, R=3, T=[900, 900, 900], W=32, B=8),      # GQA 2: 16 query rows
    dict(N=1, Hq=40, kvH=40, d=64, R=3, T=[2000], W=16, B=4),                # three CTAs per head
])
def test_heads_split_over_ctas(kw, cuda_device):
    """Fewer heads than SMs with equal lengths: each head is split into equal pieces, one per CTA.
    Two pieces are merged inside a 2-CTA cluster through shared memory; more go through global
    scratch.  Independent planes, every loop."""
    c = Case(L=1, seed=41, independent=True, **kw)
    for r in range(kw["R"]):
        c.check(0, r)
    c.close()


def test_live_caches_of_different_batch(cuda_device):
    """A cache of batch 16 stays usable after a cache of batch 1 is allocated (and used) on the
    same device: a launch asks for shared memory that grows with the batch, and allocating a
    smaller cache must not lower the kernels' limit below what the larger one asks for."""
    T16 = [130 + 37 * n for n in range(16)]
    big = Case(N=16, L=1, Hq=4, kvH=2, d=96, R=3, T=T16, W=16, B=4, seed=12, independent=True,
               oracle_seqs=[0, 7, 15])
    for r in range(3):
        big.check(0, r)
    small = Case(N=1, L=1, Hq=4, kvH=2, d=96, R=3, T=[200], W=16, B=4, seed=13, independent=True)
    for r in range(3):
        small.check(0, r)
        big.check(0, r)
    small.close()
    for r in range(3):
        big.check(0, r)
    big.close()
