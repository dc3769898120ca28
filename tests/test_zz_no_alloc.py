"""ripe_verify_attn_static, the entry point that allocates nothing.

Some callers cannot call cudaMalloc: their device memory belongs to an inference engine's
pool or to a framework that preallocates everything, or they run while a stream capture is
open.  For them the library verifies over cache buffers the caller owns, with its scratch
in a fixed device array inside the library.  This test fills such buffers (the test itself
may allocate) in the documented layout from the same synthetic planes as a regular cache,
and checks that two calls in a row give what ripe_verify_attn gives, within the tolerance of
the other parity tests.  It lives in its own file so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import numpy as np

from harness import Case, check_close, check_lse, dev_to_bits
from oracle import ripe_oracle as orc
from self_speculative_decode_b200 import ripe
from self_speculative_decode_b200.ripe import CacheView, RipeCache, RipeError
from self_speculative_decode_b200.synth import PlaneSource

pytestmark = pytest.mark.gpu


def _layout(planes, T, W, B, R, max_T, max_B):
    """Deepest-plane region and window ring of one layer in the library's documented layout."""
    K = planes  # list over planes of [N][kvH][len][d]
    N, kvH, _, d = K[0].shape
    Wc = min(W, max_T)
    S = min(Wc + max_B, max_T)
    deep = torch.zeros((N, kvH, max_T - Wc, d), dtype=torch.bfloat16, device=K[0].device)
    ring = torch.zeros((N, R, kvH, S, d), dtype=torch.bfloat16, device=K[0].device)
    for n in range(N):
        lo = max(0, T[n] - Wc)
        if lo:
            deep[n, :, :lo] = K[R - 1][n, :, :lo]
        for t in range(lo, T[n] + B):
            for pl in range(R):
                ring[n, pl, :, t % S] = K[pl][n, :, t]
    return deep, ring


@pytest.mark.parametrize("W,g,B,d", [(5, 2, 6, 96), (64, 4, 8, 128), (0, 1, 8, 64)])
def test_static_entry_matches_cache_entry(W, g, B, d, cuda_device):
    N, L, kvH, R = 3, 2, 3, 4
    T = [40, 7, 150]
    max_B, max_T = B, 170
    Hq = kvH * g
    src = [PlaneSource(N, kvH, d, R, max_T, 0.88, 21, layer=l, independent=True, backend="torch",
                       device=cuda_device) for l in range(L)]
    PK = [[src[l].plane(pl, "K") for pl in range(R)] for l in range(L)]
    PV = [[src[l].plane(pl, "V") for pl in range(R)] for l in range(L)]

    cache = RipeCache(N, L, Hq, kvH, d, R, W, max_T, max_B)
    for l in range(L):
        for pl in range(R):
            cache.load_prefix(l, pl, T, PK[l][pl], PV[l][pl])
    for l in range(L):
        for pl in range(R):
            kb = torch.stack([PK[l][pl][n, :, T[n]:T[n] + B].permute(1, 0, 2) for n in range(N)]).contiguous()
            vb = torch.stack([PV[l][pl][n, :, T[n]:T[n] + B].permute(1, 0, 2) for n in range(N)]).contiguous()
            cache.append_block(l, pl, kb, vb)

    lay = [(_layout(PK[l], T, W, B, R, max_T, max_B), _layout(PV[l], T, W, B, R, max_T, max_B)) for l in range(L)]
    k_deep = torch.stack([x[0][0] for x in lay]).contiguous()
    v_deep = torch.stack([x[1][0] for x in lay]).contiguous()
    k_ring = torch.stack([x[0][1] for x in lay]).contiguous()
    v_ring = torch.stack([x[1][1] for x in lay]).contiguous()
    lengths = torch.tensor(T, dtype=torch.int32, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    view = CacheView(batch=N, layers=L, q_heads=Hq, kv_heads=kvH, head_dim=d, loops=R, window=W, max_T=max_T,
                     max_B=max_B, window_mode=0, block_len=B,
                     k_deep=k_deep.data_ptr() if k_deep.numel() else None,
                     v_deep=v_deep.data_ptr() if v_deep.numel() else None,
                     k_ring=k_ring.data_ptr(), v_ring=v_ring.data_ptr(), lengths=lengths.data_ptr())

    for layer in range(L):
        for r in (0, R - 2, R - 1):
            q = src[layer].queries(r, B, Hq)
            lse_ref = torch.empty((N, B, Hq), dtype=torch.float32, device=cuda_device)
            ref = cache.verify_attn(layer, r, q, lse=lse_ref)
            for _ in range(2):   # two calls in a row share and reuse the static scratch
                out = torch.full_like(ref, float("nan"))
                lse = torch.empty_like(lse_ref)
                ripe.ripe_verify_attn_static(view, layer, r, q.data_ptr(), out.data_ptr(), lse.data_ptr(), 1.0,
                                             err.data_ptr())
                torch.cuda.synchronize()
                check_close(out, ref.double().cpu().numpy(), f"static layer {layer} loop {r}")
                check_lse(lse, lse_ref.double().cpu().numpy())
    # one call against the CPU oracle directly (layer 1, loop R-2: window, block and deepest keys)
    layer, r = 1, R - 2
    oc = orc.OracleCache(N, 1, kvH, d, R, W, max_T)
    for pl in range(R):
        oc.load_prefix(0, pl, T, dev_to_bits(PK[layer][pl]), dev_to_bits(PV[layer][pl]))
    for pl in range(R):
        kb = torch.stack([PK[layer][pl][n, :, T[n]:T[n] + B].permute(1, 0, 2) for n in range(N)])
        vb = torch.stack([PV[layer][pl][n, :, T[n]:T[n] + B].permute(1, 0, 2) for n in range(N)])
        oc.append(0, pl, dev_to_bits(kb), dev_to_bits(vb))
    q = src[layer].queries(r, B, Hq)
    out = torch.empty((N, B, Hq, d), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((N, B, Hq), dtype=torch.float32, device=cuda_device)
    ripe.ripe_verify_attn_static(view, layer, r, q.data_ptr(), out.data_ptr(), lse.data_ptr(), 1.0, err.data_ptr())
    ro, rl = oc.verify(0, r, np.ascontiguousarray(dev_to_bits(q)), g)
    check_close(out, ro, "static vs oracle")
    check_lse(lse, rl)
    assert int(err.item()) == 0
    assert cache.device_error() == 0
    cache.close()


def test_static_entry_rejects_problems_beyond_its_scratch(cuda_device):
    big = CacheView(batch=1024, layers=1, q_heads=64, kv_heads=64, head_dim=128, loops=4, window=8, max_T=64,
                    max_B=8, window_mode=0, block_len=8, k_deep=1 << 20, v_deep=1 << 20, k_ring=1 << 20,
                    v_ring=1 << 20, lengths=1 << 20)
    with pytest.raises(RipeError) as e:
        ripe.ripe_verify_attn_static(big, 0, 0, 1 << 20, 1 << 20)
    assert e.value.status == ripe.RIPE_ESCRATCH


def test_static_call_leaves_larger_caches_usable(cuda_device):
    """A cache of batch 16 and one of batch 1 are live; an allocation-free call at batch 1 runs;
    the batch-16 cache then still verifies within tolerance of the CPU oracle, and every call
    returns RIPE_OK.  (A launch asks for shared memory that grows with the batch: no call may
    lower the kernels' limit below what a live cache of a larger batch needs.)"""
    N, kvH, g, d, R, W, B = 1, 2, 2, 96, 3, 16, 4
    T16 = [130 + 37 * n for n in range(16)]
    big = Case(N=16, L=1, Hq=kvH * g, kvH=kvH, d=d, R=R, T=T16, W=W, B=B, seed=14, independent=True,
               oracle_seqs=[0, 9, 15])
    small = Case(N=1, L=1, Hq=kvH * g, kvH=kvH, d=d, R=R, T=[300], W=W, B=B, seed=15, independent=True,
                 backend="torch")
    # the allocation-free view of a batch-1 cache with the same planes as ``small`` (same generator
    # arguments: seed, layer 0, length, rho, tagged planes, torch backend)
    T, max_T = [300], 300 + B
    src = PlaneSource(N, kvH, d, R, max_T, 0.88, 15, independent=True, backend="torch", device=cuda_device)
    PK = [src.plane(pl, "K") for pl in range(R)]
    PV = [src.plane(pl, "V") for pl in range(R)]
    kd, kr = _layout(PK, T, W, B, R, max_T, B)
    vd, vr = _layout(PV, T, W, B, R, max_T, B)
    lengths = torch.tensor(T, dtype=torch.int32, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    view = CacheView(batch=N, layers=1, q_heads=kvH * g, kv_heads=kvH, head_dim=d, loops=R, window=W,
                     max_T=max_T, max_B=B, window_mode=0, block_len=B, k_deep=kd.data_ptr(), v_deep=vd.data_ptr(),
                     k_ring=kr.data_ptr(), v_ring=vr.data_ptr(), lengths=lengths.data_ptr())
    for r in range(R):
        q = torch.randn((N, B, kvH * g, d), device=cuda_device).div(d ** 0.5).to(torch.bfloat16)
        out = torch.empty_like(q)
        ripe.ripe_verify_attn_static(view, 0, r, q.data_ptr(), out.data_ptr(), None, 1.0, err.data_ptr())
        ref = small.gpu.verify_attn(0, r, q)
        torch.cuda.synchronize()
        check_close(out, ref.double().cpu().numpy(), f"static batch 1, loop {r}")
        big.check(0, r)          # raises RipeError (RIPE_ECUDA) if its launch were refused
    assert int(err.item()) == 0
    small.close()
    big.close()
