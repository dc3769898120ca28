"""GPU cache maintenance against the oracle's logical state, bit for bit.

Random sequences of appends (every plane of every layer) and commits with accepted lengths
drawn from U{0..B}; after every step the exported logical view (which planes of which
positions are stored, and their bf16 bits) must equal the oracle's exactly, and the
committed lengths must match.  Covers ring wrap-around, eviction into the deepest-plane
region, rollback of rejected drafts, the three layouts, and the device-side commit.
"""
import numpy as np
import pytest
import torch

from harness import bits_to_dev, dev_to_bits
from oracle import ripe_oracle as orc
from self_speculative_decode_b200 import ripe
from self_speculative_decode_b200.ripe import RipeCache, RipeError

pytestmark = pytest.mark.gpu


def _compare_state(gpu, oc, N, L, R):
    T = gpu.sync_lengths()
    assert T == [int(x) for x in oc.T]
    for n in range(N):
        for layer in range(L):
            k, v, present = gpu.export(n, layer)
            Tv = int(oc.T[n]) + oc.B
            assert present.shape == (R, Tv)
            pres = oc.present[layer, :, n, :Tv]
            np.testing.assert_array_equal(present.cpu().numpy().astype(bool), pres)
            kb, vb = dev_to_bits(k), dev_to_bits(v)
            for pl in range(R):
                ok = oc.values(layer, pl, "K")[n, :, :Tv]
                ov = oc.values(layer, pl, "V")[n, :, :Tv]
                m = pres[pl][None, :, None]
                np.testing.assert_array_equal(np.where(m, kb[pl], 0), np.where(m, ok, 0))
                np.testing.assert_array_equal(np.where(m, vb[pl], 0), np.where(m, ov, 0))
                assert not kb[pl][:, ~pres[pl]].any()   # absent planes export as zero


@pytest.mark.parametrize("W,device_commit", [(5, False), (5, True), (0, False), (1000, False), (2, False)])
def test_random_append_commit_sequences(W, device_commit, cuda_device):
    N, L, kvH, d, R, max_B, max_T = 3, 2, 2, 64, 3, 6, 90
    rng = np.random.default_rng(17 + W)
    gpu = RipeCache(N, L, 2 * kvH, kvH, d, R, W, max_T, max_B)
    oc = orc.OracleCache(N, L, kvH, d, R, W, max_T)
    T0 = [3, 0, 11]
    for layer in range(L):
        for pl in range(R):
            k = rng.integers(0, 1 << 16, size=(N, kvH, 16, d), dtype=np.uint16)
            v = rng.integers(0, 1 << 16, size=(N, kvH, 16, d), dtype=np.uint16)
            # keep the bit patterns finite: clear the exponent's top bit
            k &= 0xBFFF
            v &= 0xBFFF
            gpu.load_prefix(layer, pl, T0, bits_to_dev(k, cuda_device), bits_to_dev(v, cuda_device))
            oc.load_prefix(layer, pl, T0, k, v)
    _compare_state(gpu, oc, N, L, R)
    step = 0
    while True:
        B = int(rng.integers(1, max_B + 1))
        if int(oc.T.max()) + B > max_T:
            break
        for layer in range(L):
            for pl in range(R):
                k = (rng.integers(0, 1 << 16, size=(N, B, kvH, d), dtype=np.uint16) & 0xBFFF).astype(np.uint16)
                v = (rng.integers(0, 1 << 16, size=(N, B, kvH, d), dtype=np.uint16) & 0xBFFF).astype(np.uint16)
                gpu.append_block(layer, pl, bits_to_dev(k, cuda_device), bits_to_dev(v, cuda_device))
                oc.append(layer, pl, k, v)
        if step % 4 == 1:
            _compare_state(gpu, oc, N, L, R)   # mid-block view: the block's planes are present
        a = rng.integers(0, B + 1, size=N).astype(np.int32)
        if device_commit:
            gpu.commit_device(torch.tensor(a, dtype=torch.int32, device=cuda_device))
            assert gpu.stats()["lengths_synced"] == 0
        else:
            gpu.commit(a)
        oc.commit(a)
        _compare_state(gpu, oc, N, L, R)
        st = gpu.stats()
        Wc = min(W, max_T)
        assert st["stored_position_planes"] == sum(int(t) + min(Wc, int(t)) * (R - 1) for t in oc.T)
        for n in range(N):
            assert oc.stored_position_planes(0, n) == int(oc.T[n]) + min(W, int(oc.T[n])) * (R - 1)
        step += 1
    assert step > 10
    assert gpu.device_error() == 0
    gpu.close()


def test_state_errors_are_reported_on_the_host(cuda_device):
    N, kvH, d, R = 2, 1, 64, 3
    gpu = RipeCache(N, 2, kvH, kvH, d, R, 4, 20, 4)
    blk = torch.zeros((N, 4, kvH, d), dtype=torch.bfloat16, device=cuda_device)
    q = torch.zeros((N, 4, kvH, d), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(RipeError) as e:
        gpu.verify_attn(0, 0, q)                  # nothing appended
    assert e.value.status == ripe.RIPE_ESTATE
    gpu.append_block(0, 1, blk, blk)
    with pytest.raises(RipeError) as e:
        gpu.verify_attn(0, 0, q)                  # plane 0 not appended yet
    assert e.value.status == ripe.RIPE_ESTATE
    with pytest.raises(RipeError) as e:
        gpu.commit([1, 1])                        # other planes / layers missing
    assert e.value.status == ripe.RIPE_ESTATE
    with pytest.raises(RipeError) as e:
        gpu.append_block(0, 2, blk[:, :3].contiguous(), blk[:, :3].contiguous())   # block length changed
    assert e.value.status == ripe.RIPE_EINVAL
    for layer in range(2):
        for r in range(R):
            gpu.append_block(layer, r, blk, blk)
    with pytest.raises(RipeError) as e:
        gpu.commit([5, 0])                        # more than the block
    assert e.value.status == ripe.RIPE_EINVAL
    gpu.commit([4, 4])
    for _ in range(3):
        for layer in range(2):
            for r in range(R):
                gpu.append_block(layer, r, blk, blk)
        gpu.commit([4, 4])
    with pytest.raises(RipeError) as e:           # 16 + 5 > 20
        gpu.append_block(0, 0, torch.zeros((N, 5, kvH, d), dtype=torch.bfloat16, device=cuda_device),
                         torch.zeros((N, 5, kvH, d), dtype=torch.bfloat16, device=cuda_device))
    assert e.value.status == ripe.RIPE_EINVAL     # 5 > max_B is checked first
    for layer in range(2):
        for r in range(R):
            gpu.append_block(layer, r, blk, blk)
    gpu.commit([4, 4])                            # T = 20 = max_T
    with pytest.raises(RipeError) as e:
        gpu.append_block(0, 0, blk[:, :1].contiguous(), blk[:, :1].contiguous())
    assert e.value.status == ripe.RIPE_ECAPACITY
    assert gpu.device_error() == 0
    gpu.close()


def test_device_commit_clamps_and_flags_bad_lengths(cuda_device):
    N, kvH, d, R = 2, 1, 64, 2
    gpu = RipeCache(N, 1, kvH, kvH, d, R, 4, 40, 4)
    blk = torch.ones((N, 4, kvH, d), dtype=torch.bfloat16, device=cuda_device)
    for r in range(R):
        gpu.append_block(0, r, blk, blk)
    gpu.commit_device(torch.tensor([9, -2], dtype=torch.int32, device=cuda_device))
    assert gpu.sync_lengths() == [4, 0]
    assert gpu.device_error() == ripe.RIPE_DEVERR_ACCEPT
    assert gpu.device_error() == 0                # reading clears the word
    gpu.close()


@pytest.mark.parametrize("W", [5, 0, 1000])
def test_checkpoint_and_resume_through_export_and_load_prefix(W, cuda_device):
    """A cache's committed state, exported per (sequence, layer) and loaded plane by plane into a fresh
    cache with ripe_load_prefix, is the same state: equal exports bit for bit, and equal verification
    results bit for bit on the next block (same kernel, same inputs)."""
    N, L, kvH, d, R, max_B, max_T = 3, 2, 2, 64, 3, 6, 90
    rng = np.random.default_rng(29 + W)
    a_cache = RipeCache(N, L, 2 * kvH, kvH, d, R, W, max_T, max_B)
    rand = lambda *shape: bits_to_dev((rng.integers(0, 1 << 16, size=shape, dtype=np.uint16) & 0xBFFF).astype(np.uint16),
                                      cuda_device)
    T0 = [7, 0, 19]
    for layer in range(L):
        for pl in range(R):
            a_cache.load_prefix(layer, pl, T0, rand(N, kvH, 20, d), rand(N, kvH, 20, d))
    for step in range(9):   # ragged decode: ring wrap-around and eviction
        for layer in range(L):
            for pl in range(R):
                a_cache.append_block(layer, pl, rand(N, 5, kvH, d), rand(N, 5, kvH, d))
        a_cache.commit(rng.integers(0, 6, size=N).astype(np.int32))
    T = a_cache.sync_lengths()
    # checkpoint: the logical view of every (sequence, layer)
    views = {(n, layer): a_cache.export(n, layer) for n in range(N) for layer in range(L)}
    # resume: plane by plane, positions 0 .. T_n - 1 of every sequence
    b_cache = RipeCache(N, L, 2 * kvH, kvH, d, R, W, max_T, max_B)
    ld = max(T)
    for layer in range(L):
        for pl in range(R):
            k = torch.zeros((N, kvH, ld, d), dtype=torch.bfloat16, device=cuda_device)
            v = torch.zeros_like(k)
            for n in range(N):
                kx, vx, _ = views[(n, layer)]
                k[n, :, :T[n]] = kx[pl, :, :T[n]]
                v[n, :, :T[n]] = vx[pl, :, :T[n]]
            b_cache.load_prefix(layer, pl, T, k, v)
    assert b_cache.sync_lengths() == T
    for n in range(N):
        for layer in range(L):
            ka, va, pa = views[(n, layer)]
            kb, vb, pb = b_cache.export(n, layer)
            assert torch.equal(pa, pb)
            assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
            assert torch.equal(va.view(torch.int16), vb.view(torch.int16))
    assert a_cache.stats()["stored_position_planes"] == b_cache.stats()["stored_position_planes"]
    # the next block on both: the same outputs, bit for bit
    blk = [(rand(N, 4, kvH, d), rand(N, 4, kvH, d)) for _ in range(L * R)]
    q = rand(N, 4, 2 * kvH, d)
    outs = []
    for c in (a_cache, b_cache):
        for layer in range(L):
            for pl in range(R):
                c.append_block(layer, pl, *blk[layer * R + pl])
        outs.append([c.verify_attn(layer, r, q).view(torch.int16).clone() for layer in range(L) for r in range(R)])
    for x, y in zip(*outs):
        assert torch.equal(x, y)
    for c in (a_cache, b_cache):
        assert c.device_error() == 0
        c.close()
