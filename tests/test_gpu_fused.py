"""ripe_append_verify == ripe_append_block + ripe_verify_attn: the cache state after each commit bit
for bit, and the outputs of every call bit for bit when both calls run the same consumer (the fused
call always runs the mma.sync one; at these sizes so does the separate call, unless
RIPE_VERIFY_CONSUMER=tc puts the tcgen05 one on 9..64 query rows per kv head, and then the two
outputs agree within the parity tolerance), over several decode
steps with ragged accepted lengths (ring wrap-around, eviction, all three layouts); and
ripe_append_verify against the CPU oracle directly."""
import os

import numpy as np
import pytest
import torch

from harness import Case, assert_same_result, check_close, check_lse, dev_to_bits
from self_speculative_decode_b200.ripe import RipeCache
from self_speculative_decode_b200.synth import PlaneSource, acceptance_draws

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,B,g,d,T0", [(16, 8, 1, 96, 90), (5, 6, 2, 64, 90), (0, 4, 4, 128, 90),
                                        (10 ** 6, 8, 1, 96, 90), (64, 8, 4, 128, 90),
                                        (10 ** 6, 8, 1, 64, 60), (0, 8, 2, 96, 188)])
def test_fused_append_verify_is_bitwise_the_two_calls(W, B, g, d, T0, cuda_device):
    """T0 = 60 (full cache) and 188 (deepest only) put the block's rows across a 64-row tile edge."""
    N, L, kvH, R, steps = 3, 2, 3, 4, 6
    # the fused launch always runs the mma.sync consumer; a separate verify of these short pairs
    # runs it too unless RIPE_VERIFY_CONSUMER=tc puts the tcgen05 one on 9..64 query rows
    same_consumer = B * g <= 8 or os.environ.get("RIPE_VERIFY_CONSUMER") != "tc"
    max_T = T0 + B * (steps + 1)
    src = PlaneSource(N, kvH, d, R, T0, 0.88, 31, backend="torch", device=cuda_device)
    caches = [RipeCache(N, L, kvH * g, kvH, d, R, W, max_T, B) for _ in range(2)]
    T = [T0, 7, 45]
    for layer in range(L):
        s = PlaneSource(N, kvH, d, R, T0, 0.88, 31, layer=layer, backend="torch", device=cuda_device)
        for pl in range(R):
            k, v = s.plane(pl, "K"), s.plane(pl, "V")
            for c in caches:
                c.load_prefix(layer, pl, T, k, v)
    acc = acceptance_draws(5, steps, N, B)
    for step in range(steps):
        for r in range(R):
            for layer in range(L):
                kb, vb = src.block(step * L + layer, r, B, "K"), src.block(step * L + layer, r, B, "V")
                q = src.queries(r, B, kvH * g, step * L + layer)
                caches[0].append_block(layer, r, kb, vb)
                a = caches[0].verify_attn(layer, r, q)
                b = caches[1].append_verify(layer, r, kb, vb, q)
                if same_consumer:
                    assert torch.equal(a, b), (step, r, layer)
                else:
                    assert_same_result(a, b, f"step {step} loop {r} layer {layer}")
        for c in caches:
            c.commit(acc[step])
        for n in range(N):
            for layer in range(L):
                ka, va, pa = caches[0].export(n, layer)
                kb_, vb_, pb = caches[1].export(n, layer)
                assert torch.equal(pa, pb)
                assert np.array_equal(dev_to_bits(ka), dev_to_bits(kb_))
                assert np.array_equal(dev_to_bits(va), dev_to_bits(vb_))
    for c in caches:
        assert c.device_error() == 0
        c.close()


@pytest.mark.parametrize("W", [16, 0, 10 ** 6])
def test_fused_append_verify_against_the_oracle(W, cuda_device):
    """Each plane of the block written by the verify launch itself, then checked against the
    oracle (tagged planes: a wrong plane or a row written to the wrong slot is an O(1) error)."""
    c = Case(N=3, L=1, Hq=6, kvH=3, d=96, R=4, T=[90, 7, 45], W=W, B=8, seed=33, independent=True,
             append_block=False)
    for r in range(4):
        kb, vb = c.blocks[(0, r)]
        qd, qh = c.queries(0, r)
        lse = torch.empty((c.N, c.B, c.Hq), dtype=torch.float32, device=c.device)
        out = c.gpu.append_verify(0, r, c._dev(kb), c._dev(vb), qd, lse=lse)
        c.orc.append(0, r, c._sub_block(kb), c._sub_block(vb))
        ro, rl = c.orc.verify(0, r, qh, c.g)
        check_close(out, ro, f"fused loop {r}")
        check_lse(lse, rl)
    c.close()
