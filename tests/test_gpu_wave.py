"""GPU parity of ripe_verify_attn_wave: a loop per block position in one call (a wavefront
schedule's batched pass), against the oracle, which evaluates every position as the
single-loop verification at its own loop."""
import pytest
import torch

from harness import Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,loops", [(16, [3, 3, 2, 0]), (0, [3, 2, 1, 0]), (10 ** 6, [1, 1, 1, 1]),
                                     (5, [0, 3, 0, 3])])
def test_wave_tiny(W, loops, cuda_device):
    c = Case(N=1, L=1, Hq=2, kvH=2, d=64, R=4, T=128, W=W, B=4, rho=0.88, seed=0, independent=True)
    c.check_wave(0, loops)
    c.close()


@pytest.mark.parametrize("d,g,B,W", [(96, 2, 6, 5), (128, 4, 8, 9), (64, 1, 16, 3)])
def test_wave_ragged_tagged(d, g, B, W, cuda_device):
    kvH, R = 3, 5
    T = [0, 1, 37, 200, 129]
    c = Case(N=5, L=2, Hq=kvH * g, kvH=kvH, d=d, R=R, T=T, W=W, B=B, seed=3, independent=True,
             max_T=max(T) + B + 11)
    diag = [max(0, R - 1 - j) for j in range(B)]          # older positions deeper
    for layer in range(2):
        c.check_wave(layer, diag)
        c.check_wave(layer, [j % R for j in range(B)])    # any order is well defined
    c.close()


@pytest.mark.parametrize("layout", ["ripe", "full", "deepest"])
def test_wave_huginn_shape(layout, cuda_device):
    W = {"ripe": 64, "full": 10 ** 6, "deepest": 0}[layout]
    loops = [31, 27, 23, 19, 15, 11, 7, 3]
    c = Case(N=1, L=1, Hq=55, kvH=55, d=96, R=32, T=1024, W=W, B=8, rho=0.88, seed=1, backend="torch",
             oracle_planes=set(loops) | {31})
    c.check_wave(0, loops)
    c.close()


def test_single_loop_wave_is_the_single_loop_call(cuda_device):
    c = Case(N=2, L=1, Hq=8, kvH=2, d=128, R=6, T=[700, 300], W=32, B=8, seed=4, independent=True)
    q, _ = c.queries(0, 0)
    for r in range(5):                                     # below the deepest loop both plans coincide
        a = c.gpu.verify_attn(0, r, q)
        b = c.gpu.verify_attn_wave(0, [r] * 8, q)
        assert torch.equal(a, b)
    c.close()
