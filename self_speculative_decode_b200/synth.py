"""Seeded synthetic inputs for RIPE verification: key/value planes, draft blocks, queries.

This module only draws numbers.  It contains none of the method's arithmetic
(no plane selection, no attention, no cache bookkeeping), so the CUDA library's
tests and the CPU oracle can both consume what it produces.

Recipe (the pages give no data, only how the planes behave):
  * the deepest plane D of every position is N(0, 1) per element;
  * plane r < R-1 is D + rho**r * eps_r with eps_r ~ N(0, 1) drawn independently
    per plane, separately for keys and values, so the distance to the deepest
    plane shrinks by rho per loop (RIPE abstract, second sentence: the planes
    converge geometrically on the last one, at 0.88 per loop for Huginn-0125 and
    0.81 for Raven-Llama);
  * plane R-1 is D itself, the plane that RIPE keeps everywhere;
  * ``independent=True`` draws every plane as its own N(0, 1) sample ("tagged"
    planes): a wrong plane choice then moves an output by O(1) instead of
    O(rho**r);
  * queries are N(0, 1) / sqrt(d), to be used with softmax scale 1;
  * every value is rounded once to bf16 (round to nearest even).

Each plane, block and query tensor has its own seed tuple
``(seed, layer, stream, index...)`` so any subset can be regenerated alone.

Two backends draw the same recipe: ``numpy`` (host, bf16 returned as uint16
bit patterns) and ``torch`` (device tensors of dtype bfloat16, drawn with a
seeded ``torch.Generator`` on the tensor's device).  The two backends do not
produce equal values; a test uses one backend for both sides.
"""
from __future__ import annotations

import hashlib
import math

import numpy as np

# stream ids inside a seed tuple
K_DEEP, V_DEEP, K_NOISE, V_NOISE, QUERY, K_BLOCK, V_BLOCK = range(7)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _torch_seed(parts) -> int:
    h = hashlib.sha256(repr(tuple(int(p) for p in parts)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


class PlaneSource:
    """Synthetic planes of one recurrent layer for N sequences.

    ``plane(r, 'K')`` returns plane r of every position in [0, length):
    numpy backend -> uint16 bf16 bits [N][kvH][length][d];
    torch backend -> bfloat16 tensor of the same shape on ``device``.
    """

    def __init__(self, N, kvH, d, R, length, rho, seed, layer=0,
                 independent=False, backend="numpy", device=None):
        self.N, self.kvH, self.d, self.R, self.length = N, kvH, d, R, length
        self.rho, self.seed, self.layer = float(rho), int(seed), int(layer)
        self.independent = bool(independent)
        self.backend = backend
        self.device = device
        if backend not in ("numpy", "torch"):
            raise ValueError("backend must be 'numpy' or 'torch'")
        self.shape = (N, kvH, length, d)
        self._deep = {}

    # -- raw N(0,1) draws ------------------------------------------------------
    def _normal(self, parts, shape):
        if self.backend == "numpy":
            rng = np.random.default_rng([self.seed, self.layer, *parts])
            return rng.standard_normal(shape)  # float64
        import torch
        gen = torch.Generator(device=self.device)
        gen.manual_seed(_torch_seed((self.seed, self.layer, *parts)))
        return torch.randn(shape, generator=gen, device=self.device, dtype=torch.float32)

    def _to_bf16(self, x):
        if self.backend == "numpy":
            return f32_to_bf16_bits(x.astype(np.float32))
        import torch
        return x.to(torch.bfloat16)

    def plane(self, r: int, which: str = "K"):
        if not 0 <= r < self.R:
            raise ValueError("plane index out of range")
        deep_id, noise_id = (K_DEEP, K_NOISE) if which == "K" else (V_DEEP, V_NOISE)
        if self.independent:
            return self._to_bf16(self._normal((noise_id, r), self.shape))
        if deep_id not in self._deep:
            self._deep[deep_id] = self._normal((deep_id,), self.shape)
        D = self._deep[deep_id]
        if r == self.R - 1:
            return self._to_bf16(D)
        eps = self._normal((noise_id, r), self.shape)
        return self._to_bf16(D + (self.rho ** r) * eps)

    def release(self):
        """Drop the cached deepest-plane draws."""
        self._deep.clear()

    # -- draft blocks drawn per decoding step (streaming workloads) -------------
    def block(self, step: int, r: int, B: int, which: str = "K"):
        """Fresh block K/V for loop r of decoding step ``step``: [N][B][kvH][d]."""
        sid = K_BLOCK if which == "K" else V_BLOCK
        shape = (self.N, B, self.kvH, self.d)
        if self.independent:
            return self._to_bf16(self._normal((sid, step, r, 1), shape))
        D = self._normal((sid, step, self.R), shape)
        if r == self.R - 1:
            return self._to_bf16(D)
        eps = self._normal((sid, step, r), shape)
        return self._to_bf16(D + (self.rho ** r) * eps)

    def queries(self, r: int, B: int, Hq: int, step: int = 0):
        """Queries of loop r for a block of B positions: [N][B][Hq][d] ~ N(0,1)/sqrt(d)."""
        x = self._normal((QUERY, step, r), (self.N, B, Hq, self.d))
        return self._to_bf16(x / math.sqrt(self.d))


def block_from_planes(planes_r, T, B):
    """Positions [T, T+B) of a plane [N][kvH][len][d] rearranged to the block layout [N][B][kvH][d]."""
    blk = planes_r[:, :, T:T + B, :]
    if isinstance(blk, np.ndarray):
        return np.ascontiguousarray(blk.transpose(0, 2, 1, 3))
    return blk.permute(0, 2, 1, 3).contiguous()


def acceptance_draws(seed: int, steps: int, N: int, B: int) -> np.ndarray:
    """Accepted block length per (step, sequence), uniform on {0, ..., B}."""
    rng = np.random.default_rng([seed, 99])
    return rng.integers(0, B + 1, size=(steps, N), dtype=np.int32)
