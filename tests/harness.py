"""Shared set-up for the GPU parity tests: one seeded synthetic cache loaded into both the
CUDA library (through its C ABI) and the CPU oracle, from the same generator output.

Nothing the oracle sees comes from the CUDA library: planes, blocks and queries are drawn
by ``self_speculative_decode_b200.synth`` and copied to whichever side needs them.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import ripe_oracle as orc
from self_speculative_decode_b200.ripe import RipeCache
from self_speculative_decode_b200.synth import PlaneSource

# bf16 inputs, fp32 accumulation, bf16 output: the tolerance the benchmark spec fixes for the verify output
MAX_ABS = 2e-2
REL_L2 = 5e-3
# the log-sum-exp is returned in fp32 from an fp32 sum of up to ~33K exponentials: its error is
# bounded by the sum's rounding (< 33K * 2^-24 relative) plus the approximate exp2 / log2 (~2^-22
# relative each), well under 1e-3 in absolute terms for logits of moderate size
LSE_ABS = 1e-3


def bits_to_dev(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def seq_block(plane, T, B):
    """Block layout [N][B][kvH][d] of positions [T_n, T_n + B) of a plane [N][kvH][len][d]."""
    if isinstance(plane, np.ndarray):
        return np.ascontiguousarray(np.stack([plane[n, :, T[n]:T[n] + B].transpose(1, 0, 2)
                                              for n in range(plane.shape[0])]))
    return torch.stack([plane[n, :, T[n]:T[n] + B].permute(1, 0, 2) for n in range(plane.shape[0])]).contiguous()


def check_close(gpu_out: torch.Tensor, ref: np.ndarray, what: str = "out"):
    got = bf16_to_f64(gpu_out)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert err.max() <= MAX_ABS, f"{what}: max abs error {err.max():.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)


def check_lse(gpu_lse: torch.Tensor, ref: np.ndarray):
    got = gpu_lse.detach().double().cpu().numpy()
    err = np.abs(got - ref).max()
    assert err <= LSE_ABS, f"lse: max abs error {err:.3e}"
    return float(err)


def assert_same_result(a: torch.Tensor, b: torch.Tensor, what: str = ""):
    """Two GPU results of the same attention with a different split of the key range.

    Each is within MAX_ABS / REL_L2 of the exact value (the parity tolerance: bf16 P and
    output rounding, fp32 sums), so by the triangle inequality they are within twice that
    of each other."""
    a, b = a.double(), b.double()
    err = (a - b).abs().max().item()
    rel = (torch.linalg.vector_norm(a - b) / torch.clamp(torch.linalg.vector_norm(a), min=1e-30)).item()
    assert err <= 2 * MAX_ABS and rel <= 2 * REL_L2, f"{what}: max abs {err:.3e}, relative L2 {rel:.3e}"


class Case:
    """A synthetic cache in both implementations.

    T: committed length per sequence; W: window (>= max_T means full cache);
    oracle_seqs / oracle_kvh: subsets mirrored in the oracle (all by default);
    oracle_planes: planes whose values the oracle keeps (all by default);
    append_block=False leaves the draft block out (kept in ``blocks`` for a later append).
    """

    def __init__(self, N, L, Hq, kvH, d, R, T, W, B, rho=0.88, seed=0, mode=0, max_T=None,
                 independent=False, backend="numpy", oracle_seqs=None, oracle_kvh=None,
                 oracle_planes=None, device="cuda", append_block=True):
        self.N, self.L, self.Hq, self.kvH, self.d, self.R = N, L, Hq, kvH, d, R
        self.g = Hq // kvH
        self.T = [int(t) for t in (T if hasattr(T, "__len__") else [T] * N)]
        self.W, self.B, self.mode = W, B, mode
        self.max_T = max_T or max(self.T) + B
        self.device = torch.device(device)
        self.backend = backend
        self.oseq = list(range(N)) if oracle_seqs is None else list(oracle_seqs)
        self.okvh = list(range(kvH)) if oracle_kvh is None else list(oracle_kvh)
        self.oheads = [kh * self.g + x for kh in self.okvh for x in range(self.g)]
        self.src = [PlaneSource(N, kvH, d, R, self.max_T, rho, seed, layer=l, independent=independent,
                                backend=backend, device=self.device if backend == "torch" else None)
                    for l in range(L)]
        self.gpu = RipeCache(N, L, Hq, kvH, d, R, W, self.max_T, B, mode)
        self.orc = orc.OracleCache(len(self.oseq), L, len(self.okvh), d, R, W, self.max_T, mode,
                                   value_planes=oracle_planes)
        self._load(append_block)

    # -- helpers ---------------------------------------------------------------
    def _host(self, x):
        """Oracle-side slice (uint16 bits) of a generator tensor [N][kvH or B ...]."""
        if isinstance(x, np.ndarray):
            return x
        return dev_to_bits(x)

    def _dev(self, x):
        return bits_to_dev(x, self.device) if isinstance(x, np.ndarray) else x

    def _sub_plane(self, x):
        return np.ascontiguousarray(self._host(x)[self.oseq][:, self.okvh])

    def _sub_block(self, x):
        return np.ascontiguousarray(self._host(x)[self.oseq][:, :, self.okvh])

    def _load(self, append_block=True):
        To = [self.T[n] for n in self.oseq]
        keep = self.orc.value_planes
        blocks = []
        for l in range(self.L):
            for pl in range(self.R):
                k, v = self.src[l].plane(pl, "K"), self.src[l].plane(pl, "V")
                self.gpu.load_prefix(l, pl, self.T, self._dev(k), self._dev(v))
                kept = keep is None or pl in keep
                if kept:
                    self.orc.load_prefix(l, pl, To, self._sub_plane(k), self._sub_plane(v))
                else:
                    self.orc.load_prefix(l, pl, To, None, None)
                # the draft block of this plane: positions [T_n, T_n + B) of the same plane
                blocks.append((l, pl, kept, seq_block(k, self.T, self.B), seq_block(v, self.T, self.B)))
                del k, v
            self.src[l].release()
        self.blocks = {(l, pl): (kb, vb) for l, pl, _, kb, vb in blocks}
        if append_block:
            self.append_blocks()
        torch.cuda.synchronize()

    def append_blocks(self):
        """Append every plane of every layer's draft block on both sides."""
        keep = self.orc.value_planes
        for (l, pl), (kb, vb) in self.blocks.items():
            kept = keep is None or pl in keep
            self.gpu.append_block(l, pl, self._dev(kb), self._dev(vb))
            if kept:
                self.orc.append(l, pl, self._sub_block(kb), self._sub_block(vb))
            else:
                self.orc.append(l, pl, None, None, B=self.B)
        torch.cuda.synchronize()

    def queries(self, layer, r, step=0):
        q = self.src[layer].queries(r, self.B, self.Hq, step)
        return self._dev(q), np.ascontiguousarray(self._host(q)[self.oseq][:, :, self.oheads])

    def run(self, layer, r, scale=1.0, with_lse=True, step=0):
        """Verify on both sides; returns (gpu out [oracle subset], gpu lse, oracle out, oracle lse)."""
        qd, qh = self.queries(layer, r, step)
        lse = torch.empty((self.N, self.B, self.Hq), dtype=torch.float32, device=self.device) if with_lse else None
        out = self.gpu.verify_attn(layer, r, qd, lse=lse, scale=scale)
        ro, rl = self.orc.verify(layer, r, qh, self.g, scale)
        idx_n = torch.tensor(self.oseq, device=self.device)
        idx_h = torch.tensor(self.oheads, device=self.device)
        go = out.index_select(0, idx_n).index_select(2, idx_h)
        gl = lse.index_select(0, idx_n).index_select(2, idx_h) if with_lse else None
        return go, gl, ro, rl

    def check_wave(self, layer, loops, scale=1.0):
        """A loop per block position, against the oracle's per-position composition."""
        qd, qh = self.queries(layer, 0, step=7)
        lse = torch.empty((self.N, self.B, self.Hq), dtype=torch.float32, device=self.device)
        out = self.gpu.verify_attn_wave(layer, loops, qd, lse=lse, scale=scale)
        ro, rl = orc.verify_wave(self.orc, layer, loops, qh, self.g, scale)
        idx_n = torch.tensor(self.oseq, device=self.device)
        idx_h = torch.tensor(self.oheads, device=self.device)
        e = check_close(out.index_select(0, idx_n).index_select(2, idx_h), ro, f"layer {layer} loops {loops}")
        check_lse(lse.index_select(0, idx_n).index_select(2, idx_h), rl)
        return e

    def check(self, layer, r, scale=1.0):
        go, gl, ro, rl = self.run(layer, r, scale)
        e = check_close(go, ro, f"layer {layer} loop {r}")
        check_lse(gl, rl)
        return e

    def close(self):
        assert self.gpu.device_error() == 0
        self.gpu.close()
