"""CPU oracle for RIPE caching and verification attention (fp64).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, the package's ``smoke()`` check and
the benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library and never takes an input or an expected value from it.

Source: "Prefix Keys and Values Matter Late: RIPE Caching for Self-Speculative
Decoding in Looped Language Models" (arXiv 2610.34436), abstract; and the
WaveFront Decoding write-up (rit.work blog, section on drafting and checking in
one pass) for the accept/rollback semantics; "Windowed-MTP: Removing the
Full-Context Draft-KV Tax at Million-Token Context", abstract, for the windowed
draft attention (a sliding window plus an attention sink on the draft only).

Contents
  * ``verify``         verification attention of one loop, through the C oracle
                       (``ripe_oracle.c``), fp64, OpenMP over (sequence, position, head).
  * ``brute_verify``   an independent numpy formulation of the same quantity for
                       tiny shapes (full logical planes + explicit full-depth sets).
  * ``OracleCache``    the logical cache state machine: which (position, plane)
                       pairs RIPE stores, their bf16 bit patterns, append, accept /
                       rollback and window eviction.
  * ``memory_fraction`` stored fraction of the full cache, counted from the state
                       machine.
  * ``verify_wave``    a loop per block position: each position evaluated as the
                       single-loop verification at its own loop (definition by
                       composition).
  * ``OracleCache.draft``  one draft-phase step: plane r of block position j stored,
                       then the query of that position attends with the verification
                       rule for p = T + j (draft-then-verify builds the block one
                       position at a time at a shallow loop); optionally windowed.
  * ``windowed_draft`` draft attention restricted to an attention sink and a sliding
                       window (the Windowed-MTP abstract), planes by the RIPE rule.
Every function here is pinned by ``tests/test_oracle_*.py``; none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes

import numpy as np

from .build import build_oracle

_lib = None

QUERY_RELATIVE = 0  # window measured back from each query position (default rule)
CACHE_RELATIVE = 1  # window measured back from the end of the committed cache


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        lp = ctypes.POINTER(ctypes.c_long)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_plane.restype = ctypes.c_int
        lib.oracle_plane.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.oracle_verify.restype = ctypes.c_int
        lib.oracle_verify.argtypes = [ctypes.c_int] * 5 + [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, lp, ctypes.c_long, dp, dp, dp, dp, dp,
                                      ctypes.c_double, dp, dp]
        lib.oracle_weights.restype = ctypes.c_int
        lib.oracle_weights.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_long, ctypes.c_int, dp, dp, dp,
                                       ctypes.c_double, dp]
        _lib = lib
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def plane_of(p: int, t: int, r: int, R: int, T: int, W: int, mode: int = QUERY_RELATIVE) -> int:
    """Plane read by query position p for key t at loop r (the C oracle's rule)."""
    return _load().oracle_plane(p, t, r, R, T, W, mode)


def verify(T, B, r, R, W, g, Kr, Vr, Kl, Vl, q, scale=1.0, mode=QUERY_RELATIVE):
    """Verification attention at loop r.

    T: committed lengths [N]; Kr/Vr: plane r [N][kvH][ld][d] (NaN where not stored);
    Kl/Vl: plane R-1, same shape; q: [N][B][kvH*g][d].  All float64.
    Returns (out [N][B][Hq][d], lse [N][B][Hq]).  Raises if a selected plane is absent.
    """
    T = np.ascontiguousarray(T, dtype=np.int64)
    Kr, Vr, Kl, Vl, q = (np.ascontiguousarray(x, dtype=np.float64) for x in (Kr, Vr, Kl, Vl, q))
    N, kvH, ld, d = Kr.shape
    Hq = q.shape[2]
    if Hq != kvH * g or q.shape != (N, B, Hq, d):
        raise ValueError("query shape does not match the planes")
    out = np.zeros((N, B, Hq, d))
    lse = np.zeros((N, B, Hq))
    st = _load().oracle_verify(N, kvH, g, d, R, W, r, mode, B,
                               T.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), ld,
                               _dp(Kr), _dp(Vr), _dp(Kl), _dp(Vl), _dp(q), float(scale),
                               _dp(out), _dp(lse))
    if st == 2:
        raise RuntimeError("oracle read a plane that the cache does not store")
    if st != 0:
        raise ValueError(f"oracle_verify rejected its arguments (status {st})")
    return out, lse


def weights(T, j, r, R, W, Kr_seq, Kl_seq, qv, scale=1.0, mode=QUERY_RELATIVE):
    """Softmax weights of one query (one sequence, one key/value head): array of length T+j+1."""
    Kr_seq, Kl_seq, qv = (np.ascontiguousarray(x, dtype=np.float64) for x in (Kr_seq, Kl_seq, qv))
    w = np.zeros(T + j + 1)
    st = _load().oracle_weights(Kr_seq.shape[-1], R, W, r, mode, T, j, _dp(Kr_seq), _dp(Kl_seq),
                                _dp(qv), float(scale), _dp(w))
    if st != 0:
        raise RuntimeError("oracle read a plane that the cache does not store")
    return w


def brute_verify(Kplanes, Vplanes, T, B, r, W, g, q, scale=1.0, mode=QUERY_RELATIVE):
    """Independent numpy formulation for tiny shapes (one sequence).

    Kplanes/Vplanes: every plane of every position, float64 [R][kvH][T+B][d];
    q: [B][kvH*g][d].  For each query position p = T+j the set of keys read at
    full depth (plane r) is written out explicitly -- the draft block up to p and
    the window -- and every other key reads the deepest plane.
    """
    R, kvH, L, d = Kplanes.shape
    Hq = q.shape[1]
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for j in range(B):
        p = T + j
        block = set(range(T, p + 1))
        if mode == QUERY_RELATIVE:
            window = set(range(max(0, p - W), T))
        else:
            window = set(range(max(0, T - W), T))
        full_depth = block | window
        plane_idx = np.array([r if t in full_depth else R - 1 for t in range(p + 1)])
        pos = np.arange(p + 1)
        for h in range(Hq):
            kh = h // g
            Kp = Kplanes[plane_idx, kh, pos, :]
            Vp = Vplanes[plane_idx, kh, pos, :]
            s = scale * (Kp @ q[j, h])
            e = np.exp(s - s.max())
            out[j, h] = (e[:, None] * Vp).sum(0) / e.sum()
            lse[j, h] = s.max() + np.log(e.sum())
    return out, lse


class OracleCache:
    """Logical RIPE cache: which (position, plane) pairs are stored, and their bf16 bits.

    Rules (RIPE abstract, fourth sentence; accept/rollback from the WaveFront
    write-up, section on drafting and checking in one pass):
      * committed position t < T - W keeps only the deepest plane R-1;
      * committed position t >= T - W keeps all R planes (the window);
      * the current draft block (positions T .. T+B-1) holds the planes
        appended so far;
      * commit(a): block positions j < a_n become committed, the rest are
        discarded; then positions that left the window drop planes 0 .. R-2.
    ``W >= max_T`` is the full cache, ``W = 0`` keeps only the deepest plane.
    ``value_planes`` (optional) limits which planes keep their bf16 values, to save host
    memory on large shapes; presence is tracked for every plane either way.
    """

    def __init__(self, N, L, kvH, d, R, W, max_T, mode=QUERY_RELATIVE, value_planes=None):
        self.N, self.L, self.kvH, self.d, self.R, self.W = N, L, kvH, d, R, W
        self.max_T, self.mode = max_T, mode
        self.T = np.zeros(N, dtype=np.int64)
        self.B = 0
        self.appended = np.zeros((L, R), dtype=bool)
        self.drafted = np.zeros((L, R), dtype=np.int64)   # draft positions stored per plane
        self.present = np.zeros((L, R, N, max_T), dtype=bool)
        self._K = {}
        self._V = {}
        self._prefix_set = False
        self.value_planes = None if value_planes is None else set(int(p) for p in value_planes)

    def _keeps(self, plane):
        return self.value_planes is None or plane in self.value_planes

    def _arr(self, store, layer, plane):
        key = (layer, plane)
        if key not in store:
            store[key] = np.zeros((self.N, self.kvH, self.max_T, self.d), dtype=np.uint16)
        return store[key]

    def values(self, layer, plane, which="K"):
        """bf16 bits [N][kvH][max_T][d] of one plane (zeros where never written)."""
        store = self._K if which == "K" else self._V
        return self._arr(store, layer, plane)

    # -- maintenance ------------------------------------------------------------
    def load_prefix(self, layer, plane, T, k, v):
        """Store what RIPE keeps of one plane of a prefix: k, v bits [N][kvH][>=T][d]."""
        T = np.asarray(T, dtype=np.int64)
        if self.B or self.drafted.any():
            raise RuntimeError("load_prefix with a draft block in flight")
        if self._prefix_set and not np.array_equal(T, self.T):
            raise ValueError("prefix lengths differ between calls")
        self.T = T.copy()
        self._prefix_set = True
        keep = self._keeps(plane)
        for n in range(self.N):
            lo = 0 if plane == self.R - 1 else max(0, int(T[n]) - self.W)
            hi = int(T[n])
            if keep:
                self._arr(self._K, layer, plane)[n, :, lo:hi] = k[n, :, lo:hi]
                self._arr(self._V, layer, plane)[n, :, lo:hi] = v[n, :, lo:hi]
            self.present[layer, plane, n, lo:hi] = True

    def append(self, layer, r, k, v, B=None):
        """Plane r of the draft block for one layer: k, v bits [N][B][kvH][d].

        For a plane outside ``value_planes`` k and v may be None (then B is required).
        """
        B = k.shape[1] if k is not None else int(B)
        if self.B and B != self.B:
            raise ValueError("block length changed inside a block")
        if np.any(self.T + B > self.max_T):
            raise ValueError("capacity")
        self.B = B
        keep = self._keeps(r)
        for n in range(self.N):
            t0 = int(self.T[n])
            if keep:
                self._arr(self._K, layer, r)[n, :, t0:t0 + B] = np.transpose(k[n], (1, 0, 2))
                self._arr(self._V, layer, r)[n, :, t0:t0 + B] = np.transpose(v[n], (1, 0, 2))
            self.present[layer, r, n, t0:t0 + B] = True
        self.appended[layer, r] = True

    def commit(self, accepted):
        """Accept the first a_n block positions of each sequence, discard the rest, evict."""
        a = np.asarray(accepted, dtype=np.int64)
        if not self.appended.all():
            raise RuntimeError("commit before every plane of the block was appended")
        if np.any(a < 0) or np.any(a > self.B):
            raise ValueError("accepted length out of range")
        span = max(self.B, int(self.drafted.max()))   # drafts past the block are discarded too
        for n in range(self.N):
            t0 = int(self.T[n])
            rej = slice(t0 + int(a[n]), t0 + span)
            self.present[:, :, n, rej] = False
            for store in (self._K, self._V):
                for arr in store.values():
                    arr[n, :, rej] = 0
            self.T[n] = t0 + int(a[n])
            old = slice(0, max(0, int(self.T[n]) - self.W))
            self.present[:, : self.R - 1, n, old] = False
            for (layer, plane), arr in list(self._K.items()) + list(self._V.items()):
                if plane < self.R - 1:
                    arr[n, :, old] = 0
        self.B = 0
        self.appended[:] = False
        self.drafted[:] = 0

    # -- draft phase --------------------------------------------------------------
    def draft(self, layer, r, j, k, v, q_bits, g, scale=1.0, sink=None, window=None):
        """Draft step at loop r for block position j of every sequence.

        Stores plane r of position T_n + j (k, v bits [N][1][kvH][d]); positions after j of
        that plane become stale.  Then the query q_bits [N][1][Hq][d] of position p = T_n + j
        attends over keys t <= p: the definition of ``verify`` with a block of j + 1
        positions, row j (the drafts 0 .. j at plane r, the window from p, older keys at the
        deepest plane).  Returns (out [N][1][Hq][d], lse [N][1][Hq]) in fp64.

        With ``sink`` and ``window`` (windowed draft attention: a sliding window plus an
        attention sink on the draft's attention only, the Windowed-MTP abstract), only the
        keys t < sink and t >= p - window are attended, each at the plane the rule above
        gives it (``windowed_draft``).
        """
        if self.B:
            raise RuntimeError("draft step with a verification block in flight")
        if j < 0 or j > self.drafted[layer, r]:
            raise RuntimeError("draft positions of a plane are written in order")
        if np.any(self.T + j + 1 > self.max_T):
            raise ValueError("capacity")
        keep = self._keeps(r)
        for n in range(self.N):
            t = int(self.T[n]) + j
            stale = slice(t + 1, int(self.T[n]) + int(self.drafted[layer, r]))
            self.present[layer, r, n, stale] = False
            if keep:
                for store, x in ((self._K, k), (self._V, v)):
                    arr = self._arr(store, layer, r)
                    arr[n, :, t] = x[n, 0]
                    arr[n, :, stale] = 0
            self.present[layer, r, n, t] = True
        self.drafted[layer, r] = j + 1
        if not (keep and self._keeps(self.R - 1)):
            raise RuntimeError("a draft step needs the values of planes r and R-1")
        Kr, Vr, Kl, Vl, _ = self.verify_inputs(layer, r)
        qb = bf16_to_f64(q_bits)
        if sink is not None or window is not None:
            return windowed_draft(self.T, j, r, self.R, self.W, g, Kr, Vr, Kl, Vl, qb[:, 0],
                                  0 if sink is None else int(sink),
                                  int(self.max_T) if window is None else int(window), scale, self.mode)
        qfull = np.zeros((self.N, j + 1) + qb.shape[2:])
        qfull[:, j] = qb[:, 0]
        out, lse = verify(self.T, j + 1, r, self.R, self.W, g, Kr, Vr, Kl, Vl, qfull, scale, self.mode)
        return out[:, j:j + 1], lse[:, j:j + 1]

    # -- queries ----------------------------------------------------------------
    def stored_position_planes(self, layer, n):
        """Stored (position, plane) pairs of committed positions, per key/value head."""
        return int(self.present[layer, :, n, : int(self.T[n])].sum())

    def verify_inputs(self, layer, r):
        """fp64 planes r and R-1 with NaN where the cache stores nothing."""
        ld = self.max_T
        out = []
        for plane in (r, self.R - 1):
            for store in (self._K, self._V):
                x = bf16_to_f64(self._arr(store, layer, plane))
                mask = self.present[layer, plane][:, None, :, None]
                out.append(np.where(np.broadcast_to(mask, x.shape), x, np.nan))
        Kr, Vr, Kl, Vl = out
        return Kr, Vr, Kl, Vl, ld

    def verify(self, layer, r, q_bits, g, scale=1.0):
        """Verification attention of the current block at loop r: (out, lse) in fp64."""
        if not self.appended[layer, r]:
            raise RuntimeError("verify before plane r of the block was appended")
        if not (self._keeps(r) and self._keeps(self.R - 1)):
            raise RuntimeError("verify needs the values of planes r and R-1")
        Kr, Vr, Kl, Vl, _ = self.verify_inputs(layer, r)
        return verify(self.T, self.B, r, self.R, self.W, g, Kr, Vr, Kl, Vl,
                      bf16_to_f64(q_bits), scale, self.mode)


def windowed_draft(T, j, r, R, W, g, Kr, Vr, Kl, Vl, q, sink, window, scale=1.0, mode=QUERY_RELATIVE):
    """Windowed draft attention of one query per sequence (numpy, fp64).

    The query of position p = T_n + j attends over the keys t <= p with t < sink (the
    attention sink) or t >= p - window (the sliding window), each read at the plane the RIPE
    rule gives it (``plane_of``): plane r for the draft rows t >= T_n and the RIPE window,
    plane R-1 otherwise.  Kr/Vr/Kl/Vl as for ``verify`` (NaN where nothing is stored);
    q [N][Hq][d].  Returns (out [N][1][Hq][d], lse [N][1][Hq]).
    """
    T = np.asarray(T, dtype=np.int64)
    N, kvH, _, d = Kr.shape
    Hq = q.shape[1]
    out = np.zeros((N, 1, Hq, d))
    lse = np.zeros((N, 1, Hq))
    for n in range(N):
        Tn = int(T[n])
        p = Tn + j
        keys = [t for t in range(p + 1) if t < sink or t >= p - window]
        planes = np.array([plane_of(p, t, r, R, Tn, W, mode) for t in keys])
        idx = np.array(keys)
        deep = planes == R - 1
        for h in range(Hq):
            kh = h // g
            K = np.where(deep[:, None], Kl[n, kh, idx], Kr[n, kh, idx])
            V = np.where(deep[:, None], Vl[n, kh, idx], Vr[n, kh, idx])
            if np.isnan(K).any() or np.isnan(V).any():
                raise RuntimeError("oracle read a plane that the cache does not store")
            s = scale * (K @ q[n, h])
            m = s.max()
            e = np.exp(s - m)
            out[n, 0, h] = (e[:, None] * V).sum(0) / e.sum()
            lse[n, 0, h] = m + np.log(e.sum())
    return out, lse


def verify_wave(cache, layer, loop_of_position, q_bits, g, scale=1.0):
    """Verification with a loop per block position (several depths in one call, as in a
    wavefront schedule): block position j is evaluated exactly as a single-loop verification
    at loop loop_of_position[j] would evaluate it.  Returns (out, lse) in fp64."""
    loops = [int(x) for x in loop_of_position]
    if len(loops) != cache.B:
        raise ValueError("one loop per block position")
    out = lse = None
    for r in sorted(set(loops)):
        o, l = cache.verify(layer, r, q_bits, g, scale)
        if out is None:
            out, lse = np.zeros_like(o), np.zeros_like(l)
        for j, rj in enumerate(loops):
            if rj == r:
                out[:, j] = o[:, j]
                lse[:, j] = l[:, j]
    return out, lse


def memory_fraction(T, W, R, recurrent_layers=1, other_layers=0, B=1):
    """Stored share of the full cache after decoding T positions, counted by the state machine.

    One recurrent layer with one key/value head and d = 1 is decoded position
    by position (append every plane, accept one) and its stored (position,
    plane) pairs are counted; each of ``other_layers`` non-recurrent layers
    stores one plane per position.  The full cache stores R planes per position
    in every recurrent layer.
    """
    c = OracleCache(N=1, L=1, kvH=1, d=1, R=R, W=W, max_T=T + B)
    one = np.ones((1, 1, 1, 1), dtype=np.uint16)
    for _ in range(T):
        for r in range(R):
            c.append(0, r, one, one)
        c.commit([1])
    stored = c.stored_position_planes(0, 0)
    full = R * T
    return ((recurrent_layers * stored + other_layers * T) /
            (recurrent_layers * full + other_layers * T), stored)
