"""Python binding of libripe.so: same names as the C ABI in include/ripe.h.

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and passed as raw device pointers; every step of the work runs in the
library's CUDA kernels.  There is no fallback: if the shared library is missing
or no CUDA device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# the library to load: libripe.so, or another build of the same sources (e.g. the debug build
# lib/libripe_debug.so) named by the environment variable RIPE_LIBRARY
LIB_PATH = os.environ.get("RIPE_LIBRARY") or os.path.join(PKG, "lib", "libripe.so")

RIPE_OK, RIPE_EINVAL, RIPE_ENOMEM, RIPE_ECAPACITY, RIPE_ESTATE, RIPE_ECUDA = 0, -1, -2, -3, -4, -5
RIPE_WINDOW_QUERY_RELATIVE, RIPE_WINDOW_CACHE_RELATIVE = 0, 1
RIPE_DEVERR_WAIT_TIMEOUT, RIPE_DEVERR_CAPACITY, RIPE_DEVERR_ACCEPT, RIPE_DEVERR_BOUNDS = 1, 2, 4, 8
RIPE_BUILD_DEBUG = 1
RIPE_CONSUMER_DEFAULT, RIPE_CONSUMER_MMA, RIPE_CONSUMER_TC = 0, 1, 2

# exported entry points (kept in step with include/ripe.h; a CPU test checks both)
EXPORTS = (
    "ripe_cache_alloc", "ripe_cache_free", "ripe_load_prefix", "ripe_append_block",
    "ripe_verify_attn", "ripe_commit", "ripe_commit_device", "ripe_sync_lengths",
    "ripe_cache_stats", "ripe_cache_export", "ripe_get_device_error", "ripe_launch_count",
    "ripe_strerror", "ripe_verify_attn_static", "ripe_verify_attn_wave", "ripe_append_verify",
    "ripe_draft_attn", "ripe_draft_attn_window", "ripe_build_info", "ripe_set_verify_consumer",
    "ripe_get_verify_consumer",
)
RIPE_ESCRATCH = -6
RIPE_STATIC_SCRATCH_BYTES = 4 << 20


class RipeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} ({status})")


class _Stats(ctypes.Structure):
    _fields_ = [("stored_position_planes", ctypes.c_int64), ("full_position_planes", ctypes.c_int64),
                ("kv_bytes", ctypes.c_int64), ("scratch_bytes", ctypes.c_int64),
                ("deep_rows", ctypes.c_int32), ("ring_slots", ctypes.c_int32),
                ("block_len", ctypes.c_int32), ("lengths_synced", ctypes.c_int32)]


class CacheView(ctypes.Structure):
    """ripe_cache_view: caller-owned cache buffers for ripe_verify_attn_static."""
    _fields_ = [(name, ctypes.c_int32) for name in
                ("batch", "layers", "q_heads", "kv_heads", "head_dim", "loops", "window", "max_T",
                 "max_B", "window_mode", "block_len")] + \
               [(name, ctypes.c_void_p) for name in ("k_deep", "v_deep", "k_ring", "v_ring", "lengths")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libripe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m self_speculative_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        i32p = ctypes.POINTER(ctypes.c_int32)
        sig = {
            "ripe_cache_alloc": ([i] * 10 + [ctypes.POINTER(vp)], i),
            "ripe_cache_free": ([vp], i),
            "ripe_load_prefix": ([vp, i, i, i32p, vp, vp, i64, vp], i),
            "ripe_append_block": ([vp, i, i, i, vp, vp, vp], i),
            "ripe_verify_attn": ([vp, i, i, vp, vp, vp, ctypes.c_float, vp], i),
            "ripe_commit": ([vp, i32p, vp], i),
            "ripe_commit_device": ([vp, vp, vp], i),
            "ripe_sync_lengths": ([vp, i32p, vp], i),
            "ripe_cache_stats": ([vp, ctypes.POINTER(_Stats)], i),
            "ripe_cache_export": ([vp, i, i, vp, vp, vp, vp], i),
            "ripe_get_device_error": ([vp, ctypes.POINTER(ctypes.c_uint32), vp], i),
            "ripe_launch_count": ([vp], i64),
            "ripe_build_info": ([], i),
            "ripe_set_verify_consumer": ([i], i),
            "ripe_get_verify_consumer": ([], i),
            "ripe_strerror": ([i], ctypes.c_char_p),
            "ripe_verify_attn_static": ([ctypes.POINTER(CacheView), i, i, vp, vp, vp, ctypes.c_float, vp, vp], i),
            "ripe_verify_attn_wave": ([vp, i, i32p, vp, vp, vp, ctypes.c_float, vp], i),
            "ripe_append_verify": ([vp, i, i, i, vp, vp, vp, vp, vp, ctypes.c_float, vp], i),
            "ripe_draft_attn": ([vp, i, i, i, vp, vp, vp, vp, vp, ctypes.c_float, vp], i),
            "ripe_draft_attn_window": ([vp, i, i, i, i, i, vp, vp, vp, vp, vp, ctypes.c_float, vp], i),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes, fn.restype = args, res
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().ripe_strerror(status).decode()


def _check(status: int, where: str):
    if status != RIPE_OK:
        raise RipeError(status, where)


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype, shape, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _ints(values, n):
    arr = (ctypes.c_int32 * n)(*[int(x) for x in values])
    if len(values) != n:
        raise ValueError(f"expected {n} values")
    return arr


# ------------------------------------------------------------------ C-ABI mirrors
def ripe_cache_alloc(batch, layers, q_heads, kv_heads, head_dim, loops, window, max_T, max_B,
                     window_mode=RIPE_WINDOW_QUERY_RELATIVE):
    h = ctypes.c_void_p()
    _check(lib().ripe_cache_alloc(batch, layers, q_heads, kv_heads, head_dim, loops, window, max_T,
                                  max_B, window_mode, ctypes.byref(h)), "ripe_cache_alloc")
    return h


def ripe_cache_free(h):
    _check(lib().ripe_cache_free(h), "ripe_cache_free")


def ripe_load_prefix(h, layer, plane, T, k, v, ld_t, stream=None):
    n = len(T)
    _check(lib().ripe_load_prefix(h, layer, plane, _ints(T, n), ctypes.c_void_p(k), ctypes.c_void_p(v),
                                  ld_t, _stream(stream)), "ripe_load_prefix")


def ripe_append_block(h, layer, r, B, k, v, stream=None):
    _check(lib().ripe_append_block(h, layer, r, B, ctypes.c_void_p(k), ctypes.c_void_p(v), _stream(stream)),
           "ripe_append_block")


def ripe_verify_attn(h, layer, r, q, out, lse=None, scale=1.0, stream=None):
    _check(lib().ripe_verify_attn(h, layer, r, ctypes.c_void_p(q), ctypes.c_void_p(out),
                                  ctypes.c_void_p(lse or 0), float(scale), _stream(stream)),
           "ripe_verify_attn")


def ripe_append_verify(h, layer, r, B, k, v, q, out, lse=None, scale=1.0, stream=None):
    _check(lib().ripe_append_verify(h, layer, r, B, ctypes.c_void_p(k), ctypes.c_void_p(v), ctypes.c_void_p(q),
                                    ctypes.c_void_p(out), ctypes.c_void_p(lse or 0), float(scale),
                                    _stream(stream)), "ripe_append_verify")


def ripe_draft_attn(h, layer, r, j, k, v, q, out, lse=None, scale=1.0, stream=None):
    _check(lib().ripe_draft_attn(h, layer, r, j, ctypes.c_void_p(k), ctypes.c_void_p(v), ctypes.c_void_p(q),
                                 ctypes.c_void_p(out), ctypes.c_void_p(lse or 0), float(scale),
                                 _stream(stream)), "ripe_draft_attn")


def ripe_draft_attn_window(h, layer, r, j, sink, window, k, v, q, out, lse=None, scale=1.0, stream=None):
    _check(lib().ripe_draft_attn_window(h, layer, r, j, int(sink), int(window), ctypes.c_void_p(k), ctypes.c_void_p(v),
                                        ctypes.c_void_p(q), ctypes.c_void_p(out), ctypes.c_void_p(lse or 0),
                                        float(scale), _stream(stream)), "ripe_draft_attn_window")


def ripe_verify_attn_wave(h, layer, loop_of_position, q, out, lse=None, scale=1.0, stream=None):
    _check(lib().ripe_verify_attn_wave(h, layer, _ints(loop_of_position, len(loop_of_position)),
                                       ctypes.c_void_p(q), ctypes.c_void_p(out), ctypes.c_void_p(lse or 0),
                                       float(scale), _stream(stream)), "ripe_verify_attn_wave")


def ripe_commit(h, accepted_len, stream=None):
    _check(lib().ripe_commit(h, _ints(accepted_len, len(accepted_len)), _stream(stream)), "ripe_commit")


def ripe_commit_device(h, accepted_ptr, stream=None):
    _check(lib().ripe_commit_device(h, ctypes.c_void_p(accepted_ptr), _stream(stream)), "ripe_commit_device")


def ripe_sync_lengths(h, n, stream=None):
    out = (ctypes.c_int32 * n)()
    _check(lib().ripe_sync_lengths(h, out, _stream(stream)), "ripe_sync_lengths")
    return list(out)


def ripe_cache_stats(h):
    st = _Stats()
    _check(lib().ripe_cache_stats(h, ctypes.byref(st)), "ripe_cache_stats")
    return {name: getattr(st, name) for name, _ in _Stats._fields_}


def ripe_cache_export(h, n, layer, k_out, v_out, present, stream=None):
    _check(lib().ripe_cache_export(h, n, layer, ctypes.c_void_p(k_out), ctypes.c_void_p(v_out),
                                   ctypes.c_void_p(present), _stream(stream)), "ripe_cache_export")


def ripe_get_device_error(h, stream=None):
    e = ctypes.c_uint32()
    _check(lib().ripe_get_device_error(h, ctypes.byref(e), _stream(stream)), "ripe_get_device_error")
    return e.value


def ripe_verify_attn_static(view, layer, r, q, out, lse=None, scale=1.0, device_error=None, stream=None):
    """Allocation-free verify over caller-owned buffers (see include/ripe.h); pointers are ints."""
    _check(lib().ripe_verify_attn_static(ctypes.byref(view), layer, r, ctypes.c_void_p(q), ctypes.c_void_p(out),
                                         ctypes.c_void_p(lse or 0), float(scale),
                                         ctypes.c_void_p(device_error or 0), _stream(stream)),
           "ripe_verify_attn_static")


def ripe_launch_count(h):
    return lib().ripe_launch_count(h)


def ripe_build_info():
    return lib().ripe_build_info()


def ripe_set_verify_consumer(consumer):
    """Select the consumer of verification launches with 9..64 query rows per kv head (process-wide);
    returns the previous choice."""
    prev = lib().ripe_set_verify_consumer(int(consumer))
    _check(prev if prev < 0 else RIPE_OK, "ripe_set_verify_consumer")
    return prev


def ripe_get_verify_consumer():
    return lib().ripe_get_verify_consumer()


# ------------------------------------------------------------------ tensor-level wrapper
class RipeCache:
    """A RIPE cache on the current CUDA device, driven with torch tensors.

    Shapes (bf16, contiguous, on the cache's device):
      prefix plane  k, v [N][kvH][ld_t][d]
      block plane   k, v [N][B][kvH][d]
      queries       q, out [N][B][Hq][d]; lse fp32 [N][B][Hq]
    """

    def __init__(self, batch, layers, q_heads, kv_heads, head_dim, loops, window, max_T, max_B,
                 window_mode=RIPE_WINDOW_QUERY_RELATIVE):
        import torch
        if not torch.cuda.is_available():
            raise RuntimeError("RipeCache needs a CUDA device")
        self.N, self.L, self.Hq, self.kvH, self.d = batch, layers, q_heads, kv_heads, head_dim
        self.R, self.W, self.max_T, self.max_B, self.mode = loops, window, max_T, max_B, window_mode
        self.handle = ripe_cache_alloc(batch, layers, q_heads, kv_heads, head_dim, loops, window, max_T,
                                       max_B, window_mode)

    def close(self):
        if self.handle is not None and self.handle.value:
            ripe_cache_free(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load_prefix(self, layer, plane, T, k, v, stream=None):
        import torch
        ld_t = k.shape[2]
        shape = (self.N, self.kvH, ld_t, self.d)
        ripe_load_prefix(self.handle, layer, plane, list(T), _dev(k, torch.bfloat16, shape, "k").value,
                         _dev(v, torch.bfloat16, shape, "v").value, ld_t, stream)

    def append_block(self, layer, r, k, v, stream=None):
        import torch
        B = k.shape[1]
        shape = (self.N, B, self.kvH, self.d)
        ripe_append_block(self.handle, layer, r, B, _dev(k, torch.bfloat16, shape, "k").value,
                          _dev(v, torch.bfloat16, shape, "v").value, stream)

    def verify_attn(self, layer, r, q, out=None, lse=None, scale=1.0, stream=None):
        import torch
        B = q.shape[1]
        shape = (self.N, B, self.Hq, self.d)
        qp = _dev(q, torch.bfloat16, shape, "q").value
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
        op = _dev(out, torch.bfloat16, shape, "out").value
        lp = _dev(lse, torch.float32, shape[:3], "lse").value if lse is not None else None
        ripe_verify_attn(self.handle, layer, r, qp, op, lp, scale, stream)
        return out

    def append_verify(self, layer, r, k, v, q, out=None, lse=None, scale=1.0, stream=None):
        """append_block(layer, r, k, v) + verify_attn(layer, r, q) in one launch."""
        import torch
        B = q.shape[1]
        kshape = (self.N, B, self.kvH, self.d)
        shape = (self.N, B, self.Hq, self.d)
        kp = _dev(k, torch.bfloat16, kshape, "k").value
        vp = _dev(v, torch.bfloat16, kshape, "v").value
        qp = _dev(q, torch.bfloat16, shape, "q").value
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
        op = _dev(out, torch.bfloat16, shape, "out").value
        lp = _dev(lse, torch.float32, shape[:3], "lse").value if lse is not None else None
        ripe_append_verify(self.handle, layer, r, B, kp, vp, qp, op, lp, scale, stream)
        return out

    def draft_attn(self, layer, r, j, k, v, q, out=None, lse=None, scale=1.0, stream=None, sink=None,
                   window=None):
        """Draft step: write plane r of block position j (k, v [N][1][kvH][d]) and attend its
        query q [N][1][Hq][d] over keys up to that position; with ``sink`` / ``window`` only
        over the first ``sink`` keys and the last ``window`` + 1 (windowed draft attention)."""
        import torch
        kshape = (self.N, 1, self.kvH, self.d)
        shape = (self.N, 1, self.Hq, self.d)
        kp = _dev(k, torch.bfloat16, kshape, "k").value
        vp = _dev(v, torch.bfloat16, kshape, "v").value
        qp = _dev(q, torch.bfloat16, shape, "q").value
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
        op = _dev(out, torch.bfloat16, shape, "out").value
        lp = _dev(lse, torch.float32, shape[:3], "lse").value if lse is not None else None
        if sink is None and window is None:
            ripe_draft_attn(self.handle, layer, r, j, kp, vp, qp, op, lp, scale, stream)
        else:
            ripe_draft_attn_window(self.handle, layer, r, j, 0 if sink is None else sink,
                                   (1 << 30) if window is None else window, kp, vp, qp, op, lp, scale, stream)
        return out

    def verify_attn_wave(self, layer, loop_of_position, q, out=None, lse=None, scale=1.0, stream=None):
        """Block position j verified at loop loop_of_position[j] (one pass over the deepest plane)."""
        import torch
        B = q.shape[1]
        shape = (self.N, B, self.Hq, self.d)
        qp = _dev(q, torch.bfloat16, shape, "q").value
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
        op = _dev(out, torch.bfloat16, shape, "out").value
        lp = _dev(lse, torch.float32, shape[:3], "lse").value if lse is not None else None
        ripe_verify_attn_wave(self.handle, layer, list(loop_of_position), qp, op, lp, scale, stream)
        return out

    def commit(self, accepted_len, stream=None):
        ripe_commit(self.handle, list(accepted_len), stream)

    def commit_device(self, accepted, stream=None):
        import torch
        ripe_commit_device(self.handle, _dev(accepted, torch.int32, (self.N,), "accepted").value, stream)

    def sync_lengths(self, stream=None):
        return ripe_sync_lengths(self.handle, self.N, stream)

    def stats(self):
        return ripe_cache_stats(self.handle)

    def export(self, n, layer, stream=None):
        """Logical view of sequence n, layer: (k, v [R][kvH][Tv][d] bf16, present [R][Tv] uint8)."""
        import torch
        st = self.stats()
        if not st["lengths_synced"]:
            raise RipeError(RIPE_ESTATE, "export")
        Tv = self.sync_lengths(stream)[n] + st["block_len"]
        dev = torch.device("cuda", torch.cuda.current_device())
        k = torch.zeros((self.R, self.kvH, Tv, self.d), dtype=torch.bfloat16, device=dev)
        v = torch.zeros_like(k)
        present = torch.zeros((self.R, Tv), dtype=torch.uint8, device=dev)
        if Tv:
            ripe_cache_export(self.handle, n, layer, k.data_ptr(), v.data_ptr(), present.data_ptr(), stream)
        return k, v, present

    def device_error(self, stream=None):
        return ripe_get_device_error(self.handle, stream)

    def launch_count(self):
        return ripe_launch_count(self.handle)
