"""The C ABI: the shared library loads without a GPU and exports every entry point
declared in include/ripe.h; host-side argument checks reject bad calls before any
CUDA work."""
import ctypes
import os
import re

import pytest

from self_speculative_decode_b200 import ripe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ripe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ripe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(ripe.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ripe.lib()
    missing = [name for name in _declared() if not hasattr(lib, name)]
    assert not missing


def test_strerror_covers_every_status():
    for st in (0, -1, -2, -3, -4, -5):
        assert ripe.strerror(st) and ripe.strerror(st) != "unknown status"
    assert ripe.strerror(7) == "unknown status"


@pytest.mark.parametrize("args", [
    (0, 1, 2, 2, 64, 4, 16, 128, 4, 0),        # no sequences
    (1025, 1, 2, 2, 64, 4, 16, 128, 4, 0),     # more sequences than the kernels keep in shared memory
    (1, 1, 3, 2, 64, 4, 16, 128, 4, 0),        # q heads not a multiple of kv heads
    (1, 1, 2, 2, 80, 4, 16, 128, 4, 0),        # unsupported head_dim
    (1, 1, 2, 2, 64, 0, 16, 128, 4, 0),        # no loops
    (1, 1, 2, 2, 64, 4, -1, 128, 4, 0),        # negative window
    (1, 1, 2, 2, 64, 4, 16, 128, 0, 0),        # empty block
    (1, 1, 8, 1, 64, 4, 16, 128, 16, 0),       # block x group > 64 query rows
    (1, 1, 2, 2, 64, 4, 16, 128, 4, 2),        # unknown window mode
    (1, 1, 2, 2, 64, 4, 16, 3, 4, 0),          # block longer than the capacity
])
def test_alloc_rejects_bad_arguments_on_the_host(args):
    h = ctypes.c_void_p(123)
    st = ripe.lib().ripe_cache_alloc(*args, ctypes.byref(h))
    assert st == ripe.RIPE_EINVAL
    assert h.value is None


def test_calls_on_a_null_handle_are_rejected():
    L = ripe.lib()
    null = ctypes.c_void_p(0)
    assert L.ripe_verify_attn(null, 0, 0, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_append_block(null, 0, 0, 1, null, null, null) == ripe.RIPE_EINVAL
    assert L.ripe_commit(null, None, null) == ripe.RIPE_EINVAL
    assert L.ripe_append_verify(null, 0, 0, 1, null, null, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_draft_attn(null, 0, 0, 0, null, null, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_draft_attn_window(null, 0, 0, 0, 4, 64, null, null, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_draft_attn_window(null, 0, 0, 0, -1, 64, null, null, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_verify_attn_wave(null, 0, None, null, null, null, 1.0, null) == ripe.RIPE_EINVAL
    assert L.ripe_cache_free(null) == ripe.RIPE_OK
    assert L.ripe_launch_count(null) == -1


def test_verify_consumer_selection():
    """ripe_set_verify_consumer: returns the previous choice, refuses values outside the enum and
    changes nothing then (no device work: runs without a GPU)."""
    L = ripe.lib()
    first = L.ripe_set_verify_consumer(ripe.RIPE_CONSUMER_TC)
    assert first in (ripe.RIPE_CONSUMER_DEFAULT, ripe.RIPE_CONSUMER_MMA, ripe.RIPE_CONSUMER_TC)
    assert L.ripe_get_verify_consumer() == ripe.RIPE_CONSUMER_TC
    assert L.ripe_set_verify_consumer(ripe.RIPE_CONSUMER_MMA) == ripe.RIPE_CONSUMER_TC
    assert L.ripe_set_verify_consumer(7) == ripe.RIPE_EINVAL
    assert L.ripe_set_verify_consumer(-1) == ripe.RIPE_EINVAL
    assert ripe.ripe_get_verify_consumer() == ripe.RIPE_CONSUMER_MMA
    assert ripe.ripe_set_verify_consumer(first) == ripe.RIPE_CONSUMER_MMA
    with pytest.raises(ripe.RipeError):
        ripe.ripe_set_verify_consumer(3)
    assert L.ripe_set_verify_consumer(first) == first


def test_build_info_tells_the_release_and_debug_builds_apart():
    """ripe_build_info: 0 for libripe.so; RIPE_BUILD_DEBUG for libripe_debug.so, which exports the
    same entry points."""
    from self_speculative_decode_b200 import build
    if "RIPE_LIBRARY" not in os.environ:
        assert ripe.ripe_build_info() == 0
    if not os.path.exists(build.LIB_DEBUG):
        pytest.skip("debug build not present")
    dbg = ctypes.CDLL(build.LIB_DEBUG)
    assert dbg.ripe_build_info() == ripe.RIPE_BUILD_DEBUG
    assert not [name for name in _declared() if not hasattr(dbg, name)]
