"""Both consumers of the verify kernel for 9..64 query rows per kv head.

By default the mma.sync consumer serves every launch; the tensor-core (tcgen05) consumer serves the
launches with 9..64 query rows per kv head when the process selects it (ripe_set_verify_consumer, or
the environment variable RIPE_VERIFY_CONSUMER=tc, which sets the initial choice; =mma selects the
default explicitly).  The rest of the suite runs the default; these tests rerun the parity cases that
have more than 8 rows per kv head under each choice, in a child process, including the comparison of
the fused append with the separate calls (bitwise when both run the mma.sync consumer), and check that
the selection call itself switches the kernel in one process.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    "tests/test_gpu_verify.py::test_ragged_tagged_planes",
    "tests/test_gpu_verify.py::test_long_pair_split_over_many_ctas",
    "tests/test_gpu_verify.py::test_heads_split_over_ctas",
    "tests/test_gpu_verify.py::test_live_caches_of_different_batch",
    "tests/test_gpu_configs.py::test_edge_shapes",
    "tests/test_gpu_configs.py::test_long_context_gqa_sampled",
    "tests/test_gpu_configs.py::test_long_context_64_rows_sampled",
    "tests/test_gpu_wave.py",
    "tests/test_gpu_fused.py::test_fused_append_verify_is_bitwise_the_two_calls",
    "tests/test_zz_no_alloc.py",
]


def _rerun(consumer):
    env = dict(os.environ, RIPE_VERIFY_CONSUMER=consumer)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *CASES],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_mma_sync_consumer_parity(cuda_device):
    _rerun("mma")


def test_tcgen05_consumer_parity(cuda_device):
    _rerun("tc")


def test_selection_switches_the_kernel_in_process(cuda_device):
    """ripe_set_verify_consumer between calls on one cache (64 query rows per kv head): both results
    match the oracle, and the two consumers agree within the output rounding."""
    from harness import Case, assert_same_result, check_close, check_lse
    from self_speculative_decode_b200 import ripe
    c = Case(N=2, L=1, Hq=16, kvH=2, d=128, R=3, T=[900, 333], W=20, B=8, seed=21, independent=True)
    got = {}
    prev = ripe.ripe_set_verify_consumer(ripe.RIPE_CONSUMER_TC)
    try:
        for name, consumer in (("tc", ripe.RIPE_CONSUMER_TC), ("mma", ripe.RIPE_CONSUMER_MMA)):
            ripe.ripe_set_verify_consumer(consumer)
            go, gl, ro, rl = c.run(0, 1)
            check_close(go, ro, name)
            check_lse(gl, rl)
            got[name] = go.clone()
    finally:
        ripe.ripe_set_verify_consumer(prev)
    assert_same_result(got["tc"], got["mma"], "tcgen05 vs mma.sync")
    c.close()
