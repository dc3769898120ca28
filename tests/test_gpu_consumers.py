"""Both consumers of the verify kernel for 9..64 query rows per kv head.

By default the mma.sync consumer serves every launch except long pairs with head_dim 128 and
57..64 query rows per kv head, which the tensor-core (tcgen05) consumer serves;
RIPE_VERIFY_CONSUMER=tc or =mma puts one of them on all of 9..64 rows.  The rest of the suite runs
the default; these tests rerun the parity cases that have more than 8 rows per kv head under each
override, in a child process (the choice is
read once, when the library first launches a verify kernel), including the comparison of the fused
append with the separate calls (bitwise when both run the mma.sync consumer).
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
