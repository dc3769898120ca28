"""The debug build (libripe_debug.so, compiled with -DRIPE_DEBUG) on the parity cases.

In that build every tile the verify kernel streams is checked against its region and the plan
(outside: RIPE_DEVERR_BOUNDS in the device error word), and after every commit the ring slots
and deepest-plane rows that hold no live position are filled with the largest finite bf16, so
that a read of a dead slot with non-zero weight turns into a huge or non-finite output.  The
tiny, ragged, fused, state and draft parity tests run against that build in a child process
(the library is chosen when the binding first loads it); each of them ends by asserting that
the device error word is 0.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    "tests/test_gpu_verify.py::test_tiny_config_every_loop",
    "tests/test_gpu_verify.py::test_ragged_tagged_planes",
    "tests/test_gpu_verify.py::test_long_pair_split_over_many_ctas",
    "tests/test_gpu_verify.py::test_heads_split_over_ctas",
    "tests/test_gpu_fused.py::test_fused_append_verify_against_the_oracle",
    "tests/test_gpu_state.py",
    "tests/test_gpu_draft.py",
    "tests/test_gpu_wave.py",
]


def test_debug_build_passes_the_parity_cases(cuda_device):
    from self_speculative_decode_b200 import build
    path = build.build(debug=True)          # already built in-tree by the package build
    env = dict(os.environ, RIPE_LIBRARY=path)
    probe = subprocess.run([sys.executable, "-c", "from self_speculative_decode_b200 import ripe; "
                            "print(ripe.ripe_build_info())"], env=env, cwd=ROOT, capture_output=True,
                           text=True, timeout=300)
    assert probe.returncode == 0 and probe.stdout.strip() == "1", probe.stderr[-2000:]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *CASES],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
