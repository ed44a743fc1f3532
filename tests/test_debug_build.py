"""The bounds-checking debug library, in place of a memory checker (which cannot run on
these machines).  libattn_sink_debug.so is the same sources compiled with ATTN_SINK_DEBUG:
every global store of an output first checks that its index range lies inside the tensor
it writes, skips the store otherwise and sets bit 3 of the device status word.

The guard-region suite (test_canaries.py) runs again in a child process with that library
loaded: forward (staged, unstaged and grid schedules, head dims 64 / 128 / 256, dv 32,
fp16, fp32, dropout), backward (atomic, deterministic, dropout, every head dim and dtype)
and the packed and paged decode.  Every case must match the oracle, leave its guards intact
and leave the device status word clear."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _debug_library() -> str:
    sys.path.insert(0, ROOT)
    from softmax_attn_sink_b200 import build as B
    return B.LIB_DEBUG if os.path.exists(B.LIB_DEBUG) else B.build(debug=True)


def test_guard_suite_under_the_bounds_checking_library():
    lib = _debug_library()
    env = dict(os.environ, ATTN_SINK_LIBRARY=lib, ATTN_SINK_EXPECT_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_canaries.py"),
                        "-q", "-m", "gpu", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-6000:] + r.stderr[-3000:]
    assert " passed" in r.stdout and "skipped" not in r.stdout, r.stdout[-3000:]
