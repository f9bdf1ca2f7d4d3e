"""The bounds-checked debug build (libca2_debug.so, -DCA2_DEBUG).

Every global access a kernel addresses itself is checked there against its buffer's extent;
a failed check skips the access and records CA2_ERR_BOUNDS.  Here the GPU parity tests of the
small workloads run again in a child process that loads the debug build (CA2_LIBRARY): their
outputs must still meet the oracle and every test must leave the status word clear
(tests/conftest.py checks it after each GPU test).  The tests that plant a timeout or an
out-of-range value read their own status and are included; the large workloads are left to
the release build.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "causal_kv_cache_b200", "libca2_debug.so")


def test_library_flags():
    """The release build says it is not the debug build; the debug build says it is."""
    from causal_kv_cache_b200 import ca2
    if not os.environ.get("CA2_LIBRARY"):
        assert ca2.ca2_debug_build() is False
    r = subprocess.run([sys.executable, "-c", "from causal_kv_cache_b200 import ca2; print(ca2.ca2_debug_build())"],
                       cwd=ROOT, env=dict(os.environ, CA2_LIBRARY=DEBUG_LIB), capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "True"


def test_small_workloads_under_bounds_checks():
    if os.environ.get("CA2_LIBRARY"):
        pytest.skip("already running under another build")
    select = "not os_p41 and not os_p25 and not hires and not 28_blocks and not spatial_max_grows"
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py", "tests/test_gpu_head_shard.py", "-k", select]
    r = subprocess.run(cmd, cwd=ROOT, env=dict(os.environ, CA2_LIBRARY=DEBUG_LIB), capture_output=True, text=True,
                       timeout=1200)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, tail
    assert " passed" in tail and "failed" not in tail
    print(tail)
