"""The small-shape GPU parity tests again, on the bounds-checked build.

libmoe_bounds.so is the library compiled with MOE_BOUNDS: every index its
kernels read from data -- routed experts, task lists, assignment ids,
padded-row offsets -- is range-checked, and a value out of range is recorded
as MOE_EDEVICE in the workspace's status word.  The parity tests check the
status word after every call, so running them on this build shows that no
index leaves its range on any path (decode kernels, dp4a multi-kernel path,
tensor-core path, routers, ties, the allocation-free router).  Each group
runs in a child process with MOE_LIBRARY=bounds, which makes the package
load the checked build.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GROUPS = {
    "parity_small": ["tests/test_gpu_parity.py", "-k", "small or one_token or quantize or route"],
    "tensor_core": ["tests/test_gpu_tc.py", "-k", "not full and not prefill"],
    "ties": ["tests/test_gpu_ties.py"],
    "waits": ["tests/test_gpu_waits.py"],
}


@pytest.mark.parametrize("group", list(GROUPS))
def test_small_cases_on_the_bounds_checked_build(group):
    lib = os.path.join(ROOT, "expert_ffn_router_b200", "libmoe_bounds.so")
    assert os.path.exists(lib), "libmoe_bounds.so is not built"
    env = dict(os.environ, MOE_LIBRARY="bounds")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider"] +
                       GROUPS[group], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert "passed" in r.stdout
