"""The small GPU suite under the bounds-checking debug build (libmoe_debug.so).

The debug build checks every index that one kernel reads from another's
output; a failed check records MOE_ERR_DEVICE and skips the access.  The
parity tests clear and check the status word after every call, so this run
shows that no check fires on correct inputs and that the checked kernels
still match the oracle.  Full-size workloads are left to the release build.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_suite_passes_under_the_debug_build():
    env = dict(os.environ, MOE_LIBRARY="debug")
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           "-k", "not configs and not full_size",
           "tests/test_gpu_parity.py", "tests/test_gpu_block.py", "tests/test_gpu_backward.py",
           "tests/test_gpu_block_backward.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
    probe = subprocess.run([sys.executable, "-c", "import sparse_mixture_experts_14_b200 as m; "
                            "print(m.loaded_library_path())"], cwd=ROOT, env=env, capture_output=True, text=True)
    assert probe.stdout.strip().endswith("libmoe_debug.so")
