"""The bounds-checking debug build: it is built beside the release library,
exports the same C ABI, and MOE_LIBRARY=debug makes the package load it."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def debug_lib():
    import __graft_entry__
    return __graft_entry__._builder().build(variant="debug")


def test_debug_library_exports_the_abi(debug_lib):
    import sparse_mixture_experts_14_b200 as m
    lib = ctypes.CDLL(debug_lib)
    for name in m.SIGNATURES:
        assert hasattr(lib, name), name


def test_environment_selects_the_debug_library(debug_lib):
    code = "import sparse_mixture_experts_14_b200 as m; print(m.loaded_library_path())"
    env = dict(os.environ, MOE_LIBRARY="debug")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, check=True)
    assert out.stdout.strip().endswith("libmoe_debug.so")
    env["MOE_LIBRARY"] = "fast"
    bad = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert bad.returncode != 0 and "MOE_LIBRARY" in bad.stderr
