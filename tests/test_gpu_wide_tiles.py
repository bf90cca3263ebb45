"""Wide (256 x 512) and standard (256 x 256) tiles of the grouped GEMMs give the same bits.

The library picks the wide tile when a GEMM's reduction is 5120 or longer; the
environment variable MOE_WIDE_MIN_K moves that threshold.  Each output element
sees the same tensor-core MMAs in the same K order in both tile shapes, so the
layer (GEMM1 and GEMM2 wide here) and the backward (dXp wide) must match a run
with every tile 256 x 256 bit for bit.  The threshold is read once per process,
so the all-standard run is a child process.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE = (300, 5120, 5120, 8, 2)   # T, d, ffn, E, k: GEMM1 (K = d), GEMM2 (K = ffn) and dXp (K = 2 ffn) wide

CHILD = r"""
import sys, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import sparse_mixture_experts_14_b200 as moe, moe_inputs
from moe_testlib import upload, to_dev
T, d, F, E, k = {shape!r}
inp = moe_inputs.make_inputs(T, d, F, E, k, "bf16", seed=5)
dev = upload(inp)
dout = to_dev(moe_inputs.make_dout(T, d, "bf16", seed=5), "bf16")
ws = torch.empty(moe.moe_train_workspace_size(T, d, F, E, k), dtype=torch.uint8, device="cuda")
out = moe.moe_forward_ws(*dev, k, path=moe.MOE_PATH_TRAIN, workspace=ws)
g, _ = moe.moe_backward_ws(*dev, dout, k, ws)
assert moe.moe_get_device_status() == moe.MOE_OK
torch.save({{"out": moe.moe_forward(*dev, k).cpu(), "train_out": out.cpu(), "dx": g["dx"].cpu(),
            "dW1": g["dW1"].cpu()}}, {path!r})
"""


def _run(env_min_k, path):
    env = dict(os.environ)
    if env_min_k is None:
        env.pop("MOE_WIDE_MIN_K", None)
    else:
        env["MOE_WIDE_MIN_K"] = str(env_min_k)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), shape=SHAPE, path=str(path))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    return torch.load(str(path))


def test_wide_and_standard_tiles_give_the_same_bits(tmp_path):
    wide = _run(None, tmp_path / "wide.pt")
    std = _run(1 << 30, tmp_path / "std.pt")
    for n in ("out", "train_out", "dx", "dW1"):
        assert torch.equal(wide[n], std[n]), n
