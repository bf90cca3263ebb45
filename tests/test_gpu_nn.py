"""The autograd glue (sparse_mixture_experts_14_b200.nn) on a B200: its gradients are the
C ABI's backward, and a few SGD steps on a fixed target lower the loss."""
import pytest
import torch

import moe_inputs
from moe_testlib import to_dev, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    import sparse_mixture_experts_14_b200 as m
    import sparse_mixture_experts_14_b200.nn as nn
    return m, nn


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_autograd_matches_backward_entry(mods, dtype):
    moe, nn = mods
    T, d, F, E, k = 200, 128, 256, 8, 2
    inp = moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=51)
    dev = [t.clone().requires_grad_() for t in upload(inp)]
    dout = to_dev(moe_inputs.make_dout(T, d, dtype, seed=51), dtype)
    out = nn.MoEFunction.apply(*dev, k, 0.25)
    out.backward(dout)
    ref = moe.moe_forward(*[t.detach() for t in dev], k)
    assert torch.equal(out.detach(), ref)
    code = moe.MOE_DTYPE_BF16 if dtype == "bf16" else moe.MOE_DTYPE_F32
    ws = torch.empty(moe.moe_train_workspace_size(T, d, F, E, k, code), dtype=torch.uint8, device="cuda")
    det = [t.detach() for t in dev]
    moe.moe_forward_ws(*det, k, path=moe.MOE_PATH_TRAIN, workspace=ws)
    g, _ = moe.moe_backward_ws(*det, dout, k, ws, alpha=0.25)
    assert torch.equal(dev[0].grad, g["dx"])
    for t, n in zip(dev[1:], ("dWg", "dW1", "dW3", "dW2")):
        assert torch.equal(t.grad, g[n].to(t.dtype)), n
    assert moe.moe_get_device_status() == moe.MOE_OK


def test_sgd_steps_lower_the_loss(mods):
    moe, nn = mods
    torch.manual_seed(0)
    layer = nn.SparseMoE(d=128, ffn=256, E=8, k=2, alpha=0.01, dtype=torch.float32)
    x = torch.randn(4, 64, 128, device="cuda")
    target = torch.randn(4, 64, 128, device="cuda")
    opt = torch.optim.SGD(layer.parameters(), lr=0.2)
    losses = []
    for _ in range(5):
        opt.zero_grad()
        loss = ((layer(x) - target) ** 2).mean()
        loss.backward()
        opt.step()
        losses.append(loss.item())
    assert losses[-1] < losses[0]
    with torch.no_grad():
        assert layer(x).shape == x.shape
    assert moe.moe_get_device_status() == moe.MOE_OK
