"""Backward of the block form out = h + MoE(RMSNorm(h)) against the fp64 oracle, through the C ABI.

The forward runs moe_block_forward_ws with MOE_PATH_TRAIN; moe_block_backward_ws reads its
workspace.  Tolerances follow test_gpu_backward's per-entry and bulk rules (the MoE part carries
three bf16 roundings in series), applied to the part of each gradient the MoE layer produces:
dh - dout for dh (the residual passes dout through exactly; dh is rounded once at the end, which
adds 2^-8 |dh| (bf16) or 2^-22 |dh| (fp32) per entry).  The oracle runs the MoE backward at the
exact normalised rows; the GPU's experts see them rounded once, which is inside the same bounds.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_testlib import MARGIN, experts_reached, stratified_tokens, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5
TOL = {"bf16": 2e-2 * np.sqrt(3.0), "f32": 1e-5}
BULK = {"bf16": 1e-2, "f32": 2e-6}
FINAL = {"bf16": 2.0 ** -8, "f32": 2.0 ** -22}


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _f64(t):
    return t.double().cpu().numpy()


def _check(name, got, want, dtype, K=256, base=None):
    """Per entry |G - G*| <= tol (RMS(M*) + |M*|) + final |G*| and RMS(G - G*) <= bulk RMS(M*), where
    M* = G* - base is the MoE-produced part (base: the exact pass-through, dout for dh)."""
    scale = max(1.0, np.sqrt(K / 256.0)) if dtype == "f32" else 1.0
    tol, bulk = TOL[dtype] * scale, BULK[dtype] * scale
    m = want - base if base is not None else want
    rms = np.sqrt((m ** 2).mean())
    err = np.abs(got - want)
    excess = (err - tol * np.abs(m) - FINAL[dtype] * np.abs(want)).max()
    l2 = np.sqrt((err ** 2).mean()) / rms
    print(f"  {name}: max|err|/RMS {err.max() / rms:.3e}  excess/RMS {excess / rms:.3e}  rms err/RMS {l2:.3e}")
    assert excess <= tol * rms, f"{name}: max excess {excess:.3e} > {tol:.2e} x RMS {rms:.3e}"
    assert l2 <= bulk + FINAL[dtype] * np.sqrt((want ** 2).mean()) / rms, f"{name}: RMS error {l2:.3e}"


def _run(moe, blk, dev, dout_d, alpha=0.0, dlogits=True, wgrad=torch.float32):
    h, gamma, Wg, W1, W3, W2 = dev
    T, d, F, E, k = blk.T, blk.d, blk.F, blk.E, blk.k
    code = moe.MOE_DTYPE_BF16 if blk.dtype == "bf16" else moe.MOE_DTYPE_F32
    fws = torch.empty(moe.moe_block_train_workspace_size(T, d, F, E, k, code), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(h)
    moe.moe_block_forward_ws(h, gamma, EPS, Wg, W1, W3, W2, k, fws, out, alpha=alpha, path=moe.MOE_PATH_TRAIN)
    dl = torch.empty((T, E), dtype=torch.float32, device="cuda") if dlogits else None
    grads, n = moe.moe_block_backward_ws(h, gamma, Wg, W1, W3, W2, dout_d, k, fws, dlogits=dl, alpha=alpha,
                                         wgrad_dtype=wgrad)
    assert moe.moe_get_device_status() == moe.MOE_OK
    if dl is not None:
        grads["dlogits"] = dl
    return out, grads, n


def _upload(blk):
    dt = blk.dtype
    return [to_dev(a, dt) for a in (blk.x, blk.gamma, blk.Wg, blk.W1, blk.W3, blk.W2)]


def _blk(T, d, F, E, k, dtype, seed):
    return moe_inputs.make_block(moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=seed))


@pytest.mark.parametrize("dtype,T,d,F,E,k,alpha", [("bf16", 200, 256, 512, 8, 2, 0.0), ("bf16", 300, 192, 384, 4, 2, 0.5),
                                                   ("bf16", 90, 128, 256, 16, 4, 0.0),
                                                   ("f32", 64, 128, 256, 8, 2, 0.0), ("f32", 120, 96, 160, 5, 3, 0.5)])
def test_block_backward_small(moe, dtype, T, d, F, E, k, alpha):
    blk = _blk(T, d, F, E, k, dtype, seed=T + d + k)
    dout = moe_inputs.make_dout(T, d, dtype, seed=T + 1)
    dev = _upload(blk)
    _, g, n = _run(moe, blk, dev, to_dev(dout, dtype), alpha=alpha)
    assert n == (10 if dtype == "bf16" else 11)   # the layer backward's launches and the dgamma reduction
    ref = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, k, dtype, alpha=alpha)
    if not (ref["margin"] >= MARGIN).all():
        pytest.skip("a token sits within the routing margin; the weight gradients would include its choice")
    K = max(d, F, T)
    dout64 = dout.astype(np.float64) if dtype == "f32" else moe_inputs.bf16_bits_to_f32(dout).astype(np.float64)
    _check("dh", _f64(g["dh"]), ref["dh"], dtype, K, base=dout64)
    for name in ("dgamma", "dWg", "dW1", "dW3", "dW2", "dlogits"):
        _check(name, _f64(g[name]), ref[name], dtype, K)


def test_block_backward_run_to_run_bitwise(moe):
    blk = _blk(333, 256, 384, 8, 2, "bf16", seed=5)
    dout = to_dev(moe_inputs.make_dout(333, 256, "bf16", seed=5), "bf16")
    dev = _upload(blk)
    _, a, _ = _run(moe, blk, dev, dout)
    _, b, _ = _run(moe, blk, dev, dout)
    for name in a:
        assert torch.equal(a[name], b[name]), name


@pytest.mark.parametrize("cfg", [3])
def test_block_backward_full_size(moe, cfg):
    """Full-size workload, dout kept on a stratified token sample and zero elsewhere: dh of the
    sample and dgamma (a sum over the sample only) against the oracle's token-restricted block
    backward; every other token gets dh = 0 exactly."""
    blk = moe_inputs.make_block(moe_inputs.make_config(cfg))
    dtype = blk.dtype
    r_idx = oracle.select(oracle.block_scores(blk.x, blk.gamma, EPS, blk.Wg, dtype), blk.k)[0]
    toks = stratified_tokens(r_idx, blk.E, n_random=4, boundaries=2, odd_tail=3, seed=cfg + 20)
    assert experts_reached(r_idx, toks) == set(range(blk.E))
    dout = moe_inputs.make_dout(blk.T, blk.d, dtype, seed=blk.seed)
    mask = np.zeros(blk.T, dtype=bool)
    mask[toks] = True
    dout[~mask] = 0
    dev = _upload(blk)
    _, g, _ = _run(moe, blk, dev, to_dev(dout, dtype))
    ref = oracle.block_backward_tokens(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, blk.k, dtype, toks)
    if not (ref["margin"] >= MARGIN).all():
        pytest.skip("a sampled token sits within the routing margin")
    dout64 = moe_inputs.bf16_bits_to_f32(dout[toks]).astype(np.float64)
    _check("dh", _f64(g["dh"])[toks], ref["dh"], dtype, base=dout64)
    _check("dgamma", _f64(g["dgamma"]), ref["dgamma"], dtype)
    _check("dlogits", _f64(g["dlogits"])[toks], ref["dlogits"], dtype)
    rest = torch.from_numpy(~mask).cuda()
    assert torch.count_nonzero(g["dh"][rest]) == 0
    del dev, g
    torch.cuda.empty_cache()
