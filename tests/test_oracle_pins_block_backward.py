"""Pins of the oracle's block backward: gradients of L = sum_t <dout_t, out_t> (+ alpha E sum f p)
for out = h + MoE(RMSNorm(h)), the top-k choice held fixed.

  * fp64 operand storage: backward() on exactly widened operands equals backward() on the
    fp32 originals, bit for bit (the block backward runs the MoE part on fp64 rows)
  * finite differences: every parameter of a tiny fp32 block (h, gamma, Wg, W1, W3, W2) is
    moved by about +-2^-12 (the step actually stored is used) and the central difference of
    L, from the oracle's block forward (and balance() of block_scores() when alpha != 0), is
    compared with the gradient; moves that change the routing are skipped
  * E=1, k=1: the block is h + SwiGLU(RMSNorm(h)); torch autograd in fp64 gives dh, dgamma
    and the expert gradients, and the router gradient is zero
  * k=E: the block is h + sum_e softmax(Wg u)_e E_e(u) with u = RMSNorm(h); torch autograd of
    that expression gives every gradient, dWg and the score gradient included
  * W2 = 0: the MoE part is identically zero, so dh = dout, dgamma = 0, dW1 = dW3 = dWg = 0
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle

EPS = 1e-5


def _t64(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _f64(a, dtype):
    return moe_inputs.bf16_bits_to_f32(a).astype(np.float64) if dtype == "bf16" else np.asarray(a, np.float64)


def _block_inputs(T, d, F, E, k, dtype, seed):
    """Block operands: the residual stream h is the generator's x (rows scaled by powers of two)."""
    return moe_inputs.make_block(moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=seed))


def test_f64_storage_equals_f32():
    inp = moe_inputs.make_inputs(9, 16, 24, 4, 2, "f32", seed=61)
    dout = moe_inputs.make_dout(9, 16, "f32", 61)
    a = oracle.backward(*inp.arrays(), dout, 2, "f32", alpha=0.3)
    b = oracle.backward(*[np.asarray(t, np.float64) for t in inp.arrays()], dout.astype(np.float64), 2, "f64",
                        alpha=0.3)
    for n in ("dx", "dlogits", "dWg", "dW1", "dW3", "dW2", "g", "margin"):
        assert np.array_equal(a[n], b[n]), n
    assert np.array_equal(a["idx"], b["idx"])


def _loss(blk, dout, k, alpha):
    r = oracle.block(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, k, "f32")
    L = float((r["out"] * dout.astype(np.float64)).sum())
    if alpha:
        s = oracle.block_scores(blk.x, blk.gamma, EPS, blk.Wg, "f32")
        L += oracle.balance(s, k, alpha)[2]
    return L, r["idx"]


@pytest.mark.parametrize("alpha", [0.0, 0.7])
def test_finite_differences(alpha):
    T, d, F, E, k = 4, 8, 16, 4, 2
    blk = _block_inputs(T, d, F, E, k, "f32", seed=62)
    dout = moe_inputs.make_dout(T, d, "f32", 62)
    g = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, k, "f32", alpha=alpha)
    _, idx0 = _loss(blk, dout, k, alpha)
    step = 2.0 ** -12
    grads = {"x": g["dh"], "gamma": g["dgamma"], "Wg": g["dWg"], "W1": g["dW1"], "W3": g["dW3"], "W2": g["dW2"]}
    checked = 0
    for name, grad in grads.items():
        flat = getattr(blk, name).reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            flat[i] = np.float32(v + step)
            hp = float(flat[i]) - float(v)
            lp, ip = _loss(blk, dout, k, alpha)
            flat[i] = np.float32(v - step)
            hm = float(v) - float(flat[i])
            lm, im = _loss(blk, dout, k, alpha)
            flat[i] = v
            if not (np.array_equal(ip, idx0) and np.array_equal(im, idx0)):
                continue
            fd = (lp - lm) / (hp + hm)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (name, i, fd, an)
            checked += 1
    assert checked > 1500


def _torch_block(blk, dtype, E_all):
    h = _t64(_f64(blk.x, dtype)).requires_grad_()
    gamma = _t64(_f64(blk.gamma, dtype)).requires_grad_()
    Wg = _t64(_f64(blk.Wg, dtype)).requires_grad_()
    W1 = _t64(_f64(blk.W1, dtype)).requires_grad_()
    W3 = _t64(_f64(blk.W3, dtype)).requires_grad_()
    W2 = _t64(_f64(blk.W2, dtype)).requires_grad_()
    u = torch.nn.functional.rms_norm(h, (h.shape[1],), weight=gamma, eps=EPS)
    s = u @ Wg.T
    s.retain_grad()
    p = torch.softmax(s, dim=1) if E_all else torch.ones_like(s)
    out = h + sum(p[:, e:e + 1] * ((torch.nn.functional.silu(u @ W1[e].T) * (u @ W3[e].T)) @ W2[e].T)
                  for e in range(W1.shape[0]))
    return out, dict(dh=h, dgamma=gamma, dWg=Wg, dW1=W1, dW3=W3, dW2=W2), s


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dense_block_matches_torch_autograd(dtype):
    T, d, F = 7, 16, 24
    blk = _block_inputs(T, d, F, 1, 1, dtype, seed=63)
    dout = moe_inputs.make_dout(T, d, dtype, 63)
    g = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, 1, dtype)
    out, leaves, _ = _torch_block(blk, dtype, E_all=False)
    (out * _t64(_f64(dout, dtype))).sum().backward()
    for n in ("dh", "dgamma", "dW1", "dW3", "dW2"):
        assert np.allclose(g[n], leaves[n].grad.numpy(), rtol=1e-11, atol=1e-13), n
    assert np.all(g["dWg"] == 0.0) and np.all(g["dlogits"] == 0.0)


@pytest.mark.parametrize("E", [2, 3])
def test_softmax_mixture_block_matches_torch_autograd(E):
    T, d, F = 6, 16, 24
    blk = _block_inputs(T, d, F, E, E, "f32", seed=64 + E)
    dout = moe_inputs.make_dout(T, d, "f32", 64)
    g = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, E, "f32")
    out, leaves, s = _torch_block(blk, "f32", E_all=True)
    (out * _t64(dout)).sum().backward()
    for n in ("dh", "dgamma", "dWg", "dW1", "dW3", "dW2"):
        assert np.allclose(g[n], leaves[n].grad.numpy(), rtol=1e-10, atol=1e-12), n
    assert np.allclose(g["dlogits"], s.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_w2_passes_dout_through(dtype):
    T, d, F, E, k = 10, 16, 32, 4, 2
    blk = _block_inputs(T, d, F, E, k, dtype, seed=66)
    blk.W2[:] = 0
    dout = moe_inputs.make_dout(T, d, dtype, 66)
    g = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, k, dtype)
    assert np.array_equal(g["dh"], _f64(dout, dtype))
    for n in ("dgamma", "dWg", "dW1", "dW3", "dlogits"):
        assert np.all(g[n] == 0.0), n
    assert np.any(g["dW2"] != 0.0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_rows_equal_backward_tokens(dtype):
    """backward_rows reads its input rows as float64: given the exactly widened rows of x it is
    backward_tokens bit for bit (the same per-token arithmetic)."""
    inp = moe_inputs.make_inputs(40, 32, 48, 6, 2, dtype, seed=71)
    dout = moe_inputs.make_dout(40, 32, dtype, 71)
    toks = np.array([0, 3, 17, 39], dtype=np.int32)
    a = oracle.backward_tokens(*inp.arrays(), dout, 2, dtype, toks)
    b = oracle.backward_rows(_f64(inp.x[toks], dtype), inp.Wg, inp.W1, inp.W3, inp.W2, dout[toks], 2, dtype)
    for n in ("dx", "dlogits", "g", "margin", "mingap"):
        assert np.array_equal(a[n], b[n]), n
    assert np.array_equal(a["idx"], b["idx"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_backward_tokens_is_block_backward_restricted(dtype):
    """With dout zero on every token but the listed ones, the full block backward's dh rows of the
    listed tokens and its dgamma (a sum in which every other token adds an exact zero) are the
    token-restricted ones; the other tokens get dh = 0."""
    blk = _block_inputs(24, 32, 48, 5, 2, dtype, seed=72)
    dout = moe_inputs.make_dout(24, 32, dtype, 72)
    toks = np.array([1, 2, 11, 23], dtype=np.int64)
    mask = np.zeros(24, dtype=bool)
    mask[toks] = True
    dout[~mask] = 0
    full = oracle.block_backward(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, 2, dtype)
    part = oracle.block_backward_tokens(blk.x, blk.gamma, EPS, blk.Wg, blk.W1, blk.W3, blk.W2, dout, 2, dtype, toks)
    np.testing.assert_allclose(part["dh"], full["dh"][toks], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(part["dgamma"], full["dgamma"], rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(part["dlogits"], full["dlogits"][toks])
    assert np.all(full["dh"][~mask] == 0)
