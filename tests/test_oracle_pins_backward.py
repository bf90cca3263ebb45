"""Pins of the oracle's backward pass (gradients of L = sum_t <dout_t, out_t>).

  * finite differences: every parameter of a tiny fp32 layer (x, Wg, W1, W3,
    W2) is moved by about +-2^-12 (the step actually stored in fp32 is used)
    and the central difference of L, from the oracle's forward, is compared
    with the backward's gradient; coordinates whose move changes the routing
    are skipped
  * E=1, k=1: the layer is one dense SwiGLU FFN; torch autograd in fp64 gives
    dx, dW1, dW3, dW2, and the router gradient is zero (the gate is always 1)
  * k=E: every expert is selected and the gates are the full softmax of Wg x,
    so the layer is the dense softmax mixture sum_e softmax(Wg x)_e E_e(x);
    torch autograd of that expression gives every gradient, dWg included
  * the token-subset and weight-slice forms equal the full backward
  * load-balance part (alpha != 0): finite differences of L + alpha E sum f p
    (f computed by oracle.balance on the perturbed scores, routing unchanged);
    torch autograd of alpha E sum_e f_e mean_t softmax(s_t)_e with f fixed; with
    k = E every f_e = 1, the loss is the constant alpha E and its gradient 0
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle


def _t64(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _dout(T, d, dtype, seed):
    return moe_inputs.make_dout(T, d, dtype, seed)


def _loss(inp, dout, k):
    r = oracle.moe(*inp.arrays(), k=k, dtype="f32")
    return float((r["out"] * dout.astype(np.float64)).sum()), r["idx"]


def test_finite_differences():
    T, d, F, E, k = 4, 8, 16, 4, 2
    inp = moe_inputs.make_inputs(T, d, F, E, k, "f32", seed=31)
    dout = _dout(T, d, "f32", 31)
    g = oracle.backward(*inp.arrays(), dout, k, "f32")
    _, idx0 = _loss(inp, dout, k)
    h = 2.0 ** -12
    grads = {"x": g["dx"], "Wg": g["dWg"], "W1": g["dW1"], "W3": g["dW3"], "W2": g["dW2"]}
    checked = 0
    for name, grad in grads.items():
        arr = getattr(inp, name)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            flat[i] = np.float32(v + h)
            hp = float(flat[i]) - float(v)          # the step actually taken (fp32 rounding)
            lp, ip = _loss(inp, dout, k)
            flat[i] = np.float32(v - h)
            hm = float(v) - float(flat[i])
            lm, im = _loss(inp, dout, k)
            flat[i] = v
            if not (np.array_equal(ip, idx0) and np.array_equal(im, idx0)):
                continue
            fd = (lp - lm) / (hp + hm)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (name, i, fd, an)
            checked += 1
    assert checked > 1500


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_expert_matches_torch_autograd(dtype):
    T, d, F = 7, 16, 24
    inp = moe_inputs.make_inputs(T, d, F, 1, 1, dtype, seed=32)
    dout = _dout(T, d, dtype, 32)
    g = oracle.backward(*inp.arrays(), dout, 1, dtype)
    x = _t64(inp.as_f32("x")).requires_grad_()
    W1 = _t64(inp.as_f32("W1")[0]).requires_grad_()
    W3 = _t64(inp.as_f32("W3")[0]).requires_grad_()
    W2 = _t64(inp.as_f32("W2")[0]).requires_grad_()
    go = _t64(moe_inputs.bf16_bits_to_f32(dout) if dtype == "bf16" else dout)
    out = (torch.nn.functional.silu(x @ W1.T) * (x @ W3.T)) @ W2.T
    (out * go).sum().backward()
    assert np.allclose(g["dx"], x.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.allclose(g["dW1"][0], W1.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.allclose(g["dW3"][0], W3.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.allclose(g["dW2"][0], W2.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.all(g["dWg"] == 0.0) and np.all(g["dlogits"] == 0.0)


@pytest.mark.parametrize("E", [2, 4])
def test_all_experts_is_softmax_mixture(E):
    T, d, F = 6, 16, 24
    inp = moe_inputs.make_inputs(T, d, F, E, E, "f32", seed=33 + E)
    dout = _dout(T, d, "f32", 33)
    g = oracle.backward(*inp.arrays(), dout, E, "f32")
    x = _t64(inp.x).requires_grad_()
    Wg = _t64(inp.Wg).requires_grad_()
    W1 = _t64(inp.W1).requires_grad_()
    W3 = _t64(inp.W3).requires_grad_()
    W2 = _t64(inp.W2).requires_grad_()
    s = x @ Wg.T
    s.retain_grad()
    p = torch.softmax(s, dim=1)
    out = sum(p[:, e:e + 1] * ((torch.nn.functional.silu(x @ W1[e].T) * (x @ W3[e].T)) @ W2[e].T)
              for e in range(E))
    (out * _t64(dout)).sum().backward()
    for name, t in (("dx", x), ("dWg", Wg), ("dW1", W1), ("dW3", W3), ("dW2", W2)):
        assert np.allclose(g[name], t.grad.numpy(), rtol=1e-11, atol=1e-13), name
    assert np.allclose(g["dlogits"], s.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_token_rows_and_weight_slices_match_full_backward():
    T, d, F, E, k = 23, 32, 48, 4, 2
    inp = moe_inputs.make_inputs(T, d, F, E, k, "bf16", seed=34)
    dout = _dout(T, d, "bf16", 34)
    full = oracle.backward(*inp.arrays(), dout, k, "bf16")
    toks = [22, 0, 9]
    rows = oracle.backward_tokens(*inp.arrays(), dout, k, "bf16", toks)
    assert np.array_equal(rows["dx"], full["dx"][toks])
    assert np.array_equal(rows["dlogits"], full["dlogits"][toks])
    for e in range(E):
        fs = [0, 17, F - 1]
        r1, r3, c2 = oracle.weight_grad_slices(*inp.arrays(), dout, k, "bf16", e, fs)
        assert np.allclose(r1, full["dW1"][e][fs], rtol=1e-12, atol=1e-14)
        assert np.allclose(r3, full["dW3"][e][fs], rtol=1e-12, atol=1e-14)
        assert np.allclose(c2, full["dW2"][e][:, fs], rtol=1e-12, atol=1e-14)


def test_router_gradient_sums_to_zero_over_selected():
    """The gates are a softmax over the k selected scores, so ds sums to zero per token."""
    inp = moe_inputs.make_inputs(30, 16, 16, 6, 3, "f32", seed=35)
    g = oracle.backward(*inp.arrays(), _dout(30, 16, "f32", 35), 3, "f32")
    assert np.allclose(g["dlogits"].sum(axis=1), 0.0, atol=1e-14)
    sel = np.zeros_like(g["dlogits"], dtype=bool)
    np.put_along_axis(sel, g["idx"], True, axis=1)
    assert np.all(g["dlogits"][~sel] == 0.0)


def _loss_bal(inp, dout, k, alpha):
    r = oracle.moe(*inp.arrays(), k=k, dtype="f32")
    _, _, lb = oracle.balance(oracle.scores(inp.x, inp.Wg, "f32"), k, alpha)
    return float((r["out"] * dout.astype(np.float64)).sum()) + lb, r["idx"]


def test_finite_differences_with_balance_loss():
    T, d, F, E, k, alpha = 5, 8, 16, 4, 2, 0.7
    inp = moe_inputs.make_inputs(T, d, F, E, k, "f32", seed=36)
    dout = _dout(T, d, "f32", 36)
    g = oracle.backward(*inp.arrays(), dout, k, "f32", alpha=alpha)
    _, idx0 = _loss_bal(inp, dout, k, alpha)
    h = 2.0 ** -12
    checked = 0
    for name, grad in (("x", g["dx"]), ("Wg", g["dWg"])):
        flat = getattr(inp, name).reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            flat[i] = np.float32(v + h)
            hp = float(flat[i]) - float(v)
            lp, ip = _loss_bal(inp, dout, k, alpha)
            flat[i] = np.float32(v - h)
            hm = float(v) - float(flat[i])
            lm, im = _loss_bal(inp, dout, k, alpha)
            flat[i] = v
            if not (np.array_equal(ip, idx0) and np.array_equal(im, idx0)):
                continue
            fd = (lp - lm) / (hp + hm)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (name, i, fd, an)
            checked += 1
    assert checked > 60
    # the expert weights do not see the balance loss
    g0 = oracle.backward(*inp.arrays(), dout, k, "f32")
    for n in ("dW1", "dW3", "dW2"):
        assert np.array_equal(g[n], g0[n])


def test_balance_grad_matches_torch():
    rng = np.random.default_rng(37)
    s = rng.standard_normal((40, 6))
    k, alpha = 2, 0.3
    f, _, _ = oracle.balance(s, k, alpha)
    st = _t64(s).requires_grad_()
    loss = alpha * 6 * (_t64(f) * torch.softmax(st, dim=1).mean(dim=0)).sum()
    loss.backward()
    assert np.allclose(oracle.balance_grad(s, k, alpha), st.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_balance_grad_vanishes_when_every_expert_is_selected():
    s = np.random.default_rng(38).standard_normal((25, 5))
    assert np.allclose(oracle.balance_grad(s, 5, 1.3), 0.0, atol=1e-16)
