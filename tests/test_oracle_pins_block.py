"""Pins of the oracle's block and load-balance steps to things other than itself.

"Mistral/Mixtral architecture" page:
  * section "Mixtral 8x7B — Sparse MoEの導入", subsection "Mixtralのアーキテクチャ":
    the MoE sub-layer of a block is RMSNorm, then the MoE layer, then the
    residual connection.  The page prints no RMSNorm formula; the oracle uses
    gamma_j h_j / sqrt(mean(h^2) + eps), which torch's ``rms_norm`` also computes.
  * subsection "ロードバランス損失": f_i, p_i and L = alpha * N * sum f_i p_i.

What pins what:
  rmsnorm   torch.nn.functional.rms_norm in fp64; a 2-element example by hand;
            exact invariance under power-of-two scaling at eps = 0; unit RMS;
            a zero row stays zero
  block     E=1, k=1 reduces to h + one dense SwiGLU FFN on the normalised row;
            k=E with a zero router reduces to h + the mean of all experts (torch
            fp64); router scores equal torch's normalised row times Wg^T;
            routing is invariant under power-of-two row scaling
  balance   uniform scores give p = 1/E and L = alpha*k; the cyclic batch of
            every rotation of one score vector is perfectly balanced (f = k/E,
            p = 1/E, L = alpha*k: the page's balanced case, with f summing to k
            as in its code); brute-force top-k and torch softmax on random
            scores; a 2-token example by hand
"""
import itertools
import math

import numpy as np
import pytest
import torch

import moe_inputs
import oracle

EPS = moe_inputs.BLOCK_EPS


def _t64(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _torch_rmsnorm(h, gamma, eps):
    h = _t64(h)
    return torch.nn.functional.rms_norm(h, (h.shape[-1],), weight=_t64(gamma), eps=eps)


def _torch_swiglu(u, W1, W3, W2):
    u, W1, W3, W2 = (x if isinstance(x, torch.Tensor) else _t64(x) for x in (u, W1, W3, W2))
    return (torch.nn.functional.silu(u @ W1.T) * (u @ W3.T)) @ W2.T


def _block_inputs(T, d, F, E, k, dtype, seed):
    return moe_inputs.make_block(moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=seed))


# ---------------------------------------------------------------- rmsnorm


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rmsnorm_matches_torch(dtype):
    inp = _block_inputs(37, 96, 32, 2, 1, dtype, seed=21)
    u = oracle.rmsnorm(inp.x, inp.gamma, EPS, dtype)
    ref = _torch_rmsnorm(inp.as_f32("x"), inp.as_f32("gamma"), EPS).numpy()
    assert np.allclose(u, ref, rtol=1e-13, atol=1e-15)


def test_rmsnorm_hand_example():
    """h = (3, 4): mean square 12.5."""
    h = np.float32([[3, 4]])
    g = np.float32([2, -1])
    u0 = oracle.rmsnorm(h, g, 0.0, "f32")[0]
    assert abs(u0[0] - 6 / math.sqrt(12.5)) < 1e-15 and abs(u0[1] + 4 / math.sqrt(12.5)) < 1e-15
    u1 = oracle.rmsnorm(h, g, 0.5, "f32")[0]
    assert abs(u1[0] - 6 / math.sqrt(13.0)) < 1e-15 and abs(u1[1] + 4 / math.sqrt(13.0)) < 1e-15


def test_rmsnorm_scale_invariance_and_unit_rms():
    inp = _block_inputs(20, 64, 32, 2, 1, "f32", seed=22)
    ones = np.ones(64, dtype=np.float32)
    u = oracle.rmsnorm(inp.x, ones, 0.0, "f32")
    u4 = oracle.rmsnorm(np.ascontiguousarray(inp.x * np.float32(4.0)), ones, 0.0, "f32")
    assert np.array_equal(u, u4)
    assert np.allclose((u ** 2).mean(axis=1), 1.0, rtol=0, atol=1e-14)
    # with a gain, each column is scaled by it
    ug = oracle.rmsnorm(inp.x, inp.gamma, 0.0, "f32")
    assert np.allclose(ug, u * inp.gamma.astype(np.float64)[None, :], rtol=1e-15, atol=0)


def test_rmsnorm_zero_row():
    h = np.zeros((2, 16), dtype=np.float32)
    h[1, 3] = 2.0
    u = oracle.rmsnorm(h, np.ones(16, dtype=np.float32), EPS, "f32")
    assert np.all(u[0] == 0.0)
    assert abs(u[1, 3] - 2.0 / math.sqrt(4.0 / 16 + EPS)) < 1e-14


# ---------------------------------------------------------------- block


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_single_expert_is_dense(dtype):
    """E=1, k=1: out = h + SwiGLU(RMSNorm(h))."""
    inp = _block_inputs(19, 64, 96, 1, 1, dtype, seed=23)
    r = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=1, dtype=dtype)
    assert np.all(r["idx"] == 0) and np.all(r["g"] == 1.0)
    u = _torch_rmsnorm(inp.as_f32("x"), inp.as_f32("gamma"), EPS)
    ref = (_t64(inp.as_f32("x")) + _torch_swiglu(u, inp.as_f32("W1")[0], inp.as_f32("W3")[0],
                                                 inp.as_f32("W2")[0])).numpy()
    assert np.max(np.abs(r["out"] - ref)) < 1e-12 * np.sqrt((ref ** 2).mean())


@pytest.mark.parametrize("E", [2, 4])
def test_block_uniform_router_is_residual_plus_average(E):
    inp = _block_inputs(11, 64, 64, E, E, "f32", seed=24)
    inp.Wg[:] = 0.0
    r = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=E, dtype="f32")
    assert np.all(r["idx"] == np.arange(E)[None, :])
    u = _torch_rmsnorm(inp.x, inp.gamma, EPS)
    mean = sum(_torch_swiglu(u, inp.W1[e], inp.W3[e], inp.W2[e]) for e in range(E)) / E
    ref = (_t64(inp.x) + mean).numpy()
    assert np.max(np.abs(r["out"] - ref)) < 1e-12 * np.sqrt((ref ** 2).mean())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_scores_are_normalised_row_times_router(dtype):
    inp = _block_inputs(33, 96, 32, 6, 2, dtype, seed=25)
    s = oracle.block_scores(inp.x, inp.gamma, EPS, inp.Wg, dtype)
    ref = (_torch_rmsnorm(inp.as_f32("x"), inp.as_f32("gamma"), EPS) @ _t64(inp.as_f32("Wg")).T).numpy()
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-13)
    r = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype=dtype)
    idx, g, margin, _ = oracle.select(s, 2)
    assert np.array_equal(r["idx"], idx) and np.array_equal(r["g"], g) and np.array_equal(r["margin"], margin)


def test_block_routing_ignores_row_scale():
    """At eps = 0 a power-of-two row scale leaves the normalised row, hence the MoE part, unchanged."""
    inp = _block_inputs(24, 64, 64, 8, 2, "f32", seed=26)
    r = oracle.block(inp.x, inp.gamma, 0.0, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="f32")
    h4 = np.ascontiguousarray(inp.x * np.float32(4.0))
    r4 = oracle.block(h4, inp.gamma, 0.0, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="f32")
    assert np.array_equal(r["idx"], r4["idx"]) and np.array_equal(r["g"], r4["g"])
    m = r["out"] - inp.x.astype(np.float64)
    m4 = r4["out"] - h4.astype(np.float64)
    assert np.max(np.abs(m - m4)) < 1e-12 * (1 + np.abs(h4).max())


def test_block_zero_row_gives_zero():
    inp = _block_inputs(3, 32, 32, 4, 2, "f32", seed=27)
    inp.x[1] = 0.0
    r = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="f32")
    assert np.all(r["out"][1] == 0.0)
    assert list(r["idx"][1]) == [0, 1]          # all scores 0: ties to the lowest indices


def test_block_token_subset_matches_full_run():
    inp = _block_inputs(21, 64, 64, 8, 2, "bf16", seed=28)
    args = (inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2)
    full = oracle.block(*args, k=2, dtype="bf16")
    sub = oracle.block(*args, k=2, dtype="bf16", tokens=[20, 3])
    assert np.array_equal(sub["out"], full["out"][[20, 3]])


# ---------------------------------------------------------------- balance


def _brute_topk(s, k):
    """The k-subset whose members all dominate all non-members (higher score, or equal and lower index)."""
    E = len(s)

    def dom(a, b):
        return s[a] > s[b] or (s[a] == s[b] and a < b)

    for sub in itertools.combinations(range(E), k):
        if all(dom(a, b) for a in sub for b in range(E) if b not in sub):
            return sub
    raise AssertionError("no dominant subset")


@pytest.mark.parametrize("k", [1, 2, 3])
def test_balance_uniform_scores(k):
    E = 6
    f, p, loss = oracle.balance(np.zeros((10, E)), k, alpha=0.01)
    assert np.array_equal(f, np.array([1.0] * k + [0.0] * (E - k)))
    assert np.allclose(p, 1.0 / E, rtol=0, atol=1e-16)
    assert abs(loss - 0.01 * k) < 1e-16


@pytest.mark.parametrize("E,k", [(8, 2), (5, 2), (6, 3)])
def test_balance_cyclic_batch_is_balanced(E, k):
    v = np.random.default_rng(E * 10 + k).standard_normal(E)
    logits = np.stack([np.roll(v, r) for r in range(E)])
    f, p, loss = oracle.balance(logits, k, alpha=1.0)
    assert np.allclose(f, k / E, rtol=0, atol=1e-15)
    assert np.allclose(p, 1.0 / E, rtol=0, atol=1e-15)
    assert abs(loss - k) < 1e-13


@pytest.mark.parametrize("E,k", [(6, 3), (8, 2), (3, 1)])
def test_balance_bruteforce(E, k):
    rng = np.random.default_rng(E + 100 * k)
    logits = np.concatenate([rng.standard_normal((60, E)), rng.integers(-1, 2, size=(17, E)).astype(float)])
    f, p, loss = oracle.balance(logits, k, alpha=0.3)
    T = logits.shape[0]
    f_ref = np.zeros(E)
    for t in range(T):
        for e in _brute_topk(list(logits[t]), k):
            f_ref[e] += 1.0 / T
    p_ref = torch.softmax(_t64(logits), dim=1).mean(dim=0).numpy()
    assert np.allclose(f, f_ref, rtol=0, atol=1e-14)
    assert np.allclose(p, p_ref, rtol=0, atol=1e-15)
    assert abs(loss - 0.3 * E * float(f_ref @ p_ref)) < 1e-13
    assert abs(f.sum() - k) < 1e-13 and abs(p.sum() - 1.0) < 1e-14


def test_balance_hand_example():
    """Two tokens, E=3, k=1.  Softmaxes (1/4, 1/2, 1/4) and (3/5, 1/5, 1/5); top-1 picks 1 and 0."""
    logits = np.array([[0.0, math.log(2.0), 0.0], [math.log(3.0), 0.0, 0.0]])
    f, p, loss = oracle.balance(logits, 1, alpha=2.0)
    assert np.allclose(f, [0.5, 0.5, 0.0], rtol=0, atol=1e-16)
    assert np.allclose(p, [0.425, 0.35, 0.225], rtol=0, atol=1e-15)
    assert abs(loss - 2.0 * 3 * (0.5 * 0.425 + 0.5 * 0.35)) < 1e-14
