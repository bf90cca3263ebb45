"""Pins of the fp64 oracle to things other than itself.

Each test ties one step of the oracle to what the pages or plain mathematics
fix ("Mistral/Mixtral architecture" page, section "MoEの数学 — ルーターとゲーティング機構"):

  * selection   brute force over every k-subset with the dominance rule
                (higher score, or equal score and lower index)
  * gates       closed form g1 = 1/(1+exp(-(s1-s2))) for k=2; sum to 1; g1 >= 1/k
  * scores      numpy matmul in fp64
  * expert      E=1, k=1 reduces to one dense SwiGLU FFN, computed with torch fp64
  * combine     k=E with all-zero router reduces to the plain average of the experts
  * hand case   a 2-dim example worked out in closed form (silu(1), silu(2), sigmoid)
  * invariances token permutation, expert relabelling, exact scaling of W2 by 2

The pages print no numeric worked example of the layer, so there is no
printed-value fixture to compare against.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import moe_inputs
import oracle


# ---------------------------------------------------------------- selection


def _brute_topk(s, k):
    """The unique k-subset whose members all dominate all non-members, in dominance order."""
    E = len(s)

    def dom(a, b):
        return s[a] > s[b] or (s[a] == s[b] and a < b)

    winners = []
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(dom(a, b) for a in sub for b in rest):
            winners.append(sub)
    assert len(winners) == 1
    sub = list(winners[0])
    # order the subset: position of a = number of members that dominate it
    ordered = sorted(sub, key=lambda a: sum(dom(b, a) for b in sub))
    return ordered


@pytest.mark.parametrize("E", [1, 2, 3, 5, 8])
def test_select_matches_bruteforce(E):
    rng = np.random.default_rng(E)
    for k in range(1, E + 1):
        cont = rng.standard_normal((60, E))
        ties = rng.integers(-2, 3, size=(60, E)).astype(np.float64)  # many exact ties
        for s in (cont, ties):
            idx, g, margin, mingap = oracle.select(s, k)
            for t in range(s.shape[0]):
                assert list(idx[t]) == _brute_topk(list(s[t]), k)
                srt = sorted(s[t], reverse=True)
                want_margin = srt[k - 1] - srt[k] if k < E else math.inf
                assert margin[t] == want_margin
                gaps = [srt[j] - srt[j + 1] for j in range(k - 1)]
                assert mingap[t] == (min(gaps) if gaps else math.inf)


def test_gate_closed_form_k2():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((500, 8)) * 3
    idx, g, _, _ = oracle.select(s, 2)
    for t in range(500):
        s1, s2 = s[t, idx[t, 0]], s[t, idx[t, 1]]
        g1 = 1.0 / (1.0 + math.exp(-(s1 - s2)))
        assert abs(g[t, 0] - g1) < 1e-15
        assert abs(g[t, 1] - (1.0 - g1)) < 1e-15


@pytest.mark.parametrize("k", [1, 2, 3, 8])
def test_gate_invariants(k):
    rng = np.random.default_rng(k)
    s = rng.standard_normal((300, 8)) * 4
    idx, g, _, _ = oracle.select(s, k)
    assert np.all(g > 0)
    assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(g[:, 0] >= 1.0 / k - 1e-15)
    assert np.all(np.diff(g, axis=1) <= 1e-16)                 # descending with the scores
    for t in range(300):
        assert len(set(idx[t].tolist())) == k                  # k distinct experts
    # softmax over the selected scores, from the page's formula written out directly
    for t in range(0, 300, 7):
        ex = np.exp(s[t, idx[t]])
        assert np.allclose(g[t], ex / ex.sum(), rtol=1e-14, atol=0)


def test_gate_is_softmax_of_keep_topk():
    """The summary page's form: softmax over all E with the unselected scores at -inf."""
    rng = np.random.default_rng(9)
    s = rng.standard_normal((100, 8))
    idx, g, _, _ = oracle.select(s, 2)
    keep = np.full_like(s, -np.inf)
    rows = np.arange(100)[:, None]
    keep[rows, idx] = s[rows, idx]
    full = torch.softmax(torch.from_numpy(keep), dim=-1).numpy()
    assert np.allclose(full[rows, idx], g, rtol=1e-14, atol=0)
    mask = np.ones_like(s, dtype=bool)
    mask[rows, idx] = False
    assert np.all(full[mask] == 0.0)


# ---------------------------------------------------------------- scores


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_scores_match_numpy(dtype):
    inp = moe_inputs.make_inputs(50, 96, 32, 6, 2, dtype, seed=11, weights=False)
    s = oracle.scores(inp.x, inp.Wg, dtype)
    ref = inp.as_f32("x").astype(np.float64) @ inp.as_f32("Wg").astype(np.float64).T
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)


def test_route_equals_scores_then_select():
    inp = moe_inputs.make_inputs(64, 128, 32, 8, 2, "bf16", seed=2, weights=False)
    idx, g, m, mg = oracle.route(inp.x, inp.Wg, 2, "bf16")
    idx2, g2, m2, mg2 = oracle.select(oracle.scores(inp.x, inp.Wg, "bf16"), 2)
    assert np.array_equal(idx, idx2) and np.array_equal(g, g2) and np.array_equal(m, m2)


# ---------------------------------------------------------------- experts


def _torch_swiglu(x, W1, W3, W2):
    x, W1, W3, W2 = (torch.from_numpy(np.asarray(a, dtype=np.float64)) for a in (x, W1, W3, W2))
    return (torch.nn.functional.silu(x @ W1.T) * (x @ W3.T)) @ W2.T


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_expert_is_dense_swiglu(dtype):
    """E=1, k=1: the gate is 1 and the layer is one dense SwiGLU FFN."""
    inp = moe_inputs.make_inputs(24, 64, 160, 1, 1, dtype, seed=4)
    r = oracle.moe(*inp.arrays(), k=1, dtype=dtype)
    assert np.all(r["idx"] == 0) and np.all(r["g"] == 1.0)
    ref = _torch_swiglu(inp.as_f32("x"), inp.as_f32("W1")[0], inp.as_f32("W3")[0], inp.as_f32("W2")[0]).numpy()
    scale = np.sqrt((ref ** 2).mean())
    assert np.max(np.abs(r["out"] - ref)) < 1e-12 * scale


def test_expert_matches_torch():
    inp = moe_inputs.make_inputs(6, 48, 80, 3, 2, "bf16", seed=8)
    for e in range(3):
        for t in (0, 5):
            y = oracle.expert(inp.x, inp.W1, inp.W3, inp.W2, e, t, "bf16")
            ref = _torch_swiglu(inp.as_f32("x")[t:t + 1], inp.as_f32("W1")[e], inp.as_f32("W3")[e],
                                inp.as_f32("W2")[e]).numpy()[0]
            assert np.allclose(y, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("E", [2, 4, 8])
def test_uniform_router_all_experts_is_average(E):
    """k=E with Wg=0: every score is 0, every gate is 1/E, output = mean of all experts."""
    inp = moe_inputs.make_inputs(12, 64, 96, E, E, "f32", seed=6)
    inp.Wg[:] = 0.0
    r = oracle.moe(*inp.arrays(), k=E, dtype="f32")
    assert np.all(r["idx"] == np.arange(E)[None, :])          # ties resolved to ascending index
    assert np.allclose(r["g"], 1.0 / E, rtol=0, atol=1e-15)
    ref = sum(_torch_swiglu(inp.x, inp.W1[e], inp.W3[e], inp.W2[e]).numpy() for e in range(E)) / E
    assert np.max(np.abs(r["out"] - ref)) < 1e-12 * np.sqrt((ref ** 2).mean())


def test_top1_switch_routing():
    """k=1: gate 1 on the arg-max expert, output = that expert alone."""
    inp = moe_inputs.make_inputs(20, 64, 96, 4, 1, "f32", seed=12)
    r = oracle.moe(*inp.arrays(), k=1, dtype="f32")
    s = inp.x.astype(np.float64) @ inp.Wg.astype(np.float64).T
    assert np.array_equal(r["idx"][:, 0], np.argmax(s, axis=1))
    assert np.all(r["g"] == 1.0)
    for t in range(20):
        e = r["idx"][t, 0]
        ref = _torch_swiglu(inp.x[t:t + 1], inp.W1[e], inp.W3[e], inp.W2[e]).numpy()[0]
        assert np.allclose(r["out"][t], ref, rtol=1e-12, atol=1e-13)


def test_hand_worked_example():
    """d=2, F=2, E=3, k=2, one token x=(1,2), every value worked out by hand.

    scores s = Wg x = (0.5, 1.0, -1.0): experts 1 then 0 are kept, expert 2 dropped.
    gates: g = (1/(1+e^-0.5), 1/(1+e^0.5)).
    expert 0: W1 x = (1, 2), W3 x = (3, 0)  -> h = (3 silu(1), 0)
              W2 h = (1*h0 + 2*h1, 3*h0 + 4*h1)
    expert 1: W1 x = (2, 1), W3 x = (1, -1) -> h = (silu(2), -silu(1))
              W2 h = (h1, h0)
    silu(a) = a / (1 + e^-a).
    """
    x = np.float32([[1, 2]])
    Wg = np.float32([[0.5, 0], [0, 0.5], [-1, 0]])
    W1 = np.float32([[[1, 0], [0, 1]], [[0, 1], [1, 0]], [[5, 5], [5, 5]]])
    W3 = np.float32([[[1, 1], [0, 0]], [[0, 0.5], [-1, 0]], [[5, 5], [5, 5]]])
    W2 = np.float32([[[1, 2], [3, 4]], [[0, 1], [1, 0]], [[7, 7], [7, 7]]])
    r = oracle.moe(x, Wg, W1, W3, W2, k=2, dtype="f32")

    def silu(a):
        return a / (1 + math.exp(-a))

    g0, g1 = 1 / (1 + math.exp(-0.5)), 1 / (1 + math.exp(0.5))
    y0 = [3 * silu(1), 9 * silu(1)]
    y1 = [-silu(1), silu(2)]
    want = [g0 * y1[0] + g1 * y0[0], g0 * y1[1] + g1 * y0[1]]
    assert list(r["idx"][0]) == [1, 0]
    assert abs(r["g"][0, 0] - g0) < 1e-15 and abs(r["g"][0, 1] - g1) < 1e-15
    assert abs(r["margin"][0] - 1.5) < 1e-15 and abs(r["mingap"][0] - 0.5) < 1e-15
    assert np.allclose(r["out"][0], want, rtol=1e-15, atol=1e-15)
    assert np.allclose(oracle.expert(x, W1, W3, W2, 0, 0, "f32"), y0, rtol=1e-15)
    assert np.allclose(oracle.expert(x, W1, W3, W2, 1, 0, "f32"), y1, rtol=1e-15)


# ---------------------------------------------------------------- invariances


def test_token_permutation_equivariance():
    inp = moe_inputs.make_inputs(40, 64, 64, 8, 2, "bf16", seed=13)
    r = oracle.moe(*inp.arrays(), k=2, dtype="bf16")
    perm = np.random.default_rng(0).permutation(40)
    x2 = np.ascontiguousarray(inp.x[perm])
    r2 = oracle.moe(x2, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="bf16")
    assert np.array_equal(r2["out"], r["out"][perm])
    assert np.array_equal(r2["idx"], r["idx"][perm])


def test_expert_relabelling_invariance():
    inp = moe_inputs.make_inputs(40, 64, 64, 8, 2, "bf16", seed=14)
    r = oracle.moe(*inp.arrays(), k=2, dtype="bf16")
    relabel = np.random.default_rng(1).permutation(8)          # new expert i = old expert relabel[i]
    args = [np.ascontiguousarray(a[relabel]) for a in (inp.Wg, inp.W1, inp.W3, inp.W2)]
    r2 = oracle.moe(inp.x, *args, k=2, dtype="bf16")
    assert np.array_equal(relabel[r2["idx"]], r["idx"])
    assert np.array_equal(r2["out"], r["out"])


def test_w2_power_of_two_scaling_is_exact():
    inp = moe_inputs.make_inputs(16, 64, 64, 4, 2, "bf16", seed=15)
    r = oracle.moe(*inp.arrays(), k=2, dtype="bf16")
    W2x2 = moe_inputs.f32_to_bf16_bits(inp.as_f32("W2") * np.float32(2.0))
    r2 = oracle.moe(inp.x, inp.Wg, inp.W1, inp.W3, W2x2, k=2, dtype="bf16")
    assert np.array_equal(r2["out"], 2.0 * r["out"])


def test_token_subset_matches_full_run():
    inp = moe_inputs.make_inputs(30, 64, 64, 8, 2, "bf16", seed=16)
    full = oracle.moe(*inp.arrays(), k=2, dtype="bf16")
    sub = oracle.moe(*inp.arrays(), k=2, dtype="bf16", tokens=[29, 0, 7])
    assert np.array_equal(sub["out"], full["out"][[29, 0, 7]])


# ---------------------------------------------------------------- histogram


def test_counts_bruteforce():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((333, 8))
    idx, _, _, _ = oracle.select(s, 2)
    c = oracle.counts(idx, 8)
    assert c.sum() == 2 * 333
    for e in range(8):
        assert c[e] == sum(1 for t in range(333) for j in range(2) if idx[t, j] == e)


def test_skewed_workload_follows_zipf():
    """The stored offsets give Zipf(1.2) top-2 shares on the skewed workload's own tokens."""
    inp = moe_inputs.make_config(4, weights=False)
    idx, _, _, _ = oracle.route(inp.x, inp.Wg, 2, "bf16")
    c = oracle.counts(idx, 8).astype(np.float64)
    p = c / c.sum()
    w = np.arange(1, 9, dtype=np.float64) ** -1.2
    assert np.allclose(p, w / w.sum(), atol=2e-3)
    assert p[0] > 0.42
