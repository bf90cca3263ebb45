"""Block form (out = h + MoE(RMSNorm(h))) and load-balance statistics against the
fp64 oracle, through the C ABI on a B200.

Tolerances, derived from the arithmetic:
  * routing: the oracle's margin rule (moe_testlib).  The router sees the
    unrounded normalised row, so its scores differ from the oracle's only by
    fp32 summation and the fp32 norm factor, as in the plain layer.
  * output: out = h + m is rounded once; h can be several times larger than the
    MoE part m, so the check is on m's scale plus the final rounding:
        max_t,j (|out - out*| - c |out*|) <= tol * RMS(m*),  m* = out* - h,
    with c = 2^-8 (twice bf16's half ulp) or 2^-22 for fp32, and tol = 2e-2
    (bf16) or 1e-5 (fp32), the plain layer's tolerances.  fp32 rounding error
    of a length-K sum grows like sqrt(K); the fp32 bound holds for reductions
    up to K = 256 and is scaled by sqrt(K / 256) beyond (K = max(d, ffn)).
  * statistics: p within 1e-5 (fp32 scores and exp against fp64); each
    expert's selection count within the number of tokens the margin rule
    excludes; the loss within alpha E sum(f) 1e-5 of alpha E sum(f p*) recomputed
    from the GPU's f and the oracle's p.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_testlib import MARGIN, experts_reached, out_to_f64, stratified_tokens, to_dev

pytestmark = pytest.mark.gpu

EPS = moe_inputs.BLOCK_EPS
TOL = {"bf16": 2e-2, "f32": 1e-5}
ROUND = {"bf16": 2.0 ** -8, "f32": 2.0 ** -22}


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _status_clear(moe):
    assert moe.moe_get_device_status() == moe.MOE_OK


def _block_inputs(T, d, F, E, k, dtype, seed):
    return moe_inputs.make_block(moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=seed))


def _upload(inp):
    return {n: to_dev(getattr(inp, n), inp.dtype) for n in ("x", "gamma", "Wg", "W1", "W3", "W2")}


def _h64(inp, rows):
    return inp.as_f32("x").astype(np.float64)[rows]


def _compare_block(out_gpu, ref, h64, dtype, K=256):
    keep = ref["margin"] >= MARGIN
    assert keep.mean() > 0.9
    want = ref["out"][keep]
    m = want - h64[keep]
    excess = np.abs(out_gpu[keep] - want) - ROUND[dtype] * np.abs(want)
    rms = np.sqrt((m ** 2).mean())
    err = excess.max()
    tol = TOL[dtype] * (max(1.0, np.sqrt(K / 256.0)) if dtype == "f32" else 1.0)
    assert err <= tol * rms, f"max excess {err:.3e} > {tol:.2e} x RMS(m) {rms:.3e}"
    return err / rms


def _compare_stats(stats, logits_ref, k, alpha, E):
    f_ref, p_ref, _ = oracle.balance(logits_ref, k, alpha)
    st = stats.cpu().numpy().astype(np.float64)
    f, p, loss = st[:E], st[E:2 * E], st[2 * E]
    T = logits_ref.shape[0]
    _, _, margin, _ = oracle.select(logits_ref, k)
    near = int((margin < MARGIN).sum())
    cnt = np.rint(f * T)
    assert np.all(np.abs(f * T - cnt) < 1e-2)              # f is a count / T, rounded once to fp32
    assert np.all(np.abs(cnt - np.rint(f_ref * T)) <= near), (cnt, f_ref * T, near)
    assert np.abs(p - p_ref).max() <= 1e-5, np.abs(p - p_ref).max()
    assert abs(p.sum() - 1.0) < 1e-5 and abs(cnt.sum() - k * T) == 0
    want = alpha * E * float(f @ p_ref)
    assert abs(loss - want) <= abs(alpha) * E * f.sum() * 1e-5 + 1e-6 * abs(want), (loss, want)


# ---------------------------------------------------------------- small shapes, every element


@pytest.mark.parametrize("T,d,F,E,k", [(200, 256, 512, 8, 2), (77, 128, 256, 4, 1), (700, 256, 384, 8, 2),
                                       (650, 192, 256, 16, 4), (640, 128, 256, 32, 2), (16, 512, 256, 8, 2)])
def test_block_bf16_small(moe, T, d, F, E, k):
    inp = _block_inputs(T, d, F, E, k, "bf16", seed=T + d + E)
    dv = _upload(inp)
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device="cuda")
    out = moe.moe_block_forward(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], k,
                                alpha=0.01, stats=stats)
    _status_clear(moe)
    ref = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=k, dtype="bf16")
    rel = _compare_block(out_to_f64(out), ref, _h64(inp, slice(None)), "bf16")
    print(f"block bf16 T={T}: max excess / RMS(m) = {rel:.3e}")
    _compare_stats(stats, oracle.block_scores(inp.x, inp.gamma, EPS, inp.Wg, "bf16"), k, 0.01, E)


@pytest.mark.parametrize("T,d,F,E,k", [(64, 128, 256, 8, 2), (150, 96, 160, 5, 3), (33, 4200, 64, 8, 2)])
def test_block_f32_small(moe, T, d, F, E, k):
    inp = _block_inputs(T, d, F, E, k, "f32", seed=T * 3 + d)
    dv = _upload(inp)
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device="cuda")
    out = moe.moe_block_forward(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], k,
                                alpha=1.0, stats=stats)
    _status_clear(moe)
    ref = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=k, dtype="f32")
    _compare_block(out.double().cpu().numpy(), ref, _h64(inp, slice(None)), "f32", K=max(d, F))
    _compare_stats(stats, oracle.block_scores(inp.x, inp.gamma, EPS, inp.Wg, "f32"), k, 1.0, E)


def test_block_long_rows_bf16(moe):
    """d above 1024 16-byte chunks takes the looping router with the norm."""
    inp = _block_inputs(24, 8256 - 8256 % 64, 128, 8, 2, "bf16", seed=9)
    dv = _upload(inp)
    out = moe.moe_block_forward(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], 2)
    _status_clear(moe)
    ref = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="bf16")
    _compare_block(out_to_f64(out), ref, _h64(inp, slice(None)), "bf16")


# ---------------------------------------------------------------- full-size workloads, sampled tokens


@pytest.mark.parametrize("cfg,n", [(1, 0), (2, 0), (3, 1), (5, 1)])
def test_block_configs(moe, cfg, n):
    """n = 0: every token; n = 1: a stratified sample from the oracle's routing of the normalised
    rows (every expert's first and last row, m-tile boundaries, odd last m-tiles)."""
    inp = moe_inputs.make_block(moe_inputs.make_config(cfg))
    dv = _upload(inp)
    E, k = inp.E, inp.k
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device="cuda")
    out = moe.moe_block_forward(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], k,
                                alpha=0.01, stats=stats)
    _status_clear(moe)
    toks = None
    if n:
        r_idx = oracle.select(oracle.block_scores(inp.x, inp.gamma, EPS, inp.Wg, inp.dtype), k)[0]
        toks = stratified_tokens(r_idx, E, seed=cfg)
        assert experts_reached(r_idx, toks) == set(range(E))
    ref = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=k, dtype=inp.dtype, tokens=toks)
    sel = ref["tokens"]
    got = out_to_f64(out)[sel] if inp.dtype == "bf16" else out.double().cpu().numpy()[sel]
    rel = _compare_block(got, ref, _h64(inp, sel), inp.dtype)
    print(f"block config {cfg}: max excess / RMS(m) = {rel:.3e} over {len(sel)} tokens")
    _compare_stats(stats, oracle.block_scores(inp.x, inp.gamma, EPS, inp.Wg, inp.dtype), k, 0.01, E)
    del dv, out
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- properties of the CUDA path


@pytest.fixture(scope="module")
def mid():
    inp = _block_inputs(700, 256, 512, 8, 2, "bf16", seed=78)
    return inp, _upload(inp)


def _run(moe, dv, k=2, **kw):
    return moe.moe_block_forward(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], k, **kw)


def test_block_run_to_run_bitwise(moe, mid):
    _, dv = mid
    s1 = torch.empty(17, dtype=torch.float32, device="cuda")
    s2 = torch.empty(17, dtype=torch.float32, device="cuda")
    a = _run(moe, dv, stats=s1)
    b = _run(moe, dv, stats=s2)
    assert torch.equal(a, b) and torch.equal(s1, s2)


def test_block_in_place(moe, mid):
    _, dv = mid
    want = _run(moe, dv)
    h = dv["x"].clone()
    moe.moe_block_forward(h, dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], 2, out=h)
    assert torch.equal(h, want)


def test_block_token_permutation_equivariance(moe, mid):
    _, dv = mid
    out = _run(moe, dv)
    p = torch.randperm(dv["x"].shape[0], generator=torch.Generator().manual_seed(1)).cuda()
    dp = dict(dv, x=dv["x"][p].contiguous())
    assert torch.equal(_run(moe, dp), out[p])


def test_block_workspace_entry_matches_pooled(moe, mid):
    inp, dv = mid
    T, d, F, E, k = inp.T, inp.d, inp.F, inp.E, inp.k
    ws = torch.empty(moe.moe_block_workspace_size(T, d, F, E, k), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dv["x"])
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device="cuda")
    n = moe.moe_block_forward_ws(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], k, ws, out,
                                 alpha=0.5, stats=stats)
    assert n >= 8
    s2 = torch.empty_like(stats)
    assert torch.equal(out, _run(moe, dv, alpha=0.5, stats=s2)) and torch.equal(stats, s2)


@pytest.mark.parametrize("T", [1, 16, 64])
@pytest.mark.parametrize("path", [1, 2])
def test_block_paths_match_oracle(moe, T, path):
    """Decode (swap-AB weight streaming, fused sort + normalising gather) and prefill paths."""
    inp = _block_inputs(T, 256, 512, 8, 2, "bf16", seed=300 + T)
    dv = _upload(inp)
    ws = torch.empty(moe.moe_block_workspace_size(T, 256, 512, 8, 2), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dv["x"])
    moe.moe_block_forward_ws(dv["x"], dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], 2, ws, out,
                             path=path)
    _status_clear(moe)
    ref = oracle.block(inp.x, inp.gamma, EPS, inp.Wg, inp.W1, inp.W3, inp.W2, k=2, dtype="bf16")
    _compare_block(out_to_f64(out), ref, _h64(inp, slice(None)), "bf16")


def test_block_zero_row_and_empty_batch(moe):
    inp = _block_inputs(40, 128, 256, 8, 2, "bf16", seed=5)
    inp.x[7] = 0
    dv = _upload(inp)
    out = _run(moe, dv)
    _status_clear(moe)
    assert torch.all(out[7] == 0)
    empty = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    r = moe.moe_block_forward(empty, dv["gamma"], EPS, dv["Wg"], dv["W1"], dv["W3"], dv["W2"], 2)
    assert r.shape == (0, 128)


def test_stats_uniform_router_closed_form(moe):
    """Wg = 0, k = E = 8: f = 1, p = 1/8 exactly, loss = alpha * E * sum f p = 8 alpha."""
    inp = _block_inputs(512, 128, 128, 8, 8, "bf16", seed=6)
    dv = _upload(inp)
    dv["Wg"].zero_()
    stats = torch.empty(17, dtype=torch.float32, device="cuda")
    _run(moe, dv, k=8, alpha=0.25, stats=stats)
    st = stats.cpu().numpy()
    assert np.all(st[:8] == 1.0) and np.all(st[8:16] == 0.125) and st[16] == 2.0


# ---------------------------------------------------------------- statistics of the plain router


@pytest.mark.parametrize("dtype,T,d,E,k", [("bf16", 300, 256, 8, 2), ("bf16", 1000, 256, 8, 2),
                                           ("bf16", 2000, 320, 16, 4), ("f32", 200, 128, 6, 3)])
def test_route_stats_small(moe, dtype, T, d, E, k):
    inp = moe_inputs.make_inputs(T, d, 128, E, k, dtype, seed=T + E, weights=False)
    x, Wg = to_dev(inp.x, dtype), to_dev(inp.Wg, dtype)
    idx, w, stats = moe.moe_route_stats(x, Wg, k, alpha=0.01)
    _status_clear(moe)
    idx2, w2 = moe.moe_route(x, Wg, k)
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    _compare_stats(stats, oracle.scores(inp.x, inp.Wg, dtype), k, 0.01, E)


@pytest.mark.parametrize("cfg", [3, 4])
def test_route_stats_configs(moe, cfg):
    """Full-size batches, including the Zipf(1.2)-skewed routing (f far from uniform)."""
    inp = moe_inputs.make_config(cfg, weights=False)
    x, Wg = to_dev(inp.x, inp.dtype), to_dev(inp.Wg, inp.dtype)
    _, _, stats = moe.moe_route_stats(x, Wg, inp.k, alpha=0.01)
    _status_clear(moe)
    _compare_stats(stats, oracle.scores(inp.x, inp.Wg, inp.dtype), inp.k, 0.01, inp.E)
