"""Backward pass against the fp64 oracle, through the C ABI on a B200.

The forward runs with the grouped-GEMM (prefill) path into a caller
workspace; the backward reads that workspace.  Tokens within the routing
margin are excluded from the token-wise checks.

Tolerances, derived from the arithmetic.  On the bf16 path dy = g dout, dA
and dB are rounded to bf16 before their GEMMs, so each product term carries
up to three bf16 roundings (2^-9 each) in series where the forward output
carries one (H); independent rounding errors add in quadrature, so the
forward's 2e-2 becomes 2e-2 sqrt(3) = 3.5e-2.  An entry's error also scales
with the entry itself (weight-gradient entries are heavy-tailed: a few
tokens with large |dout| and |h| dominate them).  Two checks per gradient G
against the oracle's G*:
  * every entry:  |G - G*| <= tol (RMS(G*) + |G*|),  tol = 3.5e-2 (bf16) or
    1e-5 (fp32);
  * the bulk:     RMS(G - G*) <= bulk RMS(G*),  bulk = 1e-2 (bf16, about 4x the
    3 x 2^-9 / sqrt(3) expected) or 2e-6 (fp32).
fp32 bounds are scaled by sqrt(K / 256) for reductions longer than 256
(K = the longest of d, ffn and T).
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_testlib import MARGIN, experts_reached, out_to_f64, stratified_tokens, to_dev, upload

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2 * np.sqrt(3.0), "f32": 1e-5}
BULK = {"bf16": 1e-2, "f32": 2e-6}


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _status_clear(moe):
    assert moe.moe_get_device_status() == moe.MOE_OK


def _run(moe, inp, dev, dout_d, dlogits=False, alpha=0.0):
    x, Wg, W1, W3, W2 = dev
    code = moe.MOE_DTYPE_BF16 if inp.dtype == "bf16" else moe.MOE_DTYPE_F32
    fws = torch.empty(moe.moe_train_workspace_size(inp.T, inp.d, inp.F, inp.E, inp.k, code), dtype=torch.uint8,
                      device="cuda")
    out = moe.moe_forward_ws(x, Wg, W1, W3, W2, inp.k, path=moe.MOE_PATH_TRAIN, workspace=fws)
    dl = torch.empty((inp.T, inp.E), dtype=torch.float32, device="cuda") if dlogits else None
    grads, n = moe.moe_backward_ws(x, Wg, W1, W3, W2, dout_d, inp.k, fws, dlogits=dl, alpha=alpha)
    _status_clear(moe)
    if dl is not None:
        grads["dlogits"] = dl
    return out, grads, n


def _f64(t):
    return t.double().cpu().numpy() if t.dtype == torch.float32 else out_to_f64(t)


def _check(name, got, want, dtype, K=256):
    scale = max(1.0, np.sqrt(K / 256.0)) if dtype == "f32" else 1.0
    tol, bulk = TOL[dtype] * scale, BULK[dtype] * scale
    rms = np.sqrt((want ** 2).mean())
    err = np.abs(got - want)
    excess = (err - tol * np.abs(want)).max()
    l2 = np.sqrt((err ** 2).mean()) / rms
    print(f"  {name}: max|err|/RMS {err.max() / rms:.3e}  excess/RMS {excess / rms:.3e}  rms err/RMS {l2:.3e}")
    assert excess <= tol * rms, f"{name}: max excess {excess:.3e} > {tol:.2e} x RMS {rms:.3e}"
    assert l2 <= bulk, f"{name}: RMS error {l2:.3e} x RMS > {bulk:.2e}"
    return l2


@pytest.mark.parametrize("dtype,T,d,F,E,k", [("bf16", 200, 256, 512, 8, 2), ("bf16", 700, 192, 384, 4, 2),
                                             ("bf16", 90, 128, 256, 16, 4), ("bf16", 40, 256, 128, 8, 8),
                                             ("bf16", 160, 512, 2560, 8, 2),   # dXp on 256 x 512 tiles (K = 2F)
                                             ("f32", 64, 128, 256, 8, 2), ("f32", 150, 96, 160, 5, 3)])
def test_backward_small(moe, dtype, T, d, F, E, k):
    inp = moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=T + d + E + k)
    dout = moe_inputs.make_dout(T, d, dtype, seed=T)
    dev = upload(inp)
    _, g, n = _run(moe, inp, dev, to_dev(dout, dtype), dlogits=True)
    assert n == (9 if dtype == "bf16" else 10)   # scatter, ds, 4 or 5 GEMMs, dWg (2), dx
    ref = oracle.backward(*inp.arrays(), dout, k, dtype)
    keep = ref["margin"] >= MARGIN
    if not keep.all():
        pytest.skip("a token sits within the routing margin; the weight gradients would include its choice")
    K = max(d, F, T)
    rel = {}
    rel["dx"] = _check("dx", _f64(g["dx"]), ref["dx"], dtype, K)
    rel["dlogits"] = _check("dlogits", _f64(g["dlogits"]), ref["dlogits"], dtype, K)
    for n_ in ("dWg", "dW1", "dW3", "dW2"):
        rel[n_] = _check(n_, _f64(g[n_]), ref[n_], dtype, K)
    print(dtype, T, d, F, E, k, {a: f"{b:.2e}" for a, b in rel.items()})


def test_bf16_weight_gradients_are_the_fp32_ones_rounded(moe):
    """wgrad_dtype = bf16 rounds the same fp32 sums once in the epilogue: equal to the fp32
    gradients rounded to nearest even, bit for bit; dx and dWg are unchanged."""
    inp = moe_inputs.make_inputs(400, 256, 384, 8, 2, "bf16", seed=45)
    dev = upload(inp)
    dout = to_dev(moe_inputs.make_dout(400, 256, "bf16", seed=45), "bf16")
    ws = torch.empty(moe.moe_train_workspace_size(400, 256, 384, 8, 2), dtype=torch.uint8, device="cuda")
    moe.moe_forward_ws(*dev, 2, path=moe.MOE_PATH_TRAIN, workspace=ws)
    g32, _ = moe.moe_backward_ws(*dev, dout, 2, ws, alpha=0.1)
    g16, _ = moe.moe_backward_ws(*dev, dout, 2, ws, alpha=0.1, wgrad_dtype=torch.bfloat16)
    _status_clear(moe)
    for n in ("dW1", "dW3", "dW2"):
        assert g16[n].dtype == torch.bfloat16
        assert torch.equal(g16[n], g32[n].to(torch.bfloat16)), n
    assert torch.equal(g16["dx"], g32["dx"]) and torch.equal(g16["dWg"], g32["dWg"])


def test_backward_run_to_run_bitwise(moe):
    inp = moe_inputs.make_inputs(300, 256, 256, 8, 2, "bf16", seed=41)
    dev = upload(inp)
    dout = to_dev(moe_inputs.make_dout(300, 256, "bf16", seed=41), "bf16")
    _, a, _ = _run(moe, inp, dev, dout, dlogits=True)
    _, b, _ = _run(moe, inp, dev, dout, dlogits=True)
    for n in a:
        assert torch.equal(a[n], b[n]), n


def _close(name, got, want, rel):
    """|got - want| <= rel (RMS(want) + |want|) entrywise: sums of the same terms in another order."""
    got, want = got.double(), want.double()
    rms = want.pow(2).mean().sqrt()
    bad = (got - want).abs() > rel * (rms + want.abs())
    assert not bad.any(), f"{name}: {int(bad.sum())} entries differ by more than {rel:.1e} (RMS + |G|)"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_token_permutation_equivariance(moe, dtype):
    """Tokens are independent: permuting x and dout permutes dx and the router-score gradient bit
    for bit.  The weight gradients sum the same per-token terms in another order (each expert's
    rows follow token order), so they agree to fp32 reassociation."""
    T, d, F = 300, 256, 256
    inp = moe_inputs.make_inputs(T, d, F, 8, 2, dtype, seed=46)
    dev = upload(inp)
    dout = to_dev(moe_inputs.make_dout(T, d, dtype, seed=46), dtype)
    _, a, _ = _run(moe, inp, dev, dout, dlogits=True)
    p = torch.randperm(T, generator=torch.Generator().manual_seed(1)).cuda()
    dev_p = (dev[0][p].contiguous(),) + tuple(dev[1:])
    _, b, _ = _run(moe, inp, dev_p, dout[p].contiguous(), dlogits=True)
    assert torch.equal(b["dx"], a["dx"][p])
    assert torch.equal(b["dlogits"], a["dlogits"][p])
    for n in ("dWg", "dW1", "dW3", "dW2"):
        _close(n, b[n], a[n], 2e-4)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_expert_relabelling(moe, dtype):
    """Relabelling the experts (rows of Wg, blocks of W1, W3, W2) permutes every per-expert
    gradient bit for bit: each expert sees the same tokens in the same order.  dx adds the k
    router terms in expert-index order, so it agrees to one rounding of its output."""
    T, d, F = 300, 256, 256
    inp = moe_inputs.make_inputs(T, d, F, 8, 2, dtype, seed=47)
    dev = upload(inp)
    dout = to_dev(moe_inputs.make_dout(T, d, dtype, seed=47), dtype)
    _, a, _ = _run(moe, inp, dev, dout, dlogits=True)
    r = torch.tensor([3, 7, 0, 5, 1, 6, 2, 4], device="cuda")
    dev_r = (dev[0],) + tuple(t[r].contiguous() for t in dev[1:])
    _, b, _ = _run(moe, inp, dev_r, dout, dlogits=True)
    for n in ("dWg", "dW1", "dW3", "dW2"):
        assert torch.equal(b[n], a[n][r]), n
    assert torch.equal(b["dlogits"], a["dlogits"][:, r])
    _close("dx", b["dx"], a["dx"], 2.0 ** -7 if dtype == "bf16" else 1e-5)


def test_backward_experts_without_tokens(moe):
    """Experts no token chose get exactly zero weight gradients."""
    inp = moe_inputs.make_inputs(100, 128, 256, 8, 2, "bf16", seed=42)
    inp.Wg[:] = 0
    inp.Wg[0, :] = moe_inputs.f32_to_bf16_bits(np.full(128, 0.5, dtype=np.float32))
    inp.Wg[1, :] = moe_inputs.f32_to_bf16_bits(np.full(128, 0.25, dtype=np.float32))
    inp.x[:] = moe_inputs.f32_to_bf16_bits(np.abs(moe_inputs.bf16_bits_to_f32(inp.x)) + 0.01)
    dev = upload(inp)
    dout = moe_inputs.make_dout(100, 128, "bf16", seed=42)
    _, g, _ = _run(moe, inp, dev, to_dev(dout, "bf16"))
    for n in ("dW1", "dW3", "dW2"):
        assert torch.all(g[n][2:] == 0), n
        assert torch.any(g[n][:2] != 0), n
    ref = oracle.backward(*inp.arrays(), dout, 2, "bf16")
    for n in ("dW1", "dW3", "dW2"):   # the two experts with tokens (the zero blocks would halve the RMS)
        _check(n, _f64(g[n][:2]), ref[n][:2], "bf16")
    _check("dx", _f64(g["dx"]), ref["dx"], "bf16")


@pytest.mark.parametrize("cfg,n_tok,alpha", [(1, 0, 0.0), (1, 0, 0.5), (3, 1, 0.0), (3, 1, 0.01), (5, 1, 0.0)])
def test_backward_configs(moe, cfg, n_tok, alpha):
    """Full-size workloads (in the launch configuration bench.py --train times): dx and dlogits on
    a stratified token sample (every expert's first and last row, its m-tile boundaries, odd last
    m-tiles), slices of the weight gradients of two experts; alpha != 0 includes the load-balance
    loss.  dWg at full size is pinned by test_backward_dwg_full_size."""
    inp = moe_inputs.make_config(cfg)
    dtype = inp.dtype
    dout = moe_inputs.make_dout(inp.T, inp.d, dtype, seed=inp.seed)
    dev = upload(inp)
    _, g, _ = _run(moe, inp, dev, to_dev(dout, dtype), dlogits=True, alpha=alpha)
    K = max(inp.d, inp.F, inp.T)
    if n_tok == 0:
        ref = oracle.backward(*inp.arrays(), dout, inp.k, dtype, alpha=alpha)
        for n in ("dx", "dlogits", "dWg", "dW1", "dW3", "dW2"):
            _check(n, _f64(g[n]), ref[n], dtype, K)
        return
    r_idx = oracle.route(inp.x, inp.Wg, inp.k, dtype)[0]
    toks = stratified_tokens(r_idx, inp.E, n_random=4, boundaries=2, odd_tail=3, seed=cfg)
    assert experts_reached(r_idx, toks) == set(range(inp.E))
    ref = oracle.backward_tokens(*inp.arrays(), dout, inp.k, dtype, toks, alpha=alpha)
    keep = ref["margin"] >= MARGIN
    _check("dx", _f64(g["dx"])[toks][keep], ref["dx"][keep], dtype)
    _check("dlogits", _f64(g["dlogits"])[toks][keep], ref["dlogits"][keep], dtype)
    fs = [0, 777, inp.F - 1]
    if alpha != 0.0:   # the expert weight gradients do not see the balance loss
        del dev, g
        torch.cuda.empty_cache()
        return
    for e in (0, inp.E - 1):
        r1, r3, c2 = oracle.weight_grad_slices(*inp.arrays(), dout, inp.k, dtype, e, fs)
        _check(f"dW1[{e}]", _f64(g["dW1"][e][fs]), r1, dtype)
        _check(f"dW3[{e}]", _f64(g["dW3"][e][fs]), r3, dtype)
        _check(f"dW2[{e}]", _f64(g["dW2"][e][:, fs]), c2, dtype)
    del dev, g
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", [3, 5])
def test_backward_dwg_full_size(moe, cfg):
    """dWg at full size against the oracle.  dout is kept on a stratified sample of tokens and
    set to zero on every other token, so the loss only sees the sample: the oracle's score
    gradient of those tokens gives dWg = sum_t ds_t x_t^T exactly, while the GPU still reduces
    over all T tokens in its full-size launch configuration.  Tokens with dout = 0 get dx = 0
    and a zero score gradient exactly (dy = 0 and dg = 0)."""
    inp = moe_inputs.make_config(cfg)
    dtype = inp.dtype
    r_idx = oracle.route(inp.x, inp.Wg, inp.k, dtype)[0]
    toks = stratified_tokens(r_idx, inp.E, n_random=4, boundaries=2, odd_tail=3, seed=cfg + 10)
    assert experts_reached(r_idx, toks) == set(range(inp.E))
    dout = moe_inputs.make_dout(inp.T, inp.d, dtype, seed=inp.seed)
    mask = np.zeros(inp.T, dtype=bool)
    mask[toks] = True
    dout[~mask] = 0
    dev = upload(inp)
    _, g, _ = _run(moe, inp, dev, to_dev(dout, dtype), dlogits=True)
    ref = oracle.backward_tokens(*inp.arrays(), dout, inp.k, dtype, toks)
    if not (ref["margin"] >= MARGIN).all():
        pytest.skip("a sampled token sits within the routing margin")
    x_s = moe_inputs.bf16_bits_to_f32(inp.x[toks]).astype(np.float64) if dtype == "bf16" else \
        inp.x[toks].astype(np.float64)
    want = ref["dlogits"].T @ x_s
    _check("dWg", _f64(g["dWg"]), want, dtype, len(toks))
    _check("dx", _f64(g["dx"])[toks], ref["dx"], dtype)
    rest = torch.from_numpy(~mask).cuda()
    assert torch.count_nonzero(g["dx"][rest]) == 0
    assert torch.count_nonzero(g["dlogits"][rest]) == 0
    del dev, g
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_training_forward_output_equals_prefill(moe, dtype):
    """The training path only keeps more state: its output is the grouped-GEMM path's, bit for bit."""
    inp = moe_inputs.make_inputs(333, 256, 384, 8, 2, dtype, seed=43) if dtype == "bf16" else \
        moe_inputs.make_inputs(100, 96, 160, 8, 2, dtype, seed=43)
    dev = upload(inp)
    code = moe.MOE_DTYPE_BF16 if dtype == "bf16" else moe.MOE_DTYPE_F32
    ws = torch.empty(moe.moe_train_workspace_size(inp.T, inp.d, inp.F, inp.E, inp.k, code), dtype=torch.uint8,
                     device="cuda")
    a = moe.moe_forward_ws(*dev, inp.k, path=moe.MOE_PATH_TRAIN, workspace=ws)
    b = moe.moe_forward_ws(*dev, inp.k, path=moe.MOE_PATH_PREFILL)
    _status_clear(moe)
    assert torch.equal(a, b)


def test_backward_rejects_inference_workspace(moe):
    """A workspace sized for inference cannot hold the training state: the backward refuses it."""
    inp = moe_inputs.make_inputs(200, 256, 512, 8, 2, "bf16", seed=44)
    dev = upload(inp)
    ws = torch.empty(moe.moe_workspace_size(inp.T, inp.d, inp.F, inp.E, inp.k), dtype=torch.uint8, device="cuda")
    moe.moe_forward_ws(*dev, inp.k, path=moe.MOE_PATH_PREFILL, workspace=ws)
    dout = to_dev(moe_inputs.make_dout(inp.T, inp.d, "bf16", seed=44), "bf16")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_backward_ws(*dev, dout, inp.k, ws)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE



@pytest.mark.parametrize("dtype,T,d,F,E,k", [("bf16", 300, 256, 384, 8, 2), ("f32", 96, 128, 160, 6, 2)])
def test_backward_with_balance_loss(moe, dtype, T, d, F, E, k):
    """alpha != 0 adds the load-balance loss: the router-score gradient gains its part on every
    expert (dx and dWg follow), the expert weight gradients stay bit for bit the same."""
    alpha = 0.5
    inp = moe_inputs.make_inputs(T, d, F, E, k, dtype, seed=T + 7)
    dout = moe_inputs.make_dout(T, d, dtype, seed=T + 7)
    dev = upload(inp)
    _, g0, _ = _run(moe, inp, dev, to_dev(dout, dtype), dlogits=True)
    _, g, _ = _run(moe, inp, dev, to_dev(dout, dtype), dlogits=True, alpha=alpha)
    for n in ("dW1", "dW3", "dW2"):
        assert torch.equal(g[n], g0[n]), n
    ref = oracle.backward(*inp.arrays(), dout, k, dtype, alpha=alpha)
    if not (ref["margin"] >= MARGIN).all():
        pytest.skip("a token sits within the routing margin")
    K = max(d, F, T)
    for n in ("dx", "dlogits", "dWg"):
        _check(n, _f64(g[n]), ref[n], dtype, K)
    assert torch.count_nonzero(g["dlogits"]) > torch.count_nonzero(g0["dlogits"])
