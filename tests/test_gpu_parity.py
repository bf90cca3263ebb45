"""CUDA path against the fp64 oracle, through the C ABI (sm_100a, B200).

Small shapes compare every output element; the full-size workloads compare
sampled tokens (the oracle evaluates them one by one) in the same launch
configuration the bench times.  Rules are in moe_testlib.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_testlib import compare_outputs, compare_routing, experts_reached, out_to_f64, stratified_tokens, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _status_clear(moe):
    assert moe.moe_get_device_status() == moe.MOE_OK


# ---------------------------------------------------------------- routing


@pytest.mark.parametrize("dtype,d", [("bf16", 256), ("f32", 128)])
@pytest.mark.parametrize("E,k", [(1, 1), (3, 2), (8, 1), (8, 2), (8, 8), (16, 4), (32, 2)])
def test_route_small(moe, dtype, d, E, k):
    inp = moe_inputs.make_inputs(300, d, 128, E, k, dtype, seed=100 + E * 7 + k, weights=False)
    x, Wg = upload(inp)[:2]
    idx, w = moe.moe_route(x, Wg, k)
    ref = oracle.route(inp.x, inp.Wg, k, dtype)
    compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    _status_clear(moe)


@pytest.mark.parametrize("d", [192, 320, 1024])
@pytest.mark.parametrize("E,k", [(3, 2), (8, 2), (16, 4), (32, 2)])
def test_route_large_batches(moe, d, E, k):
    """Batches above 4 x SMs take the tensor-core score path (16-token tiles, warps split d)."""
    inp = moe_inputs.make_inputs(1000, d, 128, E, k, "bf16", seed=500 + d + E, weights=False)
    x, Wg = upload(inp)[:2]
    idx, w = moe.moe_route(x, Wg, k)
    ref = oracle.route(inp.x, inp.Wg, k, "bf16")
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    assert keep.mean() > 0.98
    _status_clear(moe)


@pytest.mark.parametrize("dtype,d", [("bf16", 8256), ("f32", 4200)])
def test_route_long_rows(moe, dtype, d):
    """Rows longer than 1024 16-byte chunks take the looping router."""
    inp = moe_inputs.make_inputs(40, d, 64, 8, 2, dtype, seed=d, weights=False)
    x, Wg = upload(inp)[:2]
    idx, w = moe.moe_route(x, Wg, 2)
    ref = oracle.route(inp.x, inp.Wg, 2, dtype)
    compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    _status_clear(moe)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_route_configs(moe, cfg):
    inp = moe_inputs.make_config(cfg, weights=False)
    x, Wg = upload(inp)[:2]
    idx, w = moe.moe_route(x, Wg, inp.k)
    ref = oracle.route(inp.x, inp.Wg, inp.k, inp.dtype)
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    assert keep.mean() > 0.99
    _status_clear(moe)


def test_route_tie_break_lowest_index(moe):
    # every score equal: the k lowest expert ids in ascending order, uniform gates
    x = torch.randn(50, 128, device="cuda").to(torch.bfloat16)
    Wg = torch.zeros(8, 128, device="cuda", dtype=torch.bfloat16)
    idx, w = moe.moe_route(x, Wg, 3)
    assert torch.equal(idx.cpu(), torch.tensor([[0, 1, 2]] * 50, dtype=torch.int32))
    assert torch.allclose(w.cpu(), torch.full((50, 3), 1 / 3), atol=1e-7)


# ---------------------------------------------------------------- dispatch


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (1000, 8, 2), (2500, 5, 3), (4097, 32, 4), (300, 1, 1)])
def test_dispatch_stable_counting_sort(moe, T, E, k):
    rng = np.random.default_rng(T + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = moe.moe_dispatch(torch.from_numpy(idx).cuda(), E)
    counts, offsets, perm, inv = (a.cpu().numpy() for a in (counts, offsets, perm, inv))
    assert np.array_equal(counts, oracle.counts(idx, E))
    seg = (counts + 127) // 128 * 128
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(seg)]))
    for e in range(E):
        rows = perm[offsets[e]:offsets[e] + counts[e]]
        toks = rows // k
        assert np.all(idx.reshape(-1)[rows] == e)
        assert np.all(np.diff(toks) > 0)                        # stable: token order kept
        assert np.all(perm[offsets[e] + counts[e]:offsets[e + 1]] == -1)
    assert np.array_equal(perm[inv.reshape(-1)], np.arange(T * k))   # inverse permutation
    _status_clear(moe)


def test_dispatch_bad_expert_id_is_reported(moe):
    idx = torch.tensor([[0, 1], [2, 99], [3, 4]], dtype=torch.int32, device="cuda")
    moe.moe_dispatch(idx, 8)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE
    _status_clear(moe)                                          # cleared, context still usable
    counts, _, _, _ = moe.moe_dispatch(idx.clamp(max=7), 8)
    assert int(counts.sum()) == 6


# ---------------------------------------------------------------- whole layer, small shapes

SMALL_BF16 = [
    (1, 128, 256, 8, 2),
    (7, 128, 256, 4, 2),
    (130, 128, 256, 8, 2),
    (300, 256, 512, 8, 2),
    (1000, 128, 256, 8, 2),
    (257, 192, 384, 5, 3),
    (64, 128, 128, 1, 1),
    (100, 128, 256, 4, 4),
    (333, 320, 256, 32, 2),
]


@pytest.mark.parametrize("T,d,F,E,k", SMALL_BF16)
def test_forward_bf16_small(moe, T, d, F, E, k):
    inp = moe_inputs.make_inputs(T, d, F, E, k, "bf16", seed=T + d + E)
    dev = upload(inp)
    out = moe.moe_forward(*dev, k)
    _status_clear(moe)
    ref = oracle.moe(*inp.arrays(), k=k, dtype="bf16")
    idx, w = moe.moe_route(dev[0], dev[1], k)
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    compare_outputs(out_to_f64(out), ref["out"], keep, "bf16")


@pytest.mark.parametrize("T,d,F,E,k", [(517, 5120, 5120, 8, 2), (300, 6144, 1024, 8, 2), (301, 1024, 6144, 6, 2),
                                       (257, 5184, 5248, 8, 2)])
def test_forward_wide_tiles(moe, T, d, F, E, k):
    """Reductions of 5120 and more run on 256 x 512 tiles (GEMM1 when d >= 5120, GEMM2 when
    ffn >= 5120): both wide, GEMM1 only, GEMM2 only (ffn = 6144 is 12 wide n-blocks, d = 1024
    two of GEMM2's), and both wide with ragged last n-blocks (ffn = 5248: GEMM1's last 256
    features half past ffn; d = 5184: GEMM2's last 512 columns mostly past d); ragged expert counts.  Rows this long are compared on the stratified token
    sample of the full-size workloads (every expert's first and last rows, its m-tile boundaries
    and odd last m-tile): over every token of these shapes (1.5-1.8 M outputs, the largest at
    5.5 x RMS) rounding the exact result to bf16 alone costs up to 1.8% of the 2% bound."""
    inp = moe_inputs.make_inputs(T, d, F, E, k, "bf16", seed=T + d + F)
    dev = upload(inp)
    out = moe.moe_forward(*dev, k)
    _status_clear(moe)
    r_idx = oracle.route(inp.x, inp.Wg, k, inp.dtype)[0]
    toks = stratified_tokens(r_idx, E, seed=T)
    ref = oracle.moe(*inp.arrays(), k=k, dtype="bf16", tokens=toks, nthreads=oracle.max_threads())
    idx, w = moe.moe_route(dev[0], dev[1], k)
    keep = compare_routing(idx.cpu().numpy()[toks], w.cpu().numpy()[toks], ref)
    rel = compare_outputs(out_to_f64(out)[toks], ref["out"], keep, "bf16")
    print(f"wide {T}x{d}x{F}: max|err|/RMS = {rel:.3e} over {keep.sum()} tokens")


@pytest.mark.parametrize("T,d,F,E,k", [(64, 128, 256, 8, 2), (1, 4, 1, 1, 1), (37, 12, 20, 3, 2),
                                       (200, 64, 100, 8, 8), (129, 132, 70, 6, 1)])
def test_forward_f32_small(moe, T, d, F, E, k):
    inp = moe_inputs.make_inputs(T, d, F, E, k, "f32", seed=T + d + F)
    dev = upload(inp)
    out = moe.moe_forward(*dev, k)
    _status_clear(moe)
    ref = oracle.moe(*inp.arrays(), k=k, dtype="f32")
    idx, w = moe.moe_route(dev[0], dev[1], k)
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    compare_outputs(out_to_f64(out), ref["out"], keep, "f32")


def test_forward_zero_tokens(moe):
    inp = moe_inputs.make_inputs(1, 128, 256, 4, 2, "bf16", seed=1)
    dev = upload(inp)
    x0 = dev[0][:0]
    out = moe.moe_forward(x0, *dev[1:], 2)
    assert out.shape == (0, 128)
    _status_clear(moe)


# ---------------------------------------------------------------- full-size workloads, sampled tokens


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_forward_configs(moe, cfg):
    """Full-size workloads in the launch configuration bench.py times.  Workloads 1 and 2 are
    compared on every token; the prefill ones on a stratified sample chosen from the oracle's
    routing: every expert's first and last row, rows on both sides of its 128-row m-tile
    boundaries, and its last m-tile when it has an odd number of them (so every expert and every
    tile case is reached, the skewed workload's rare experts included)."""
    inp = moe_inputs.make_config(cfg)
    dev = upload(inp)
    out = moe.moe_forward(*dev, inp.k)
    _status_clear(moe)
    toks = None
    if inp.T > 64:
        r_idx = oracle.route(inp.x, inp.Wg, inp.k, inp.dtype)[0]
        toks = stratified_tokens(r_idx, inp.E, seed=cfg)
        assert experts_reached(r_idx, toks) == set(range(inp.E))
    ref = oracle.moe(*inp.arrays(), k=inp.k, dtype=inp.dtype, tokens=toks)
    sel = ref["tokens"]
    idx, w = moe.moe_route(dev[0], dev[1], inp.k)
    keep = compare_routing(idx.cpu().numpy()[sel], w.cpu().numpy()[sel], ref)
    got = out_to_f64(out)[sel]
    rel = compare_outputs(got, ref["out"], keep, inp.dtype)
    print(f"config {cfg}: max|err|/RMS = {rel:.3e} over {keep.sum()} tokens")
    del dev, out
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- invariants of the CUDA path


@pytest.fixture(scope="module")
def mid():
    inp = moe_inputs.make_inputs(700, 256, 512, 8, 2, "bf16", seed=77)
    return inp, upload(inp)


def test_run_to_run_bitwise(moe, mid):
    _, dev = mid
    a = moe.moe_forward(*dev, 2)
    b = moe.moe_forward(*dev, 2)
    assert torch.equal(a, b)


def test_token_permutation_equivariance(moe, mid):
    _, dev = mid
    out = moe.moe_forward(*dev, 2)
    p = torch.randperm(dev[0].shape[0], generator=torch.Generator().manual_seed(0)).cuda()
    out_p = moe.moe_forward(dev[0][p].contiguous(), *dev[1:], 2)
    assert torch.equal(out_p, out[p])


def test_expert_relabelling_invariance(moe, mid):
    _, dev = mid
    out = moe.moe_forward(*dev, 2)
    r = torch.tensor([3, 7, 0, 5, 1, 6, 2, 4], device="cuda")
    out_r = moe.moe_forward(dev[0], *[t[r].contiguous() for t in dev[1:]], 2)
    assert torch.equal(out_r, out)


def test_w2_scaling_by_two_is_exact(moe, mid):
    _, dev = mid
    out = moe.moe_forward(*dev, 2)
    out2 = moe.moe_forward(*dev[:4], (dev[4].float() * 2).to(torch.bfloat16), 2)
    assert torch.equal(out2, (out.float() * 2).to(torch.bfloat16))


def test_workspace_entry_matches_pooled(moe, mid):
    _, dev = mid
    a = moe.moe_forward(*dev, 2)
    b = moe.moe_forward_ws(*dev, 2, path=moe.MOE_PATH_PREFILL)
    assert torch.equal(a, b)


def test_host_entry_matches_device(moe, mid):
    _, dev = mid
    a = moe.moe_forward(*dev, 2)
    x_host = dev[0].cpu().pin_memory()
    b = moe.moe_forward_host(x_host, *dev[1:], 2)
    assert torch.equal(a.cpu(), b)


def test_wait_timeout_is_reported_not_hung(moe):
    moe.moe_selftest_wait_timeout(2_000_000)          # 2 ms on a barrier nobody arrives at
    assert moe.moe_get_device_status() == moe.MOE_ERR_TIMEOUT
    assert moe.moe_get_device_status() == moe.MOE_OK
    x = torch.randn(8, 128, device="cuda").to(torch.bfloat16)   # context still usable
    idx, _ = moe.moe_route(x, torch.randn(4, 128, device="cuda").to(torch.bfloat16), 2)
    assert idx.shape == (8, 2)


# ---------------------------------------------------------------- both expert paths


@pytest.mark.parametrize("T,d,F,E,k", [(1, 128, 256, 8, 2), (16, 256, 512, 8, 2), (40, 192, 384, 5, 3),
                                       (64, 128, 256, 4, 1), (64, 320, 256, 32, 2), (9, 128, 128, 1, 1)])
@pytest.mark.parametrize("path", ["prefill", "decode"])
def test_forward_paths_match_oracle(moe, T, d, F, E, k, path):
    inp = moe_inputs.make_inputs(T, d, F, E, k, "bf16", seed=900 + T + E)
    dev = upload(inp)
    code = moe.MOE_PATH_DECODE if path == "decode" else moe.MOE_PATH_PREFILL
    out = moe.moe_forward_ws(*dev, k, path=code)
    _status_clear(moe)
    ref = oracle.moe(*inp.arrays(), k=k, dtype="bf16")
    idx, w = moe.moe_route(dev[0], dev[1], k)
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    compare_outputs(out_to_f64(out), ref["out"], keep, "bf16")


def test_decode_path_rejects_large_batches(moe):
    inp = moe_inputs.make_inputs(65, 128, 256, 4, 2, "bf16", seed=3)
    dev = upload(inp)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward_ws(*dev, 2, path=moe.MOE_PATH_DECODE)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_decode_max_tokens() == 64


# ---------------------------------------------------------------- experts with no tokens, decode invariants


@pytest.mark.parametrize("T,path", [(16, "decode"), (48, "decode"), (48, "prefill"), (900, "prefill")])
def test_experts_without_tokens(moe, T, path):
    """Experts 5..7 never win (feature 0 pinned to 1.0 and a -30 offset on their scores)."""
    inp = moe_inputs.make_inputs(T, 256, 512, 8, 2, "bf16", seed=31 + T,
                                 bias=[0.5, 0.25, 0.0, -0.25, -0.5, -30.0, -30.0, -30.0])
    dev = upload(inp)
    code = moe.MOE_PATH_DECODE if path == "decode" else moe.MOE_PATH_PREFILL
    out = moe.moe_forward_ws(*dev, 2, path=code)
    _status_clear(moe)
    ref = oracle.moe(*inp.arrays(), k=2, dtype="bf16")
    assert not np.isin(ref["idx"], [5, 6, 7]).any()
    idx, w = moe.moe_route(dev[0], dev[1], 2)
    keep = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), ref)
    compare_outputs(out_to_f64(out), ref["out"], keep, "bf16")


@pytest.fixture(scope="module")
def small():
    inp = moe_inputs.make_inputs(24, 512, 1024, 8, 2, "bf16", seed=55)
    return inp, upload(inp)


def test_decode_run_to_run_bitwise(moe, small):
    _, dev = small
    a = moe.moe_forward(*dev, 2)
    b = moe.moe_forward(*dev, 2)
    assert torch.equal(a, b)


def test_decode_token_permutation_equivariance(moe, small):
    _, dev = small
    out = moe.moe_forward(*dev, 2)
    p = torch.randperm(24, generator=torch.Generator().manual_seed(1)).cuda()
    out_p = moe.moe_forward(dev[0][p].contiguous(), *dev[1:], 2)
    assert torch.equal(out_p, out[p])


def test_decode_host_entry_matches_device(moe, small):
    _, dev = small
    a = moe.moe_forward(*dev, 2)
    b = moe.moe_forward_host(dev[0].cpu().pin_memory(), *dev[1:], 2)
    assert torch.equal(a.cpu(), b)


def test_decode_host_entry_pageable_buffers(moe, small):
    """Pageable host buffers go through the same copies, with the same result."""
    _, dev = small
    a = moe.moe_forward(*dev, 2)
    x_host = dev[0].cpu()
    out_host = torch.empty_like(x_host)
    assert not x_host.is_pinned() and not out_host.is_pinned()
    b = moe.moe_forward_host(x_host, *dev[1:], 2, out_host=out_host)
    assert torch.equal(a.cpu(), b)


def test_paths_agree_closely(moe, small):
    """Decode and grouped-GEMM paths compute the same function (different summation order)."""
    _, dev = small
    a = moe.moe_forward_ws(*dev, 2, path=moe.MOE_PATH_DECODE).float()
    b = moe.moe_forward_ws(*dev, 2, path=moe.MOE_PATH_PREFILL).float()
    rms = b.pow(2).mean().sqrt()
    assert (a - b).abs().max() <= 1e-2 * rms


@pytest.mark.parametrize("T", [16, 700])
def test_forward_ws_graph_capture(moe, T):
    """moe_forward_ws with a caller workspace can be captured into a CUDA graph and replayed
    (decode path at T=16, grouped GEMMs at T=700); the replay gives the eager result bit for bit."""
    inp = moe_inputs.make_inputs(T, 256, 512, 8, 2, "bf16", seed=900 + T)
    dev = upload(inp)
    ws = torch.empty(moe.moe_workspace_size(T, 256, 512, 8, 2), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dev[0])
    moe.moe_forward_ws(*dev, 2, workspace=ws, out=out)   # first call: per-device set-up outside capture
    torch.cuda.synchronize()
    want = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward_ws(*dev, 2, workspace=ws, out=out)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    _status_clear(moe)
    assert torch.equal(out, want)
    del g


@pytest.mark.parametrize("d,E,k", [(1024, 8, 2), (4096, 8, 2), (2048, 32, 2), (6144, 16, 4)])
def test_route_is_batch_invariant(moe, d, E, k):
    """The tensor-core router adds its 256-wide K chunks in the same order whatever cluster split a
    batch size picks: a token's gates and experts are the same bits in a batch of 1000 and of 9000."""
    inp = moe_inputs.make_inputs(9000, d, 128, E, k, "bf16", seed=d + E, weights=False)
    x, Wg = upload(inp)[:2]
    idx_big, w_big = moe.moe_route(x, Wg, k)
    idx_small, w_small = moe.moe_route(x[:1000].contiguous(), Wg, k)
    _status_clear(moe)
    assert torch.equal(idx_small, idx_big[:1000])
    assert torch.equal(w_small, w_big[:1000])


@pytest.mark.parametrize("T", [4096, 6143, 8192, 10001, 12288, 16384, 30000])
def test_chunked_host_entry_matches_device(moe, T):
    """Batches of 4096 tokens and more go through the host entry point in pipelined chunks (two
    halves below 8192 tokens, then short first and last chunks around middle ones, by
    moe_host_chunk_plan); the result equals the one-call device path bit for bit, from pinned and
    pageable buffers."""
    inp = moe_inputs.make_inputs(T, 256, 512, 8, 2, "bf16", seed=T)
    dev = upload(inp)
    a = moe.moe_forward(*dev, 2).cpu()
    b = moe.moe_forward_host(dev[0].cpu().pin_memory(), *dev[1:], 2)
    assert torch.equal(a, b)
    out = torch.empty_like(a)
    c = moe.moe_forward_host(dev[0].cpu(), *dev[1:], 2, out_host=out)
    assert torch.equal(a, c)
    _status_clear(moe)
