"""Helpers shared by the parity tests: upload seeded inputs, compare with the oracle.

Comparison rules (fixed by the layer's contract):
  * routing: expert ids must equal the oracle's bit for bit, except tokens whose
    oracle margin between the k-th and (k+1)-th score is below 1e-4 (excluded:
    either choice is within rounding of a tie); when two selected scores are
    within 1e-4 of each other the ids are compared as a set.
  * gates: |w - g| <= 2e-5 (fp32 scores and exp against fp64).
  * outputs: max |out - out*| <= tol * RMS(out*) over the compared tokens, with
    tol = 2e-2 for bf16 and 1e-5 for fp32.
"""
from __future__ import annotations

import numpy as np
import torch

MARGIN = 1e-4
TOL = {"bf16": 2e-2, "f32": 1e-5}


def to_dev(a: np.ndarray, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def upload(inp, device="cuda"):
    return [None if a is None else to_dev(a, inp.dtype, device) for a in inp.arrays()]


def out_to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def compare_routing(idx_gpu, w_gpu, ref, tokens=None):
    """idx_gpu/w_gpu: numpy [n][k] for the same tokens as ref (oracle dict or tuple)."""
    if isinstance(ref, dict):
        r_idx, r_g, r_margin, r_gap = ref["idx"], ref["g"], ref["margin"], ref["mingap"]
    else:
        r_idx, r_g, r_margin, r_gap = ref
    keep = r_margin >= MARGIN
    ordered = keep & (r_gap >= MARGIN)
    bad_ordered = np.nonzero(ordered & np.any(idx_gpu != r_idx, axis=1))[0]
    unordered = keep & ~ordered
    bad_set = [t for t in np.nonzero(unordered)[0] if sorted(idx_gpu[t]) != sorted(r_idx[t])]
    assert len(bad_ordered) == 0, f"expert ids differ on tokens {bad_ordered[:10]}"
    assert len(bad_set) == 0, f"expert id sets differ on tokens {bad_set[:10]}"
    gerr = np.abs(w_gpu[ordered] - r_g[ordered]).max() if ordered.any() else 0.0
    assert gerr <= 2e-5, f"gate error {gerr}"
    return keep


def compare_outputs(out_gpu, out_ref, keep, dtype):
    """out_gpu/out_ref [n][d] (f64); keep: tokens outside the margin rule."""
    if not np.any(keep):
        return 0.0
    ref = out_ref[keep]
    err = np.abs(out_gpu[keep] - ref).max()
    rms = np.sqrt((ref ** 2).mean())
    assert err <= TOL[dtype] * rms, f"max|err| {err:.3e} > {TOL[dtype]} x RMS {rms:.3e}"
    return err / rms


def sample_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n, T), replace=False).tolist())
    s.update({0, T - 1})
    return np.array(sorted(s), dtype=np.int32)


def stratified_tokens(idx, E, n_random=8, boundaries=3, odd_tail=8, seed=0, tile=128):
    """Tokens that reach every tile case of the grouped GEMMs, chosen from a routing idx [T][k]
    (the oracle's, so the choice never depends on the CUDA path).

    Within expert e's segment the rows are the tokens that chose e, in increasing token order
    (the dispatch is a stable counting sort), so row r of the segment is the r-th such token.
    For every expert with tokens this takes:
      * its first and last row;
      * the rows on both sides of up to `boundaries` of its 128-row m-tile boundaries, always
        including the first and the last boundary;
      * up to `odd_tail` rows spread over its last m-tile when it has an odd number of m-tiles
        (the CTA pair's second half is then empty);
    plus `n_random` tokens drawn uniformly, and tokens 0 and T - 1.
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    picked = {0, T - 1}
    for e in range(E):
        rows = np.nonzero((idx == e).any(axis=1))[0]
        n = len(rows)
        if n == 0:
            continue
        want = {0, n - 1}
        mt = (n + tile - 1) // tile
        bnds = list(range(tile, n, tile))
        if bnds:
            sel = sorted({bnds[0], bnds[-1], bnds[len(bnds) // 2]})[:max(boundaries, 2)]
            for b in sel:
                want.update({b - 1, b})
        if mt % 2 == 1:
            lo = (mt - 1) * tile
            want.update(np.linspace(lo, n - 1, min(odd_tail, n - lo)).astype(np.int64).tolist())
        picked.update(int(rows[r]) for r in want)
    rng = np.random.default_rng(seed)
    picked.update(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    return np.array(sorted(picked), dtype=np.int32)


def experts_reached(idx, tokens):
    """Experts chosen by at least one of `tokens` (routing idx [T][k])."""
    return set(np.unique(np.asarray(idx)[tokens]).tolist())
