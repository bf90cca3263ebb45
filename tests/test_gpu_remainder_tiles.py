"""The last rows of each expert in the expert GEMMs.

An expert's rows run as 256-row CTA-pair tiles (two 128-row m-tiles); its last
r = n mod 256 rows share a tile with padding rows, and when its 128-row m-tiles
are odd in number the pair's second CTA holds padding only.  The expert counts
are set directly through the expert-side entry point of expert parallelism on
one rank (rows arrive grouped by expert), so every remainder of interest is
reached: r = 1, a multiple of 16, one past it, 128, 129, 255 and none at all.
Every row is compared with the oracle's expert (subsection "各エキスパートの構造"
of the Mistral/Mixtral architecture page), and a row's result must not depend
on where in a tile it lands.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_testlib import TOL, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _oracle_rows(inp, counts):
    ref, row = [], 0
    for e, c in enumerate(counts):
        for _ in range(c):
            ref.append(oracle.expert(inp.x, inp.W1, inp.W3, inp.W2, e, row, inp.dtype))
            row += 1
    return np.stack(ref)


@pytest.mark.parametrize("counts,d,F", [
    ([1, 17, 128, 129, 255, 256, 300, 543], 256, 512),
    ([0, 16, 31, 112, 240, 257, 0, 2], 320, 384),
    ([513, 0, 0, 0, 0, 0, 0, 79], 256, 256),
])
def test_remainder_rows_match_oracle(moe, counts, d, F):
    E = len(counts)
    rows = sum(counts)
    inp = moe_inputs.make_inputs(rows, d, F, E, 2, "bf16", seed=rows + d)
    x, _, W1, W3, W2 = upload(inp)
    y = moe.moe_ep_experts(x, np.array([counts]), 0, W1, W3, W2)
    assert moe.moe_get_device_status() == moe.MOE_OK
    got = y.double().cpu().numpy()
    ref = _oracle_rows(inp, counts)
    at = 0
    for e, c in enumerate(counts):
        if c == 0:
            continue
        g, r = got[at:at + c], ref[at:at + c]
        err = np.abs(g - r).max()
        rms = np.sqrt((r ** 2).mean())
        assert err <= TOL["bf16"] * rms, f"expert {e} ({c} rows): max|err| {err:.3e} vs RMS {rms:.3e}"
        at += c


@pytest.mark.parametrize("n", [16, 100, 200, 255])
def test_row_result_does_not_depend_on_the_tile_kind(moe, n):
    """The same n rows of one expert, once inside a full 256-row pair tile (the expert holds 256
    rows) and once as the expert's only, partly padded tile (it holds just these n): equal bits."""
    d, F = 256, 512
    inp = moe_inputs.make_inputs(256, d, F, 1, 2, "bf16", seed=n)
    x, _, W1, W3, W2 = upload(inp)
    full = moe.moe_ep_experts(x, np.array([[256]]), 0, W1, W3, W2)
    part = moe.moe_ep_experts(x[:n].contiguous(), np.array([[n]]), 0, W1, W3, W2)
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert torch.equal(full[:n], part)
