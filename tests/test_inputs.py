"""The seeded input generator: SplitMix64 known answers, bf16 rounding, moments, layout."""
import json
import os

import numpy as np
import pytest
import torch

import moe_inputs

M64 = (1 << 64) - 1


def _mix64_py(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_splitmix64_known_answer():
    # First outputs of SplitMix64 started at state 0, as published with the
    # reference implementation (Vigna's splitmix64.c seeded with 0).
    out = moe_inputs.splitmix64(0, 3)
    assert int(out[0]) == 0xE220A8397B1DCDAF
    assert int(out[1]) == 0x6E789E6AA1B965F4
    assert int(out[2]) == 0x06C45D188009454F


def test_splitmix64_matches_python_statement():
    state = 0x0123456789ABCDEF
    out = moe_inputs.splitmix64(state, 64)
    for i in range(64):
        assert int(out[i]) == _mix64_py((state + (i + 1) * 0x9E3779B97F4A7C15) & M64)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = rng.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    # exact ties between two bf16 neighbours: low 16 bits == 0x8000
    ties = (rng.integers(0, 1 << 15, 1000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    ties = ties[np.isfinite(ties)]          # the generator never produces nan/inf
    a = np.concatenate([a, ties, np.float32([0.0, -0.0, 1e-40, 3.0e38])])
    ours = moe_inputs.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_normal_moments():
    z = moe_inputs.normal((1 << 20,), seed=7, tensor_id=0, sigma=1.0, dtype="f32").astype(np.float64)
    n = z.size
    assert abs(z.mean()) < 5 / np.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    # fourth moment of N(0,1) is 3
    assert abs((z ** 4).mean() - 3.0) < 0.05
    s = moe_inputs.normal((1 << 16,), seed=7, tensor_id=2, sigma=0.125, dtype="bf16")
    sf = moe_inputs.bf16_bits_to_f32(s).astype(np.float64)
    assert abs(sf.std() - 0.125) < 0.005


def test_streams_are_distinct_and_deterministic():
    a = moe_inputs.normal((4096,), 1, 2, 1.0, "f32")
    b = moe_inputs.normal((4096,), 1, 2, 1.0, "f32")
    c = moe_inputs.normal((4096,), 1, 3, 1.0, "f32")
    d = moe_inputs.normal((4096,), 2, 2, 1.0, "f32")
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    assert not np.array_equal(a, d)


def test_bf16_is_rounded_f32_stream():
    f = moe_inputs.normal((5000,), 3, 1, 0.5, "f32")
    h = moe_inputs.normal((5000,), 3, 1, 0.5, "bf16")
    assert np.array_equal(moe_inputs.f32_to_bf16_bits(f), h)


def test_token_prefix_property():
    big = moe_inputs.make_inputs(40, 64, 128, 4, 2, "bf16", seed=5)
    small = moe_inputs.make_inputs(17, 64, 128, 4, 2, "bf16", seed=5)
    assert np.array_equal(big.x[:17], small.x)
    assert np.array_equal(big.W1, small.W1)


def test_shapes_and_scales():
    inp = moe_inputs.make_inputs(32, 256, 512, 8, 2, "bf16", seed=1)
    assert inp.x.shape == (32, 256) and inp.Wg.shape == (8, 256)
    assert inp.W1.shape == (8, 512, 256) and inp.W3.shape == (8, 512, 256) and inp.W2.shape == (8, 256, 512)
    assert abs(inp.as_f32("W1").std() - 1 / 16) < 0.002
    assert abs(inp.as_f32("W2").std() - 1 / np.sqrt(512)) < 0.002


def test_skew_recipe():
    inp = moe_inputs.make_inputs(8, 64, 128, 8, 2, "bf16", seed=3, skew=True, weights=False)
    assert np.all(inp.x[:, 0] == moe_inputs.BF16_ONE)
    b = moe_inputs.skew_bias(8)
    assert np.array_equal(moe_inputs.bf16_bits_to_f32(inp.Wg[:, 0]), np.float32(b))


def test_skew_bias_file_is_bf16_exact():
    with open(os.path.join(os.path.dirname(moe_inputs.__file__), "skew_bias.json")) as f:
        doc = json.load(f)
    b = np.float32(doc["b"])
    assert np.array_equal(moe_inputs.bf16_bits_to_f32(moe_inputs.f32_to_bf16_bits(b)), b)
    assert abs(sum(doc["achieved_shares"]) - 1.0) < 1e-5


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_config_table(cfg):
    c = moe_inputs.WORKLOADS[cfg]
    assert c["k"] == 2 and c["E"] == 8
    assert c["dtype"] == ("f32" if cfg == 1 else "bf16")


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_mixtral_shapes_match_printed_parameter_counts(cfg):
    """The Mixtral 8x7B workloads' sizes against the figures the Mistral/Mixtral page prints
    (tests/golden/mixtral_8x7b_printed_sizes.json, each figure with its section): d_ff, d_model,
    the layer count, 8 experts with top-2, and the parameter totals, from which one expert's
    parameters over all layers follow as (total - active) / (experts - top_k).  A SwiGLU expert
    holds three d x F matrices in each layer."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "mixtral_8x7b_printed_sizes.json")) as f:
        g = json.load(f)
    c = moe_inputs.WORKLOADS[cfg]
    d, F, E, k = c["d"], c["F"], c["E"], c["k"]
    assert (d, F, E, k) == (g["d_model"], g["d_ff"], g["experts"], g["top_k"])
    p_ffn = g["layers"] * 3 * d * F
    from_totals = (g["total_params"] - g["active_params"]) / (E - k)
    assert abs(p_ffn - from_totals) / from_totals < 0.005
    assert abs(p_ffn - g["p_ffn_estimate"]) / g["p_ffn_estimate"] < 0.005
    # the pin separates: two matrices per expert instead of three would be a third short
    assert abs(g["layers"] * 2 * d * F - from_totals) / from_totals > 0.3
