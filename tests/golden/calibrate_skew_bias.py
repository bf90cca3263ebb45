"""Fit the per-expert router offsets of the skewed workload; writes moe_inputs/skew_bias.json.

The skewed workload (T=8192 tokens, d=4096, ffn=14336, E=8, k=2, seed 3) wants
top-2 assignment shares that follow Zipf(s=1.2) over the 8 experts.  The router
has no bias term ("Mistral/Mixtral architecture" page, "Top-2ゲーティングの定式化":
the router's only parameter is Wg), so the offset b_e rides on input feature 0,
which the workload pins to 1.0: Wg[e][0] = b_e adds exactly b_e to the score of
expert e.

Fit: the scores without offsets come from the oracle (Wg[:, 0] = 0); then 50
fixed-point steps b_e += 0.5 (ln p_e - ln phat_e) with phat from the oracle's
own top-2 selection of s + b; then b is rounded to bf16 (the storage type) and
the achieved shares are recorded.  Only ``oracle/`` and the input generator
are called.

Run from the repository root:  python tests/golden/calibrate_skew_bias.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402
import oracle  # noqa: E402


def zipf_shares(E, s):
    w = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    return w / w.sum()


def shares(z, b, k):
    idx, _, _, _ = oracle.select(z + b[None, :], k)
    c = oracle.counts(idx, z.shape[1]).astype(np.float64)
    return c / c.sum()


def main():
    c = moe_inputs.WORKLOADS[4]
    T, d, E, k = c["T"], c["d"], c["E"], c["k"]
    inp = moe_inputs.make_inputs(T, d, c["F"], E, k, c["dtype"], c["seed"], bias=[0.0] * E, weights=False)
    z = oracle.scores(inp.x, inp.Wg, c["dtype"])
    target = zipf_shares(E, 1.2)
    b = np.zeros(E)
    for _ in range(50):
        p = shares(z, b, k)
        b += 0.5 * (np.log(target) - np.log(np.maximum(p, 1e-9)))
        b -= b.mean()
    b_stored = moe_inputs.bf16_bits_to_f32(moe_inputs.f32_to_bf16_bits(b.astype(np.float32))).astype(np.float64)
    achieved = shares(z, b_stored, k)
    doc = {
        "workload": c["name"],
        "recipe": "x[:,0]=1.0, Wg[e][0]=b[e] (bf16); fitted to Zipf(1.2) top-2 assignment shares",
        "zipf_s": 1.2,
        "target_shares": [round(float(v), 6) for v in target],
        "achieved_shares": [round(float(v), 6) for v in achieved],
        "b": [float(v) for v in b_stored],
    }
    path = os.path.join(ROOT, "moe_inputs", "skew_bias.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print(json.dumps(doc, indent=1))


if __name__ == "__main__":
    main()
