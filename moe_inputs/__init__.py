"""Seeded synthetic inputs for the sparse MoE feed-forward layer.

This module holds no arithmetic of the layer: it only draws the seeded normal
samples (see ``gen.c`` for the generator's definition) and lays them out as the
layer's operands.  The fp64 oracle and the CUDA path both consume the arrays it
returns, so both sides see byte-identical inputs.

Operand layouts (row-major, the ``nn.Linear`` weight convention of the
"Mistral/Mixtral architecture" page, section "MoEレイヤー全体の実装"):

    x  [T][d]       Wg [E][d]
    W1 [E][F][d]    W3 [E][F][d]    W2 [E][d][F]

Initialisation: x ~ N(0, 1), Wg, W1, W3 ~ N(0, 1/d), W2 ~ N(0, 1/F).  bf16
operands are returned as uint16 bit patterns, fp32 operands as float32.

Backward workloads add dout = dL/dout [T][d] (id 6): N(0, 1).

Block operands (the MoE sub-layer with its pre-norm and residual): the
residual stream h is x with row t scaled by 2^((t mod 5) - 2), an exact
power-of-two scale in bf16 and fp32, so rows span a 16x range of norms; the
norm gain is gamma_j = 1 + 0.2 N(0, 1), rounded to the operand dtype.

The skewed workload sets feature 0 of every token to exactly 1.0 and
Wg[e][0] to a stored per-expert constant b_e, which adds b_e to the logit of
expert e (the router has no bias term, so the bias rides on a constant input
feature).  The constants live in ``skew_bias.json``; they were fitted so that
top-2 assignment shares follow Zipf(s=1.2) over the 8 experts.
"""
from __future__ import annotations

import ctypes
import json
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_inputs.so")
_lock = threading.Lock()
_lib = None

TENSOR_IDS = {"x": 0, "Wg": 1, "W1": 2, "W3": 3, "W2": 4, "gamma": 5, "dout": 6}
BLOCK_EPS = 1e-5      # eps of the block's RMSNorm in every test and workload
BF16_ONE = 0x3F80


def build(force: bool = False) -> str:
    """Compile gen.c into libmoe_inputs.so beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, u64, dbl, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
            lib.moe_gen_normal_f32.argtypes = [vp, i64, u64, u64, dbl]
            lib.moe_gen_normal_bf16.argtypes = [vp, i64, u64, u64, dbl]
            lib.moe_gen_splitmix64.argtypes = [vp, i64, u64]
            lib.moe_gen_f32_to_bf16.argtypes = [vp, vp, i64]
            lib.moe_gen_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def normal(shape, seed: int, tensor_id: int, sigma: float, dtype: str) -> np.ndarray:
    """sigma * N(0,1) samples of one tensor stream; uint16 bf16 bits or float32."""
    lib = _load()
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "bf16":
        out = np.empty(shape, dtype=np.uint16)
        lib.moe_gen_normal_bf16(out.ctypes.data, n, seed, tensor_id, float(sigma))
    elif dtype == "f32":
        out = np.empty(shape, dtype=np.float32)
        lib.moe_gen_normal_f32(out.ctypes.data, n, seed, tensor_id, float(sigma))
    else:
        raise ValueError(f"unknown dtype {dtype!r}")
    return out


def splitmix64(state: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().moe_gen_splitmix64(out.ctypes.data, n, state)
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().moe_gen_f32_to_bf16(a.ctypes.data, out.ctypes.data, a.size)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def generator_threads() -> int:
    return int(_load().moe_gen_num_threads())


def skew_bias(E: int = 8) -> list:
    with open(os.path.join(_HERE, "skew_bias.json")) as f:
        doc = json.load(f)
    b = [float(v) for v in doc["b"]]
    if len(b) != E:
        raise ValueError(f"skew_bias.json holds {len(b)} biases, workload has E={E}")
    return b


@dataclass
class MoEInputs:
    T: int
    d: int
    F: int
    E: int
    k: int
    dtype: str           # "bf16" or "f32"
    seed: int
    skew: bool = False
    x: np.ndarray = field(default=None, repr=False)
    Wg: np.ndarray = field(default=None, repr=False)
    W1: np.ndarray = field(default=None, repr=False)
    W3: np.ndarray = field(default=None, repr=False)
    W2: np.ndarray = field(default=None, repr=False)
    gamma: np.ndarray = field(default=None, repr=False)   # block operands only

    def arrays(self):
        return self.x, self.Wg, self.W1, self.W3, self.W2

    def as_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return bf16_bits_to_f32(a) if self.dtype == "bf16" else a


def make_inputs(T: int, d: int, F: int, E: int, k: int, dtype: str = "bf16", seed: int = 0,
                skew: bool = False, bias=None, weights: bool = True) -> MoEInputs:
    """Generate all operands of one layer call.

    ``bias`` overrides the skew constants (a list of E floats) and implies the
    skew recipe; ``weights=False`` leaves W1/W3/W2 out (routing-only uses).
    """
    inp = MoEInputs(T=T, d=d, F=F, E=E, k=k, dtype=dtype, seed=seed, skew=skew or bias is not None)
    inp.x = normal((T, d), seed, TENSOR_IDS["x"], 1.0, dtype)
    inp.Wg = normal((E, d), seed, TENSOR_IDS["Wg"], 1.0 / np.sqrt(d), dtype)
    if inp.skew:
        b = list(bias) if bias is not None else skew_bias(E)
        if dtype == "bf16":
            inp.x[:, 0] = BF16_ONE
            inp.Wg[:, 0] = f32_to_bf16_bits(np.asarray(b, dtype=np.float32))
        else:
            inp.x[:, 0] = 1.0
            inp.Wg[:, 0] = np.asarray(b, dtype=np.float32)
    if weights:
        inp.W1 = normal((E, F, d), seed, TENSOR_IDS["W1"], 1.0 / np.sqrt(d), dtype)
        inp.W3 = normal((E, F, d), seed, TENSOR_IDS["W3"], 1.0 / np.sqrt(d), dtype)
        inp.W2 = normal((E, d, F), seed, TENSOR_IDS["W2"], 1.0 / np.sqrt(F), dtype)
    return inp


def make_dout(T: int, d: int, dtype: str, seed: int) -> np.ndarray:
    """The upstream gradient dL/dout [T][d] of the backward workloads: N(0, 1)."""
    return normal((T, d), seed, TENSOR_IDS["dout"], 1.0, dtype)


def row_scales(T: int) -> np.ndarray:
    """The block recipe's per-row power-of-two scales of the residual stream."""
    return np.ldexp(np.float32(1.0), (np.arange(T) % 5) - 2).astype(np.float32)


def make_block(inp: MoEInputs) -> MoEInputs:
    """Turn one layer's operands into block operands: x becomes the residual h, gamma is added."""
    sc = row_scales(inp.T)[:, None]
    if inp.dtype == "bf16":
        inp.x = f32_to_bf16_bits(bf16_bits_to_f32(inp.x) * sc)          # exact: power-of-two scales
        g = normal((inp.d,), inp.seed, TENSOR_IDS["gamma"], 0.2, "f32")
        inp.gamma = f32_to_bf16_bits(np.float32(1.0) + g)
    else:
        inp.x = np.ascontiguousarray(inp.x * sc, dtype=np.float32)
        inp.gamma = (np.float32(1.0) + normal((inp.d,), inp.seed, TENSOR_IDS["gamma"], 0.2, "f32")).astype(np.float32)
    return inp


# The five named workloads (sizes, dtype, seed, routing recipe).
WORKLOADS = {
    1: dict(name="tiny-f32", T=64, d=128, F=256, E=8, k=2, dtype="f32", seed=0, skew=False),
    2: dict(name="mixtral-8x7b-decode", T=16, d=4096, F=14336, E=8, k=2, dtype="bf16", seed=1, skew=False),
    3: dict(name="mixtral-8x7b-prefill", T=4096, d=4096, F=14336, E=8, k=2, dtype="bf16", seed=2, skew=False),
    4: dict(name="mixtral-8x7b-skewed-zipf1.2", T=8192, d=4096, F=14336, E=8, k=2, dtype="bf16", seed=3, skew=True),
    5: dict(name="8x22b-shape-prefill", T=16384, d=6144, F=16384, E=8, k=2, dtype="bf16", seed=4, skew=False),
}


def make_config(cfg: int, weights: bool = True, T: int | None = None) -> MoEInputs:
    c = WORKLOADS[cfg]
    return make_inputs(T if T is not None else c["T"], c["d"], c["F"], c["E"], c["k"], c["dtype"],
                       c["seed"], c["skew"], weights=weights)
