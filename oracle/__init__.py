"""fp64 CPU oracle of the Mixtral-style sparse MoE feed-forward layer.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path never
does, and this package never imports the product package.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, no BLAS);
this file only compiles it with gcc and marshals numpy arrays.  Which passage
of the pages each step follows is stated in the C file's header:
"Mistral/Mixtral architecture" page, section "MoEの数学 — ルーターとゲーティング機構"
(score, Top-2, gate, expert and output equations).

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  scores / route / select  pinned: brute force over all k-subsets, closed
                           form of the k=2 gate, invariants, hand example
  expert                   pinned: E=1 dense SwiGLU against torch fp64, hand example
  moe                      pinned: k=E uniform average, E=1 dense FFN, hand
                           example, permutation/relabelling invariances
  counts                   pinned: sums to k*T, brute-force histogram
  rmsnorm                  pinned: torch's rms_norm in fp64, hand example,
                           power-of-two homogeneity, unit RMS at eps = 0
  block / block_scores     pinned: E=1 dense block and k=E uniform block
                           against torch fp64, scale invariance of the
                           routing, zero row
  balance                  pinned: uniform scores (loss = alpha*k), cyclic
                           balanced batch, brute force against torch,
                           sums of f and p
  backward / backward_tokens / weight_grad_slices / balance_grad
                           pinned: central finite differences of moe() (and
                           of moe() + balance() for the load-balance part);
                           torch autograd of the E=1 dense FFN and of the
                           k=E softmax mixture; slices and token rows equal
                           the full backward
  block_backward           pinned (tests/test_oracle_pins_block_backward.py):
                           central finite differences of block() (+ balance()
                           of block_scores()) on every parameter; torch
                           autograd of the E=1 dense block and of the k=E
                           softmax-mixture block; W2 = 0 passes dout to h
                           unchanged; fp64 operand storage equals fp32

The block and balance steps follow the same page, section "Mixtral 8x7B —
Sparse MoEの導入" (subsection "Mixtralのアーキテクチャ": RMSNorm, MoE layer,
residual) and subsection "ロードバランス損失" (f, p and loss equations).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODE = {"f32": 0, "bf16": 1, "f64": 2}   # f64: operands that are exact fp64 results (block backward)


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc -O2, OpenMP; no -ffast-math)."""
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
            vp, ci = ctypes.c_void_p, ctypes.c_int
            lib.oracle_scores.argtypes = [ci, ci, ci, vp, vp, ci, vp, ci]
            lib.oracle_select.argtypes = [ci, ci, ci, vp, vp, vp, vp, vp]
            lib.oracle_route.argtypes = [ci, ci, ci, ci, vp, vp, ci, vp, vp, vp, vp, ci]
            lib.oracle_expert.argtypes = [ci, ci, vp, vp, vp, vp, ci, ci, ci, vp]
            lib.oracle_moe.argtypes = [ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, ci, vp, ci, vp, vp, vp, vp,
                                       vp, ci]
            lib.oracle_counts.argtypes = [ci, ci, ci, vp, vp]
            cd = ctypes.c_double
            lib.oracle_rmsnorm.argtypes = [ci, ci, vp, vp, cd, ci, vp]
            lib.oracle_block_scores.argtypes = [ci, ci, ci, vp, vp, cd, vp, ci, vp, ci]
            lib.oracle_block.argtypes = [ci, ci, ci, ci, ci, vp, vp, cd, vp, vp, vp, vp, ci, vp, ci, vp, vp, vp,
                                         vp, vp, ci]
            lib.oracle_balance.argtypes = [ci, ci, ci, vp, cd, vp, vp, vp]
            lib.oracle_backward.argtypes = [ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, ci, vp, cd] + [vp] * 10
            lib.oracle_backward_tokens.argtypes = [ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, ci, vp, cd, vp, ci] + \
                [vp] * 6 + [ci]
            lib.oracle_backward_rows.argtypes = [ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, ci, vp] + [vp] * 6 + [ci]
            lib.oracle_balance_grad.argtypes = [ci, ci, ci, vp, cd, vp]
            lib.oracle_weight_grad_slices.argtypes = [ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, ci, vp, ci, vp, ci,
                                                      vp, vp, vp, ci]
            lib.oracle_max_threads.restype = ci
            _lib = lib
    return _lib


def _arr(a, dtype):
    want = {"bf16": np.uint16, "f32": np.float32, "f64": np.float64}[dtype]
    a = np.ascontiguousarray(a)
    if a.dtype != want:
        raise TypeError(f"expected {want} storage for dtype {dtype}, got {a.dtype}")
    return a


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def scores(x, Wg, dtype: str, nthreads: int = 0) -> np.ndarray:
    x, Wg = _arr(x, dtype), _arr(Wg, dtype)
    T, d = x.shape
    E = Wg.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    _check(_load().oracle_scores(T, d, E, x.ctypes.data, Wg.ctypes.data, DTYPE_CODE[dtype],
                                 out.ctypes.data, nthreads), "scores")
    return out


def select(logits, k: int):
    """Top-k selection + gate softmax from given fp64 scores [T][E]."""
    s = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = s.shape
    idx = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float64)
    margin = np.empty(T, dtype=np.float64)
    mingap = np.empty(T, dtype=np.float64)
    _check(_load().oracle_select(T, E, k, s.ctypes.data, idx.ctypes.data, g.ctypes.data, margin.ctypes.data,
                                 mingap.ctypes.data), "select")
    return idx, g, margin, mingap


def route(x, Wg, k: int, dtype: str, nthreads: int = 0):
    """Steps 1-3 for every token: (idx [T][k] int32, g [T][k] f64, margin [T], mingap [T])."""
    x, Wg = _arr(x, dtype), _arr(Wg, dtype)
    T, d = x.shape
    E = Wg.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float64)
    margin = np.empty(T, dtype=np.float64)
    mingap = np.empty(T, dtype=np.float64)
    _check(_load().oracle_route(T, d, E, k, x.ctypes.data, Wg.ctypes.data, DTYPE_CODE[dtype], idx.ctypes.data,
                                g.ctypes.data, margin.ctypes.data, mingap.ctypes.data, nthreads), "route")
    return idx, g, margin, mingap


def expert(x, W1, W3, W2, e: int, t: int, dtype: str) -> np.ndarray:
    """Step 4 alone: expert e applied to token row t of x, in double."""
    x, W1, W3, W2 = (_arr(a, dtype) for a in (x, W1, W3, W2))
    d = x.shape[1]
    F = W1.shape[1]
    y = np.empty(d, dtype=np.float64)
    _check(_load().oracle_expert(d, F, x.ctypes.data, W1.ctypes.data, W3.ctypes.data, W2.ctypes.data,
                                 DTYPE_CODE[dtype], e, t, y.ctypes.data), "expert")
    return y


def moe(x, Wg, W1, W3, W2, k: int, dtype: str, tokens=None, nthreads: int = 0) -> dict:
    """The whole layer for all tokens, or for the listed token ids only.

    Returns dict(out [n][d] f64, idx [n][k], g [n][k], margin [n], mingap [n], tokens [n]).
    """
    x, Wg, W1, W3, W2 = (_arr(a, dtype) for a in (x, Wg, W1, W3, W2))
    T, d = x.shape
    E, F = W1.shape[0], W1.shape[1]
    if tokens is None:
        tok = None
        n = T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tok.size
    out = np.empty((n, d), dtype=np.float64)
    idx = np.empty((n, k), dtype=np.int32)
    g = np.empty((n, k), dtype=np.float64)
    margin = np.empty(n, dtype=np.float64)
    mingap = np.empty(n, dtype=np.float64)
    _check(_load().oracle_moe(T, d, F, E, k, x.ctypes.data, Wg.ctypes.data, W1.ctypes.data, W3.ctypes.data,
                              W2.ctypes.data, DTYPE_CODE[dtype], None if tok is None else tok.ctypes.data, n,
                              out.ctypes.data, idx.ctypes.data, g.ctypes.data, margin.ctypes.data,
                              mingap.ctypes.data, nthreads), "moe")
    return dict(out=out, idx=idx, g=g, margin=margin, mingap=mingap,
                tokens=np.arange(T, dtype=np.int32) if tok is None else tok)


def counts(idx, E: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    c = np.empty(E, dtype=np.int64)
    _check(_load().oracle_counts(T, k, E, idx.ctypes.data, c.ctypes.data), "counts")
    return c


def rmsnorm(h, gamma, eps: float, dtype: str) -> np.ndarray:
    """RMSNorm of every row, in double: gamma_j h_j / sqrt(mean(h^2) + eps)."""
    h, gamma = _arr(h, dtype), _arr(gamma, dtype)
    T, d = h.shape
    if gamma.shape != (d,):
        raise ValueError("gamma must have shape [d]")
    u = np.empty((T, d), dtype=np.float64)
    _check(_load().oracle_rmsnorm(T, d, h.ctypes.data, gamma.ctypes.data, float(eps), DTYPE_CODE[dtype],
                                  u.ctypes.data), "rmsnorm")
    return u


def block_scores(h, gamma, eps: float, Wg, dtype: str, nthreads: int = 0) -> np.ndarray:
    """Router scores of the normalised rows: [T][E] = Wg RMSNorm(h_t)."""
    h, gamma, Wg = _arr(h, dtype), _arr(gamma, dtype), _arr(Wg, dtype)
    T, d = h.shape
    E = Wg.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    _check(_load().oracle_block_scores(T, d, E, h.ctypes.data, gamma.ctypes.data, float(eps), Wg.ctypes.data,
                                       DTYPE_CODE[dtype], out.ctypes.data, nthreads), "block_scores")
    return out


def block(h, gamma, eps: float, Wg, W1, W3, W2, k: int, dtype: str, tokens=None, nthreads: int = 0) -> dict:
    """out = h + MoE(RMSNorm(h)) for all tokens or the listed ones; same dict as moe()."""
    h, gamma, Wg, W1, W3, W2 = (_arr(a, dtype) for a in (h, gamma, Wg, W1, W3, W2))
    T, d = h.shape
    E, F = W1.shape[0], W1.shape[1]
    if tokens is None:
        tok = None
        n = T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tok.size
    out = np.empty((n, d), dtype=np.float64)
    idx = np.empty((n, k), dtype=np.int32)
    g = np.empty((n, k), dtype=np.float64)
    margin = np.empty(n, dtype=np.float64)
    mingap = np.empty(n, dtype=np.float64)
    _check(_load().oracle_block(T, d, F, E, k, h.ctypes.data, gamma.ctypes.data, float(eps), Wg.ctypes.data,
                                W1.ctypes.data, W3.ctypes.data, W2.ctypes.data, DTYPE_CODE[dtype],
                                None if tok is None else tok.ctypes.data, n, out.ctypes.data, idx.ctypes.data,
                                g.ctypes.data, margin.ctypes.data, mingap.ctypes.data, nthreads), "block")
    return dict(out=out, idx=idx, g=g, margin=margin, mingap=mingap,
                tokens=np.arange(T, dtype=np.int32) if tok is None else tok)


def balance(logits, k: int, alpha: float):
    """Load-balance statistics from fp64 scores [T][E]: (f [E], p [E], loss)."""
    s = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = s.shape
    f = np.empty(E, dtype=np.float64)
    p = np.empty(E, dtype=np.float64)
    loss = np.empty(1, dtype=np.float64)
    _check(_load().oracle_balance(T, E, k, s.ctypes.data, float(alpha), f.ctypes.data, p.ctypes.data,
                                  loss.ctypes.data), "balance")
    return f, p, float(loss[0])


def backward(x, Wg, W1, W3, W2, dout, k: int, dtype: str, alpha: float = 0.0) -> dict:
    """Every gradient of L = sum <dout, out> + alpha E sum f p (small shapes): dict(dx, dlogits, dWg, dW1, dW3,
    dW2, idx, g, margin, mingap), all float64."""
    x, Wg, W1, W3, W2, dout = (_arr(a, dtype) for a in (x, Wg, W1, W3, W2, dout))
    T, d = x.shape
    E, F = W1.shape[0], W1.shape[1]
    r = dict(dx=np.empty((T, d)), dlogits=np.empty((T, E)), dWg=np.empty((E, d)), dW1=np.empty((E, F, d)),
             dW3=np.empty((E, F, d)), dW2=np.empty((E, d, F)), idx=np.empty((T, k), dtype=np.int32),
             g=np.empty((T, k)), margin=np.empty(T), mingap=np.empty(T))
    _check(_load().oracle_backward(T, d, F, E, k, x.ctypes.data, Wg.ctypes.data, W1.ctypes.data, W3.ctypes.data,
                                   W2.ctypes.data, DTYPE_CODE[dtype], dout.ctypes.data, float(alpha),
                                   *[r[n].ctypes.data for n in ("dx", "dlogits", "dWg", "dW1", "dW3", "dW2", "idx",
                                                                "g", "margin", "mingap")]), "backward")
    return r


def backward_tokens(x, Wg, W1, W3, W2, dout, k: int, dtype: str, tokens, nthreads: int = 0,
                    alpha: float = 0.0) -> dict:
    """dx and the router-score gradient of the listed tokens only: dict(dx, dlogits, idx, g, margin, mingap, tokens)."""
    x, Wg, W1, W3, W2, dout = (_arr(a, dtype) for a in (x, Wg, W1, W3, W2, dout))
    T, d = x.shape
    E, F = W1.shape[0], W1.shape[1]
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tok.size
    r = dict(dx=np.empty((n, d)), dlogits=np.empty((n, E)), idx=np.empty((n, k), dtype=np.int32),
             g=np.empty((n, k)), margin=np.empty(n), mingap=np.empty(n))
    _check(_load().oracle_backward_tokens(T, d, F, E, k, x.ctypes.data, Wg.ctypes.data, W1.ctypes.data,
                                          W3.ctypes.data, W2.ctypes.data, DTYPE_CODE[dtype], dout.ctypes.data,
                                          float(alpha), tok.ctypes.data, n,
                                          *[r[m].ctypes.data for m in ("dx", "dlogits", "idx", "g", "margin",
                                                                       "mingap")], nthreads), "backward_tokens")
    r["tokens"] = tok
    return r


def weight_grad_slices(x, Wg, W1, W3, W2, dout, k: int, dtype: str, e: int, fs, nthreads: int = 0):
    """Rows fs of dW1_e and dW3_e ([n][d] each) and columns fs of dW2_e ([d][n]) over all tokens."""
    x, Wg, W1, W3, W2, dout = (_arr(a, dtype) for a in (x, Wg, W1, W3, W2, dout))
    T, d = x.shape
    E, F = W1.shape[0], W1.shape[1]
    f = np.ascontiguousarray(fs, dtype=np.int32)
    n = f.size
    r1, r3, c2 = np.empty((n, d)), np.empty((n, d)), np.empty((d, n))
    _check(_load().oracle_weight_grad_slices(T, d, F, E, k, x.ctypes.data, Wg.ctypes.data, W1.ctypes.data,
                                             W3.ctypes.data, W2.ctypes.data, DTYPE_CODE[dtype], dout.ctypes.data,
                                             int(e), f.ctypes.data, n, r1.ctypes.data, r3.ctypes.data,
                                             c2.ctypes.data, nthreads), "weight_grad_slices")
    return r1, r3, c2


def balance_grad(logits, k: int, alpha: float) -> np.ndarray:
    """Gradient of alpha E sum f p with respect to every score [T][E] (f held fixed)."""
    s = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = s.shape
    out = np.empty((T, E), dtype=np.float64)
    _check(_load().oracle_balance_grad(T, E, k, s.ctypes.data, float(alpha), out.ctypes.data), "balance_grad")
    return out


def _widen(a, dtype) -> np.ndarray:
    """Exact float64 copy of an operand stored as `dtype`."""
    a = _arr(a, dtype)
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def backward_rows(u, Wg, W1, W3, W2, dout_rows, k: int, dtype: str, nthreads: int = 0) -> dict:
    """dx and the router-score gradient (output path, alpha = 0) of given input rows u [n][d] held in
    float64, with Wg, W1, W3, W2 and dout_rows [n][d] stored as `dtype`: dict(dx, dlogits, idx, g, margin,
    mingap).  The block form's MoE input is the exact normalised row, which no stored dtype holds."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    Wg, W1, W3, W2, dout_rows = (_arr(a, dtype) for a in (Wg, W1, W3, W2, dout_rows))
    n, d = u.shape
    E, F = W1.shape[0], W1.shape[1]
    r = dict(dx=np.empty((n, d)), dlogits=np.empty((n, E)), idx=np.empty((n, k), dtype=np.int32),
             g=np.empty((n, k)), margin=np.empty(n), mingap=np.empty(n))
    _check(_load().oracle_backward_rows(n, d, F, E, k, u.ctypes.data, Wg.ctypes.data, W1.ctypes.data,
                                        W3.ctypes.data, W2.ctypes.data, DTYPE_CODE[dtype], dout_rows.ctypes.data,
                                        *[r[m].ctypes.data for m in ("dx", "dlogits", "idx", "g", "margin",
                                                                     "mingap")], nthreads), "backward_rows")
    return r


def _block_chain(h64, g64, dout64, du, eps: float):
    """The RMSNorm and residual part of the block backward (see block_backward): (dh, dgamma)."""
    d = h64.shape[1]
    rho = 1.0 / np.sqrt((h64 * h64).sum(axis=1) / d + eps)
    proj = (du * g64 * h64).sum(axis=1)
    dh = dout64 + rho[:, None] * g64 * du - (rho ** 3 / d)[:, None] * h64 * proj[:, None]
    dgamma = (du * h64 * rho[:, None]).sum(axis=0)
    return dh, dgamma


def block_backward_tokens(h, gamma, eps: float, Wg, W1, W3, W2, dout, k: int, dtype: str, tokens,
                          nthreads: int = 0) -> dict:
    """block_backward (alpha = 0) restricted to the listed tokens, for full-size layers: dh of those rows
    and dgamma summed over them, plus their score gradients and routing: dict(dh, dgamma, dlogits, idx, g,
    margin, mingap, tokens).  Equal to block_backward's dh rows, and to its dgamma when dout is zero on
    every other token.  Without the load-balance part the tokens are independent."""
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    h_s = _arr(h, dtype)[tok]
    dout_s = _arr(dout, dtype)[tok]
    u = rmsnorm(h_s, gamma, eps, dtype)
    r = backward_rows(u, Wg, W1, W3, W2, dout_s, k, dtype, nthreads)
    du = r.pop("dx")
    r["dh"], r["dgamma"] = _block_chain(_widen(h_s, dtype), _widen(gamma, dtype), _widen(dout_s, dtype), du, eps)
    r["tokens"] = tok
    return r


def block_backward(h, gamma, eps: float, Wg, W1, W3, W2, dout, k: int, dtype: str, alpha: float = 0.0) -> dict:
    """Every gradient of L = sum <dout, out> + alpha E sum f p for out = h + MoE(RMSNorm(h)), with the
    top-k choice held fixed (small shapes): dict(dh, dgamma, dWg, dW1, dW3, dW2, dlogits, idx, g,
    margin, mingap), all float64.

    The MoE part is backward() at x = u = RMSNorm(h), the exact fp64 rows block() evaluates, which
    gives du = dL/du (the load-balance part, on the scores Wg u, included).  With
    rho_t = (mean_i h_ti^2 + eps)^(-1/2) and u_tj = gamma_j h_tj rho_t, d rho_t / d h_ti = -rho_t^3 h_ti / d:
        dh_ti    = dout_ti + rho_t gamma_i du_ti - (rho_t^3 / d) h_ti sum_j du_tj gamma_j h_tj
        dgamma_j = sum_t du_tj h_tj rho_t
    (the residual passes dout to h unchanged).
    """
    u = rmsnorm(h, gamma, eps, dtype)
    h64, g64, dout64 = _widen(h, dtype), _widen(gamma, dtype), _widen(dout, dtype)
    Wg64, W1_64, W3_64, W2_64 = (_widen(a, dtype) for a in (Wg, W1, W3, W2))
    r = backward(u, Wg64, W1_64, W3_64, W2_64, dout64, k, "f64", alpha=alpha)
    du = r.pop("dx")
    r["dh"], r["dgamma"] = _block_chain(h64, g64, dout64, du, eps)
    return r
