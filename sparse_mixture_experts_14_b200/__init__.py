"""B200 (sm_100a) sparse mixture-of-experts feed-forward layer: Python binding.

A thin ctypes layer over ``libmoe.so`` (the C ABI declared in include/moe.h):
the functions below carry the C names, check shapes/dtypes/devices, pass raw
device pointers and torch's current CUDA stream, and turn a non-zero status
into ``MoEError``.  Every step of the layer runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or cannot load,
importing this package raises.

bf16 tensors are torch.bfloat16; the layer's operand layouts are
    x [T][d], Wg [E][d], W1 [E][F][d], W3 [E][F][d], W2 [E][d][F], out [T][d].
The block form adds h [T][d] (the residual stream, in place of x) and
gamma [d]; load-balance statistics come back as a float32 [2E+1] tensor
(f, p, loss).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=debug loads the bounds-checking build (libmoe_debug.so): the same kernels with every
# index read from another kernel checked; a failed check records MOE_ERR_DEVICE and skips the access
_VARIANT = os.environ.get("MOE_LIBRARY", "release")
if _VARIANT not in ("release", "debug"):
    raise ImportError(f"MOE_LIBRARY must be 'release' or 'debug', got {_VARIANT!r}")
LIB_PATH = os.path.join(_HERE, "libmoe_debug.so" if _VARIANT == "debug" else "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python sparse_mixture_experts_14_b200/build.py` "
                      f"(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_WORKSPACE, \
    MOE_ERR_DEVICE = range(7)
MOE_PATH_AUTO, MOE_PATH_PREFILL, MOE_PATH_DECODE, MOE_PATH_TRAIN = 0, 1, 2, 3
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1
MOE_NUM_STAGES = 6
STAGE_NAMES = ("route", "dispatch", "gather", "expert1", "expert2", "combine")
MOE_BWD_NUM_STAGES = 7
BWD_STAGE_NAMES = ("scatter", "dgrad_h", "swiglu_bwd", "dgrad_x", "wgrad2", "wgrad13", "router")

# every symbol include/moe.h declares, with its ctypes signature
_vp, _ci, _sz, _ll, _cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong, ctypes.c_float
SIGNATURES = {
    "moe_route": (_ci, [_vp, _vp, _ci, _ci, _ci, _ci, _vp, _vp, _vp]),
    "moe_route_f32": (_ci, [_vp, _vp, _ci, _ci, _ci, _ci, _vp, _vp, _vp]),
    "moe_slots_capacity": (_sz, [_ci, _ci, _ci]),
    "moe_dispatch": (_ci, [_vp, _ci, _ci, _ci, _vp, _vp, _vp, _vp, _vp]),
    "moe_dispatch_noalloc": (_ci, [_vp, _ci, _ci, _ci, _vp, _vp, _vp, _vp, _vp]),
    "moe_forward": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _vp]),
    "moe_forward_f32": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _vp]),
    "moe_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_forward_ws": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _vp, _sz, _vp]),
    "moe_forward_profiled": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _vp, _sz, _vp,
                                   _vp, _vp]),
    "moe_forward_host": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _vp]),
    "moe_host_chunk_plan": (_ci, [_ci, _vp, _ci]),
    "moe_get_device_status": (_ci, [_vp]),
    "moe_selftest_wait_timeout": (_ci, [_ll, _vp]),
    "moe_status_string": (ctypes.c_char_p, [_ci]),
    "moe_decode_max_tokens": (_ci, []),
    "moe_block_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_block_forward": (_ci, [_vp, _vp, _cf, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp]),
    "moe_block_forward_f32": (_ci, [_vp, _vp, _cf, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp,
                                    _vp]),
    "moe_block_forward_ws": (_ci, [_vp, _vp, _cf, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _ci,
                                   _ci, _vp, _sz, _vp, _vp, _vp]),
    "moe_route_stats": (_ci, [_vp, _vp, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp]),
    "moe_backward_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_train_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_backward_ws": (_ci, [_vp] * 12 + [_cf] + [_ci] * 7 + [_vp, _sz, _vp, _sz, _vp, _vp, _vp]),
    "moe_route_stats_f32": (_ci, [_vp, _vp, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp]),
    "moe_pool_stats": (_ci, [_ci, _vp, _vp]),
    "moe_block_train_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_block_backward_workspace_size": (_sz, [_ci, _ci, _ci, _ci, _ci, _ci]),
    "moe_block_backward_ws": (_ci, [_vp] * 14 + [_cf] + [_ci] * 7 + [_vp, _sz, _vp, _sz, _vp, _vp, _vp]),
    "moe_ep_plan": (_ci, [_vp, _ci, _ci, _ci] + [_vp] * 9),
    "moe_ep_dispatch": (_ci, [_vp, _vp, _ci, _ci, _ci, _ci, _vp, _vp, _vp, _vp]),
    "moe_ep_experts": (_ci, [_vp, _vp, _ci, _ci, _ci, _vp, _vp, _vp, _ci, _ci, _vp, _vp]),
    "moe_ep_combine": (_ci, [_vp, _vp, _vp, _ci, _ci, _ci, _vp, _vp]),
}
for _name, (_res, _args) in SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {moe_status_string(status)} (status {status})")


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what)


def _stream(stream=None, *tensors):
    """The stream to launch on: `stream`, else torch's current stream of the device that holds
    the call's CUDA tensors.  Tensors on several devices (or a stream of another device) raise:
    a kernel cannot address another device's memory through them."""
    devs = {t.device for t in tensors if isinstance(t, torch.Tensor) and t.is_cuda}
    if len(devs) > 1:
        raise ValueError(f"tensors on several devices: {sorted(str(v) for v in devs)}")
    dev = devs.pop() if devs else None
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and stream.device != dev:
        raise ValueError(f"stream of {stream.device} for tensors on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _room(t, numel, name):
    """A caller-supplied output must hold at least `numel` elements: the kernels write that many and
    trust the pointer.  Checked before the device and dtype checks, and before anything launches."""
    if isinstance(t, torch.Tensor) and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {numel}")
    return t


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    if t.dtype == torch.float32:
        return MOE_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _router_shapes(x, Wg):
    """Tokens x [T][d] and router weights Wg [E][d]: the kernels trust these sizes."""
    if x.dim() != 2 or Wg.dim() != 2 or Wg.shape[1] != x.shape[1]:
        raise ValueError(f"inconsistent shapes x{tuple(x.shape)} Wg{tuple(Wg.shape)}")
    return x.shape[0], x.shape[1], Wg.shape[0]


def _layer_shapes(x, Wg, W1, W3, W2):
    if x.dim() != 2 or W1.dim() != 3:
        raise ValueError(f"x must be [T][d] and W1 [E][F][d], got x{tuple(x.shape)} W1{tuple(W1.shape)}")
    T, d = x.shape
    E, F, d1 = W1.shape
    if Wg.shape != (E, d) or d1 != d or W3.shape != (E, F, d) or W2.shape != (E, d, F):
        raise ValueError(f"inconsistent shapes x{tuple(x.shape)} Wg{tuple(Wg.shape)} W1{tuple(W1.shape)} "
                         f"W3{tuple(W3.shape)} W2{tuple(W2.shape)}")
    return T, d, F, E


def moe_route(x, Wg, k, topk_idx=None, topk_w=None, stream=None):
    """Router scores, top-k (lowest index on ties), softmax over the k: (topk_idx int32 [T][k], topk_w f32 [T][k])."""
    T, d, E = _router_shapes(x, Wg)
    code = _dtype_code(x)
    _dev(x, x.dtype, "x")
    _dev(Wg, x.dtype, "Wg")
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _room(topk_idx, T * k, "topk_idx")
    _room(topk_w, T * k, "topk_w")
    _dev(topk_idx, torch.int32, "topk_idx")
    _dev(topk_w, torch.float32, "topk_w")
    fn = _lib.moe_route if code == MOE_DTYPE_BF16 else _lib.moe_route_f32
    _check(fn(_ptr(x), _ptr(Wg), T, d, E, k, _ptr(topk_idx), _ptr(topk_w),
              _stream(stream, x, Wg, topk_idx, topk_w)), "moe_route")
    return topk_idx, topk_w


def moe_slots_capacity(T, E, k) -> int:
    return int(_lib.moe_slots_capacity(T, E, k))


def moe_dispatch(topk_idx, E, stream=None):
    """Stable counting sort of assignments into 128-padded expert segments: (counts, offsets, perm, inv)."""
    _dev(topk_idx, torch.int32, "topk_idx")
    T, k = topk_idx.shape
    dev = topk_idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(moe_slots_capacity(T, E, k), 1), dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    _check(_lib.moe_dispatch(_ptr(topk_idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                             _stream(stream, topk_idx)), "moe_dispatch")
    return counts, offsets, perm, inv


def moe_dispatch_noalloc(topk_idx, E, counts, offsets, perm, inv, stream=None):
    """moe_dispatch into caller-provided outputs, using the library's fixed scratch array instead of
    any allocation (for callers that may not allocate device memory); raises MoEError above its limit."""
    if not isinstance(topk_idx, torch.Tensor) or topk_idx.dim() != 2:
        raise ValueError("topk_idx must be a 2-D [T][k] tensor")
    T, k = topk_idx.shape
    for t, numel, n in ((counts, E, "counts"), (offsets, E + 1, "offsets"),
                        (perm, moe_slots_capacity(T, E, k) if E > 0 and 0 < k <= E else 0, "perm"),
                        (inv, T * k, "inv")):
        _room(t, numel, n)
    _dev(topk_idx, torch.int32, "topk_idx")
    for t, n in ((counts, "counts"), (offsets, "offsets"), (perm, "perm"), (inv, "inv")):
        _dev(t, torch.int32, n)
    _check(_lib.moe_dispatch_noalloc(_ptr(topk_idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                                     _stream(stream, topk_idx, counts, offsets, perm, inv)), "moe_dispatch_noalloc")
    return counts, offsets, perm, inv


def moe_forward(x, Wg, W1, W3, W2, k, out=None, stream=None):
    """The whole layer; bf16 tensors use moe_forward, float32 tensors moe_forward_f32."""
    code = _dtype_code(x)
    for t, n in ((x, "x"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2")):
        _dev(t, x.dtype, n)
    T, d, F, E = _layer_shapes(x, Wg, W1, W3, W2)
    if out is None:
        out = torch.empty((T, d), dtype=x.dtype, device=x.device)
    _room(out, T * d, "out")
    _dev(out, x.dtype, "out")
    fn = _lib.moe_forward if code == MOE_DTYPE_BF16 else _lib.moe_forward_f32
    _check(fn(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out), T, d, F, E, k,
              _stream(stream, x, Wg, W1, W3, W2, out)), "moe_forward")
    return out


moe_forward_f32 = moe_forward


def moe_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_workspace_size(T, d, ffn, E, k, dtype))


def moe_forward_ws(x, Wg, W1, W3, W2, k, path=MOE_PATH_AUTO, workspace=None, out=None, stream=None):
    """moe_forward with an explicit workspace (a uint8 CUDA tensor) and path."""
    code = _dtype_code(x)
    for t, n in ((x, "x"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2")):
        _dev(t, x.dtype, n)
    T, d, F, E = _layer_shapes(x, Wg, W1, W3, W2)
    need = (moe_train_workspace_size if path == MOE_PATH_TRAIN else moe_workspace_size)(T, d, F, E, k, code)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _dev(workspace, torch.uint8, "workspace")
    if out is None:
        out = torch.empty((T, d), dtype=x.dtype, device=x.device)
    _room(out, T * d, "out")
    _dev(out, x.dtype, "out")
    _check(_lib.moe_forward_ws(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out), T, d, F, E, k, code,
                               path, _ptr(workspace), workspace.numel(),
                               _stream(stream, x, Wg, W1, W3, W2, out, workspace)), "moe_forward_ws")
    return out


def moe_forward_profiled(x, Wg, W1, W3, W2, k, workspace, out, events=None, path=MOE_PATH_AUTO, stream=None):
    """moe_forward_ws recording torch.cuda.Event objects (MOE_NUM_STAGES + 1 of them, timing enabled)
    at the stage boundaries; returns the number of kernels launched."""
    code = _dtype_code(x)
    T, d, F, E = _layer_shapes(x, Wg, W1, W3, W2)
    _room(out, T * d, "out")
    for t, n in ((x, "x"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2"), (out, "out")):
        _dev(t, x.dtype, n)
    _dev(workspace, torch.uint8, "workspace")
    ev_arr = _events(events)
    n = ctypes.c_int(0)
    _check(_lib.moe_forward_profiled(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out), T, d, F, E, k, code,
                                     path, _ptr(workspace), workspace.numel(), ev_arr, ctypes.byref(n),
                                     _stream(stream, x, Wg, W1, W3, W2, out, workspace)), "moe_forward_profiled")
    return n.value


def moe_forward_host(x_host, Wg, W1, W3, W2, k, out_host=None, stream=None):
    """End to end from host memory: x_host / out_host are CPU bf16 tensors (pinned for full speed)."""
    if x_host.is_cuda or x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
        raise TypeError("x_host must be a contiguous CPU bfloat16 tensor")
    T, d, F, E = _layer_shapes(x_host, Wg, W1, W3, W2)
    if out_host is not None:
        _room(out_host, T * d, "out_host")
        if out_host.is_cuda or out_host.dtype != torch.bfloat16 or not out_host.is_contiguous():
            raise TypeError("out_host must be a contiguous CPU bfloat16 tensor")
    for t, n in ((Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2")):
        _dev(t, torch.bfloat16, n)
    if out_host is None:
        out_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    _check(_lib.moe_forward_host(_ptr(x_host), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out_host), T, d, F, E,
                                 k, _stream(stream, Wg, W1, W3, W2)), "moe_forward_host")
    return out_host


def _events(events, n=MOE_NUM_STAGES):
    if events is None:
        return None
    if len(events) != n + 1:
        raise ValueError(f"need {n + 1} events")
    return (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])


def _block_args(h, gamma, Wg, W1, W3, W2, stats):
    for t, n in ((h, "h"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2"), (gamma, "gamma")):
        _dev(t, h.dtype, n)
    T, d, F, E = _layer_shapes(h, Wg, W1, W3, W2)
    if gamma.shape != (d,):
        raise ValueError(f"gamma must have shape ({d},), got {tuple(gamma.shape)}")
    if stats is not None:
        _dev(stats, torch.float32, "stats")
        if stats.numel() < 2 * E + 1:
            raise ValueError(f"stats needs {2 * E + 1} floats")
    return T, d, F, E


def moe_block_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_block_workspace_size(T, d, ffn, E, k, dtype))


def moe_block_forward(h, gamma, eps, Wg, W1, W3, W2, k, alpha=1.0, stats=None, out=None, stream=None):
    """out = h + MoE(RMSNorm(h)); bf16 tensors use moe_block_forward, float32 moe_block_forward_f32.
    stats (float32 [2E+1] CUDA tensor or None) receives f, p and the load-balance loss.  out may be h."""
    code = _dtype_code(h)
    T, d, F, E = _block_args(h, gamma, Wg, W1, W3, W2, stats)
    if out is None:
        out = torch.empty((T, d), dtype=h.dtype, device=h.device)
    _room(out, T * d, "out")
    _dev(out, h.dtype, "out")
    fn = _lib.moe_block_forward if code == MOE_DTYPE_BF16 else _lib.moe_block_forward_f32
    _check(fn(_ptr(h), _ptr(gamma), float(eps), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out), T, d, F, E, k,
              float(alpha), _ptr(stats), _stream(stream, h, gamma, Wg, W1, W3, W2, stats, out)), "moe_block_forward")
    return out


moe_block_forward_f32 = moe_block_forward


def moe_block_forward_ws(h, gamma, eps, Wg, W1, W3, W2, k, workspace, out, alpha=1.0, stats=None,
                         path=MOE_PATH_AUTO, events=None, stream=None):
    """moe_block_forward with an explicit workspace, path and optional stage events; returns the launch count."""
    code = _dtype_code(h)
    T, d, F, E = _block_args(h, gamma, Wg, W1, W3, W2, stats)
    _room(out, T * d, "out")
    _dev(workspace, torch.uint8, "workspace")
    _dev(out, h.dtype, "out")
    n = ctypes.c_int(0)
    _check(_lib.moe_block_forward_ws(_ptr(h), _ptr(gamma), float(eps), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2),
                                     _ptr(out), T, d, F, E, k, float(alpha), _ptr(stats), code, path,
                                     _ptr(workspace), workspace.numel(), _events(events), ctypes.byref(n),
                                     _stream(stream, h, gamma, Wg, W1, W3, W2, stats, out, workspace)),
           "moe_block_forward_ws")
    return n.value


def moe_route_stats(x, Wg, k, alpha=1.0, stream=None):
    """moe_route plus load-balance statistics: (topk_idx, topk_w, stats [2E+1] = f, p, loss)."""
    T, d, E = _router_shapes(x, Wg)
    code = _dtype_code(x)
    _dev(x, x.dtype, "x")
    _dev(Wg, x.dtype, "Wg")
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    stats = torch.empty(2 * E + 1, dtype=torch.float32, device=x.device)
    fn = _lib.moe_route_stats if code == MOE_DTYPE_BF16 else _lib.moe_route_stats_f32
    _check(fn(_ptr(x), _ptr(Wg), T, d, E, k, float(alpha), _ptr(idx), _ptr(w), _ptr(stats), _stream(stream, x, Wg)),
           "moe_route_stats")
    return idx, w, stats


def moe_train_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_train_workspace_size(T, d, ffn, E, k, dtype))


def moe_backward_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_backward_workspace_size(T, d, ffn, E, k, dtype))


def moe_backward_ws(x, Wg, W1, W3, W2, dout, k, fwd_workspace, workspace=None, grads=None, dlogits=None,
                    alpha=0.0, wgrad_dtype=torch.float32, events=None, stream=None):
    """Gradients of the layer given dout = dL/dout, after moe_forward_ws(..., path=MOE_PATH_TRAIN,
    workspace=fwd_workspace) on the same operands (fwd_workspace: moe_train_workspace_size bytes).  Returns (grads, launches) with grads a dict of
    dx (layer dtype), dWg, dW1, dW3, dW2 (float32); pass `grads` to reuse buffers, `dlogits` (float32
    [T][E]) to also get the router-score gradient.  alpha != 0 adds the load-balance loss
    alpha E sum f p of the forward's routing to the loss.  wgrad_dtype=torch.bfloat16 (bf16 layers)
    returns dW1, dW3, dW2 rounded once to bf16."""
    code = _dtype_code(x)
    for t, n in ((x, "x"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2"), (dout, "dout")):
        _dev(t, x.dtype, n)
    T, d, F, E = _layer_shapes(x, Wg, W1, W3, W2)
    if dout.shape != (T, d):
        raise ValueError("dout must have the shape of x")
    dev = x.device
    if grads is None:
        f32 = torch.float32
        wd = wgrad_dtype
        grads = dict(dx=torch.empty((T, d), dtype=x.dtype, device=dev), dWg=torch.empty((E, d), dtype=f32, device=dev),
                     dW1=torch.empty((E, F, d), dtype=wd, device=dev), dW3=torch.empty((E, F, d), dtype=wd, device=dev),
                     dW2=torch.empty((E, d, F), dtype=wd, device=dev))
    for n, numel in (("dx", T * d), ("dWg", E * d), ("dW1", E * F * d), ("dW3", E * F * d), ("dW2", E * d * F)):
        _room(grads[n], numel, n)
    if dlogits is not None:
        _room(dlogits, T * E, "dlogits")
    _dev(grads["dx"], x.dtype, "dx")
    _dev(grads["dWg"], torch.float32, "dWg")
    for n in ("dW1", "dW3", "dW2"):
        _dev(grads[n], grads["dW1"].dtype, n)
    wcode = _dtype_code(grads["dW1"])
    if dlogits is not None:
        _dev(dlogits, torch.float32, "dlogits")
    _dev(fwd_workspace, torch.uint8, "fwd_workspace")
    if workspace is None:
        workspace = torch.empty(max(moe_backward_workspace_size(T, d, F, E, k, code), 1), dtype=torch.uint8,
                                device=dev)
    _dev(workspace, torch.uint8, "workspace")
    n = ctypes.c_int(0)
    _check(_lib.moe_backward_ws(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dout), _ptr(grads["dx"]),
                                _ptr(grads["dWg"]), _ptr(grads["dW1"]), _ptr(grads["dW3"]), _ptr(grads["dW2"]),
                                _ptr(dlogits), float(alpha), wcode, T, d, F, E, k, code, _ptr(fwd_workspace),
                                fwd_workspace.numel(),
                                _ptr(workspace), workspace.numel(), _events(events, MOE_BWD_NUM_STAGES),
                                ctypes.byref(n),
                                _stream(stream, x, Wg, W1, W3, W2, dout, fwd_workspace, workspace, dlogits,
                                        *grads.values())), "moe_backward_ws")
    return grads, n.value


def moe_block_train_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_block_train_workspace_size(T, d, ffn, E, k, dtype))


def moe_block_backward_workspace_size(T, d, ffn, E, k, dtype=MOE_DTYPE_BF16) -> int:
    return int(_lib.moe_block_backward_workspace_size(T, d, ffn, E, k, dtype))


def moe_block_backward_ws(h, gamma, Wg, W1, W3, W2, dout, k, fwd_workspace, workspace=None, grads=None,
                          dlogits=None, alpha=0.0, wgrad_dtype=torch.float32, events=None, stream=None):
    """Gradients of the block out = h + MoE(RMSNorm(h)) given dout, after moe_block_forward_ws(...,
    path=MOE_PATH_TRAIN, workspace=fwd_workspace) on the same h, gamma and weights.  Returns (grads,
    launches) with grads a dict of dh (layer dtype), dgamma, dWg (float32), dW1, dW3, dW2 (wgrad_dtype)."""
    code = _dtype_code(h)
    T, d, F, E = _layer_shapes(h, Wg, W1, W3, W2)
    if dout.shape != (T, d) or gamma.shape != (d,):
        raise ValueError("dout must have the shape of h and gamma shape (d,)")
    dev = h.device
    if grads is None:
        f32, wd = torch.float32, wgrad_dtype
        grads = dict(dh=torch.empty((T, d), dtype=h.dtype, device=dev), dgamma=torch.empty(d, dtype=f32, device=dev),
                     dWg=torch.empty((E, d), dtype=f32, device=dev), dW1=torch.empty((E, F, d), dtype=wd, device=dev),
                     dW3=torch.empty((E, F, d), dtype=wd, device=dev), dW2=torch.empty((E, d, F), dtype=wd, device=dev))
    for n, numel in (("dh", T * d), ("dgamma", d), ("dWg", E * d), ("dW1", E * F * d), ("dW3", E * F * d),
                     ("dW2", E * d * F)):
        _room(grads[n], numel, n)
    if dlogits is not None:
        _room(dlogits, T * E, "dlogits")
    for t, n in ((h, "h"), (gamma, "gamma"), (Wg, "Wg"), (W1, "W1"), (W3, "W3"), (W2, "W2"), (dout, "dout")):
        _dev(t, h.dtype, n)
    _dev(grads["dh"], h.dtype, "dh")
    _dev(grads["dgamma"], torch.float32, "dgamma")
    _dev(grads["dWg"], torch.float32, "dWg")
    for n in ("dW1", "dW3", "dW2"):
        _dev(grads[n], grads["dW1"].dtype, n)
    wcode = _dtype_code(grads["dW1"])
    if dlogits is not None:
        _dev(dlogits, torch.float32, "dlogits")
    _dev(fwd_workspace, torch.uint8, "fwd_workspace")
    if workspace is None:
        workspace = torch.empty(max(moe_block_backward_workspace_size(T, d, F, E, k, code), 1), dtype=torch.uint8,
                                device=dev)
    _dev(workspace, torch.uint8, "workspace")
    n = ctypes.c_int(0)
    _check(_lib.moe_block_backward_ws(_ptr(h), _ptr(gamma), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dout),
                                      _ptr(grads["dh"]), _ptr(grads["dgamma"]), _ptr(grads["dWg"]),
                                      _ptr(grads["dW1"]), _ptr(grads["dW3"]), _ptr(grads["dW2"]), _ptr(dlogits),
                                      float(alpha), wcode, T, d, F, E, k, code, _ptr(fwd_workspace),
                                      fwd_workspace.numel(), _ptr(workspace), workspace.numel(),
                                      _events(events, MOE_BWD_NUM_STAGES), ctypes.byref(n),
                                      _stream(stream, h, gamma, Wg, W1, W3, W2, dout, fwd_workspace, workspace,
                                              dlogits, *grads.values())), "moe_block_backward_ws")
    return grads, n.value


def moe_ep_plan(counts_all, rank):
    """Expert-parallel dispatch plan of `rank` from every rank's expert counts (int array [R][E]):
    dict(send_counts, send_offsets, recv_counts, recv_offsets, experts (lo, hi), seg_counts, seg_offsets,
    block_recv [R][EL], block_seg [R][EL]) as numpy int32 arrays.  Host only: no device is touched."""
    import numpy as np
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    if c.ndim != 2:
        raise ValueError("counts_all must be [R][E]")
    R, E = c.shape
    a = {n: np.zeros(sz, dtype=np.int32) for n, sz in (("send_counts", R), ("send_offsets", R + 1),
                                                         ("recv_counts", R), ("recv_offsets", R + 1),
                                                         ("experts", 2), ("seg_counts", E), ("seg_offsets", E + 1),
                                                         ("block_recv", R * E), ("block_seg", R * E))}
    p = lambda n: ctypes.c_void_p(a[n].ctypes.data)
    _check(_lib.moe_ep_plan(ctypes.c_void_p(c.ctypes.data), R, E, int(rank), p("send_counts"), p("send_offsets"),
                            p("recv_counts"), p("recv_offsets"), p("experts"), p("seg_counts"), p("seg_offsets"),
                            p("block_recv"), p("block_seg")), "moe_ep_plan")
    EL = int(a["experts"][1] - a["experts"][0])
    a["seg_counts"] = a["seg_counts"][:EL]
    a["seg_offsets"] = a["seg_offsets"][:EL + 1]
    a["block_recv"] = a["block_recv"][:R * EL].reshape(R, EL)
    a["block_seg"] = a["block_seg"][:R * EL].reshape(R, EL)
    return a


def moe_ep_dispatch(x, topk_idx, E, send=None, send_pos=None, stream=None):
    """Route side of expert parallelism: (send [T*k][d] bf16 rows in send order, send_pos int32 [T][k],
    counts numpy int32 [E]).  Synchronises the stream (the counts come back to the host)."""
    import numpy as np
    T, k = topk_idx.shape
    if x.dim() != 2 or x.shape[0] != T:
        raise ValueError(f"x must be [T][d] with T = {T} rows (topk_idx), got {tuple(x.shape)}")
    d = x.shape[1]
    if send is None:
        send = torch.empty((T * k, d), dtype=x.dtype, device=x.device)
    if send_pos is None:
        send_pos = torch.empty((T, k), dtype=torch.int32, device=x.device)
    _room(send, T * k * d, "send")
    _room(send_pos, T * k, "send_pos")
    _dev(x, torch.bfloat16, "x")
    _dev(topk_idx, torch.int32, "topk_idx")
    _dev(send, torch.bfloat16, "send")
    _dev(send_pos, torch.int32, "send_pos")
    counts = np.zeros(E, dtype=np.int32)
    _check(_lib.moe_ep_dispatch(_ptr(x), _ptr(topk_idx), T, d, E, k, _ptr(send), _ptr(send_pos),
                                ctypes.c_void_p(counts.ctypes.data), _stream(stream, x, topk_idx, send, send_pos)),
           "moe_ep_dispatch")
    return send, send_pos, counts


def moe_ep_experts(recv, counts_all, rank, W1, W3, W2, yrecv=None, stream=None):
    """Expert side: the received rows (receive order of moe_ep_plan) through this rank's experts
    (W1, W3 [EL][F][d], W2 [EL][d][F]); returns yrecv float32 [rows][d] in the receive order."""
    import numpy as np
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    R, E = c.shape
    EL, F, d = W1.shape
    plan = moe_ep_plan(c, rank)
    rows = int(plan["recv_offsets"][-1])
    if recv.shape[0] < rows or recv.shape[1] != d:
        raise ValueError(f"recv must hold {rows} rows of {d}")
    if int(plan["experts"][1] - plan["experts"][0]) != EL or W3.shape != W1.shape or W2.shape != (EL, d, F):
        raise ValueError("W1, W3, W2 must hold exactly this rank's experts")
    if yrecv is None:
        yrecv = torch.empty((rows, d), dtype=torch.float32, device=recv.device)
    _room(yrecv, rows * d, "yrecv")
    for t, n in ((recv, "recv"), (W1, "W1"), (W3, "W3"), (W2, "W2")):
        _dev(t, torch.bfloat16, n)
    _dev(yrecv, torch.float32, "yrecv")
    _check(_lib.moe_ep_experts(_ptr(recv), ctypes.c_void_p(c.ctypes.data), R, E, int(rank), _ptr(W1), _ptr(W3),
                               _ptr(W2), d, F, _ptr(yrecv), _stream(stream, recv, W1, W3, W2, yrecv)),
           "moe_ep_experts")
    return yrecv


def moe_ep_combine(ysend, topk_w, send_pos, out=None, stream=None):
    """Route side, after the return all-to-all: out[t] = sum_j topk_w[t][j] ysend[send_pos[t][j]] (bf16)."""
    T, k = send_pos.shape
    d = ysend.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=ysend.device)
    _room(out, T * d, "out")
    _room(ysend, T * k * d, "ysend")
    _room(topk_w, T * k, "topk_w")
    _dev(ysend, torch.float32, "ysend")
    _dev(topk_w, torch.float32, "topk_w")
    _dev(send_pos, torch.int32, "send_pos")
    _dev(out, torch.bfloat16, "out")
    _check(_lib.moe_ep_combine(_ptr(ysend), _ptr(topk_w), _ptr(send_pos), T, d, k, _ptr(out),
                               _stream(stream, ysend, topk_w, send_pos, out)), "moe_ep_combine")
    return out


def moe_get_device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the device fault word (MOE_OK if none)."""
    return int(_lib.moe_get_device_status(_stream(stream)))


def moe_selftest_wait_timeout(limit_ns: int, stream=None):
    _check(_lib.moe_selftest_wait_timeout(int(limit_ns), _stream(stream)), "moe_selftest_wait_timeout")


def moe_pool_stats(device=None):
    """(reserved, used) bytes of the library's memory pool on `device` (default: torch's current device)."""
    if device is None:
        device = torch.cuda.current_device()
    elif isinstance(device, torch.device):
        device = device.index if device.index is not None else torch.cuda.current_device()
    r, u = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_lib.moe_pool_stats(int(device), ctypes.byref(r), ctypes.byref(u)), "moe_pool_stats")
    return r.value, u.value


def moe_decode_max_tokens() -> int:
    return int(_lib.moe_decode_max_tokens())


def moe_host_chunk_plan(T: int, max_chunks: int = 64) -> list:
    """Token boundaries [0, ..., T] of the chunks moe_forward_host runs a T-token batch in."""
    starts = (ctypes.c_int * (max_chunks + 1))()
    n = int(_lib.moe_host_chunk_plan(int(T), starts, int(max_chunks)))
    if n < 1:
        raise ValueError(f"no chunk plan for T={T} within {max_chunks} chunks")
    return list(starts[: n + 1])


def loaded_library_path() -> str:
    return LIB_PATH
