"""The C-ABI library without a GPU: it loads, exports every declared symbol, and
rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    path = __graft_entry__._builder().build()
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for must in ("moe_route", "moe_forward", "moe_forward_f32", "moe_dispatch", "moe_forward_ws",
                 "moe_forward_host", "moe_get_device_status", "moe_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in moe.h but not exported"


def test_binding_signatures_cover_header():
    import sparse_mixture_experts_14_b200 as m
    assert set(declared_symbols()) == set(m.SIGNATURES)


def _vp(v=0x1000):
    return ctypes.c_void_p(v)


def _fwd(lib, T=8, d=128, F=256, E=8, k=2, x=0x1000, out=0x2000, f32=False):
    fn = lib.moe_forward_f32 if f32 else lib.moe_forward
    fn.restype = ctypes.c_int
    return fn(_vp(x), _vp(), _vp(), _vp(), _vp(), _vp(out), T, d, F, E, k, ctypes.c_void_p(0))


def test_forward_argument_checks(lib):
    assert _fwd(lib, k=9) == 1                 # k > E
    assert _fwd(lib, k=0) == 1
    assert _fwd(lib, T=-1) == 1
    assert _fwd(lib, E=33, k=2) == 2           # more experts than supported
    assert _fwd(lib, d=100) == 2               # bf16 path wants d % 64 == 0
    assert _fwd(lib, F=200) == 2               # and F % 128 == 0
    assert _fwd(lib, d=102, f32=True) == 2     # fp32 path wants d % 4 == 0
    assert _fwd(lib, x=0) == 1                 # null pointer
    assert _fwd(lib, x=0x1008) == 1            # not 16-byte aligned
    assert _fwd(lib, T=0, x=0, out=0) == 0     # empty batch: no-op


def test_route_argument_checks(lib):
    f = lib.moe_route
    f.restype = ctypes.c_int
    assert f(_vp(), _vp(), 4, 128, 8, 9, _vp(), _vp(), None) == 1
    assert f(_vp(), _vp(), 4, 100, 8, 2, _vp(), _vp(), None) == 2
    assert f(None, _vp(), 4, 128, 8, 2, _vp(), _vp(), None) == 1
    assert f(_vp(), _vp(), 0, 128, 8, 2, _vp(), _vp(), None) == 0


def test_workspace_and_slots(lib):
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_slots_capacity.restype = ctypes.c_size_t
    assert lib.moe_slots_capacity(16, 8, 2) == 32 + 8 * 127 + (128 - (32 + 8 * 127) % 128) % 128
    assert lib.moe_slots_capacity(16, 8, 2) % 128 == 0
    assert lib.moe_slots_capacity(4, 2, 3) == 0              # k > E
    ws = lib.moe_workspace_size(4096, 4096, 14336, 8, 2, 1)
    slots = lib.moe_slots_capacity(4096, 8, 2)
    assert ws >= slots * (4096 * 2 + 14336 * 2 + 4096 * 4)
    assert lib.moe_workspace_size(4096, 4096, 14336, 8, 2, 7) == 0


def test_forward_ws_checks(lib):
    f = lib.moe_forward_ws
    f.restype = ctypes.c_int
    args = [_vp(), _vp(), _vp(), _vp(), _vp(), _vp(), 8, 128, 256, 8, 2]
    assert f(*args, 1, 5, _vp(0x10000), ctypes.c_size_t(1 << 30), None) == 1    # unknown path
    assert f(*args, 0, 2, _vp(0x10000), ctypes.c_size_t(1 << 30), None) == 2    # decode path is bf16 only
    assert f(*args, 1, 0, None, ctypes.c_size_t(1 << 30), None) == 5            # no workspace
    assert f(*args, 1, 0, _vp(0x10000), ctypes.c_size_t(16), None) == 5         # too small


def test_status_strings(lib):
    lib.moe_status_string.restype = ctypes.c_char_p
    for code in range(7):
        assert lib.moe_status_string(code)
    assert lib.moe_status_string(4) == b"device wait timed out"


def test_selftest_rejects_bad_limit(lib):
    f = lib.moe_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_longlong, ctypes.c_void_p]
    assert f(10, None) == 1
    assert f(10 ** 12, None) == 1


def _block(lib, T=8, d=128, F=256, E=8, k=2, h=0x1000, gamma=0x3000, out=0x100000, eps=1e-5, alpha=1.0,
           stats=0x5000, f32=False):
    fn = lib.moe_block_forward_f32 if f32 else lib.moe_block_forward
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float] + [ctypes.c_void_p] * 5 + \
        [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    return fn(_vp(h), _vp(gamma) if gamma else None, eps, _vp(), _vp(), _vp(), _vp(), _vp(out), T, d, F, E, k,
              alpha, _vp(stats) if stats else None, None)


def test_block_argument_checks(lib):
    assert _block(lib, k=9) == 1                      # k > E
    assert _block(lib, d=100) == 2                    # bf16 needs d % 64 == 0
    assert _block(lib, gamma=0) == 1                  # no gain
    assert _block(lib, gamma=0x3004) == 1             # misaligned gain
    assert _block(lib, eps=-1e-5) == 1                # negative eps
    assert _block(lib, eps=float("inf")) == 1
    assert _block(lib, eps=float("nan")) == 1
    assert _block(lib, alpha=float("nan")) == 1
    assert _block(lib, alpha=float("inf")) == 1
    assert _block(lib, stats=0x5002) == 1             # misaligned stats
    assert _block(lib, out=0x1000 + 256) == 1         # out overlaps h partly (rows are 256 bytes)
    assert _block(lib, T=0, h=0, gamma=0, out=0) == 0  # empty batch: no-op
    assert _block(lib, d=102, f32=True) == 2          # fp32 needs d % 4 == 0


def test_block_workspace_size(lib):
    lib.moe_block_workspace_size.restype = ctypes.c_size_t
    lib.moe_workspace_size.restype = ctypes.c_size_t
    plain = lib.moe_workspace_size(4096, 4096, 14336, 8, 2, 1)
    blk = lib.moe_block_workspace_size(4096, 4096, 14336, 8, 2, 1)
    assert blk >= plain + 4096 * 4 + 4096 * 8 * 4     # row factors and fp32 scores on top
    assert lib.moe_block_workspace_size(4096, 4096, 14336, 8, 2, 7) == 0


def test_route_stats_argument_checks(lib):
    f = lib.moe_route_stats
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 4
    assert f(_vp(), _vp(), 4, 128, 8, 9, 1.0, _vp(), _vp(), _vp(), None) == 1
    assert f(_vp(), _vp(), 4, 128, 8, 2, 1.0, _vp(), _vp(), None, None) == 1   # stats required
    assert f(_vp(), _vp(), 4, 128, 8, 2, float("nan"), _vp(), _vp(), _vp(), None) == 1
    assert f(_vp(), _vp(), 0, 128, 8, 2, 1.0, None, None, None, None) == 0


def test_training_workspace_sizes(lib):
    for name in ("moe_workspace_size", "moe_train_workspace_size", "moe_backward_workspace_size"):
        getattr(lib, name).restype = ctypes.c_size_t
    T, d, F, E, k = 4096, 4096, 14336, 8, 2
    plain = lib.moe_workspace_size(T, d, F, E, k, 1)
    train = lib.moe_train_workspace_size(T, d, F, E, k, 1)
    S = (T * k + E * 127 + 127) // 128 * 128               # expert-segment rows
    assert train >= plain + 2 * S * F * 4 + T * E * 4   # the kept a, b (fp32) and the scores on top
    bwd = lib.moe_backward_workspace_size(T, d, F, E, k, 1)
    assert bwd >= S * 2 * F * 2 + S * d * 4              # dA | dB (bf16) and dXp (fp32)
    assert lib.moe_train_workspace_size(T, d, F, E, k, 7) == 0
    assert lib.moe_backward_workspace_size(T, d, F, E, 9, 1) == 0   # k > E


def _bwd(lib, T=8, d=128, F=256, E=8, k=2, dtype=1, wgrad=0, alpha=0.0, dout=0x7000, dW1=0x8000, dlogits=None,
         fws=0x10000, fws_bytes=None, ws=0x20000, ws_bytes=None):
    for name in ("moe_train_workspace_size", "moe_backward_workspace_size"):
        getattr(lib, name).restype = ctypes.c_size_t
    if fws_bytes is None:
        fws_bytes = lib.moe_train_workspace_size(max(T, 1), d, F, E, min(k, E), dtype)
    if ws_bytes is None:
        ws_bytes = lib.moe_backward_workspace_size(max(T, 1), d, F, E, min(k, E), dtype)
    fn = lib.moe_backward_ws
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 12 + [ctypes.c_float] + [ctypes.c_int] * 7 + \
        [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t] + [ctypes.c_void_p] * 3
    return fn(_vp(0x1000), _vp(0x2000), _vp(0x3000), _vp(0x4000), _vp(0x5000), _vp(dout) if dout else None,
              _vp(0x6000), _vp(0x9000), _vp(dW1) if dW1 else None, _vp(0xa000), _vp(0xb000),
              _vp(dlogits) if dlogits else None, alpha, wgrad, T, d, F, E, k, dtype,
              _vp(fws) if fws else None, fws_bytes, _vp(ws) if ws else None, ws_bytes, None, None, None)


def test_backward_argument_checks(lib):
    """Every check here returns before the library touches CUDA."""
    assert _bwd(lib, k=9) == 1                          # k > E
    assert _bwd(lib, d=100) == 2                        # bf16 needs d % 64 == 0
    assert _bwd(lib, dout=0) == 1                       # upstream gradient required
    assert _bwd(lib, dW1=0x8008) == 1                   # misaligned gradient buffer
    assert _bwd(lib, dlogits=0x9002) == 1               # misaligned score gradient
    assert _bwd(lib, alpha=float("nan")) == 1
    assert _bwd(lib, alpha=float("inf")) == 1
    assert _bwd(lib, wgrad=5) == 1                      # unknown weight-gradient type
    assert _bwd(lib, dtype=0, d=128, wgrad=1) == 2      # bf16 weight gradients of an fp32 layer
    assert _bwd(lib, fws=0) == 5                        # no forward workspace
    assert _bwd(lib, fws=0x10040) == 5                  # not 256-byte aligned
    assert _bwd(lib, fws_bytes=1024) == 5               # an inference-sized workspace cannot hold a, b
    assert _bwd(lib, ws=0) == 5
    assert _bwd(lib, ws_bytes=1024) == 5
    assert _bwd(lib, T=0) == 0                          # empty batch: no-op


def _noalloc_outputs(T, E, k, m, short=None):
    """CPU int32 tensors sized as moe_dispatch_noalloc needs them, one of them a single element short."""
    need = {"counts": E, "offsets": E + 1, "perm": m.moe_slots_capacity(T, E, k), "inv": T * k}
    return [torch.zeros(need[n] - (1 if n == short else 0), dtype=torch.int32)
            for n in ("counts", "offsets", "perm", "inv")]


def test_noalloc_binding_rejects_undersized_outputs():
    """The wrapper checks the room in every caller buffer before anything reaches the library: a
    buffer one element short raises ValueError; buffers of the right size pass the size checks and
    only then meet the device check (CPU tensors here)."""
    import sparse_mixture_experts_14_b200 as m
    T, E, k = 3000, 8, 2
    idx = torch.zeros((T, k), dtype=torch.int32)
    for short in ("counts", "offsets", "perm", "inv"):
        with pytest.raises(ValueError, match=short):
            m.moe_dispatch_noalloc(idx, E, *_noalloc_outputs(T, E, k, m, short))
    with pytest.raises(ValueError, match="2-D"):
        m.moe_dispatch_noalloc(idx.reshape(-1), E, *_noalloc_outputs(T, E, k, m))
    with pytest.raises(TypeError, match="CUDA"):
        m.moe_dispatch_noalloc(idx, E, *_noalloc_outputs(T, E, k, m))


def test_binding_rejects_undersized_layer_outputs():
    import sparse_mixture_experts_14_b200 as m
    T, d, F, E, k = 8, 64, 128, 4, 2
    bf = torch.bfloat16
    x, Wg = torch.zeros((T, d), dtype=bf), torch.zeros((E, d), dtype=bf)
    W1, W3, W2 = torch.zeros((E, F, d), dtype=bf), torch.zeros((E, F, d), dtype=bf), torch.zeros((E, d, F), dtype=bf)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="out"):
        m.moe_forward_profiled(x, Wg, W1, W3, W2, k, ws, torch.zeros(T * d - 1, dtype=bf))
    with pytest.raises(ValueError, match="out_host"):
        m.moe_forward_host(x, Wg, W1, W3, W2, k, out_host=torch.zeros(T * d - 1, dtype=bf))


def test_binding_rejects_inconsistent_shapes():
    """The sizes the kernels trust come from the tensors' shapes: the wrappers refuse shapes that do
    not fit together (ValueError, CPU tensors, nothing reaches the library)."""
    import sparse_mixture_experts_14_b200 as m
    T, d, F, E, k = 8, 64, 128, 4, 2
    bf = torch.bfloat16
    x, Wg = torch.zeros((T, d), dtype=bf), torch.zeros((E, d), dtype=bf)
    W1, W3, W2 = torch.zeros((E, F, d), dtype=bf), torch.zeros((E, F, d), dtype=bf), torch.zeros((E, d, F), dtype=bf)
    short_Wg = torch.zeros((E, d // 2), dtype=bf)
    for route in (m.moe_route, m.moe_route_stats):
        with pytest.raises(ValueError, match="inconsistent"):
            route(x, short_Wg, k)
        with pytest.raises(ValueError, match="inconsistent"):
            route(x.reshape(-1), Wg, k)
    for bad in ((short_Wg, W1, W3, W2), (Wg, W1[:, :, : d // 2], W3, W2), (Wg, W1, W3[:, : F // 2], W2),
                (Wg, W1, W3, W2.transpose(1, 2).contiguous())):
        with pytest.raises(ValueError, match="inconsistent"):
            m.moe_forward_host(x, *bad, k)
    with pytest.raises(ValueError, match="rows"):
        m.moe_ep_dispatch(x[: T - 1], torch.zeros((T, k), dtype=torch.int32), E)
    with pytest.raises(ValueError, match="topk_w"):
        m.moe_ep_combine(torch.zeros((T * k, d)), torch.zeros((T, k - 1)), torch.zeros((T, k), dtype=torch.int32))


def test_pool_stats_argument_checks(lib):
    fn = lib.moe_pool_stats
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    r, u = ctypes.c_size_t(7), ctypes.c_size_t(7)
    assert fn(0, None, ctypes.byref(u)) == 1
    assert fn(-1, ctypes.byref(r), ctypes.byref(u)) == 1
    assert fn(64, ctypes.byref(r), ctypes.byref(u)) == 1
    assert fn(0, ctypes.byref(r), ctypes.byref(u)) == 0     # no pool created in this process: zeros
    assert (r.value, u.value) == (0, 0)


def test_host_chunk_plan(lib):
    """The host entry point's chunk plan: runs of consecutive tokens covering [0, T), each split
    batch's chunks large enough for the prefill kernels, short first and last chunks around
    near-equal middle ones."""
    import numpy as np
    import sparse_mixture_experts_14_b200 as m
    plan = m.moe_host_chunk_plan
    assert plan(0) == [0, 0]
    assert plan(4095) == [0, 4095]
    assert plan(4096) == [0, 2048, 4096]
    assert plan(8191) == [0, 4095, 8191]
    assert plan(8192) == [0, 1024, 7168, 8192]
    assert plan(12287) == [0, 1024, 6144, 11263, 12287]
    assert plan(12288) == [0, 2560, 9728, 12288]
    assert plan(16384) == [0, 2560, 13824, 16384]
    decode_max = m.moe_decode_max_tokens()
    for T in [4096, 4097, 6143, 8191, 8192, 8193, 10001, 12287, 12288, 16385, 30000, 100_000, 1 << 20,
              2_000_000]:
        s = plan(T)
        sizes = np.diff(s)
        assert s[0] == 0 and s[-1] == T and len(s) - 1 <= 64
        assert sizes.min() >= 1024 and sizes.min() > decode_max
        if T < 8192:
            assert len(sizes) == 2 and abs(int(sizes[0]) - int(sizes[1])) <= 1
        else:
            edge, mid_max = (1024, 7168) if T < 12288 else (2560, 11264)
            assert sizes[0] == edge and sizes[-1] == edge
            mids = sizes[1:-1]
            assert mids.max() - mids.min() <= 1
            if len(sizes) < 64:
                assert mids.max() <= mid_max
    buf = (ctypes.c_int * 65)()
    lib.moe_host_chunk_plan.restype = ctypes.c_int
    assert lib.moe_host_chunk_plan(-1, buf, 64) == 0
    assert lib.moe_host_chunk_plan(16384, None, 64) == 0
    assert lib.moe_host_chunk_plan(8192, buf, 2) == 0           # three chunks do not fit in two
    assert lib.moe_host_chunk_plan(8192, buf, 3) == 3
    assert list(buf[:4]) == [0, 1024, 7168, 8192]


def test_header_serves_a_plain_c_program(lib, tmp_path):
    """include/moe.h compiles as C99 with warnings as errors, and a C program links libmoe.so and
    calls its host-only entry points (no device is touched)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda_inc = next((p for p in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include"))
                     if os.path.exists(os.path.join(p, "cuda_runtime_api.h"))), None)
    if cuda_inc is None:
        pytest.skip("no CUDA headers")
    src = tmp_path / "client.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
    int s[65];
    if (moe_host_chunk_plan(16384, s, 64) != 3 || s[1] != 2560 || s[3] != 16384) return 1;
    if (moe_slots_capacity(16, 8, 2) % 128 != 0) return 2;
    if (strcmp(moe_status_string(MOE_ERR_TIMEOUT), "device wait timed out") != 0) return 3;
    if (moe_forward(NULL, NULL, NULL, NULL, NULL, NULL, 8, 128, 256, 8, 9, 0) != MOE_ERR_INVALID_ARG) return 4;
    printf("ok\n");
    return 0;
}
''')
    libdir = os.path.dirname(lib._name)
    exe = tmp_path / "client"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                    str(src), "-L", libdir, "-lmoe", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
