"""Expert-parallel data plane on one B200.

R ranks are emulated in one process: each rank's route, dispatch, expert and
combine calls run as they would on its own GPU, and the two all-to-alls are
device copies between the ranks' buffers in the plan's order (no kernel waits
on another).  Every rank's output must equal the single-GPU layer on its own
tokens bit for bit.  A one-rank NCCL group runs moe_forward_ep itself.
"""
import os
import socket

import numpy as np
import pytest
import torch

import moe_inputs
from moe_testlib import upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _emulate(moe, xs, Wg, W1, W3, W2, k, R):
    from sparse_mixture_experts_14_b200.ep import expert_range
    E = Wg.shape[0]
    d = xs[0].shape[1]
    routes = [moe.moe_route(x, Wg, k) for x in xs]
    disp = [moe.moe_ep_dispatch(x, idx, E) for x, (idx, _) in zip(xs, routes)]
    counts_all = np.stack([c for _, _, c in disp])
    plans = [moe.moe_ep_plan(counts_all, r) for r in range(R)]
    # rows: rank s receives, from each source r in order, r's run for s
    recvs = []
    for s in range(R):
        parts = [disp[r][0][plans[r]["send_offsets"][s]:plans[r]["send_offsets"][s + 1]] for r in range(R)]
        recvs.append(torch.cat(parts) if parts else torch.empty((0, d), dtype=torch.bfloat16, device="cuda"))
    yrecvs = []
    for s in range(R):
        lo, hi = expert_range(E, R, s)
        assert (lo, hi) == tuple(int(v) for v in plans[s]["experts"])
        if hi == lo or recvs[s].shape[0] == 0:
            yrecvs.append(torch.empty((0, d), dtype=torch.float32, device="cuda"))
            continue
        yrecvs.append(moe.moe_ep_experts(recvs[s], counts_all, s, W1[lo:hi].contiguous(), W3[lo:hi].contiguous(),
                                         W2[lo:hi].contiguous()))
    outs = []
    for r in range(R):
        T = xs[r].shape[0]
        parts = [yrecvs[s][plans[s]["recv_offsets"][r]:plans[s]["recv_offsets"][r + 1]] for s in range(R)]
        ysend = torch.zeros((T * k, d), dtype=torch.float32, device="cuda")
        back = torch.cat(parts)
        ysend[:back.shape[0]] = back
        outs.append(moe.moe_ep_combine(ysend, routes[r][1], disp[r][1]))
    return outs


@pytest.mark.parametrize("R,sizes,E,k", [(1, (333,), 8, 2), (2, (300, 217), 8, 2), (4, (200, 64, 1, 129), 8, 2),
                                         (3, (150, 90, 77), 16, 4)])
def test_emulated_ranks_equal_the_single_gpu_layer(moe, R, sizes, E, k):
    d, F = 256, 512
    full = moe_inputs.make_inputs(sum(sizes), d, F, E, k, "bf16", seed=R * 10 + E)
    dev = upload(full)
    x_all, Wg, W1, W3, W2 = dev
    xs, at = [], 0
    for n in sizes:
        xs.append(x_all[at:at + n].contiguous())
        at += n
    outs = _emulate(moe, xs, Wg, W1, W3, W2, k, R)
    assert moe.moe_get_device_status() == moe.MOE_OK
    for r, x in enumerate(xs):
        ref = moe.moe_forward_ws(x, Wg, W1, W3, W2, k, path=moe.MOE_PATH_PREFILL)
        assert torch.equal(outs[r], ref), f"rank {r}"


def test_dispatch_send_order(moe):
    """send rows are the token rows sorted by expert (stable in token order); send_pos inverts it."""
    T, d, E, k = 300, 128, 8, 2
    inp = moe_inputs.make_inputs(T, d, 256, E, k, "bf16", seed=5)
    x, Wg = upload(inp)[:2]
    idx, _ = moe.moe_route(x, Wg, k)
    send, pos, counts = moe.moe_ep_dispatch(x, idx, E)
    i = idx.cpu().numpy()
    assert np.array_equal(counts, np.bincount(i.ravel(), minlength=E))
    order = [t for e in range(E) for t in range(T) if e in i[t]]
    assert torch.equal(send[:len(order)], x[torch.tensor(order, device="cuda")])
    p = pos.cpu().numpy()
    for t in range(T):
        for j in range(k):
            assert order[p[t, j]] == t


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_forward_ep_one_rank_nccl(moe):
    import torch.distributed as dist
    from datetime import timedelta
    from sparse_mixture_experts_14_b200.ep import moe_forward_ep
    inp = moe_inputs.make_inputs(500, 256, 512, 8, 2, "bf16", seed=9)
    x, Wg, W1, W3, W2 = upload(inp)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True, timeout=timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        out = moe_forward_ep(x, Wg, W1, W3, W2, 2)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = moe.moe_forward_ws(x, Wg, W1, W3, W2, 2, path=moe.MOE_PATH_PREFILL)
    assert torch.equal(out, ref)
