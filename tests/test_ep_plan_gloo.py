"""The expert-parallel dispatch plan (moe_ep_plan, host code) on CPU.

Pure invariants for several rank and expert counts, then the plan driven by
real ranks: gloo, world size 2, each rank routing its own batch, the counts
exchanged with all_gather and the rows (global token ids) with all_to_all.
Every rank's expert segments, built from the rows it received and the plan's
block offsets, must equal bit for bit the single-GPU dispatch's segments of
the concatenated batch (tokens numbered rank-major): the same rows in the same
stable order, padded to 128 rows.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SEG = 128


def _routing(T, E, k, seed):
    """Seeded top-k choices (k distinct experts per token), skewed toward low expert ids."""
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _segments(idx, E, experts):
    """The single-GPU dispatch's segments of the listed experts: the tokens that chose each expert in
    increasing order, padded with -1 to a multiple of 128 rows."""
    out = []
    for e in experts:
        rows = np.nonzero((idx == e).any(axis=1))[0]
        pad = (len(rows) + SEG - 1) // SEG * SEG - len(rows)
        out.append(np.concatenate([rows, np.full(pad, -1)]).astype(np.int64))
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


def _send_rows(idx, E, token_base):
    """A rank's send order: its assignments sorted by expert, stable in token order (global token ids)."""
    return np.concatenate([np.nonzero((idx == e).any(axis=1))[0] + token_base for e in range(E)]).astype(np.int64)


@pytest.mark.parametrize("R,E", [(1, 8), (2, 8), (3, 8), (4, 32), (3, 1), (5, 3)])
def test_plan_invariants(R, E):
    import sparse_mixture_experts_14_b200 as m
    rng = np.random.default_rng(R * 100 + E)
    counts = rng.integers(0, 300, size=(R, E)).astype(np.int32)
    plans = [m.moe_ep_plan(counts, r) for r in range(R)]
    owned = np.concatenate([np.arange(p["experts"][0], p["experts"][1]) for p in plans])
    assert np.array_equal(owned, np.arange(E))                 # contiguous groups cover every expert once
    for r, p in enumerate(plans):
        assert p["send_offsets"][-1] == counts[r].sum()
        for s in range(R):
            assert p["send_counts"][s] == plans[s]["recv_counts"][r]
        lo, hi = p["experts"]
        EL = hi - lo
        assert np.array_equal(p["seg_counts"], counts[:, lo:hi].sum(axis=0))
        assert np.array_equal(np.diff(p["seg_offsets"]), (p["seg_counts"] + SEG - 1) // SEG * SEG)
        # blocks tile the receive buffer in order and fill each segment's rows exactly
        recv = np.zeros(p["recv_offsets"][-1], dtype=np.int32)
        segs = np.zeros(p["seg_offsets"][-1] if EL else 0, dtype=np.int32)
        for s in range(R):
            for l in range(EL):
                n = counts[s, lo + l]
                recv[p["block_recv"][s, l]:p["block_recv"][s, l] + n] += 1
                segs[p["block_seg"][s, l]:p["block_seg"][s, l] + n] += 1
        assert np.all(recv == 1)
        for l in range(EL):
            a, n = p["seg_offsets"][l], p["seg_counts"][l]
            assert np.all(segs[a:a + n] == 1) and np.all(segs[a + n:p["seg_offsets"][l + 1]] == 0)


def test_plan_argument_checks():
    import sparse_mixture_experts_14_b200 as m
    with pytest.raises(m.MoEError):
        m.moe_ep_plan(np.zeros((2, 8), dtype=np.int32), 2)     # rank outside [0, R)
    with pytest.raises(m.MoEError):
        m.moe_ep_plan(-np.ones((2, 8), dtype=np.int32), 0)     # negative count
    with pytest.raises(m.MoEError):
        m.moe_ep_plan(np.zeros((2, 33), dtype=np.int32), 0)    # more experts than supported


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, sizes, E, k, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    import sparse_mixture_experts_14_b200 as m
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        idx = _routing(sizes[rank], E, k, seed=1000 + rank)
        counts = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
        gathered = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(counts))
        counts_all = torch.stack(gathered).numpy()
        plan = m.moe_ep_plan(counts_all, rank)
        send = torch.from_numpy(_send_rows(idx, E, token_base=sum(sizes[:rank])))
        assert send.numel() == plan["send_offsets"][-1]
        recv = torch.empty(int(plan["recv_offsets"][-1]), dtype=torch.int64)
        dist.all_to_all_single(recv, send, output_split_sizes=plan["recv_counts"].tolist(),
                               input_split_sizes=plan["send_counts"].tolist())
        lo, hi = (int(v) for v in plan["experts"])
        segs = np.full(int(plan["seg_offsets"][-1]), -1, dtype=np.int64)
        rv = recv.numpy()
        for s in range(world):
            for l in range(hi - lo):
                n = counts_all[s, lo + l]
                a, b = plan["block_recv"][s, l], plan["block_seg"][s, l]
                segs[b:b + n] = rv[a:a + n]
        q.put((rank, lo, hi, segs))
    finally:
        dist.destroy_process_group()


def test_plan_drives_two_gloo_ranks_to_the_single_gpu_segments():
    world, E, k, sizes = 2, 8, 2, (300, 217)
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, sizes, E, k, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    full = np.concatenate([_routing(sizes[r], E, k, seed=1000 + r) for r in range(world)])
    for rank, lo, hi, segs in res:
        assert np.array_equal(segs, _segments(full, E, range(lo, hi))), rank
