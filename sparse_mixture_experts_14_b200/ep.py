"""Expert-parallel forward of the MoE layer over a torch.distributed process group.

Experts are split into R contiguous groups (rank s holds the weights of
experts [s E / R, (s+1) E / R) only); every rank routes its own tokens with
the full router Wg.  One forward is:

  route (moe_route) -> dispatch (moe_ep_dispatch: rows in send order, counts)
  -> all_gather of the counts -> plan (moe_ep_plan)
  -> all_to_all of the rows -> experts (moe_ep_experts: this rank's experts)
  -> all_to_all of the outputs back -> combine (moe_ep_combine)

The all-to-alls are torch.distributed's (NCCL between GPUs); every step in
between runs in the library's kernels.  Each rank's output equals the
single-GPU layer's on its tokens bit for bit: each expert segment holds the
rows the single-GPU dispatch of the concatenated batch would give it, and
every row's arithmetic is the same wherever it sits in a tile.
"""
from __future__ import annotations

import numpy as np
import torch

from . import moe_ep_combine, moe_ep_dispatch, moe_ep_experts, moe_ep_plan, moe_route


def expert_range(E: int, R: int, rank: int):
    """The experts [lo, hi) rank `rank` of R holds."""
    return rank * E // R, (rank + 1) * E // R


def moe_forward_ep(x, Wg, W1_local, W3_local, W2_local, k: int, group=None):
    """out [T][d] bf16 for this rank's tokens x [T][d]; Wg [E][d] is the full router, W1_local /
    W3_local [EL][F][d] and W2_local [EL][d][F] this rank's experts (expert_range)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    E = Wg.shape[0]
    T, d = x.shape
    idx, w = moe_route(x, Wg, k)
    send, send_pos, counts = moe_ep_dispatch(x, idx, E)
    mine = torch.from_numpy(counts).to(x.device)
    gathered = [torch.empty_like(mine) for _ in range(R)]
    dist.all_gather(gathered, mine, group=group)
    counts_all = torch.stack(gathered).cpu().numpy()
    plan = moe_ep_plan(counts_all, rank)
    recv = torch.empty((int(plan["recv_offsets"][-1]), d), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send[:int(plan["send_offsets"][-1])],
                           output_split_sizes=plan["recv_counts"].tolist(),
                           input_split_sizes=plan["send_counts"].tolist(), group=group)
    yrecv = moe_ep_experts(recv, counts_all, rank, W1_local, W3_local, W2_local)
    ysend = torch.empty((T * k, d), dtype=torch.float32, device=x.device)
    dist.all_to_all_single(ysend[:int(plan["send_offsets"][-1])], yrecv,
                           output_split_sizes=plan["send_counts"].tolist(),
                           input_split_sizes=plan["recv_counts"].tolist(), group=group)
    return moe_ep_combine(ysend, w, send_pos)
