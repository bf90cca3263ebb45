"""moe_dispatch_noalloc: the dispatch for callers that may not allocate device memory.

It must give exactly what moe_dispatch gives (integer outputs: bit for bit),
on two calls in a row that leave different contents in the shared fixed
scratch array, and refuse sizes past that array's limit.  It must leave the
library's memory pool exactly as it found it, and an empty batch (T = 0) must
give all-zero counts and offsets even after an earlier call left data in the
array.  This file is collected last so a stop-at-first-failure run has
already run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_14_b200 as m
    return m


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    return torch.from_numpy(idx).cuda()


def _outputs(T, E, k, moe):
    dev = "cuda"
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((max(moe.moe_slots_capacity(T, E, k), 1),), -7, dtype=torch.int32, device=dev),
            torch.full((T, k), -7, dtype=torch.int32, device=dev))


def _compare(moe, T, E, k, seed):
    idx = _routing(T, E, k, seed)
    ref = moe.moe_dispatch(idx, E)
    got = moe.moe_dispatch_noalloc(idx, E, *_outputs(T, E, k, moe))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    counts, offsets, perm, inv = (a.cpu() for a in got)
    r_counts, r_offsets, r_perm, r_inv = (a.cpu() for a in ref)
    assert torch.equal(counts, r_counts)
    assert torch.equal(offsets, r_offsets)
    n = int(offsets[-1])
    assert torch.equal(perm[:n], r_perm[:n])       # rows past offsets[E] are left untouched by both
    assert torch.equal(inv, r_inv)


@pytest.mark.parametrize("shape", [(3000, 8, 2), (700, 8, 2), (5000, 32, 4), (1, 4, 1)])
def test_noalloc_matches_pooled_twice_in_a_row(moe, shape):
    T, E, k = shape
    _compare(moe, T, E, k, seed=T)          # first call
    _compare(moe, T, E, k, seed=T + 1)      # second call finds the first one's contents in the array


def test_noalloc_alternating_sizes(moe):
    _compare(moe, 9000, 8, 2, seed=1)       # multi-block path fills much of the histogram
    _compare(moe, 50, 6, 3, seed=2)         # single-block path afterwards


def test_noalloc_refuses_past_its_limit(moe):
    T, E, k = 126977, 32, 2                 # ceil(T/1024) * E = 4000 > 3968
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    idx[:, 1] = 1
    outs = _outputs(T, E, k, moe)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch_noalloc(idx, E, *outs)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert int(outs[0][0]) == -7            # nothing launched
    _compare(moe, 126976, 32, 2, seed=5)    # the largest accepted size still matches


def test_noalloc_empty_batch_after_a_full_one(moe):
    _compare(moe, 3000, 8, 2, seed=11)      # leaves counts and offsets of 6000 assignments in the array
    E, k = 8, 2
    idx = torch.empty((0, k), dtype=torch.int32, device="cuda")
    counts, offsets, perm, inv = _outputs(0, E, k, moe)
    moe.moe_dispatch_noalloc(idx, E, counts, offsets, perm, inv)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert torch.equal(counts.cpu(), torch.zeros(E, dtype=torch.int32))
    assert torch.equal(offsets.cpu(), torch.zeros(E + 1, dtype=torch.int32))


def test_noalloc_leaves_the_pool_untouched(moe):
    T, E, k = 9000, 8, 2
    idx = _routing(T, E, k, seed=3)
    outs = _outputs(T, E, k, moe)
    moe.moe_dispatch(idx, E)                # the pooled call may create or grow the pool
    moe.moe_dispatch_noalloc(idx, E, *outs)  # a first call loads the array's module (lazy loading)
    torch.cuda.synchronize()
    pool_before = moe.moe_pool_stats()
    torch_before = torch.cuda.memory_reserved()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        moe.moe_dispatch_noalloc(idx, E, *outs)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK
    assert moe.moe_pool_stats() == pool_before
    assert torch.cuda.memory_reserved() == torch_before
    assert torch.cuda.mem_get_info()[0] == free_before
