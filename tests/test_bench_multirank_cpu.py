"""The multi-rank plumbing of bench.py on CPU: gloo, world size 2, no GPU.

The layer shards by tokens with no exchange (replicas), so the only
cross-rank steps are the barrier and the max-over-ranks of the timings.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        m = bench.reduce_max(ms, world)
        v = bench.weak_scaling_value(16, 100, world, m)
        torch.distributed.barrier()
        q.put((rank, m, v))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in res:
        assert m == 15.0                             # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 16 * 100 / 0.015)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.weak_scaling_value(16, 10, 1, 100.0) == pytest.approx(1600.0)


def test_reference_arm_under_torchrun_two_ranks():
    """Rank 0 prints one JSON line for the reference arm; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1", "--gpus", "2",
           "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("mode", ["--block", "--train"])
def test_reference_arm_block_and_train(mode):
    """The oracle arm of the block form and of the training step (tiny fp32 workload, short budget)."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1", mode,
           "--steps", "2", "--warmup", "1", "--ref-seconds", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"]["workload"].endswith("+block" if mode == "--block" else "+train")


def test_reference_arm_json_contract():
    """The one JSON line carries every key of the bench contract, with the reference arm's own
    cpu_baseline and a zero-transfer e2e in the line's metric and unit."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
           "--steps", "3", "--warmup", "3", "--ref-seconds", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert "workload" in d["config"] and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_seed_option_changes_the_inputs_and_tags_the_workload():
    """--seed runs a workload's recipe with another seed; the workload name carries it, so a
    traffic figure recorded for the standard seed is never looked up for it."""
    sys.path.insert(0, ROOT)
    import bench
    a = bench.make_workload(1, False)
    b = bench.make_workload(1, False, seed=7)
    assert b.seed == 7 and a.seed != 7
    assert (a.T, a.d, a.F, a.E, a.k) == (b.T, b.d, b.F, b.E, b.k)
    assert not (a.x == b.x).all()
    assert bench.workload_name(1) != bench.workload_name(1, seed=7)
    assert bench.workload_name(3, "4096,4096,4096", 5).endswith("@shape=4096,4096,4096@seed=5")


@pytest.mark.parametrize("extra", [["--train"], ["--block"], ["--impl", "reference"]])
def test_ep_mode_refuses_other_modes(extra):
    """--ep times the plain layer's forward on the library's kernels only."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--ep"] + extra
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0 and "--ep" in r.stderr
