"""The N > 1 path on the CPU: world-size-2 gloo process groups.

bench.py runs one rank per GPU with no data-path collective (every rank owns an
independent layer, or with --shard heads a disjoint run of the layer's KV
heads); the only cross-rank steps are the barrier and the max-over-ranks
reduction of the timed region. These tests run that reduction, the head-shard
assignment and the reference arm's rank handling with two gloo ranks.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, dist)      # each rank's own timed-region ms
    dist.barrier()
    value = bench.weak_scaling_value(1.0e12, world, slowest)
    queue.put((rank, slowest, value))
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [15.0, 15.0]            # every rank sees the slowest rank's time
    for _, _, value in results:
        assert abs(value - 2 * 1.0e12 / 15e-3 / 1e12) < 1e-9     # both ranks' FLOPs over the slowest time


def _shard_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    begin, count = bench.head_shard(rank, world, 8)
    mine = torch.tensor([begin, count])
    every = [torch.zeros(2, dtype=mine.dtype) for _ in range(world)]
    dist.all_gather(every, mine)
    queue.put((rank, [tuple(t.tolist()) for t in every]))
    dist.destroy_process_group()


def test_head_shards_cover_the_kv_heads_once_with_two_gloo_ranks():
    """--shard heads: each rank takes a disjoint run of KV heads; together all of them."""
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, shards in results:
        assert shards == [(0, 4), (4, 4)]
    sys.path.insert(0, ROOT)
    import bench
    import pytest
    with pytest.raises(ValueError):
        bench.head_shard(0, 3, 8)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


def test_bench_flop_accounting_from_block_codes():
    """Executed FLOPs count QK^T for every visited tile and PV for kept ones; the
    dense-equivalent count takes both for every visited tile (a tile is 2*Bq*Bk*D)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from threshold_gated_block_b200.inputs import CONFIGS
    cfg = CONFIGS["c2"]
    codes = np.array([[[[2, 3, 3], [0, 2, 3], [1, 0, 2]]]], dtype=np.uint8)   # 6 visited: 3 forced, 1 kept, 2 skipped
    visited = int((codes != 3).sum())
    kept = int(np.isin(codes, (1, 2)).sum())
    tile = 2.0 * cfg.Bq * cfg.Bk * cfg.D
    exec_f, dense_f = bench.mask_flops(codes, cfg)
    assert exec_f == (visited + kept) * tile and dense_f == 2 * visited * tile
    assert bench.weak_scaling_value(1e12, 4, 10.0) == 4 * 1e12 / 10e-3 / 1e12
