"""Multi-process (world size 2, gloo, CPU) checks of the bench's rank logic:
per-rank replicas with distinct seeds, MAX-over-ranks timing, and the reference
arm printing only on rank 0."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(float(10 + rank), world)
        bench.barrier(world)
        from attention_causal_gqa_b200.synthetic import prefill_inputs
        q_, _, _ = prefill_inputs(1, 2, 1, 8, 64, "bf16", 1.0, seed=bench.rank_seed(rank), device="cpu")
        q.put((rank, mx, bench.rank_seed(rank), float(q_.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [11.0, 11.0]          # both ranks see the slowest value
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]  # independent replicas


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
