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


def _split_worker(rank, world, port, q):
    """The sequence split of decode and MLA and the prefill unit split, run over a gloo
    group with the float64 oracle as the per-rank attention and the oracle's LSE merge,
    against the unsplit oracle."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np
    from attention_causal_gqa_b200 import sharding
    from attention_causal_gqa_b200.synthetic import decode_inputs, mla_inputs, prefill_inputs
    from oracle import decode_paged_ref, lse_merge, mla_decode_ref, prefill_ref
    dist.init_process_group("gloo", rank=rank, world_size=world)
    errs = {}
    try:
        def merge_rows(o_parts, l_parts):
            o_parts, l_parts = o_parts.numpy(), l_parts.numpy()
            lead = l_parts.shape[1:]
            o = np.zeros(o_parts.shape[1:])
            lse = np.zeros(lead)
            for idx in np.ndindex(*lead):
                o[idx], lse[idx] = lse_merge(o_parts[(slice(None),) + idx], l_parts[(slice(None),) + idx])
            return o, lse

        # paged decode: one sequence shorter than a page per rank, one empty
        lens = [1, 100, 37, 0, 700]
        d = decode_inputs(len(lens), 8, 2, 64, seq_lens=lens, seed=31, device="cpu")
        f = lambda t: t.float().numpy()  # noqa: E731
        table, lr = sharding.local_block_table(d["block_table"], d["seq_lens"], rank, world)

        def attend_dec():
            o, l = decode_paged_ref(f(d["q"]), f(d["k_pages"]), f(d["v_pages"]), table.numpy(), lr.numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        o, l = sharding.split_and_merge(attend_dec, merge_rows)
        ro, rl = decode_paged_ref(f(d["q"]), f(d["k_pages"]), f(d["v_pages"]), d["block_table"].numpy(),
                                  d["seq_lens"].numpy())
        assert np.array_equal(np.isneginf(l), np.isneginf(rl))
        fin = np.isfinite(rl)
        errs["decode"] = max(float(np.abs(o - ro).max()), float(np.abs(l[fin] - rl[fin]).max()))

        # MLA over a cache sharded by 64-token tiles: rank r keeps rows [0, n) of its slice
        mlens = [200, 70, 1, 129]
        m = mla_inputs(len(mlens), 128, 512, 64, seq_lens=mlens, T_max=256, seed=32, device="cpu")
        sl = [sharding.kv_slice(L, rank, world, 64) for L in mlens]
        tl = max(1, max(n for _, n in sl))
        kv = np.zeros((len(mlens), tl, 512))
        pe = np.zeros((len(mlens), tl, 64))
        for b, (s0, n) in enumerate(sl):
            kv[b, :n] = f(m["kv_cache"][b, s0:s0 + n])
            pe[b, :n] = f(m["pe_cache"][b, s0:s0 + n])

        def attend_mla():
            o, l = mla_decode_ref(f(m["q_nope"]), f(m["q_pe"]), kv, pe, [n for _, n in sl], 0.07)
            return torch.from_numpy(o), torch.from_numpy(l)

        o, l = sharding.split_and_merge(attend_mla, merge_rows)
        ro, rl = mla_decode_ref(f(m["q_nope"]), f(m["q_pe"]), f(m["kv_cache"]), f(m["pe_cache"]), mlens, 0.07)
        errs["mla"] = max(float(np.abs(o - ro).max()), float(np.abs(l - rl).max()))

        # prefill: disjoint (b, kv head) units, combined by a sum of zero-padded results
        qq, kk, vv = prefill_inputs(2, 6, 3, 40, 64, "bf16", 1.0, seed=33, device="cpu")
        qq, kk, vv = f(qq), f(kk), f(vv)
        out = torch.zeros(2, 6, 40, 64, dtype=torch.float64)
        lse = torch.zeros(2, 6, 40, dtype=torch.float64)
        for b, kvh in sharding.prefill_units(2, 3, rank, world):
            hs = slice(2 * kvh, 2 * kvh + 2)
            o_, l_ = prefill_ref(qq[b:b + 1, hs], kk[b:b + 1, kvh:kvh + 1], vv[b:b + 1, kvh:kvh + 1],
                                 rope_theta=1e4)
            out[b, hs], lse[b, hs] = torch.from_numpy(o_[0]), torch.from_numpy(l_[0])
        dist.all_reduce(out)
        dist.all_reduce(lse)
        ro, rl = prefill_ref(qq, kk, vv, rope_theta=1e4)
        errs["prefill"] = max(float(np.abs(out.numpy() - ro).max()), float(np.abs(lse.numpy() - rl).max()))
        q.put((rank, errs))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_sequence_and_merge_to_the_unsplit_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    for _ in range(2):
        rank, errs = q.get(timeout=10)
        for what, e in errs.items():
            assert e < 1e-10, (rank, what, e)


def test_slices_cover_every_token_once():
    from attention_causal_gqa_b200.sharding import kv_slice, prefill_units, unit_range
    for L in (0, 1, 15, 16, 17, 1000, 32768):
        for W in (1, 2, 3, 8):
            for unit in (16, 64):
                got = [kv_slice(L, r, W, unit) for r in range(W)]
                pos = 0
                for s, n in got:
                    if n:
                        assert s == pos and s % unit == 0
                        pos += n
                assert pos == L
    for n in (0, 5, 64):
        for W in (1, 3, 8):
            assert sum(b - a for a, b in (unit_range(n, r, W) for r in range(W))) == n
    assert sorted(u for r in range(3) for u in prefill_units(2, 5, r, 3)) == [(b, h) for b in range(2) for h in range(5)]
