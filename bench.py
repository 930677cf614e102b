#!/usr/bin/env python
"""Benchmark: prefill attention TFLOP/s (headline) plus paged-decode and MLA-decode
KV-read GB/s, each against the B200 roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline step: one attn_prefill call (RoPE prologue + tcgen05 prefill kernel) on the
causal GQA workload B=2, Hq=32, Hkv=8, S=4096, D=128, bf16; L2 is flushed between
timed steps. The paged-decode (B=64, Hq=32, Hkv=8, D=128, lengths U[1024, 32768],
16-token pages) and MLA-decode (B=32, H=128, Dc=512, Dr=64, T U[4096, 32768])
workloads are timed the same way in their own regions and reported beside it.
Under torchrun every rank runs its own replica (independent batches, no data-path
collective): weak scaling; times are device times, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PREFILL = "gqa_prefill_b2_hq32_hkv8_s4096_d128"
DECODE = "paged_decode_b64_hq32_hkv8_d128"
MLA = "mla_decode_b32_h128_dc512_dr64"
DSA = "dsa_mla_decode_b32_h128_dc512_dr64_hi64_di128_top2048"
PREFILL_LONG = "gqa_prefill_b1_hq32_hkv8_s32768_d128"
CHUNK = "chunk_prefill_b8_hq32_hkv8_d128_n2048_cache4k_28k"
METRIC = "prefill attn TFLOP/s & decode KV-read GB/s, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def prefill_flops(p):
    # exact causal: Q K^T and P V over the lower triangle incl. the diagonal
    return p["B"] * p["Hq"] * 4.0 * p["D"] * p["S"] * (p["S"] + 1) / 2.0


# ------------------------------------------------------------------ clocks
class Clocks:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[3:7]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- helpers
def traffic_for(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, only if taken on this kernel's exact source."""
    from attention_causal_gqa_b200.build import kernel_fingerprint
    fingerprint = kernel_fingerprint(kernel)
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel and parts[1] == fingerprint:
                return float(parts[2])
    return None


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (device times are combined by MAX, never by wall clock)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank runs its own replica of the workload: same shapes, its own seeded values."""
    return 20261202 + 1000 * rank


def timed_region(fn, steps, warmup, world, flush=None):
    """Runs warmup + steps calls of fn; returns (summed device ms of the steps, max over ranks)."""
    import torch
    for _ in range(warmup):
        if flush is not None:
            flush()
        fn()
    barrier(world)
    evs = []
    st = torch.cuda.current_stream()
    for _ in range(steps):
        if flush is not None:
            flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        fn()
        e1.record(st)
        evs.append((e0, e1))
    barrier(world)
    ms = sum(a.elapsed_time(b) for a, b in evs)
    return max_over_ranks(ms, world)


def hooked_kernel_ms(fn, steps, world, flush=None):
    """Average device time per launch of a call's main kernel, from the library's timing
    hook (CUDA events recorded around that kernel on its launch stream). Taken on steps of
    their own: while a call is timed the hook is off, so no event sits between the call's
    dependent launches and the programmatic launch overlap stays as a caller gets it."""
    import torch
    from attention_causal_gqa_b200 import binding as B_
    B_.profile_enable(True)
    B_.profile_collect()
    for _ in range(steps):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    k_ms, n = B_.profile_collect()
    B_.profile_enable(False)
    return max_over_ranks(k_ms / max(n, 1), world)


# ----------------------------------------------------------- CPU oracle leg
def oracle_prefill_sample(q, k, v, p, budget_s):
    """Times the float64 oracle on whole heads of the workload until ~budget_s elapsed."""
    import numpy as np
    from oracle import prefill_ref
    qn = q.float().cpu().numpy()
    kn = k.float().cpu().numpy()
    vn = v.float().cpu().numpy()
    G = p["Hq"] // p["Hkv"]
    heads, t0 = 0, time.perf_counter()
    for b in range(p["B"]):
        for h in range(p["Hq"]):
            kvh = h // G
            prefill_ref(qn[b:b + 1, h:h + 1], kn[b:b + 1, kvh:kvh + 1], vn[b:b + 1, kvh:kvh + 1], causal=True,
                        rope_theta=p["theta"], scale=p["scale"])
            heads += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    flops = heads * 4.0 * p["D"] * p["S"] * (p["S"] + 1) / 2.0
    return flops / dt / 1e12, heads, dt


def oracle_prefill_rows(q, k, v, p, budget_s):
    """Times the float64 oracle on the last query rows of head 0 of the workload (the rows
    that see the most keys), 32 rows per call, until ~budget_s elapsed."""
    from oracle import prefill_ref
    qn, kn, vn = (x[0:1, 0:1].float().cpu().numpy() for x in (q, k, v))
    S, D = p["S"], p["D"]
    flops, rows, hi, t0 = 0.0, 0, S, time.perf_counter()
    while hi > 0 and time.perf_counter() - t0 < budget_s:
        chunk = list(range(max(0, hi - 32), hi))
        prefill_ref(qn, kn, vn, causal=True, rope_theta=p["theta"], scale=p["scale"],
                    rows=[(0, 0, i) for i in chunk])
        flops += sum(4.0 * D * (i + 1) for i in chunk)
        rows += len(chunk)
        hi -= 32
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"the last {rows} query rows of head (0, 0) ({rows} of {S} rows, each against all "
                      f"earlier keys), float64, {dt:.1f} s"}


def oracle_decode_seqs(d, dp, budget_s):
    """Times the float64 paged-decode oracle on whole sequences (all Hq heads), one at a
    time in order, until ~budget_s of oracle time; the pages a sequence uses are copied to
    the host first (outside the timed part)."""
    import numpy as np
    import torch
    from oracle import decode_paged_ref
    lens = d["seq_lens"].cpu().tolist()
    dt, nbytes, nseq = 0.0, 0, 0
    for b, L in enumerate(lens):
        if dt > budget_s:
            break
        n = (L + 15) // 16
        pages = d["block_table"][b, :n].long()
        kp = d["k_pages"][pages].float().cpu().numpy()
        vp = d["v_pages"][pages].float().cpu().numpy()
        qb = d["q"][b:b + 1].float().cpu().numpy()
        t0 = time.perf_counter()
        decode_paged_ref(qb, kp, vp, np.arange(n, dtype=np.int64)[None, :], [L], dp["scale"])
        dt += time.perf_counter() - t0
        nbytes += L * dp["Hkv"] * dp["D"] * 2 * 2
        nseq += 1
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{nseq} whole sequences of {len(lens)} ({sum(lens[:nseq])} cached tokens, all heads), "
                      f"float64, {dt:.2f} s of oracle time"}


def oracle_mla_seqs(m, mp, budget_s):
    """Times the float64 MLA oracle on whole sequences (all heads) until ~budget_s."""
    from oracle import mla_decode_ref
    lens = m["seq_lens"].cpu().tolist()
    dt, nbytes, nseq = 0.0, 0, 0
    for b, L in enumerate(lens):
        if dt > budget_s:
            break
        kv = m["kv_cache"][b:b + 1, :L].float().cpu().numpy()
        pe = m["pe_cache"][b:b + 1, :L].float().cpu().numpy()
        qn, qp = m["q_nope"][b:b + 1].float().cpu().numpy(), m["q_pe"][b:b + 1].float().cpu().numpy()
        t0 = time.perf_counter()
        mla_decode_ref(qn, qp, kv, pe, [L], mp["scale"])
        dt += time.perf_counter() - t0
        nbytes += L * (mp["Dc"] + mp["Dr"]) * 2
        nseq += 1
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{nseq} whole sequences of {len(lens)} ({sum(lens[:nseq])} cached tokens, all 128 heads), "
                      f"float64, {dt:.2f} s of oracle time"}


def oracle_decode_fp8_seqs(d, dp, budget_s):
    """Times the float64 FP8 paged-decode oracle (E4M3 codes times their page scales, then
    the decode) on whole sequences, one at a time, until ~budget_s of oracle time."""
    import numpy as np
    from oracle import decode_paged_fp8_ref
    lens = d["seq_lens"].cpu().tolist()
    dt, nbytes, nseq = 0.0, 0, 0
    for b, L in enumerate(lens):
        if dt > budget_s:
            break
        n = (L + 15) // 16
        pages = d["block_table"][b, :n].long()
        kc, vc = d["k_pages"][pages].cpu().numpy(), d["v_pages"][pages].cpu().numpy()
        ks, vs = d["k_scale"][pages].cpu().numpy(), d["v_scale"][pages].cpu().numpy()
        qb = d["q"][b:b + 1].float().cpu().numpy()
        t0 = time.perf_counter()
        decode_paged_fp8_ref(qb, kc, vc, ks, vs, np.arange(n, dtype=np.int64)[None, :], [L], dp["scale"])
        dt += time.perf_counter() - t0
        nbytes += L * dp["Hkv"] * dp["D"] * 2 + n * dp["Hkv"] * 8
        nseq += 1
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{nseq} whole sequences of {len(lens)} ({sum(lens[:nseq])} cached tokens, all heads), "
                      f"float64, {dt:.2f} s of oracle time"}


def oracle_chunk_sample(d, p, budget_s):
    """Times the float64 chunked-prefill oracle on the first sequences of the workload, one
    KV head group at a time (its G query heads, all new rows, the whole cache), until
    ~budget_s of oracle time; the group's pages are copied to the host first."""
    import numpy as np
    from oracle import chunk_prefill_ref
    G = p["Hq"] // p["Hkv"]
    S, D = p["S_new"], p["D"]
    lens = d["cache_lens"].cpu().tolist()
    dt, flops, done = 0.0, 0.0, 0
    for b, L in enumerate(lens):
        for kvh in range(p["Hkv"]):
            if dt > budget_s:
                break
            n = (L + S + 15) // 16
            pages = d["block_table"][b, :n].long()
            kp = d["k_pages"][pages][:, :, kvh:kvh + 1].float().cpu().numpy()
            vp = d["v_pages"][pages][:, :, kvh:kvh + 1].float().cpu().numpy()
            qb = d["q"][b:b + 1, kvh * G:(kvh + 1) * G].float().cpu().numpy()
            kb = d["k"][b:b + 1, kvh:kvh + 1].float().cpu().numpy()
            vb = d["v"][b:b + 1, kvh:kvh + 1].float().cpu().numpy()
            t0 = time.perf_counter()
            chunk_prefill_ref(qb, kb, vb, kp, vp, np.arange(n, dtype=np.int64)[None, :], [L], rope_theta=p["theta"],
                              scale=p["scale"])
            dt += time.perf_counter() - t0
            flops += G * 4 * D * (S * L + S * (S + 1) / 2)
            done += 1
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} (sequence, kv head) groups of {len(lens) * p['Hkv']} ({G} query heads x {S} new rows "
                      f"over the whole cache each), float64, {dt:.2f} s of oracle time"}


def oracle_dsa_seqs(d, p, top_k, budget_s):
    """Times the float64 oracle of the whole sparse step (indexer scores, top-k, MLA over the
    selected tokens) on whole sequences, until ~budget_s of oracle time."""
    from oracle import dsa_index_scores_ref, dsa_mla_decode_ref, dsa_topk_ref
    lens = d["seq_lens"].cpu().tolist()
    dt, tokens, nseq = 0.0, 0, 0
    for b, L in enumerate(lens):
        if dt > budget_s:
            break
        qi, wi = d["q_idx"][b:b + 1].float().cpu().numpy(), d["w_idx"][b:b + 1].float().cpu().numpy()
        ki = d["k_idx"][b:b + 1, :L].float().cpu().numpy()
        kv = d["kv_cache"][b:b + 1, :L].float().cpu().numpy()
        pe = d["pe_cache"][b:b + 1, :L].float().cpu().numpy()
        qn, qp = d["q_nope"][b:b + 1].float().cpu().numpy(), d["q_pe"][b:b + 1].float().cpu().numpy()
        t0 = time.perf_counter()
        sc = dsa_index_scores_ref(qi, wi, ki, [L])
        sel = dsa_topk_ref(sc, [L], top_k)
        dsa_mla_decode_ref(qn, qp, kv, pe, sel, p["scale"])
        dt += time.perf_counter() - t0
        tokens += L
        nseq += 1
    return {"value": tokens / dt, "unit": "cached tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{nseq} whole sequences of {len(lens)} ({tokens} cached tokens: indexer, top-{top_k}, MLA over "
                      f"the selection, all heads), float64, {dt:.2f} s of oracle time"}


def want_cpu(args, world, rank):
    return rank == 0 and world == 1 and not args.no_cpu_baseline


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args):
    """Reference arm: the float64 CPU oracle, timed as it stands on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    from attention_causal_gqa_b200.synthetic import WORKLOADS, prefill_inputs
    from oracle import prefill_ref
    p = WORKLOADS[PREFILL].params
    q, k, v = prefill_inputs(p["B"], p["Hq"], p["Hkv"], p["S"], p["D"], p["dtype"], p["std"], seed=20261202,
                             device="cpu")
    qn, kn, vn = (x.float().numpy() for x in (q, k, v))
    G = p["Hq"] // p["Hkv"]
    per_head = 4.0 * p["D"] * p["S"] * (p["S"] + 1) / 2.0
    times = []
    for i in range(args.warmup + args.steps):
        b, h = divmod(i % (p["B"] * p["Hq"]), p["Hq"])
        t0 = time.perf_counter()
        prefill_ref(qn[b:b + 1, h:h + 1], kn[b:b + 1, h // G:h // G + 1], vn[b:b + 1, h // G:h // G + 1],
                    causal=True, rope_theta=p["theta"], scale=p["scale"])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    val = per_head * len(times) / tot / 1e12
    sample = f"one (b, head) of the {PREFILL} workload per step: all {p['S']} causal rows, float64"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": PREFILL, "sample": "one head per step"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def prefill_e2e(args, world, dev, p, q, k, v, out, lse, flops):
    """End to end through the public call: every step copies its own q, k, v from pinned host
    memory, runs attn_prefill and reads its out and lse back into pinned host memory. Steps
    are pipelined the way a streaming caller runs them: inputs and outputs are
    double-buffered on the device, host-to-device copies run on one stream, the call on a
    second and device-to-host copies on a third, ordered by events, so step i's upload and
    step i-1's download overlap step i-1's and step i's compute (the two copy directions use
    separate engines). Timed from the first upload to the last download (CUDA events),
    max over ranks."""
    import torch
    from attention_causal_gqa_b200 import binding as B_
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    torch.cuda.synchronize()
    ref_out, ref_lse = out.cpu(), lse.cpu()  # the plain call's result on the same inputs
    dq = [(q, k, v), tuple(torch.empty_like(x) for x in (q, k, v))]
    do = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
    hout = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(), torch.empty(lse.shape, dtype=lse.dtype).pin_memory())
            for _ in range(2)]
    ws = torch.empty(B_.prefill_workspace_size(p["B"], p["Hkv"], p["S"], p["D"]), dtype=torch.uint8, device=dev)
    s_up, s_run, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run_steps(n):
        up = [torch.cuda.Event() for _ in range(n)]
        ran = [torch.cuda.Event() for _ in range(n)]
        down = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            slot = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ran[i - 2])  # the slot's inputs were read by step i - 2
                for dst, src in zip(dq[slot], (qh, kh, vh)):
                    dst.copy_(src, non_blocking=True)
                up[i].record(s_up)
            with torch.cuda.stream(s_run):
                s_run.wait_event(up[i])
                if i >= 2:
                    s_run.wait_event(down[i - 2])  # the slot's outputs were read back by step i - 2
                B_.attn_prefill(*dq[slot], causal=True, rope_theta=p["theta"], scale=p["scale"], out=do[slot][0],
                                lse=do[slot][1], workspace=ws, stream=s_run)
                ran[i].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ran[i])
                hout[slot][0].copy_(do[slot][0], non_blocking=True)
                hout[slot][1].copy_(do[slot][1], non_blocking=True)
                down[i].record(s_down)
        return down[-1]

    run_steps(2)  # warm-up
    torch.cuda.synchronize()
    barrier(world)
    n = max(4, args.steps // 2)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    last = run_steps(n)
    s_down.wait_event(last)
    e1.record(s_down)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    B_.profile_collect()
    # every downloaded result equals the plain call's (the kernels are deterministic), so no
    # step read an input before its upload or downloaded an output before its call ended
    for ho, hl in hout:
        if not (torch.equal(ho, ref_out) and torch.equal(hl, ref_lse)):
            raise RuntimeError("pipelined end-to-end steps returned a result that differs from the plain call")
    return {"value": world * flops * n / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (qh, kh, vh)),
            "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in hout[0]),
            "pipelined": "double-buffered steps: uploads, calls and downloads on three streams"}


def bench_prefill(args, world, dev, seed, flush, pk, pk_kind, fp, name=None, with_e2e=True):
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    name = name or PREFILL
    p = WORKLOADS[name].params
    q, k, v = workload_inputs(name, seed=seed, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((p["B"], p["Hq"], p["S"]), dtype=torch.float32, device=dev)
    ws = torch.empty(B_.prefill_workspace_size(p["B"], p["Hkv"], p["S"], p["D"]), dtype=torch.uint8, device=dev)

    def step():
        B_.attn_prefill(q, k, v, causal=True, rope_theta=p["theta"], scale=p["scale"], out=out, lse=lse,
                        workspace=ws)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world, flush=flush)
    kern_avg = hooked_kernel_ms(step, args.steps, world, flush=flush)
    flops = prefill_flops(p)
    value = world * flops * args.steps / (ms * 1e-3) / 1e12
    achieved = flops / (kern_avg * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / pk["bf16_tflops"], "traffic": traffic_for("prefill_kernel"),
            "kernel": "prefill_kernel", "kernel_ms": kern_avg, "peak_kind": f"{pk_kind} dense bf16 (burst)",
            "algorithmic": f"{flops:.4g} flop per launch = B*Hq*4*D*S(S+1)/2 (exact causal)"}
    res = {"value": value, "ms": ms, "roofline": roof, "flops": flops, "p": p}
    if with_e2e and not args.no_e2e:
        res["e2e"] = prefill_e2e(args, world, dev, p, q, k, v, out, lse, flops)
    res["inputs"] = (q, k, v)
    return res


def bench_chunk(args, world, dev, seed, pk, pk_kind):
    """Chunked prefill into the paged cache: every step appends the same chunk at the same
    positions (idempotent) and attends over the whole cache."""
    import numpy as np
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    p = WORKLOADS[CHUNK].params
    d = workload_inputs(CHUNK, seed=seed, device=dev)
    B, Hq, S, D = p["B"], p["Hq"], p["S_new"], p["D"]
    out = torch.empty_like(d["q"])
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    ws = torch.empty(B_.prefill_chunk_workspace_size(B, p["Hkv"], S, d["max_cache_len"], D), dtype=torch.uint8,
                     device=dev)

    def step():
        B_.attn_prefill_chunk(d["q"], d["k"], d["v"], d["k_pages"], d["v_pages"], d["block_table"], d["cache_lens"],
                              d["max_cache_len"], rope_theta=p["theta"], scale=p["scale"], out=out, lse=lse,
                              workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world)
    kern_avg = hooked_kernel_ms(step, args.steps, world)
    lens = d["cache_lens"].cpu().numpy().astype(np.float64)
    # exact causal work: query i of sequence b sees cache_lens[b] + i + 1 keys; QK^T and P V
    flops = float(np.sum(Hq * 4 * D * (S * lens + S * (S + 1) / 2)))
    achieved = flops / (kern_avg * 1e-3) / 1e12
    cpu = None
    if want_cpu(args, world, int(os.environ.get("RANK", "0"))):
        cpu = oracle_chunk_sample(d, p, args.cpu_budget * 0.75)
    return {"workload": CHUNK, "cpu_baseline": cpu, "value": world * flops * args.steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms / args.steps, "cached_tokens": int(lens.sum()), "gpu_launches": 5 * args.steps,
            "l2": "cache (1.2 GB of pages) larger than L2",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "traffic": None, "kernel": "prefill_kernel",
                         "kernel_ms": kern_avg, "peak_kind": f"{pk_kind} dense bf16 (burst)",
                         "algorithmic": f"{flops:.4g} flop per launch = sum over rows of 4*D*(keys seen)"}}


def bench_decode(args, world, dev, seed, pk, pk_kind, fp):
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    dp = dict(WORKLOADS[DECODE].params)
    if args.small:
        from attention_causal_gqa_b200.synthetic import decode_inputs
        dp["B"] = 8
        d = decode_inputs(8, dp["Hq"], dp["Hkv"], dp["D"], dp["lmin"], dp["lmax"], dp["std"], seed, dev)
    else:
        d = workload_inputs(DECODE, seed=seed, device=dev)
    out = torch.empty_like(d["q"])
    lse = torch.empty((dp["B"], dp["Hq"]), dtype=torch.float32, device=dev)
    ws = torch.empty(B_.decode_workspace_size(dp["B"], dp["Hq"], dp["D"], d["max_pages_per_seq"]),
                     dtype=torch.uint8, device=dev)

    def step():
        B_.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                             scale=dp["scale"], out=out, lse=lse, workspace=ws)

    tokens = int(d["seq_lens"].sum().item())
    kv_bytes = tokens * dp["Hkv"] * dp["D"] * 2 * 2
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world)
    k_avg = hooked_kernel_ms(step, args.steps, world)
    ach = kv_bytes / (k_avg * 1e-3) / 1e9
    res = {"workload": DECODE + ("_small_b8" if args.small else ""), "value": world * kv_bytes * args.steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
           "ms_per_step": ms / args.steps, "kv_tokens": tokens, "kv_bytes_per_step": kv_bytes,
           "gpu_launches": 2 * args.steps, "l2": "inputs (4.4 GB) larger than L2",
           "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": traffic_for("decode_kernel"),
                        "kernel": "decode_kernel", "kernel_ms": k_avg, "peak_kind": f"{pk_kind} HBM copy",
                        "algorithmic": "4096 B per cached token (K+V, 8 heads x 128 x bf16)"}}
    if want_cpu(args, world, int(os.environ.get("RANK", "0"))):
        res["cpu_baseline"] = oracle_decode_seqs(d, dp, args.cpu_budget * 0.75)
    del d, out, lse, ws
    torch.cuda.empty_cache()
    return res


def bench_decode_fp8(args, world, dev, seed, pk, pk_kind):
    """The paged decode workload with its K/V pages quantised to E4M3 (one scale per page
    and kv head): same sequences, half the cache bytes."""
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, decode_inputs_fp8
    dp = dict(WORKLOADS[DECODE].params)
    B = 8 if args.small else dp["B"]
    d = decode_inputs_fp8(B, dp["Hq"], dp["Hkv"], dp["D"], dp["lmin"], dp["lmax"], dp["std"], seed, dev)
    out = torch.empty_like(d["q"])
    lse = torch.empty((B, dp["Hq"]), dtype=torch.float32, device=dev)
    ws = torch.empty(B_.decode_fp8_workspace_size(B, dp["Hq"], dp["D"], d["max_pages_per_seq"]), dtype=torch.uint8,
                     device=dev)

    def step():
        B_.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"], d["v_scale"], d["block_table"],
                                 d["seq_lens"], scale=dp["scale"], out=out, lse=lse, workspace=ws)

    tokens = int(d["seq_lens"].sum().item())
    # codes: Hkv * D bytes each for K and V; scales: 2 * Hkv * 4 bytes per 16-token page
    kv_bytes = tokens * dp["Hkv"] * dp["D"] * 2 + ((tokens + 15) // 16) * dp["Hkv"] * 8
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world)
    k_avg = hooked_kernel_ms(step, args.steps, world)
    ach = kv_bytes / (k_avg * 1e-3) / 1e9
    res = {"workload": DECODE + "_fp8_e4m3" + ("_small_b8" if args.small else ""),
           "value": world * kv_bytes * args.steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
           "ms_per_step": ms / args.steps, "kv_tokens": tokens, "kv_bytes_per_step": kv_bytes,
           "gpu_launches": 2 * args.steps, "l2": "inputs (2.2 GB) larger than L2",
           "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": traffic_for("decode_fp8_kernel"),
                        "kernel": "decode_fp8_kernel",
                        "kernel_ms": k_avg, "peak_kind": f"{pk_kind} HBM copy",
                        "algorithmic": "2048 B of codes per cached token + 64 B of scales per 16-token page"}}
    if want_cpu(args, world, int(os.environ.get("RANK", "0"))):
        res["cpu_baseline"] = oracle_decode_fp8_seqs(d, dp, args.cpu_budget * 0.75)
    del d, out, lse, ws
    torch.cuda.empty_cache()
    return res


def bench_mla(args, world, dev, seed, pk, pk_kind, fp):
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    mp = dict(WORKLOADS[MLA].params)
    if args.small:
        from attention_causal_gqa_b200.synthetic import mla_inputs
        mp["B"] = 8
        m = mla_inputs(8, mp["H"], mp["Dc"], mp["Dr"], mp["lmin"], mp["lmax"], mp["std"], seed, dev)
    else:
        m = workload_inputs(MLA, seed=seed, device=dev)
    out = torch.empty_like(m["q_nope"])
    lse = torch.empty((mp["B"], 1, mp["H"]), dtype=torch.float32, device=dev)
    ws = torch.empty(B_.mla_workspace_size(mp["B"], mp["H"], mp["Dc"], mp["Dr"], m["T_max"]),
                     dtype=torch.uint8, device=dev)

    def step():
        B_.mla_decode(m["q_nope"], m["q_pe"], m["kv_cache"], m["pe_cache"], m["seq_lens"], mp["scale"],
                      out=out, lse=lse, workspace=ws)

    tokens = int(m["seq_lens"].sum().item())
    nbytes = tokens * (mp["Dc"] + mp["Dr"]) * 2
    flops = tokens * mp["H"] * (2.0 * (mp["Dc"] + mp["Dr"]) + 2.0 * mp["Dc"])
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world)
    k_avg = hooked_kernel_ms(step, args.steps, world)
    ach = nbytes / (k_avg * 1e-3) / 1e9
    res = {"workload": MLA + ("_small_b8" if args.small else ""), "value": world * nbytes * args.steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
           "ms_per_step": ms / args.steps, "kv_tokens": tokens, "kv_bytes_per_step": nbytes,
           "tflops": world * flops * args.steps / (ms * 1e-3) / 1e12, "gpu_launches": 2 * args.steps,
           "l2": "kv/pe caches (1.2 GB) larger than L2",
           "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": traffic_for("mla_kernel"),
                        "kernel": "mla_kernel", "kernel_ms": k_avg, "peak_kind": f"{pk_kind} HBM copy",
                        "algorithmic": "1152 B per cached token (kv 512 + pe 64, bf16)",
                        "tensor_tflops": flops / (k_avg * 1e-3) / 1e12,
                        "tensor_frac": flops / (k_avg * 1e-3) / 1e12 / pk["bf16_tflops"]}}
    if want_cpu(args, world, int(os.environ.get("RANK", "0"))):
        res["cpu_baseline"] = oracle_mla_seqs(m, mp, args.cpu_budget * 0.75)
    del m, out, lse, ws
    torch.cuda.empty_cache()
    return res


def bench_dsa(args, world, dev, seed, pk, pk_kind, dense_ms=None):
    """DeepSeek sparse attention on the MLA workload: lightning indexer + top-k over every
    cached token, then the MLA decode over the 2048 selected tokens per sequence."""
    import torch
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.synthetic import WORKLOADS, dsa_inputs, workload_inputs
    p = dict(WORKLOADS[DSA].params)
    if args.small:
        p["B"] = 8
        d = dsa_inputs(8, p["H"], p["Dc"], p["Dr"], p["HI"], p["dI"], p["lmin"], p["lmax"], p["std"], seed, dev)
    else:
        d = workload_inputs(DSA, seed=seed, device=dev)
    B, T, K = p["B"], d["T_max"], p["top_k"]
    scores = torch.empty((B, T), dtype=torch.float32, device=dev)
    idx = torch.empty((B, K), dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q_nope"])
    lse = torch.empty((B, 1, p["H"]), dtype=torch.float32, device=dev)
    ws1 = torch.empty(256, dtype=torch.uint8, device=dev)
    ws2 = torch.empty(B_.dsa_mla_workspace_size(B, p["H"], p["Dc"], p["Dr"], K), dtype=torch.uint8, device=dev)

    def index():
        B_.dsa_index_topk(d["q_idx"], d["w_idx"], d["k_idx"], d["seq_lens"], K, scores=scores, topk_idx=idx,
                          workspace=ws1)

    def attend():
        B_.dsa_mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], idx, p["scale"],
                          out=out, lse=lse, workspace=ws2)

    def step():
        index()
        attend()

    tokens = int(d["seq_lens"].sum().item())
    selected = int(d["seq_lens"].clamp(max=K).sum().item())
    idx_bytes = tokens * (p["dI"] * 2 + 4)  # indexer keys read + scores written
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = timed_region(step, args.steps, 0, world)
    ms_index = timed_region(index, args.steps, 0, world)
    k_idx = hooked_kernel_ms(index, args.steps, world)
    ms_attend = timed_region(attend, args.steps, 0, world)
    k_mla = hooked_kernel_ms(attend, args.steps, world)
    # the same selection attended over an E4M3 latent cache (one scale per token and 128-wide block)
    from attention_causal_gqa_b200.synthetic import quantize_e4m3_rows
    kv_codes, kv_scale = quantize_e4m3_rows(d["kv_cache"])

    def attend_fp8():
        B_.dsa_mla_decode_fp8(d["q_nope"], d["q_pe"], kv_codes, kv_scale, d["pe_cache"], d["seq_lens"], idx,
                              p["scale"], out=out, lse=lse, workspace=ws2)

    for _ in range(args.warmup):
        attend_fp8()
    ms_attend_fp8 = timed_region(attend_fp8, args.steps, 0, world)
    del kv_codes, kv_scale
    ach = idx_bytes / (k_idx * 1e-3) / 1e9
    res = {"workload": DSA + ("_small_b8" if args.small else ""), "value": world * tokens * args.steps / (ms * 1e-3),
           "unit": "cached tokens/s", "ms_per_step": ms / args.steps, "kv_tokens": tokens,
           "selected_tokens": selected, "index_call_ms": ms_index / args.steps,
           "sparse_mla_call_ms": ms_attend / args.steps, "mla_kernel_ms": k_mla,
           "sparse_mla_fp8_latent_call_ms": ms_attend_fp8 / args.steps,
           "dense_mla_ms_per_step": dense_ms, "gpu_launches": 5 * args.steps,
           "l2": "indexer keys (268 MB) and caches larger than L2",
           "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": traffic_for("dsa_index_kernel"),
                        "kernel": "dsa_index_kernel", "kernel_ms": k_idx, "peak_kind": f"{pk_kind} HBM copy",
                        "algorithmic": "260 B per cached token (128 bf16 indexer key + fp32 score)"}}
    if want_cpu(args, world, int(os.environ.get("RANK", "0"))):
        res["cpu_baseline"] = oracle_dsa_seqs(d, p, K, args.cpu_budget * 0.75)
    del d, scores, idx, out, lse, ws1, ws2
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    from attention_causal_gqa_b200 import binding as B_
    from attention_causal_gqa_b200.build import _fingerprint

    pk, pk_kind = peaks()
    fp = _fingerprint()[:16]
    dev = torch.device("cuda", local if world > 1 else 0)
    seed = rank_seed(rank)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    def do(w):
        return args.only is None or args.only == w

    smi_index = local if world > 1 else int((os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0"))
    clocks = Clocks(smi_index)
    B_.profile_enable(False)  # on only inside hooked_kernel_ms
    clocks.start()
    pre = bench_prefill(args, world, dev, seed, flush, pk, pk_kind, fp) if do("prefill") else None
    sub = {}
    if do("prefill") and not args.small:
        # long-context prefill (inputs of 640 MB, larger than L2): call and kernel rates
        lp = bench_prefill(args, world, dev, seed, flush, pk, pk_kind, fp, name=PREFILL_LONG, with_e2e=False)
        lp["roofline"]["traffic"] = None  # the committed capture is of the S=4096 workload only
        sub["prefill_long"] = {"workload": PREFILL_LONG, "value": lp["value"], "unit": "TFLOP/s",
                               "ms_per_step": lp["ms"] / args.steps, "roofline": lp["roofline"],
                               "gpu_launches": 4 * args.steps}
        if want_cpu(args, world, rank):
            sub["prefill_long"]["cpu_baseline"] = oracle_prefill_rows(*lp["inputs"], lp["p"], args.cpu_budget * 0.75)
        del lp
    if do("prefill") and not args.small:
        sub["prefill_chunk"] = bench_chunk(args, world, dev, seed, pk, pk_kind)
    if do("decode"):
        sub["decode"] = bench_decode(args, world, dev, seed, pk, pk_kind, fp)
        sub["decode_fp8"] = bench_decode_fp8(args, world, dev, seed, pk, pk_kind)
    if do("mla"):
        sub["mla"] = bench_mla(args, world, dev, seed, pk, pk_kind, fp)
    if do("mla") or do("dsa"):
        dense = sub["mla"]["ms_per_step"] if "mla" in sub else None
        sub["dsa"] = bench_dsa(args, world, dev, seed, pk, pk_kind, dense_ms=dense)
    clk = clocks.stop()
    B_.profile_enable(False)

    cpu = None
    if pre is not None and rank == 0 and world == 1 and not args.no_cpu_baseline:
        q, k, v = pre["inputs"]
        tf, heads, dt = oracle_prefill_sample(q, k, v, pre["p"], budget_s=args.cpu_budget)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{heads} whole heads (all {pre['p']['S']} causal rows each) of {PREFILL}, "
                         f"float64, {dt:.1f} s"}
    if pre is not None:
        p = pre["p"]
        line = {"metric": METRIC, "value": pre["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": pre["ms"] / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": PREFILL, "B": p["B"], "Hq": p["Hq"], "Hkv": p["Hkv"], "S": p["S"],
                           "D": p["D"], "causal": True, "rope_theta": p["theta"],
                           "l2": "flushed (256 MB write) between steps", "parallelism": f"replicas x{world}"},
                "roofline": pre["roofline"], "cpu_baseline": cpu, "e2e": pre.get("e2e"),
                "gpu_launches": 4 * args.steps}
    else:
        w = sub[args.only]
        line = {"metric": METRIC, "value": w["value"], "unit": w["unit"], "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": w["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": w["workload"]}, "roofline": w["roofline"], "cpu_baseline": None,
                "e2e": None, "gpu_launches": w["gpu_launches"]}
    line["clocks"] = clk
    line["source_fingerprint"] = fp
    line.update(sub)
    # one compact entry per workload, last in the line: rate, kernel time, roofline fraction
    # and the oracle's rate on the host cores where it was measured
    summ = {}
    if pre is not None:
        summ["prefill"] = {"value": round(pre["value"], 2), "unit": "TFLOP/s",
                           "kernel_ms": round(pre["roofline"]["kernel_ms"], 4),
                           "frac": round(pre["roofline"]["frac"], 3),
                           "cpu": round(cpu["value"], 5) if cpu else None}
    for name, w in sub.items():
        cb = w.get("cpu_baseline")
        summ[name] = {"value": round(w["value"], 2), "unit": w["unit"],
                      "kernel_ms": round(w["roofline"]["kernel_ms"], 4), "frac": round(w["roofline"]["frac"], 3),
                      "cpu": round(cb["value"], 5) if cb else None}
    line["summary"] = summ
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", choices=["prefill", "decode", "mla", "dsa"], default=None,
                    help="run one workload (for profiling); the JSON line then carries that workload only")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--small", action="store_true",
                    help="profiling case: decode and MLA with B=8 sequences (inputs still larger than L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
