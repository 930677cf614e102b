"""GPU parity: mla_decode (C-ABI via the binding) against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import mla_decode_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")
SCALE = 1.0 / math.sqrt(192)


def _run(d, scale=SCALE):
    from attention_causal_gqa_b200 import mla_decode
    out, lse = mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], scale)
    torch.cuda.synchronize()
    return out, lse


def _oracle(d, pairs=None, scale=SCALE):
    sl = d["seq_lens"].cpu().numpy()
    if pairs is None:
        return mla_decode_ref(to_np(d["q_nope"]), to_np(d["q_pe"]), to_np(d["kv_cache"]), to_np(d["pe_cache"]), sl,
                              scale)
    outs, lses, order = [], [], []
    for b in sorted({b for b, _ in pairs}):
        L = int(sl[b])
        hs = [h for bb, h in pairs if bb == b]
        o, l = mla_decode_ref(to_np(d["q_nope"][b:b + 1]), to_np(d["q_pe"][b:b + 1]),
                              to_np(d["kv_cache"][b:b + 1, :L]), to_np(d["pe_cache"][b:b + 1, :L]),
                              sl[b:b + 1], scale, pairs=[(0, h) for h in hs])
        outs.append(o)
        lses.append(l)
        order += [(b, h) for h in hs]
    return np.concatenate(outs), np.concatenate(lses), order


@cuda
@pytest.mark.parametrize("lens,T_max", [([1, 31, 32, 33], 64), ([600, 1500, 513, 511, 512], 1536),
                                        ([2048, 100], 2048),
                                        # 64-token tile edges, half tiles, and a cache length that
                                        # is not a multiple of the tile (last box read past T_max)
                                        ([1, 63, 64, 65, 96, 97, 127, 129, 160], 160)])
def test_mla_matches_oracle_small(lens, T_max):
    from attention_causal_gqa_b200.synthetic import mla_inputs
    d = mla_inputs(len(lens), 128, 512, 64, seq_lens=lens, T_max=T_max, seed=T_max + len(lens), device="cuda")
    out, lse = _run(d)
    ro, rl = _oracle(d)
    check(out, ro, lse, rl, what=f"mla {lens}")


@cuda
def test_mla_empty_sequence_and_poison_past_length():
    from attention_causal_gqa_b200.synthetic import mla_inputs
    lens = [0, 45, 700]
    d = mla_inputs(3, 128, 512, 64, seq_lens=lens, T_max=1024, seed=9, device="cuda")
    ro, rl = _oracle(d)
    for b, L in enumerate(lens):
        d["kv_cache"][b, L:] = float("nan")
        d["pe_cache"][b, L:] = float("inf")
    out, lse = _run(d)
    check(out, ro, lse, rl, what="mla poison")
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@cuda
def test_mla_empty_sequences_inside_a_cluster_range():
    """Empty sequences between long ones: the clusters whose tile ranges straddle them
    write no partial for them, so the merge must not read those slots (the workspace is
    poisoned with NaN first, so a stray read shows up)."""
    from attention_causal_gqa_b200 import binding
    from attention_causal_gqa_b200.synthetic import mla_inputs
    lens = [2000, 0, 2000, 0, 0, 3000, 0]
    d = mla_inputs(len(lens), 128, 512, 64, seq_lens=lens, T_max=3072, seed=21, device="cuda")
    ws = torch.full((binding.mla_workspace_size(len(lens), 128, 512, 64, 3072),), 255, dtype=torch.uint8,
                    device="cuda")
    out, lse = binding.mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], SCALE,
                                  workspace=ws)
    torch.cuda.synchronize()
    ro, rl = _oracle(d)
    check(out, ro, lse, rl, what="mla empty inside")
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(out[b] == 0) and torch.all(torch.isneginf(lse[b]))


@cuda
def test_mla_full_size_sampled():
    from attention_causal_gqa_b200.synthetic import workload_inputs
    d = workload_inputs("mla_decode_b32_h128_dc512_dr64", device="cuda")
    out, lse = _run(d)
    rng = np.random.default_rng(8)
    pairs = sorted({(int(rng.integers(32)), int(rng.integers(128))) for _ in range(40)} | {(0, 0), (31, 127)})
    ro, rl, order = _oracle(d, pairs)
    idx = torch.tensor(order, device="cuda")
    check(out[idx[:, 0], 0, idx[:, 1]], ro, lse[idx[:, 0], 0, idx[:, 1]], rl, what="mla full")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


@cuda
def test_mla_deterministic():
    from attention_causal_gqa_b200.synthetic import mla_inputs
    d = mla_inputs(2, 128, 512, 64, seq_lens=[3000, 777], T_max=3072, seed=1, device="cuda")
    o1, l1 = _run(d)
    o2, l2 = _run(d)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@cuda
def test_mla_many_segments_deterministic_and_exact():
    """100 sequences of 0-2999 tokens: each cluster walks several sequences, so segment
    ends (partial-result writes, the next Q) and the score exchange across them are
    exercised many times per launch. Repeated launches must agree bit for bit (a block
    of partial scores read before it is fully staged shows up as run-to-run noise), and
    the sequences that end in a partial tile must match the oracle."""
    from attention_causal_gqa_b200.synthetic import mla_inputs
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 3000, 100).tolist()
    d = mla_inputs(len(lens), 128, 512, 64, seq_lens=lens, T_max=3072, seed=4, device="cuda")
    runs = [_run(d) for _ in range(4)]
    for o, l in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(l, runs[0][1])
    out, lse = runs[0]
    sl = d["seq_lens"].cpu().numpy()
    picks = [b for b in range(len(lens)) if lens[b] % 64 not in (0, 32)][:8]  # partial last tiles
    for b in picks:
        L = int(sl[b])
        ro, rl = mla_decode_ref(to_np(d["q_nope"][b:b + 1]), to_np(d["q_pe"][b:b + 1]),
                                to_np(d["kv_cache"][b:b + 1, :max(L, 1)]), to_np(d["pe_cache"][b:b + 1, :max(L, 1)]),
                                sl[b:b + 1], SCALE)
        check(out[b:b + 1], ro, lse[b:b + 1], rl, what=f"mla segments b={b} L={L}")


@cuda
@pytest.mark.parametrize("B,lo,hi,T_max,seed", [(1, 1, 5000, 5000, 31), (3, 0, 200, 257, 32), (74, 0, 1500, 1500, 33),
                                                 (150, 1, 130, 130, 34)])
def test_mla_random_layouts(B, lo, hi, T_max, seed):
    """Random batches (one sequence; fewer, as many as, and twice as many sequences as
    clusters; cache lengths that are not tile multiples): sampled sequences against the
    oracle, every output finite, empty sequences exactly 0 / -inf."""
    from attention_causal_gqa_b200.synthetic import mla_inputs
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, B).tolist()
    d = mla_inputs(B, 128, 512, 64, seq_lens=lens, T_max=T_max, seed=seed, device="cuda")
    out, lse = _run(d)
    assert torch.isfinite(out).all()
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(out[b] == 0) and torch.all(torch.isneginf(lse[b]))
    sl = d["seq_lens"].cpu().numpy()
    picks = sorted(set(rng.integers(0, B, 5).tolist()) | {0, B - 1})
    for b in picks:
        L = int(sl[b])
        if L == 0:
            continue
        ro, rl = mla_decode_ref(to_np(d["q_nope"][b:b + 1]), to_np(d["q_pe"][b:b + 1]),
                                to_np(d["kv_cache"][b:b + 1, :L]), to_np(d["pe_cache"][b:b + 1, :L]), sl[b:b + 1], SCALE)
        check(out[b:b + 1], ro, lse[b:b + 1], rl, what=f"mla random B={B} b={b} L={L}")
