"""GPU parity: attn_decode_paged (C-ABI via the binding) against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import decode_paged_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def _run(d, scale=None):
    from attention_causal_gqa_b200 import attn_decode_paged
    out, lse = attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], scale=scale)
    torch.cuda.synchronize()
    return out, lse


def _oracle(d, pairs=None, scale=None):
    bt = d["block_table"].cpu().numpy()
    sl = d["seq_lens"].cpu().numpy()
    if pairs is None:
        return decode_paged_ref(to_np(d["q"]), to_np(d["k_pages"]), to_np(d["v_pages"]), bt, sl, scale=scale)
    # only the pages of the sampled sequences come back to the host
    bs = sorted({b for b, _ in pairs})
    outs, lses = [], []
    for b in bs:
        n = int(math.ceil(int(sl[b]) / 16))
        ids = torch.from_numpy(bt[b, :n].astype(np.int64)).to(d["k_pages"].device)
        kp, vp = to_np(d["k_pages"][ids]), to_np(d["v_pages"][ids])
        table = np.arange(n)[None, :]
        hs = [h for bb, h in pairs if bb == b]
        o, l = decode_paged_ref(to_np(d["q"][b:b + 1]), kp, vp, table, sl[b:b + 1], scale=scale,
                                pairs=[(0, h) for h in hs])
        outs.append(o)
        lses.append(l)
    order = [(b, h) for b in bs for h in [h for bb, h in pairs if bb == b]]
    return np.concatenate(outs), np.concatenate(lses), order


@cuda
@pytest.mark.parametrize(
    "lens,Hq,Hkv,D",
    [
        ([1, 15, 16, 17, 511, 512, 513, 1000], 32, 8, 128),
        ([5, 300, 2049], 8, 8, 128),     # MHA-shaped (G = 1)
        ([700, 33], 4, 1, 128),          # MQA
        ([1200, 64, 9], 16, 2, 64),      # G = 8, D = 64
        ([257, 4096], 32, 2, 128),       # G = 16
        ([3000, 1, 64], 32, 32, 128),    # MHA with 32 KV heads: four 8-head TMA groups
        ([900, 17], 12, 12, 64),         # 12 KV heads: the second group is half past the end
        ([1500, 40], 32, 1, 128),        # MQA with 32 query heads: two 16-row query tiles
        ([2000, 100], 40, 2, 128),       # G = 20: a full and a partial query tile
    ],
)
def test_decode_matches_oracle_small(lens, Hq, Hkv, D):
    from attention_causal_gqa_b200.synthetic import decode_inputs
    d = decode_inputs(len(lens), Hq, Hkv, D, seq_lens=lens, seed=sum(lens), device="cuda", extra_pages=3)
    out, lse = _run(d)
    ro, rl = _oracle(d)
    check(out, ro, lse, rl, what=f"decode {lens} {Hq}/{Hkv} D{D}")


@cuda
def test_decode_empty_sequence_and_poison():
    from attention_causal_gqa_b200.synthetic import decode_inputs
    lens = [0, 37, 16, 1]
    d = decode_inputs(len(lens), 32, 8, 128, seq_lens=lens, seed=11, device="cuda")
    ro, rl = _oracle(d)
    # poison every slot past each sequence end, and the table entries past the end
    bt = d["block_table"].cpu().numpy()
    for b, L in enumerate(lens):
        if L % 16:
            pg = int(bt[b, L // 16])
            d["k_pages"][pg, L % 16:] = float("nan")
            d["v_pages"][pg, L % 16:] = float("nan")
    d["block_table"][d["block_table"] < 0] = 2 ** 30
    out, lse = _run(d)
    check(out, ro, lse, rl, what="decode poison")
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@cuda
def test_decode_full_size_sampled():
    from attention_causal_gqa_b200.synthetic import workload_inputs, WORKLOADS
    name = "paged_decode_b64_hq32_hkv8_d128"
    p = WORKLOADS[name].params
    d = workload_inputs(name, device="cuda")
    out, lse = _run(d, scale=p["scale"])
    rng = np.random.default_rng(5)
    pairs = sorted({(int(rng.integers(p["B"])), int(rng.integers(p["Hq"]))) for _ in range(48)} | {(0, 0), (63, 31)})
    ro, rl, order = _oracle(d, pairs, scale=p["scale"])
    idx = torch.tensor(order, device="cuda")
    check(out[idx[:, 0], idx[:, 1]], ro, lse[idx[:, 0], idx[:, 1]], rl, what=name)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


@cuda
def test_decode_bad_page_is_flagged_not_faulted():
    from attention_causal_gqa_b200 import attn_decode_paged, read_status, decode_workspace_size
    from attention_causal_gqa_b200.synthetic import decode_inputs
    d = decode_inputs(2, 8, 2, 128, seq_lens=[40, 20], seed=2, device="cuda")
    d["block_table"][1, 0] = d["num_pages"] + 5  # outside the page pool
    ws = torch.empty(decode_workspace_size(2, 8, 128, d["max_pages_per_seq"]), dtype=torch.uint8, device="cuda")
    attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], workspace=ws)
    assert read_status(ws) & 2
    # the context is still usable
    d2 = decode_inputs(1, 8, 2, 128, seq_lens=[40], seed=3, device="cuda")
    out, lse = _run(d2)
    ro, rl = _oracle(d2)
    check(out, ro, lse, rl, what="after flagged call")


@cuda
def test_decode_deterministic():
    from attention_causal_gqa_b200.synthetic import decode_inputs
    d = decode_inputs(4, 32, 8, 128, seq_lens=[3000, 17, 900, 5000], seed=4, device="cuda")
    o1, l1 = _run(d)
    o2, l2 = _run(d)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
