"""GPU: the sequence split of decode and MLA on one device, with the CUDA kernels as
each slice's attention and attn_lse_merge combining the partials, against the float64
oracle of the unsplit problem (the multi-GPU path minus the all-gather)."""
import numpy as np
import pytest
import torch

from oracle import decode_paged_ref, mla_decode_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


@cuda
@pytest.mark.parametrize("world", [2, 3])
def test_decode_split_over_slices_merges_to_the_oracle(world):
    from attention_causal_gqa_b200 import binding, sharding
    from attention_causal_gqa_b200.synthetic import decode_inputs
    lens = [1, 17, 3000, 0, 1024, 5000]
    d = decode_inputs(len(lens), 32, 8, 128, seq_lens=lens, seed=41, device="cuda")
    outs, lses = [], []
    for r in range(world):
        table, lr = sharding.local_block_table(d["block_table"], d["seq_lens"], r, world)
        o, l = binding.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], table, lr)
        outs.append(o)
        lses.append(l)
    out, lse = binding.lse_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    ro, rl = decode_paged_ref(to_np(d["q"]), to_np(d["k_pages"]), to_np(d["v_pages"]), d["block_table"].cpu().numpy(),
                              d["seq_lens"].cpu().numpy())
    check(out, ro, lse, rl, what=f"decode split x{world}")
    assert torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))


@cuda
def test_mla_split_over_a_sharded_cache_merges_to_the_oracle():
    from attention_causal_gqa_b200 import binding, sharding
    from attention_causal_gqa_b200.synthetic import mla_inputs
    lens = [2000, 65, 1, 700]
    m = mla_inputs(len(lens), 128, 512, 64, seq_lens=lens, T_max=2048, seed=42, device="cuda")
    sc = 1.0 / np.sqrt(192)
    outs, lses = [], []
    for r in range(2):
        sl = [sharding.kv_slice(L, r, 2, 64) for L in lens]
        tl = max(64, max(n for _, n in sl))
        kv = torch.zeros((len(lens), tl, 512), dtype=torch.bfloat16, device="cuda")
        pe = torch.zeros((len(lens), tl, 64), dtype=torch.bfloat16, device="cuda")
        for b, (s0, n) in enumerate(sl):
            kv[b, :n] = m["kv_cache"][b, s0:s0 + n]
            pe[b, :n] = m["pe_cache"][b, s0:s0 + n]
        lr = torch.tensor([n for _, n in sl], dtype=torch.int32, device="cuda")
        o, l = binding.mla_decode(m["q_nope"], m["q_pe"], kv, pe, lr, sc)
        outs.append(o)
        lses.append(l)
    out, lse = binding.lse_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    ro, rl = mla_decode_ref(to_np(m["q_nope"]), to_np(m["q_pe"]), to_np(m["kv_cache"]), to_np(m["pe_cache"]),
                            m["seq_lens"].cpu().numpy(), sc)
    check(out, ro, lse, rl, what="mla split x2")
