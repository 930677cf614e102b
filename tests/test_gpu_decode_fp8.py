"""GPU parity: attn_decode_paged_fp8 (paged decode over an E4M3 cache with per-(page, head)
scales) against the float64 oracle over the dequantised cache, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import decode_paged_fp8_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def _run(d, ws=None):
    from attention_causal_gqa_b200 import binding
    out, lse = binding.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"], d["v_scale"],
                                             d["block_table"], d["seq_lens"], workspace=ws)
    torch.cuda.synchronize()
    return out, lse


def _oracle(d, pairs=None):
    return decode_paged_fp8_ref(to_np(d["q"]), d["k_pages"].cpu().numpy(), d["v_pages"].cpu().numpy(),
                                d["k_scale"].cpu().numpy(), d["v_scale"].cpu().numpy(),
                                d["block_table"].cpu().numpy(), d["seq_lens"].cpu().numpy(), pairs=pairs)


@cuda
@pytest.mark.parametrize("lens,Hq,Hkv", [
    ([1, 15, 16, 17, 511, 512, 513, 1000], 32, 8),
    ([5, 300, 2049], 8, 8),      # G = 1
    ([700, 33], 4, 1),           # MQA
    ([257, 4096], 32, 2),        # G = 16
    ([33, 800, 1601], 48, 8),    # G = 6: a lane's second head column past the group
    ([100, 1500], 12, 1),        # G = 12: the second 8-head tile half used
])
@pytest.mark.parametrize("D", [128, 64])
def test_fp8_decode_matches_oracle(lens, Hq, Hkv, D):
    from attention_causal_gqa_b200.synthetic import decode_inputs_fp8
    d = decode_inputs_fp8(len(lens), Hq, Hkv, D, seq_lens=lens, seed=len(lens) * 31 + Hq + D, device="cuda",
                          extra_pages=3)
    out, lse = _run(d)
    ro, rl = _oracle(d)
    check(out, ro, lse, rl, what=f"fp8 decode {lens},{Hq},{Hkv},D={D}")


@cuda
@pytest.mark.parametrize("D", [128, 64])
def test_fp8_decode_empty_sequence_and_poisoned_tail(D):
    from attention_causal_gqa_b200.synthetic import decode_inputs_fp8
    lens = [0, 37, 70]
    d = decode_inputs_fp8(3, 16, 4, D, seq_lens=lens, seed=12, device="cuda")
    ro, rl = _oracle(d)
    # slots past each length hold the largest finite code: they must not reach the result
    bt = d["block_table"].cpu().numpy()
    for b, L in enumerate(lens):
        if L % 16:
            page = int(bt[b, L // 16])
            d["v_pages"][page, L % 16:] = 0x7E
            d["k_pages"][page, L % 16:] = 0x7E
    out, lse = _run(d)
    check(out, ro, lse, rl, what="fp8 decode poison")
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@cuda
@pytest.mark.parametrize("D", [128, 64])
def test_fp8_decode_full_size_sampled(D):
    from attention_causal_gqa_b200.synthetic import decode_inputs_fp8
    d = decode_inputs_fp8(64, 32, 8, D, seed=20261202, device="cuda")
    out, lse = _run(d)
    rng = np.random.default_rng(4)
    bs = sorted({int(x) for x in rng.integers(0, 64, size=6)} | {0, 63})
    pairs = [(b, h) for b in bs for h in (0, 5, 31)]
    ro, rl = _oracle(d, pairs)
    idx = torch.tensor(pairs, device="cuda")
    check(out[idx[:, 0], idx[:, 1]], ro, lse[idx[:, 0], idx[:, 1]], rl, what=f"fp8 decode full D={D}")
