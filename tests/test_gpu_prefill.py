"""GPU parity: attn_prefill (C-ABI via the binding) against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import prefill_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def _run(q, k, v, causal=True, theta=1e4, scale=None):
    from attention_causal_gqa_b200 import attn_prefill
    out, lse = attn_prefill(q, k, v, causal=causal, rope_theta=theta, scale=scale)
    torch.cuda.synchronize()
    return out, lse


def _inputs(B, Hq, Hkv, S, D, dtype="bf16", std=1.0, seed=0):
    from attention_causal_gqa_b200.synthetic import prefill_inputs
    return prefill_inputs(B, Hq, Hkv, S, D, dtype=dtype, std=std, seed=seed, device="cuda")


@cuda
@pytest.mark.parametrize(
    "B,Hq,Hkv,S,D,dtype,causal,theta",
    [
        (1, 4, 4, 256, 64, "f32", True, 1e4),      # MHA fp32 (tf32 tensor cores), the small workload
        (1, 8, 2, 300, 128, "bf16", True, 1e4),    # GQA G=4, ragged tail
        (2, 4, 1, 129, 128, "bf16", True, 1e4),    # MQA, one row past a tile
        (1, 3, 3, 200, 64, "bf16", True, 1e4),     # MHA (G=1): row-pair work items, odd row blocks
        (1, 6, 2, 257, 64, "bf16", True, 500.0),   # G=3 (odd), ragged
        (1, 4, 2, 1, 128, "bf16", True, 1e4),      # S = 1
        (1, 4, 2, 384, 128, "bf16", False, 1e4),   # non-causal
        (1, 4, 4, 160, 64, "f32", False, 0.0),     # fp32, no RoPE, non-causal, ragged
        (3, 16, 8, 640, 128, "bf16", True, 1e6),   # G=2, theta 1e6, several tiles
        (1, 2, 1, 1000, 128, "bf16", True, 1e4),   # long row pair, many KV tiles
        (1, 4, 2, 333, 128, "bf16", True, 0.0),    # bf16 without RoPE (Q read straight from q), ragged
        (2, 8, 8, 200, 64, "bf16", False, 0.0),    # bf16 without RoPE, D=64, non-causal
        (2, 32, 8, 768, 128, "bf16", True, 1e4),   # 192 work items: CTAs of the persistent grid take two
        (2, 32, 8, 640, 64, "bf16", False, 0.0),   # 160 work items, no RoPE, D=64, non-causal
    ],
)
def test_prefill_matches_oracle_small(B, Hq, Hkv, S, D, dtype, causal, theta):
    q, k, v = _inputs(B, Hq, Hkv, S, D, dtype, seed=B * 1000 + S)
    out, lse = _run(q, k, v, causal=causal, theta=theta)
    ro, rl = prefill_ref(to_np(q), to_np(k), to_np(v), causal=causal, rope_theta=theta)
    check(out, ro, lse, rl, what=f"prefill {B},{Hq},{Hkv},{S},{D},{dtype},{causal}")


def _sample_rows(B, Hq, S, n, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(B):
        for h in (0, Hq - 1):
            for i in (0, 1, 127, 128, 129, 255, 256, S // 2, S - 129, S - 128, S - 2, S - 1):
                if 0 <= i < S:
                    rows.add((b, h, i))
    while len(rows) < n:
        rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(S))))
    return sorted(rows)


@cuda
@pytest.mark.parametrize("name,nrows", [("gqa_prefill_b2_hq32_hkv8_s4096_d128", 160),
                                        ("gqa_prefill_b1_hq32_hkv8_s32768_d128", 64)])
def test_prefill_full_size_sampled_rows(name, nrows):
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    p = WORKLOADS[name].params
    q, k, v = workload_inputs(name, device="cuda")
    out, lse = _run(q, k, v, causal=True, theta=p["theta"], scale=p["scale"])
    rows = _sample_rows(p["B"], p["Hq"], p["S"], nrows, seed=7)
    idx = torch.tensor(rows, device="cuda")
    o_s = out[idx[:, 0], idx[:, 1], idx[:, 2]]
    l_s = lse[idx[:, 0], idx[:, 1], idx[:, 2]]
    ro, rl = prefill_ref(to_np(q), to_np(k), to_np(v), causal=True, rope_theta=p["theta"], scale=p["scale"],
                         rows=rows)
    check(o_s, ro, l_s, rl, what=name)
    # every output finite; every LSE within the trivial bounds of a causal row
    assert torch.isfinite(out).all()
    assert torch.isfinite(lse).all()


@cuda
def test_prefill_deterministic_and_poison_free():
    q, k, v = _inputs(1, 8, 2, 700, 128, seed=3)
    o1, l1 = _run(q, k, v)
    o2, l2 = _run(q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@cuda
def test_prefill_rejects_bad_arguments():
    from attention_causal_gqa_b200 import AttnError, attn_prefill
    q, k, v = _inputs(1, 6, 4, 64, 128)  # 6 % 4 != 0
    with pytest.raises(AttnError) as e:
        attn_prefill(q, k, v)
    assert e.value.code == 1
    q, k, v = _inputs(1, 4, 4, 64, 96)   # D = 96 unsupported
    with pytest.raises(AttnError) as e:
        attn_prefill(q, k, v)
    assert e.value.code == 2


@cuda
@pytest.mark.parametrize(
    "B,Hq,Hkv,S,D,dtype,causal,theta,fscale,layout",
    [
        (1, 8, 2, 300, 128, "bf16", True, 1e4, 0.25, "interleaved"),   # positions interpolated by 4
        (1, 8, 2, 300, 128, "bf16", True, 1e4, 1.0, "half"),           # half-split pairs
        (2, 4, 4, 257, 64, "bf16", False, 500.0, 0.5, "half"),          # D = 64, non-causal
        (1, 4, 4, 200, 64, "f32", True, 1e4, 1.0, "half"),             # fp32 operands (hi/lo split)
        (1, 4, 2, 640, 128, "bf16", True, 8.1e4, 2.0, "half"),         # an NTK-style base, frequencies stretched
    ],
)
def test_prefill_rope_variants(B, Hq, Hkv, S, D, dtype, causal, theta, fscale, layout):
    from attention_causal_gqa_b200 import attn_prefill
    q, k, v = _inputs(B, Hq, Hkv, S, D, dtype, seed=B * 7 + S)
    out, lse = attn_prefill(q, k, v, causal=causal, rope_theta=theta, rope_freq_scale=fscale, rope_layout=layout)
    torch.cuda.synchronize()
    ro, rl = prefill_ref(to_np(q), to_np(k), to_np(v), causal=causal, rope_theta=theta, rope_freq_scale=fscale,
                         rope_layout=layout)
    check(out, ro, lse, rl, what=f"prefill rope {fscale} {layout} {dtype} D={D}")
