"""GPU: device-side status and the library's own numerics checks.

The bounded-wait mechanism gives up on its own and the context stays usable; the
FMA-pipe exponential of the prefill softmax meets its stated bound against CUDA's
exp2f; rotated operands beyond the fp16 range are flagged (and served in bf16 on
request); the binding's check=True turns device flags into exceptions."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


@cuda
def test_wait_that_nothing_completes_times_out_with_a_status():
    from attention_causal_gqa_b200 import selftest_wait_timeout, attn_prefill
    flags = selftest_wait_timeout(50_000_000)  # 50 ms limit on an mbarrier nobody arrives at
    assert flags & 1
    # the CUDA context is still healthy: a normal call runs and gives finite results
    q = torch.randn(1, 2, 64, 64, device="cuda").bfloat16()
    out, lse = attn_prefill(q, q[:, :1].contiguous(), q[:, :1].contiguous())
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@cuda
def test_clean_call_reports_no_flags():
    from attention_causal_gqa_b200 import attn_prefill, read_status, prefill_workspace_size
    q = torch.randn(1, 4, 100, 128, device="cuda").bfloat16()
    k = torch.randn(1, 2, 100, 128, device="cuda").bfloat16()
    ws = torch.empty(prefill_workspace_size(1, 2, 100, 128), dtype=torch.uint8, device="cuda")
    attn_prefill(q, k, k, workspace=ws)
    assert read_status(ws) == 0


@cuda
def test_fma_exp2_meets_its_bound_against_exp2f():
    """The FMA-pipe exponential of the prefill softmax (attn_selftest_exp2) against the exact
    2^z and against CUDA's exp2f: a dense grid over [-126, 8] (the softmax feeds it
    z = s - m <= 8), both sides of every rounding boundary n +- 1/2, and the clamp below -126."""
    from attention_causal_gqa_b200.binding import selftest_exp2
    bound = 7.5e-5 + 2.0 ** -23  # the polynomial's error plus the final fp32 rounding
    grid = torch.linspace(-125.5, 8.0, 2_000_001, dtype=torch.float64).float()
    half = torch.arange(-125, 8, dtype=torch.float64) + 0.5
    edges = torch.cat([half, torch.nextafter(half, half + 1), torch.nextafter(half, half - 1)]).float()
    ints = torch.arange(-125, 9, dtype=torch.float32)
    z = torch.cat([grid, edges, ints]).cuda()
    y = selftest_exp2(z)
    exact = torch.exp2(z.double())
    rel = ((y.double() - exact) / exact).abs()
    assert float(rel.max()) <= bound, float(rel.max())
    cuda_exp2 = torch.exp2(z)  # CUDA's exp2f (a few ulp)
    rel_c = ((y.double() - cuda_exp2.double()) / cuda_exp2.double()).abs()
    assert float(rel_c.max()) <= bound + 4 * 2.0 ** -23
    # [-126, -125.5): results near the bottom of the normal range may be subnormal;
    # below -126 the argument is clamped: every result is that of -126
    tiny = 2.0 ** -126 * 2e-4
    zl = torch.linspace(-126.0, -125.5, 10_001, dtype=torch.float64).float().cuda()
    assert float((selftest_exp2(zl).double() - torch.exp2(zl.double())).abs().max()) <= tiny
    zc = torch.tensor([-126.0, -126.25, -127.0, -200.0, -1e4, -3.0e38], device="cuda")
    yc = selftest_exp2(zc).double()
    assert torch.all(yc == yc[0]) and abs(float(yc[0]) - 2.0 ** -126) <= tiny


def _big_pair(x, b, h, pos, value=1.0e5):
    """A pair (2i, 2i+1) of magnitude ~1e5 (representable in bf16, beyond fp16) at position
    0, where the rotation is the identity, so the rotated operand is out of fp16 range."""
    x[b, h, pos, 0] = value
    x[b, h, pos, 1] = -value
    return x


@cuda
def test_prefill_flags_rotated_values_beyond_fp16_and_serves_them_in_bf16():
    from attention_causal_gqa_b200 import attn_prefill, read_status, prefill_workspace_size
    from oracle import prefill_ref
    from tests.parity import MAX_ABS, MEAN_ABS, to_np
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 4, 96, 128, generator=g).bfloat16()
    k = torch.randn(1, 2, 96, 128, generator=g).bfloat16()
    v = torch.randn(1, 2, 96, 128, generator=g).bfloat16()
    q = _big_pair(q, 0, 1, 0).cuda()
    k, v = k.cuda(), v.cuda()
    ws = torch.empty(prefill_workspace_size(1, 2, 96, 128), dtype=torch.uint8, device="cuda")
    attn_prefill(q, k, v, workspace=ws)
    assert read_status(ws) & 8  # ATTN_DEV_RANGE: the fp16 operand could not hold the value
    # check=True re-runs with bf16 operands and leaves no flag
    out, lse = attn_prefill(q, k, v, workspace=ws, check=True)
    assert read_status(ws) == 0
    ro, rl = prefill_ref(to_np(q), to_np(k), to_np(v), causal=True, rope_theta=1e4)
    err = np.abs(to_np(out) - ro)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
    # bf16 operands round 8x coarser than fp16 ones: LSE within 1e-2 relative (floored at 1)
    lerr = np.abs(to_np(lse) - rl) / np.maximum(1.0, np.abs(rl))
    assert lerr.max() <= 1e-2


@cuda
def test_chunk_and_fp8_decode_flag_fp16_range_and_check_raises():
    from attention_causal_gqa_b200 import binding
    from attention_causal_gqa_b200.binding import AttnError
    from attention_causal_gqa_b200.synthetic import decode_inputs_fp8
    # chunked prefill: a new query pair beyond fp16 at the first new position of a sequence
    # with an empty cache (position 0: the rotation is the identity)
    g = torch.Generator().manual_seed(12)
    B, Hq, Hkv, D, S_new = 1, 4, 2, 128, 20
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)  # noqa: E731
    q, k, v = mk(B, Hq, S_new, D), mk(B, Hkv, S_new, D), mk(B, Hkv, S_new, D)
    q = _big_pair(q, 0, 2, 0)
    kp, vp = mk(4, 16, Hkv, D), mk(4, 16, Hkv, D)
    table = torch.tensor([[2, 0, 3]], dtype=torch.int32)
    cl = torch.tensor([0], dtype=torch.int32)
    dev = [t.cuda() for t in (q, k, v, kp, vp, table, cl)]
    ws = torch.empty(binding.prefill_chunk_workspace_size(B, Hkv, S_new, 16, D), dtype=torch.uint8, device="cuda")
    binding.attn_prefill_chunk(*dev, 16, workspace=ws)
    assert binding.read_status(ws) & 8
    with pytest.raises(AttnError) as e:
        binding.attn_prefill_chunk(*dev, 16, workspace=ws, check=True)
    assert e.value.code == 5 and "range" in str(e.value)
    # FP8 paged decode: the query is converted to fp16 for the products
    d = decode_inputs_fp8(2, 32, 8, 128, seq_lens=[33, 90], seed=13, device="cuda")
    d["q"][1, 5, 7] = 1.0e5
    ws = torch.empty(binding.decode_fp8_workspace_size(2, 32, 128, d["block_table"].shape[1]), dtype=torch.uint8,
                     device="cuda")
    args = (d["q"], d["k_pages"], d["v_pages"], d["k_scale"], d["v_scale"], d["block_table"], d["seq_lens"])
    binding.attn_decode_paged_fp8(*args, workspace=ws)
    assert binding.read_status(ws) & 8
    with pytest.raises(AttnError) as e:
        binding.attn_decode_paged_fp8(*args, workspace=ws, check=True)
    assert e.value.code == 5
