"""GPU: the bounded-wait mechanism gives up on its own and the context stays usable."""
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
