"""GPU: the allocation-free paged decode entry point (attn_decode_paged_noalloc).

For callers that cannot allocate device memory: it keeps its split partials in a
fixed file-scope device array instead of a caller workspace. This file is named
to be collected last. The parity test calls the entry point through the C ABI twice
in a row (the array keeps the previous call's contents) and compares with
attn_decode_paged given its own workspace and with the float64 oracle, at the
tolerance of the other parity tests; device-side flags come back through
attn_decode_paged_noalloc_status.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import decode_paged_ref
from tests.parity import MAX_ABS, MEAN_ABS, LSE_REL, check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def _noalloc_fn():
    from attention_causal_gqa_b200.binding import lib
    f = lib.attn_decode_paged_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.restype = i32
    f.argtypes = [vp] * 7 + [i32] * 7 + [ctypes.c_float, i32, vp]
    return f, lib


def _call_noalloc(d, out, lse):
    f, lib = _noalloc_fn()
    B, Hq, D = d["q"].shape
    P, ps, Hkv, _ = d["k_pages"].shape
    rc = f(d["q"].data_ptr(), d["k_pages"].data_ptr(), d["v_pages"].data_ptr(), d["block_table"].data_ptr(),
           d["seq_lens"].data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, D, ps,
           d["block_table"].shape[1], P, 0.0, 1, torch.cuda.current_stream().cuda_stream)
    return rc, lib.attn_last_error().decode()


def _status():
    """Waits for the stream and returns the device flags of the last call (0 when clean)."""
    from attention_causal_gqa_b200.binding import lib
    g = lib.attn_decode_paged_noalloc_status
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    flags = ctypes.c_int(-1)
    rc = g(ctypes.byref(flags), torch.cuda.current_stream().cuda_stream)
    assert rc in (0, 5), lib.attn_last_error().decode()
    return flags.value


def _close(a, b, la, lb):
    a, b, la, lb = to_np(a), to_np(b), to_np(la), to_np(lb)
    err = np.abs(a - b)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
    fin = np.isfinite(lb)
    assert np.array_equal(np.isneginf(la), np.isneginf(lb))
    assert np.all(np.abs(la[fin] - lb[fin]) <= LSE_REL * np.maximum(1.0, np.abs(lb[fin])))


@cuda
def test_noalloc_matches_workspace_entry_point_twice():
    from attention_causal_gqa_b200 import attn_decode_paged
    from attention_causal_gqa_b200.synthetic import decode_inputs
    for seed, lens in ((1, [3000, 17, 0, 1200]), (2, [511, 4097, 64])):
        d = decode_inputs(len(lens), 32, 8, 128, seq_lens=lens, seed=seed, device="cuda")
        ref_o, ref_l = attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"])
        ora_o, ora_l = decode_paged_ref(to_np(d["q"]), to_np(d["k_pages"]), to_np(d["v_pages"]),
                                        d["block_table"].cpu().numpy(), d["seq_lens"].cpu().numpy())
        for _ in range(2):  # the second call runs over the first call's leftovers
            out = torch.full_like(d["q"], float("nan"))
            lse = torch.full((len(lens), 32), float("nan"), device="cuda")
            rc, msg = _call_noalloc(d, out, lse)
            assert rc == 0, msg
            assert _status() == 0
            _close(out, ref_o, lse, ref_l)
            check(out, ora_o, lse, ora_l, what="noalloc vs oracle")


@cuda
def test_noalloc_rejects_problems_beyond_the_array():
    from attention_causal_gqa_b200.synthetic import decode_inputs
    d = decode_inputs(2, 32, 8, 128, seq_lens=[40, 20], seed=3, device="cuda")
    # a block table wide enough to need more scratch than the fixed array holds
    d["block_table"] = torch.full((2, 1 << 16), -1, dtype=torch.int32, device="cuda")
    d["block_table"][0, :3] = torch.arange(3, device="cuda")
    d["block_table"][1, :2] = torch.arange(3, 5, device="cuda")
    out = torch.empty_like(d["q"])
    lse = torch.empty(2, 32, device="cuda")
    rc, msg = _call_noalloc(d, out, lse)
    assert rc == 3 and "scratch" in msg


@cuda
def test_noalloc_flags_a_bad_page_through_its_status_reader():
    """A block-table entry outside the page pool is clamped and flagged on the device; a
    caller of the allocation-free entry point sees the flag through its status reader,
    and the next clean call clears it."""
    from attention_causal_gqa_b200.synthetic import decode_inputs
    d = decode_inputs(2, 8, 2, 128, seq_lens=[40, 20], seed=5, device="cuda")
    d["block_table"][1, 0] = d["num_pages"] + 5  # outside the page pool
    out = torch.empty_like(d["q"])
    lse = torch.empty(2, 8, device="cuda")
    rc, msg = _call_noalloc(d, out, lse)
    assert rc == 0, msg
    assert _status() & 2  # ATTN_DEV_BAD_PAGE
    d2 = decode_inputs(2, 8, 2, 128, seq_lens=[40, 20], seed=6, device="cuda")
    rc, msg = _call_noalloc(d2, out, lse)
    assert rc == 0, msg
    assert _status() == 0
