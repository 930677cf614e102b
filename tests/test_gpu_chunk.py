"""GPU parity: attn_prefill_chunk (append a chunk to the paged KV cache and attend) against
the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import apply_rope, chunk_prefill_ref, to_bf16
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def _setup(B, Hq, Hkv, D, cache_lens, S_new, seed, extra_pages=5):
    """Pages in a seeded random physical order; every slot (cached prefix and the rest)
    holds bf16 noise; new q/k/v in bf16."""
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    need = [(L + S_new + 15) // 16 for L in cache_lens]
    n_pages = sum(need) + extra_pages
    perm = rng.permutation(n_pages)
    maxp = max(need) + 1
    table = np.zeros((B, maxp), dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    return dict(q=mk(B, Hq, S_new, D), k=mk(B, Hkv, S_new, D), v=mk(B, Hkv, S_new, D),
                k_pages=mk(n_pages, 16, Hkv, D), v_pages=mk(n_pages, 16, Hkv, D),
                table=torch.from_numpy(table), cache_lens=torch.tensor(cache_lens, dtype=torch.int32))


def _run(d, theta, max_cache_len=None):
    from attention_causal_gqa_b200 import binding
    dev = {k: v.cuda() for k, v in d.items()}
    mcl = max(d["cache_lens"].tolist()) if max_cache_len is None else max_cache_len
    ws = torch.full((binding.prefill_chunk_workspace_size(d["q"].shape[0], d["k"].shape[1], d["q"].shape[2], mcl,
                                                          d["q"].shape[3]),), 255, dtype=torch.uint8, device="cuda")
    out, lse = binding.attn_prefill_chunk(dev["q"], dev["k"], dev["v"], dev["k_pages"], dev["v_pages"], dev["table"],
                                          dev["cache_lens"], mcl, rope_theta=theta, workspace=ws)
    torch.cuda.synchronize()
    return out, lse, dev, ws


def _within_one_bf16_step(a, b):
    """a and b (bf16 values) differ by at most one bf16 spacing of the larger magnitude
    (rounding of a rotation computed in fp32 versus fp64 may land on either neighbour)."""
    return bool(np.all(np.abs(a - b) <= np.maximum(np.abs(a), np.abs(b)) * 2.0 ** -7 + 1e-30))


@cuda
@pytest.mark.parametrize("B,Hq,Hkv,D,cache_lens,S_new,theta", [
    (3, 8, 2, 128, [0, 100, 1000], 77, 1e4),     # G=4, empty and long caches, ragged chunk
    (2, 4, 4, 64, [33, 0], 300, 1e4),            # G=1 (row-pair work items), several query tiles
    (2, 32, 8, 128, [500, 17], 1, 1e4),          # one new token (decode-shaped)
    (2, 6, 2, 128, [200, 64], 129, 0.0),         # no RoPE, G=3
    (1, 16, 8, 128, [1535], 513, 1e6),           # long cache, chunk over five query tiles
])
def test_chunk_prefill_matches_oracle(B, Hq, Hkv, D, cache_lens, S_new, theta):
    d = _setup(B, Hq, Hkv, D, cache_lens, S_new, seed=S_new * 7 + B)
    out, lse, dev, ws = _run(d, theta)
    kp, vp, ro, rl = chunk_prefill_ref(to_np(d["q"]), to_np(d["k"]), to_np(d["v"]), to_np(d["k_pages"]),
                                       to_np(d["v_pages"]), d["table"].numpy(), cache_lens, rope_theta=theta)
    check(out, ro, lse, rl, what=f"chunk {B},{Hq},{Hkv},{D},{cache_lens},{S_new}")
    from attention_causal_gqa_b200 import binding
    assert binding.read_status(ws) == 0
    got_k, got_v = to_np(dev["k_pages"]), to_np(dev["v_pages"])
    assert np.array_equal(got_v, vp)                  # values stored exactly; untouched slots unchanged
    assert _within_one_bf16_step(got_k, kp)           # keys rotated in fp32 on the GPU, fp64 in the oracle


@cuda
def test_chunk_last_row_agrees_with_paged_decode_on_the_updated_cache():
    from attention_causal_gqa_b200 import binding
    B, Hq, Hkv, D, S_new = 2, 32, 8, 128, 40
    cache_lens = [300, 1000]
    d = _setup(B, Hq, Hkv, D, cache_lens, S_new, seed=5)
    out, lse, dev, _ = _run(d, 1e4)
    q_last = np.stack([apply_rope(to_np(d["q"][b, :, -1]), 1e4, positions=np.full(Hq, cache_lens[b] + S_new - 1))
                       for b in range(B)])
    qd = torch.from_numpy(q_last).to(torch.bfloat16).cuda()
    lens = torch.tensor([c + S_new for c in cache_lens], dtype=torch.int32, device="cuda")
    do, dl = binding.attn_decode_paged(qd, dev["k_pages"], dev["v_pages"], dev["table"], lens)
    torch.cuda.synchronize()
    # the decode query was rounded to bf16 after rotation: agreement within the bf16 tolerances
    assert (out[:, :, -1].float() - do.float()).abs().max().item() <= 2e-2
    assert ((lse[:, :, -1] - dl).abs() / dl.abs().clamp(min=1)).max().item() <= 5e-3


@cuda
def test_chunk_bad_page_is_flagged_not_faulted():
    from attention_causal_gqa_b200 import binding
    d = _setup(1, 4, 2, 64, [20], 30, seed=9)
    d["table"][0, 2] = 10 ** 6  # the page of positions 32..47 lies outside the pool
    out, lse, dev, ws = _run(d, 1e4)
    assert binding.read_status(ws) & 2


@cuda
@pytest.mark.parametrize("B,Hq,Hkv,D,cache_lens,S_new,fscale,layout", [
    (2, 8, 2, 128, [0, 300], 77, 1.0, "half"),          # half-split pairs
    (2, 4, 4, 64, [33, 200], 129, 0.25, "half"),        # D = 64, frequencies scaled
    (1, 8, 2, 128, [500], 64, 0.5, "interleaved"),      # interpolated positions
])
def test_chunk_prefill_rope_variants(B, Hq, Hkv, D, cache_lens, S_new, fscale, layout):
    from attention_causal_gqa_b200 import binding
    d = _setup(B, Hq, Hkv, D, cache_lens, S_new, seed=S_new * 11 + D)
    dev = {k: v.cuda() for k, v in d.items()}
    mcl = max(cache_lens)
    ws = torch.empty(binding.prefill_chunk_workspace_size(B, Hkv, S_new, mcl, D), dtype=torch.uint8, device="cuda")
    out, lse = binding.attn_prefill_chunk(dev["q"], dev["k"], dev["v"], dev["k_pages"], dev["v_pages"], dev["table"],
                                          dev["cache_lens"], mcl, rope_theta=1e4, workspace=ws,
                                          rope_freq_scale=fscale, rope_layout=layout)
    torch.cuda.synchronize()
    kp, vp, ro, rl = chunk_prefill_ref(to_np(d["q"]), to_np(d["k"]), to_np(d["v"]), to_np(d["k_pages"]),
                                       to_np(d["v_pages"]), d["table"].numpy(), cache_lens, rope_theta=1e4,
                                       rope_freq_scale=fscale, rope_layout=layout)
    check(out, ro, lse, rl, what=f"chunk rope {fscale} {layout} D={D}")
    assert binding.read_status(ws) == 0
    assert np.array_equal(to_np(dev["v_pages"]), vp)
    assert _within_one_bf16_step(to_np(dev["k_pages"]), kp)


@cuda
@pytest.mark.parametrize("B,Hq,Hkv,D,cache_lens,S_new,new_lens,theta", [
    (4, 8, 2, 128, [0, 100, 1000, 37], 300, [300, 0, 129, 1], 1e4),   # full, empty, ragged, one token
    (3, 4, 4, 64, [33, 0, 500], 200, [128, 200, 127], 1e6),            # G = 1 items, tile edges
    (2, 6, 2, 128, [64, 5], 130, [65, 130], 0.0),                      # no RoPE, G = 3
])
def test_chunk_prefill_varlen_matches_oracle(B, Hq, Hkv, D, cache_lens, S_new, new_lens, theta):
    """Chunks of different lengths padded to S_new (attn_prefill_chunk_varlen): appended
    pages, outputs and LSE against the oracle; rows past a chunk are exactly 0 / -inf and
    pages a sequence does not reach stay as they were (the padding rows are poisoned)."""
    from attention_causal_gqa_b200 import binding
    d = _setup(B, Hq, Hkv, D, cache_lens, S_new, seed=S_new * 13 + B)
    for b, n in enumerate(new_lens):  # padding rows hold NaN: they must never be read
        d["q"][b, :, n:] = float("nan")
        d["k"][b, :, n:] = float("nan")
        d["v"][b, :, n:] = float("nan")
    dev = {k: v.cuda() for k, v in d.items()}
    nl = torch.tensor(new_lens, dtype=torch.int32, device="cuda")
    mcl = max(cache_lens)
    ws = torch.empty(binding.prefill_chunk_workspace_size(B, Hkv, S_new, mcl, D), dtype=torch.uint8, device="cuda")
    out, lse = binding.attn_prefill_chunk(dev["q"], dev["k"], dev["v"], dev["k_pages"], dev["v_pages"], dev["table"],
                                          dev["cache_lens"], mcl, rope_theta=theta, workspace=ws, new_lens=nl)
    torch.cuda.synchronize()
    kp, vp, ro, rl = chunk_prefill_ref(to_np(d["q"]), to_np(d["k"]), to_np(d["v"]), to_np(d["k_pages"]),
                                       to_np(d["v_pages"]), d["table"].numpy(), cache_lens, rope_theta=theta,
                                       new_lens=new_lens)
    check(out, ro, lse, rl, what=f"chunk varlen {new_lens}")
    for b, n in enumerate(new_lens):
        assert torch.all(out[b, :, n:] == 0) and torch.all(torch.isneginf(lse[b, :, n:]))
    assert binding.read_status(ws) == 0
    assert np.array_equal(to_np(dev["v_pages"]), vp)
    assert _within_one_bf16_step(to_np(dev["k_pages"]), kp)
