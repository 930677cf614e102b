"""GPU parity: DeepSeek sparse attention (dsa_index_topk, dsa_mla_decode) against the float64
oracle, through the C ABI.

The top-k decision is taken on the kernel's fp32 index scores, so the selection is checked
exactly against those scores (the same precision on both sides), the scores themselves
against the oracle's within a bound derived from fp32 accumulation, and the attention
output against the oracle run on the selected tokens."""
import math

import numpy as np
import pytest
import torch

from oracle import dsa_index_scores_ref, dsa_mla_decode_ref, dsa_topk_ref
from tests.parity import check, to_np

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")
SCALE = 1.0 / math.sqrt(192)
# fp32 sums of 128 products per head, then of <= 64 weighted heads: a relative bound on
# the magnitude sum_j |w_j| sum_i |q_ji k_si| with ample room over 200 roundings of 2^-24
SCORE_REL = 5e-5


def _index(d, top_k):
    from attention_causal_gqa_b200 import dsa_index_topk
    s, ix = dsa_index_topk(d["q_idx"], d["w_idx"], d["k_idx"], d["seq_lens"], top_k)
    torch.cuda.synchronize()
    return s, ix


def _check_scores(d, scores, rows=None):
    sl = d["seq_lens"].cpu().numpy()
    rows = range(len(sl)) if rows is None else rows
    q, w = to_np(d["q_idx"]), to_np(d["w_idx"])
    for b in rows:
        L = int(sl[b])
        k = to_np(d["k_idx"][b])
        ref = dsa_index_scores_ref(q[b:b + 1], w[b:b + 1], k[None], [L])[0]
        got = scores[b].cpu().numpy().astype(np.float64)
        assert np.all(np.isneginf(got[L:])), f"b={b}: scores past the length must be -inf"
        if L:
            mag = np.abs(w[b]) @ (np.abs(q[b]) @ np.abs(k[:L]).T)
            err = np.abs(got[:L] - ref[:L])
            assert np.all(err <= SCORE_REL * mag + 1e-6), f"b={b}: index score error {float((err / (mag + 1e-6)).max()):.2e}"


def _check_selection(scores, idx, lens, top_k, rows=None):
    """The kernel's selection is exactly the top-k of its own scores (ties: smaller index)."""
    rows = range(len(lens)) if rows is None else rows
    for b in rows:
        L = int(lens[b])
        want = dsa_topk_ref(scores[b:b + 1].cpu().numpy().astype(np.float64), [L], top_k)[0]
        got = idx[b].cpu().numpy()
        n = len(want)
        assert np.array_equal(got[:n], want), f"b={b}: selection differs from the top-{top_k} of the kernel's scores"
        assert np.all(got[n:] == -1)


def _oracle_out(d, idx, pairs=None, compact=False):
    """The oracle on the kernel's selection. compact: hand it only the selected rows
    (gathered here with torch indexing, a copy) so a full-size cache need not be converted."""
    sl = d["seq_lens"].cpu().numpy()
    n = [min(int(L), idx.shape[1]) for L in sl]
    if not compact:
        ix = [idx[b, :n[b]].cpu().numpy().astype(np.int64) for b in range(len(sl))]
        return dsa_mla_decode_ref(to_np(d["q_nope"]), to_np(d["q_pe"]), to_np(d["kv_cache"]), to_np(d["pe_cache"]),
                                  ix, SCALE, pairs=pairs)
    t = max([1] + n)
    kv = np.zeros((len(sl), t, d["kv_cache"].shape[2]))
    pe = np.zeros((len(sl), t, d["pe_cache"].shape[2]))
    for b in sorted({b for b, _ in pairs}):
        sel = idx[b, :n[b]].long()
        kv[b, :n[b]] = to_np(d["kv_cache"][b, sel])
        pe[b, :n[b]] = to_np(d["pe_cache"][b, sel])
    return dsa_mla_decode_ref(to_np(d["q_nope"]), to_np(d["q_pe"]), kv, pe, [np.arange(m) for m in n], SCALE,
                              pairs=pairs)


@cuda
@pytest.mark.parametrize("lens,T,HI,top_k", [
    ([1, 63, 64, 65, 1000], 1000, 64, 100),   # ragged blocks, short sequences keep everything
    ([3000, 0, 2048, 700], 3072, 16, 512),    # one indexer warp, an empty sequence
    ([1500, 1499], 1536, 48, 1499),           # top_k at the length boundary
])
def test_index_scores_and_selection(lens, T, HI, top_k):
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    d = dsa_inputs(len(lens), 128, 512, 64, HI, 128, seq_lens=lens, T_max=T, seed=T + HI, device="cuda")
    scores, idx = _index(d, top_k)
    _check_scores(d, scores)
    _check_selection(scores, idx, lens, top_k)
    # against the oracle's scores: nothing left out scores clearly above what was kept
    ref = dsa_index_scores_ref(to_np(d["q_idx"]), to_np(d["w_idx"]), to_np(d["k_idx"]), lens)
    for b, L in enumerate(lens):
        n = min(L, top_k)
        if 0 < n < L:
            kept = np.zeros(L, bool)
            kept[idx[b, :n].cpu().numpy()] = True
            mag = float(np.abs(ref[b, :L]).max()) + 1.0
            assert ref[b, :L][kept].min() >= ref[b, :L][~kept].max() - 1e-4 * mag


@cuda
def test_many_short_sequences():
    """300 sequences of 0-700 tokens: the indexer's CTAs each walk many sequences (a new
    Q and head weights per segment) and the top-k clusters meet every short-sequence case."""
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    rng = np.random.default_rng(12)
    lens = rng.integers(0, 701, 300).tolist()
    d = dsa_inputs(len(lens), 128, 512, 64, 32, 128, seq_lens=lens, T_max=704, seed=12, device="cuda")
    scores, idx = _index(d, 64)
    _check_scores(d, scores)
    _check_selection(scores, idx, lens, 64)


@cuda
def test_selection_ties_take_the_smaller_index():
    """Identical key rows give bit-identical scores; the kept ones must be the earliest."""
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    lens = [700, 300]
    d = dsa_inputs(2, 128, 512, 64, 32, 128, seq_lens=lens, T_max=768, seed=5, device="cuda")
    d["k_idx"][0, 100:600] = d["k_idx"][0, 50]  # 501 tokens share one score
    d["k_idx"][1, :] = d["k_idx"][1, 7]         # every token ties
    scores, idx = _index(d, 64)
    _check_selection(scores, idx, lens, 64)
    assert idx[1].cpu().tolist() == list(range(64))


@cuda
@pytest.mark.parametrize("lens,T,top_k", [([40, 900, 2000], 2048, 256), ([33, 0, 1025], 1088, 1024)])
def test_sparse_mla_matches_oracle(lens, T, top_k):
    from attention_causal_gqa_b200 import dsa_mla_decode
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    d = dsa_inputs(len(lens), 128, 512, 64, 64, 128, seq_lens=lens, T_max=T, seed=T + top_k, device="cuda")
    scores, idx = _index(d, top_k)
    out, lse = dsa_mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], idx, SCALE)
    torch.cuda.synchronize()
    ro, rl = _oracle_out(d, idx)
    check(out, ro, lse, rl, what=f"dsa {lens}")


@cuda
def test_sparse_mla_with_every_token_kept_equals_dense_mla():
    from attention_causal_gqa_b200 import dsa_mla_decode, mla_decode
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    lens = [500, 1000, 3]
    d = dsa_inputs(3, 128, 512, 64, 64, 128, seq_lens=lens, T_max=1024, seed=77, device="cuda")
    _, idx = _index(d, 1024)
    out, lse = dsa_mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], idx, SCALE)
    dout, dlse = mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], SCALE)
    torch.cuda.synchronize()
    # the same tokens in the same order: the same kernel sees identical operands
    assert torch.equal(out, dout) and torch.equal(lse, dlse)


@cuda
def test_bad_index_is_flagged_not_read():
    from attention_causal_gqa_b200 import binding
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    lens = [300, 200]
    d = dsa_inputs(2, 128, 512, 64, 16, 128, seq_lens=lens, T_max=320, seed=8, device="cuda")
    _, idx = _index(d, 64)
    idx[1, 5] = 250  # past that sequence's 200 tokens
    ws = torch.empty(binding.dsa_mla_workspace_size(2, 128, 512, 64, 64), dtype=torch.uint8, device="cuda")
    out, lse = binding.dsa_mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], idx,
                                      SCALE, workspace=ws)
    assert binding.read_status(ws) & binding.ATTN_DEV_BAD_INDEX
    assert torch.isfinite(out.float()).all()


@cuda
def test_dsa_full_size_sampled():
    from attention_causal_gqa_b200 import dsa_mla_decode
    from attention_causal_gqa_b200.synthetic import WORKLOADS, workload_inputs
    name = "dsa_mla_decode_b32_h128_dc512_dr64_hi64_di128_top2048"
    p = WORKLOADS[name].params
    d = workload_inputs(name, seed=20261202, device="cuda")
    scores, idx = _index(d, p["top_k"])
    out, lse = dsa_mla_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["seq_lens"], idx, SCALE)
    torch.cuda.synchronize()
    lens = d["seq_lens"].cpu().numpy()
    rows = [0, 13, 31]
    _check_scores(d, scores, rows)
    _check_selection(scores, idx, lens, p["top_k"], rows)
    pairs = [(b, h) for b in rows for h in (0, 77, 127)]
    ro, rl = _oracle_out(d, idx, pairs, compact=True)
    ix = torch.tensor(pairs, device="cuda")
    check(out[ix[:, 0], 0, ix[:, 1]], ro, lse[ix[:, 0], 0, ix[:, 1]], rl, what="dsa full")


@cuda
def test_selection_past_the_shared_memory_staging_limit():
    """A cache longer than the top-k kernel stages in shared memory (four slices of at most
    48,128 tokens per sequence) takes the path that re-reads the scores on every pass."""
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    lens = [200000, 7000]
    d = dsa_inputs(2, 128, 512, 64, 64, 128, seq_lens=lens, T_max=200000, seed=99, device="cuda")
    scores, idx = _index(d, 2048)
    _check_scores(d, scores, rows=[0])
    _check_selection(scores, idx, lens, 2048)


# ------------------------------------------------ FP8 (E4M3) latent cache, sparse MLA
def _oracle_fp8(d, idx, pairs=None):
    from oracle import dsa_mla_decode_fp8_ref
    sl = d["seq_lens"].cpu().numpy()
    ix = [idx[b, :min(int(sl[b]), idx.shape[1])].cpu().numpy().astype(np.int64) for b in range(len(sl))]
    return dsa_mla_decode_fp8_ref(to_np(d["q_nope"]), to_np(d["q_pe"]), d["kv_codes"].cpu().numpy(),
                                  d["kv_scale"].cpu().numpy(), to_np(d["pe_cache"]), ix, SCALE, pairs=pairs)


@cuda
@pytest.mark.parametrize("lens,T,top_k", [([40, 900, 2000], 2048, 256), ([33, 0, 1025], 1088, 2048)])
def test_sparse_mla_fp8_latent_matches_oracle(lens, T, top_k):
    from attention_causal_gqa_b200 import dsa_mla_decode_fp8
    from attention_causal_gqa_b200.synthetic import dsa_inputs_fp8
    d = dsa_inputs_fp8(len(lens), 128, 512, 64, 64, 128, seq_lens=lens, T_max=T, seed=T + 3 * top_k, device="cuda")
    _, idx = _index(d, top_k)
    out, lse = dsa_mla_decode_fp8(d["q_nope"], d["q_pe"], d["kv_codes"], d["kv_scale"], d["pe_cache"],
                                  d["seq_lens"], idx, SCALE)
    torch.cuda.synchronize()
    ro, rl = _oracle_fp8(d, idx)
    check(out, ro, lse, rl, what=f"dsa fp8 {lens}")


@cuda
def test_sparse_mla_fp8_bad_index_is_flagged():
    from attention_causal_gqa_b200 import binding
    from attention_causal_gqa_b200.synthetic import dsa_inputs_fp8
    lens = [300, 200]
    d = dsa_inputs_fp8(2, 128, 512, 64, 16, 128, seq_lens=lens, T_max=320, seed=8, device="cuda")
    _, idx = _index(d, 64)
    idx[0, 3] = -5
    ws = torch.empty(binding.dsa_mla_workspace_size(2, 128, 512, 64, 64), dtype=torch.uint8, device="cuda")
    out, _ = binding.dsa_mla_decode_fp8(d["q_nope"], d["q_pe"], d["kv_codes"], d["kv_scale"], d["pe_cache"],
                                        d["seq_lens"], idx, SCALE, workspace=ws)
    assert binding.read_status(ws) & binding.ATTN_DEV_BAD_INDEX
    assert torch.isfinite(out.float()).all()


@cuda
@pytest.mark.parametrize("B,lo,hi,T_max,HI,top_k,seed", [(1, 3000, 3000, 3000, 64, 512, 51),
                                                         (40, 0, 2500, 2600, 32, 300, 52),
                                                         (160, 100, 400, 400, 16, 128, 53)])
def test_index_random_layouts(B, lo, hi, T_max, HI, top_k, seed):
    """Random batches for the persistent indexer (one sequence; some and many sequences per
    CTA; T_max not a multiple of the 128-token tile) and the cluster top-k: sampled scores
    against the oracle, every selection exactly the top-k of the kernel's scores."""
    from attention_causal_gqa_b200.synthetic import dsa_inputs
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, B).tolist()
    d = dsa_inputs(B, 128, 512, 64, HI, 128, seq_lens=lens, T_max=T_max, seed=seed, device="cuda")
    scores, idx = _index(d, top_k)
    rows = sorted(set(rng.integers(0, B, 6).tolist()) | {0, B - 1})
    _check_scores(d, scores, rows=rows)
    _check_selection(scores, idx, lens, top_k)
