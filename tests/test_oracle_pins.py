"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a value printed
on the pages (tests/golden), a closed form, an invariant, a special case that
reduces to a different computation, or a brute-force pure-Python evaluation.
Several tests also plant a plausible mistake in a local copy of the arithmetic
and check that the pin would catch it.
"""
import math
import os

import numpy as np
import pytest

from oracle import (
    apply_rope,
    decode_paged_ref,
    gather_pages,
    lse_merge,
    mla_decode_ref,
    mla_naive_ref,
    online_softmax_merge,
    prefill_ref,
    rope_cache,
    two_pass_softmax_rows,
)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------- RoPE pins
def test_rope_theta_matches_printed_formula_values():
    rows = _golden_rows("rope_theta_d8_base1e4.txt")
    p = 7
    cs = rope_cache(p + 1, 8, 1e4)
    for i, th in rows:
        i, th = int(i), float(th)
        assert cs[p, i, 0] == pytest.approx(math.cos(p * th), abs=1e-14)
        assert cs[p, i, 1] == pytest.approx(math.sin(p * th), abs=1e-14)


def test_rope_cache_layout_matches_page():
    (row,) = _golden_rows("rope_cache_layout.txt")
    max_len, hd = int(row[0]), int(row[1])
    shape = tuple(int(x) for x in row[2].split(","))
    cs = rope_cache(max_len, hd, 1e4)
    assert cs.shape == shape
    # cos first, then sin, and cos^2 + sin^2 = 1 everywhere
    assert np.allclose(cs[..., 0] ** 2 + cs[..., 1] ** 2, 1.0, atol=1e-13)
    # large-position angle is computed directly: compare with math at p = 32767, i = 0
    assert cs[32767, 0, 0] == pytest.approx(math.cos(32767.0), abs=1e-12)


def test_rope_2d_closed_form_rotation():
    # D = 2: the single pair has theta_0 = 1; (1, 0) at position p becomes (cos p, sin p)
    x = np.zeros((5, 2))
    x[:, 0] = 1.0
    y = apply_rope(x, 1e4)
    for p in range(5):
        assert y[p, 0] == pytest.approx(math.cos(p), abs=1e-15)
        assert y[p, 1] == pytest.approx(math.sin(p), abs=1e-15)
    # (0, 1) becomes (-sin p, cos p): pins the sign of the cross term
    x = np.zeros((5, 2))
    x[:, 1] = 1.0
    y = apply_rope(x, 1e4)
    for p in range(5):
        assert y[p, 0] == pytest.approx(-math.sin(p), abs=1e-15)
        assert y[p, 1] == pytest.approx(math.cos(p), abs=1e-15)


def test_rope_interleaved_pairs_not_half_split():
    # D = 4, theta = 1e4: pair 0 = (x0, x1) with freq 1, pair 1 = (x2, x3) with freq 0.01
    x = np.array([[0.0, 0.0, 1.0, 0.0]] * 3)
    y = apply_rope(x, 1e4)
    p = 2
    assert y[p, 2] == pytest.approx(math.cos(p * 0.01), abs=1e-15)
    assert y[p, 3] == pytest.approx(math.sin(p * 0.01), abs=1e-15)
    assert y[p, 0] == 0.0 and y[p, 1] == 0.0


def test_rope_identity_at_zero_norm_and_relative_position():
    D, S = 16, 64
    q = RNG.standard_normal((S, D))
    k = RNG.standard_normal((S, D))
    qr, kr = apply_rope(q, 1e4), apply_rope(k, 1e4)
    assert np.allclose(qr[0], q[0], atol=0)  # position 0 is the identity
    assert np.allclose(np.linalg.norm(qr, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    # the score depends only on n - m: shift both positions by 17
    m, n = 5, 40
    s1 = apply_rope(q[m:m + 1], 1e4, positions=np.array([m])) @ apply_rope(k[n:n + 1], 1e4, positions=np.array([n])).T
    s2 = apply_rope(q[m:m + 1], 1e4, positions=np.array([m + 17])) @ apply_rope(k[n:n + 1], 1e4, positions=np.array([n + 17])).T
    assert s1[0, 0] == pytest.approx(s2[0, 0], rel=1e-11, abs=1e-12)


# -------------------------------------------------------------- prefill pins
def test_constant_v_gives_constant_output_and_lse_independent_of_v():
    B, Hq, Hkv, S, D = 1, 4, 2, 40, 8
    q = RNG.standard_normal((B, Hq, S, D))
    k = RNG.standard_normal((B, Hkv, S, D))
    c = RNG.standard_normal(D)
    v = np.broadcast_to(c, (B, Hkv, S, D)).copy()
    o, lse = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    assert np.allclose(o, c, atol=1e-13)
    _, lse2 = prefill_ref(q, k, RNG.standard_normal((B, Hkv, S, D)), causal=True, rope_theta=1e4)
    assert np.array_equal(lse, lse2)


def test_single_key_row_zero_closed_form():
    B, H, S, D = 1, 2, 9, 8
    q = RNG.standard_normal((B, H, S, D))
    k = RNG.standard_normal((B, H, S, D))
    v = RNG.standard_normal((B, H, S, D))
    scale = 0.3
    o, lse = prefill_ref(q, k, v, causal=True, rope_theta=1e4, scale=scale)
    for h in range(H):
        # causal row 0 sees only key 0; position 0 is unrotated
        assert np.allclose(o[0, h, 0], v[0, h, 0], atol=1e-14)
        assert lse[0, h, 0] == pytest.approx(scale * float(q[0, h, 0] @ k[0, h, 0]), abs=1e-13)
    # S = 1, non-causal: same closed form
    o1, l1 = prefill_ref(q[:, :, :1], k[:, :, :1], v[:, :, :1], causal=False, rope_theta=1e4, scale=scale)
    assert np.allclose(o1[0, :, 0], v[0, :, 0], atol=1e-14)


def test_zero_query_gives_prefix_mean_and_log_count():
    B, H, S, D = 1, 1, 33, 4
    q = np.zeros((B, H, S, D))
    k = RNG.standard_normal((B, H, S, D))
    v = RNG.standard_normal((B, H, S, D))
    o, lse = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    for i in range(S):
        assert np.allclose(o[0, 0, i], v[0, 0, : i + 1].mean(axis=0), atol=1e-13)
        assert lse[0, 0, i] == pytest.approx(math.log(i + 1), abs=1e-13)
    # non-causal: every row is the mean of all values
    o, lse = prefill_ref(q, k, v, causal=False, rope_theta=0)
    assert np.allclose(o[0, 0], v[0, 0].mean(axis=0), atol=1e-13)
    assert np.allclose(lse, math.log(S), atol=1e-13)


def _pure_python_attention(q, k, v, causal, theta, scale):
    """Independent scalar evaluation: RoPE with math.cos/sin, scores, softmax."""
    S, D = len(q), len(q[0])

    def rope(x, p):
        out = list(x)
        if theta <= 0:
            return out
        for i in range(D // 2):
            a = p * theta ** (-2.0 * i / D)
            c, s = math.cos(a), math.sin(a)
            out[2 * i] = x[2 * i] * c - x[2 * i + 1] * s
            out[2 * i + 1] = x[2 * i] * s + x[2 * i + 1] * c
        return out

    qr = [rope(q[i], i) for i in range(S)]
    kr = [rope(k[j], j) for j in range(S)]
    outs, lses = [], []
    for i in range(S):
        js = range(i + 1) if causal else range(S)
        sc = [scale * sum(qr[i][d] * kr[j][d] for d in range(D)) for j in js]
        m = max(sc)
        e = [math.exp(s - m) for s in sc]
        tot = sum(e)
        outs.append([sum(e[n] * v[j][d] for n, j in enumerate(js)) / tot for d in range(D)])
        lses.append(m + math.log(tot))
    return outs, lses


@pytest.mark.parametrize("causal", [True, False])
def test_tiny_brute_force_matches(causal):
    B, Hq, Hkv, S, D = 1, 4, 2, 7, 6
    q = RNG.standard_normal((B, Hq, S, D))
    k = RNG.standard_normal((B, Hkv, S, D))
    v = RNG.standard_normal((B, Hkv, S, D))
    o, lse = prefill_ref(q, k, v, causal=causal, rope_theta=100.0, scale=0.7)
    for h in range(Hq):
        kvh = h // 2
        bo, bl = _pure_python_attention(q[0, h].tolist(), k[0, kvh].tolist(), v[0, kvh].tolist(), causal, 100.0, 0.7)
        assert np.allclose(o[0, h], np.array(bo), atol=1e-12)
        assert np.allclose(lse[0, h], np.array(bl), atol=1e-12)


def test_row_sampled_prefill_equals_full():
    B, Hq, Hkv, S, D = 2, 4, 2, 50, 8
    q = RNG.standard_normal((B, Hq, S, D))
    k = RNG.standard_normal((B, Hkv, S, D))
    v = RNG.standard_normal((B, Hkv, S, D))
    o, lse = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    rows = [(0, 0, 0), (1, 3, 49), (0, 2, 17), (1, 1, 31)]
    os_, ls_ = prefill_ref(q, k, v, causal=True, rope_theta=1e4, rows=rows)
    for n, (b, h, i) in enumerate(rows):
        assert np.allclose(os_[n], o[b, h, i], atol=1e-13)
        assert ls_[n] == pytest.approx(lse[b, h, i], abs=1e-13)


# ------------------------------------------------------------ GQA head map
def test_gqa_head_map_matches_page_table():
    rows = _golden_rows("gqa_head_map_h4_g2.txt")
    B, Hq, Hkv, S, D = 1, 4, 2, 12, 4
    q = RNG.standard_normal((B, Hq, S, D))
    k = RNG.standard_normal((B, Hkv, S, D))
    v = RNG.standard_normal((B, Hkv, S, D))
    o, _ = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    for qh, kvh in rows:
        qh, kvh = int(qh) - 1, int(kvh) - 1
        # single-head attention against exactly that kv head
        o1, _ = prefill_ref(q[:, qh:qh + 1], k[:, kvh:kvh + 1], v[:, kvh:kvh + 1], causal=True, rope_theta=1e4)
        assert np.allclose(o[:, qh], o1[:, 0], atol=1e-13)
        other = 1 - kvh
        o2, _ = prefill_ref(q[:, qh:qh + 1], k[:, other:other + 1], v[:, other:other + 1], causal=True, rope_theta=1e4)
        assert not np.allclose(o[:, qh], o2[:, 0], atol=1e-3)


def test_gqa_equals_mha_with_replicated_kv_and_mha_special_case():
    B, Hq, Hkv, S, D = 2, 8, 2, 20, 8
    q = RNG.standard_normal((B, Hq, S, D))
    k = RNG.standard_normal((B, Hkv, S, D))
    v = RNG.standard_normal((B, Hkv, S, D))
    o, lse = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    G = Hq // Hkv
    kr = np.repeat(k, G, axis=1)  # contiguous groups, like repeat_interleave
    vr = np.repeat(v, G, axis=1)
    o2, lse2 = prefill_ref(q, kr, vr, causal=True, rope_theta=1e4)  # Hkv = Hq (MHA)
    assert np.allclose(o, o2, atol=1e-13) and np.allclose(lse, lse2, atol=1e-13)
    # MQA: Hkv = 1 equals every head attending to the single kv head
    oq, _ = prefill_ref(q, k[:, :1], v[:, :1], causal=True, rope_theta=1e4)
    om, _ = prefill_ref(q, np.repeat(k[:, :1], Hq, axis=1), np.repeat(v[:, :1], Hq, axis=1), causal=True, rope_theta=1e4)
    assert np.allclose(oq, om, atol=1e-13)


# ---------------------------------------------------- online softmax / merge
def test_online_recurrence_equals_two_pass_and_catches_missing_rescale():
    n, D = 300, 5
    s = RNG.standard_normal(n) * 4.0
    v = RNG.standard_normal((n, D))
    p, l_ = two_pass_softmax_rows(s[None, :])
    o_ref, lse_ref = (p @ v)[0], l_[0]
    cuts = [0, 17, 64, 65, 200, n]
    bs = [s[a:b] for a, b in zip(cuts[:-1], cuts[1:])]
    bv = [v[a:b] for a, b in zip(cuts[:-1], cuts[1:])]
    o_on, lse_on = online_softmax_merge(bs, bv)
    assert np.allclose(o_on, o_ref, atol=1e-13)
    assert lse_on == pytest.approx(lse_ref, abs=1e-12)
    # planted mistake: per-block softmax summed without rescaling (the long-context
    # page's chunked pseudo-code) must NOT match
    wrong = sum(two_pass_softmax_rows(a[None, :])[0] @ b for a, b in zip(bs, bv))[0]
    assert not np.allclose(wrong, o_ref, atol=1e-3)


def test_lse_merge_of_arbitrary_split_equals_unsplit_decode():
    Hq, Hkv, D, ps = 4, 2, 8, 16
    L = 203
    d = _tiny_paged(1, Hq, Hkv, D, [L], seed=5)
    o, lse = decode_paged_ref(d["q"], d["k"], d["v"], d["table"], d["lens"])
    k_seq = gather_pages(d["k"], d["table"][0], L, ps)
    v_seq = gather_pages(d["v"], d["table"][0], L, ps)
    cuts = [0, 1, 33, 34, 150, L]
    for h in range(Hq):
        kvh = h // 2
        pos, pls = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            s = (k_seq[a:b, kvh] @ d["q"][0, h]) / math.sqrt(D)
            pp, ll = two_pass_softmax_rows(s[None, :])
            pos.append((pp @ v_seq[a:b, kvh])[0])
            pls.append(ll[0])
        pos.append(np.zeros(D))  # an empty chunk carries no weight
        pls.append(-np.inf)
        om, lm = lse_merge(pos, pls)
        assert np.allclose(om, o[0, h], atol=1e-13)
        assert lm == pytest.approx(lse[0, h], abs=1e-12)


# -------------------------------------------------------------- paged decode
def _tiny_paged(B, Hq, Hkv, D, lens, seed, ps=16, identity=False):
    rng = np.random.default_rng(seed)
    npg = [math.ceil(L / ps) for L in lens]
    tot = sum(npg)
    perm = np.arange(tot) if identity else rng.permutation(tot)
    maxp = max(npg + [1])
    table = np.full((B, maxp), -1, dtype=np.int64)
    off = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[off:off + n]
        off += n
    k = rng.standard_normal((max(tot, 1), ps, Hkv, D))
    v = rng.standard_normal((max(tot, 1), ps, Hkv, D))
    q = rng.standard_normal((B, Hq, D))
    return dict(q=q, k=k, v=v, table=table, lens=np.array(lens), perm=perm)


def test_paged_equals_contiguous_and_last_row_of_causal_prefill():
    B, Hq, Hkv, D = 3, 4, 2, 8
    lens = [1, 16, 45]
    d = _tiny_paged(B, Hq, Hkv, D, lens, seed=9)
    o, lse = decode_paged_ref(d["q"], d["k"], d["v"], d["table"], d["lens"])
    # identity layout holding the same logical tokens
    for b, L in enumerate(lens):
        ks = gather_pages(d["k"], d["table"][b], L, 16)  # [L, Hkv, D]
        vs = gather_pages(d["v"], d["table"][b], L, 16)
        # decode = last row of a causal prefill over the same (already rotated) K/V
        qq = np.zeros((1, Hq, L, D))
        qq[0, :, L - 1] = d["q"][b]
        kk = ks.transpose(1, 0, 2)[None]
        vv = vs.transpose(1, 0, 2)[None]
        op, lp = prefill_ref(qq, kk, vv, causal=True, rope_theta=0, scale=1 / math.sqrt(D))
        assert np.allclose(op[0, :, L - 1], o[b], atol=1e-13)
        assert np.allclose(lp[0, :, L - 1], lse[b], atol=1e-12)
    # relabelling the physical pages does not change the result
    d2 = _tiny_paged(B, Hq, Hkv, D, lens, seed=9)
    inv = np.empty_like(d2["perm"])
    inv[d2["perm"]] = np.arange(len(inv))
    k_id = d2["k"][d2["perm"]]
    v_id = d2["v"][d2["perm"]]
    table_id = np.where(d2["table"] >= 0, inv[np.maximum(d2["table"], 0)], -1)
    o3, l3 = decode_paged_ref(d2["q"], k_id, v_id, table_id, d2["lens"])
    assert np.allclose(o3, o, atol=1e-13) and np.allclose(l3, lse, atol=1e-13)


def test_decode_empty_sequence_and_poisoned_tail():
    B, Hq, Hkv, D = 2, 2, 1, 4
    d = _tiny_paged(B, Hq, Hkv, D, [0, 5], seed=3)
    o, lse = decode_paged_ref(d["q"], d["k"], d["v"], d["table"], d["lens"])
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    k = d["k"].copy()
    v = d["v"].copy()
    pg = d["table"][1, 0]
    k[pg, 5:] = 1e4
    v[pg, 5:] = np.nan
    o2, l2 = decode_paged_ref(d["q"], k, v, d["table"], d["lens"])
    assert np.allclose(o2[1], o[1]) and np.allclose(l2[1], lse[1])


# ------------------------------------------------------------------ MLA pins
def test_mla_split_form_equals_concatenated_heads_brute_force():
    B, H, Dc, Dr, T = 2, 3, 6, 2, 9
    rng = np.random.default_rng(11)
    qn = rng.standard_normal((B, 1, H, Dc))
    qp = rng.standard_normal((B, 1, H, Dr))
    kv = rng.standard_normal((B, T, Dc))
    pe = rng.standard_normal((B, T, Dr))
    lens = np.array([9, 4])
    scale = 1 / math.sqrt(Dc + Dr)
    o, lse = mla_decode_ref(qn, qp, kv, pe, lens, scale)
    for b in range(B):
        for h in range(H):
            qc = list(qn[b, 0, h]) + list(qp[b, 0, h])
            sc = [scale * sum(a * c for a, c in zip(qc, list(kv[b, t]) + list(pe[b, t]))) for t in range(lens[b])]
            m = max(sc)
            e = [math.exp(s - m) for s in sc]
            tot = sum(e)
            ref = [sum(e[t] * kv[b, t, d] for t in range(lens[b])) / tot for d in range(Dc)]
            assert np.allclose(o[b, 0, h], ref, atol=1e-12)
            assert lse[b, 0, h] == pytest.approx(m + math.log(tot), abs=1e-12)


def test_mla_absorbed_equals_naive_with_random_up_projections():
    H, Dc, Dr, dk, T = 4, 8, 2, 5, 11
    rng = np.random.default_rng(13)
    c_kv = rng.standard_normal((T, Dc))
    k_pe = rng.standard_normal((T, Dr))
    w_uk = rng.standard_normal((H, Dc, dk))
    w_uv = rng.standard_normal((H, Dc, dk))
    x_q = rng.standard_normal((H, dk))
    q_pe = rng.standard_normal((H, Dr))
    scale = 1 / math.sqrt(dk + Dr)
    o_naive, l_naive = mla_naive_ref(x_q, c_kv, k_pe, w_uk, w_uv, q_pe, scale)
    # absorb W^K_up into the query: q_nope,h = W_uk,h x_q,h (so q_nope . c = x_q . (c W_uk))
    q_nope = np.einsum("hcd,hd->hc", w_uk, x_q)[None, None]
    o_lat, l_abs = mla_decode_ref(q_nope, q_pe[None, None], c_kv[None], k_pe[None], np.array([T]), scale)
    # W^V_up applied after attention (folded into the output projection)
    o_abs = np.einsum("hc,hcd->hd", o_lat[0, 0], w_uv)
    assert np.allclose(o_abs, o_naive, atol=1e-12)
    assert np.allclose(l_abs[0, 0], l_naive, atol=1e-12)


def test_mla_ignores_cache_beyond_length():
    B, H, Dc, Dr, T = 1, 2, 4, 2, 10
    rng = np.random.default_rng(17)
    qn = rng.standard_normal((B, 1, H, Dc))
    qp = rng.standard_normal((B, 1, H, Dr))
    kv = rng.standard_normal((B, T, Dc))
    pe = rng.standard_normal((B, T, Dr))
    o, l = mla_decode_ref(qn, qp, kv, pe, np.array([6]), 0.5)
    kv[:, 6:] = np.nan
    pe[:, 6:] = 1e6
    o2, l2 = mla_decode_ref(qn, qp, kv, pe, np.array([6]), 0.5)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


# ------------------------------------------- chunked prefill into the paged cache
def _paged_setup(rng, B, Hkv, D, cache_lens, S_new, page_size=16, extra=3):
    """A cache whose pages sit in a random physical order, filled with (rotated, stored)
    keys for the cached prefix and garbage everywhere else."""
    from oracle import to_bf16
    need = [(L + S_new + page_size - 1) // page_size for L in cache_lens]
    n_pages = sum(need) + extra
    perm = rng.permutation(n_pages)
    max_pages = max(need)
    table = np.zeros((B, max_pages), dtype=np.int64)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    kp = to_bf16(rng.standard_normal((n_pages, page_size, Hkv, D)))
    vp = to_bf16(rng.standard_normal((n_pages, page_size, Hkv, D)))
    return kp, vp, table


def test_to_bf16_matches_torch_and_ties_to_even():
    import torch
    from oracle import to_bf16
    x = np.array([1.0, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -2.5, 1e-30, 3.0e38])
    r = to_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2.0**-6 and r[3] == -2.5
    y = np.random.default_rng(3).standard_normal(10000) * 7
    ref = torch.tensor(y, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(to_bf16(y), ref)


def test_chunk_prefill_empty_cache_unrounded_equals_prefill():
    from oracle import chunk_prefill_ref, prefill_ref
    rng = np.random.default_rng(40)
    B, Hq, Hkv, S, D = 2, 4, 2, 37, 16
    q = rng.standard_normal((B, Hq, S, D))
    k = rng.standard_normal((B, Hkv, S, D))
    v = rng.standard_normal((B, Hkv, S, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, [0, 0], S)
    _, _, o, lse = chunk_prefill_ref(q, k, v, kp, vp, table, [0, 0], rope_theta=1e4, store=lambda x: x)
    ro, rl = prefill_ref(q, k, v, causal=True, rope_theta=1e4)
    assert np.allclose(o, ro, atol=1e-12) and np.allclose(lse, rl, atol=1e-12)


def test_chunk_prefill_two_chunks_equal_one():
    from oracle import chunk_prefill_ref
    rng = np.random.default_rng(41)
    B, Hq, Hkv, D = 2, 6, 2, 16
    cache = [5, 40]
    n1, n2 = 9, 14
    q = rng.standard_normal((B, Hq, n1 + n2, D))
    k = rng.standard_normal((B, Hkv, n1 + n2, D))
    v = rng.standard_normal((B, Hkv, n1 + n2, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, cache, n1 + n2)
    kp1, vp1, o1, l1 = chunk_prefill_ref(q, k, v, kp, vp, table, cache)
    kpa, vpa, oa, la = chunk_prefill_ref(q[:, :, :n1], k[:, :, :n1], v[:, :, :n1], kp, vp, table, cache)
    kpb, vpb, ob, lb = chunk_prefill_ref(q[:, :, n1:], k[:, :, n1:], v[:, :, n1:], kpa, vpa, table,
                                         [c + n1 for c in cache])
    assert np.array_equal(kpb, kp1) and np.array_equal(vpb, vp1)
    assert np.allclose(np.concatenate([oa, ob], axis=2), o1, atol=1e-12)
    assert np.allclose(np.concatenate([la, lb], axis=2), l1, atol=1e-12)


def test_chunk_prefill_appends_rotated_keys_at_their_pages():
    from oracle import apply_rope, chunk_prefill_ref, gather_pages, to_bf16
    rng = np.random.default_rng(42)
    B, Hq, Hkv, D, S_new = 2, 2, 2, 8, 20
    cache = [3, 17]
    q = rng.standard_normal((B, Hq, S_new, D))
    k = rng.standard_normal((B, Hkv, S_new, D))
    v = rng.standard_normal((B, Hkv, S_new, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, cache, S_new)
    kp2, vp2, _, _ = chunk_prefill_ref(q, k, v, kp, vp, table, cache, rope_theta=500.0)
    for b in range(B):
        L = cache[b]
        got_k = gather_pages(kp2, table[b], L + S_new, 16)
        got_v = gather_pages(vp2, table[b], L + S_new, 16)
        assert np.array_equal(got_k[:L], gather_pages(kp, table[b], L, 16))  # the cached prefix is untouched
        for kvh in range(Hkv):
            rot = apply_rope(k[b, kvh], 500.0, positions=L + np.arange(S_new))
            assert np.array_equal(got_k[L:, kvh], to_bf16(rot))
            assert np.array_equal(got_v[L:, kvh], to_bf16(v[b, kvh]))


def test_chunk_prefill_last_row_equals_decode_over_the_updated_cache():
    from oracle import apply_rope, chunk_prefill_ref, decode_paged_ref
    rng = np.random.default_rng(43)
    B, Hq, Hkv, D, S_new = 3, 8, 2, 16, 7
    cache = [0, 30, 64]
    q = rng.standard_normal((B, Hq, S_new, D))
    k = rng.standard_normal((B, Hkv, S_new, D))
    v = rng.standard_normal((B, Hkv, S_new, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, cache, S_new)
    kp2, vp2, o, lse = chunk_prefill_ref(q, k, v, kp, vp, table, cache)
    q_last = np.stack([apply_rope(q[b, :, -1], 1e4, positions=np.full(Hq, cache[b] + S_new - 1))
                       for b in range(B)])
    do, dl = decode_paged_ref(q_last, kp2, vp2, table, [c + S_new for c in cache])
    assert np.allclose(o[:, :, -1], do, atol=1e-12) and np.allclose(lse[:, :, -1], dl, atol=1e-12)


# ------------------------------------------------------ FP8 (E4M3) paged decode
def test_e4m3_decoding_matches_torch_for_every_code():
    import torch
    from oracle import e4m3_to_float
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0  # max, smallest subnormal, one


def test_fp8_decode_equals_decode_over_the_dequantised_cache():
    from oracle import decode_paged_fp8_ref, decode_paged_ref, e4m3_to_float
    rng = np.random.default_rng(50)
    B, Hq, Hkv, D, P = 2, 8, 2, 16, 9
    kc = rng.integers(0, 256, size=(P, 16, Hkv, D), dtype=np.uint8) & 0x77  # no NaN codes
    vc = rng.integers(0, 256, size=(P, 16, Hkv, D), dtype=np.uint8) & 0x77
    ks = rng.uniform(0.01, 2.0, size=(P, Hkv))
    vs = rng.uniform(0.01, 2.0, size=(P, Hkv))
    table = rng.permutation(P)[:8].reshape(2, 4)
    lens = [37, 64]
    q = rng.standard_normal((B, Hq, D))
    o, l = decode_paged_fp8_ref(q, kc, vc, ks, vs, table, lens)
    kf = np.stack([[e4m3_to_float(kc[p, :, h]) * ks[p, h] for h in range(Hkv)] for p in range(P)]).transpose(0, 2, 1, 3)
    vf = np.stack([[e4m3_to_float(vc[p, :, h]) * vs[p, h] for h in range(Hkv)] for p in range(P)]).transpose(0, 2, 1, 3)
    ro, rl = decode_paged_ref(q, kf, vf, table, lens)
    assert np.allclose(o, ro, atol=1e-12) and np.allclose(l, rl, atol=1e-12)


# ------------------------------------------- DSA: lightning indexer + top-k MLA
def test_indexer_hand_worked_example():
    """Attention study note, "Lighting Indexer": score = sum_j w_j * ReLU(q_j . k_s).
    Two heads q1 = (1, 0), q2 = (0, 1), weights (0.5, 2); keys (2, -3), (-1, 1), (1, 1):
    token 0: 0.5*2 + 2*ReLU(-3) = 1; token 1: 0.5*ReLU(-1) + 2*1 = 2; token 2: 0.5 + 2 = 2.5."""
    from oracle import dsa_index_scores_ref, dsa_topk_ref
    q = np.array([[[1.0, 0.0], [0.0, 1.0]]])
    w = np.array([[0.5, 2.0]])
    k = np.array([[[2.0, -3.0], [-1.0, 1.0], [1.0, 1.0], [9.0, 9.0]]])
    s = dsa_index_scores_ref(q, w, k, [3])
    assert s[0, :3].tolist() == [1.0, 2.0, 2.5] and s[0, 3] == -np.inf  # slot past the length never counts
    assert dsa_topk_ref(s, [3], 2)[0].tolist() == [1, 2]


def test_indexer_matches_scalar_brute_force():
    from oracle import dsa_index_scores_ref
    rng = np.random.default_rng(60)
    B, HI, d, T = 2, 3, 4, 6
    q, w, k = rng.standard_normal((B, HI, d)), rng.standard_normal((B, HI)), rng.standard_normal((B, T, d))
    lens = [6, 4]
    s = dsa_index_scores_ref(q, w, k, lens)
    for b in range(B):
        for t in range(T):
            if t >= lens[b]:
                assert s[b, t] == -np.inf
                continue
            acc = 0.0
            for j in range(HI):
                dot = sum(float(q[b, j, i]) * float(k[b, t, i]) for i in range(d))
                acc += float(w[b, j]) * (dot if dot > 0 else 0.0)
            assert abs(s[b, t] - acc) < 1e-12


def test_topk_ties_prefer_the_smaller_index_and_short_sequences_keep_everything():
    from oracle import dsa_topk_ref
    s = np.array([[3.0, 1.0, 3.0, 2.0, 3.0, -np.inf], [0.5, 0.5, 0.5, 0.5, 0.5, 0.5]])
    got = dsa_topk_ref(s, [5, 6], 2)
    assert got[0].tolist() == [0, 2] and got[1].tolist() == [0, 1]
    assert dsa_topk_ref(s, [5, 6], 4)[0].tolist() == [0, 2, 3, 4]
    assert dsa_topk_ref(s, [5, 0], 99)[0].tolist() == [0, 1, 2, 3, 4] and len(dsa_topk_ref(s, [5, 0], 99)[1]) == 0
    # brute force over every subset on a small random row: the chosen set has the largest sum
    rng = np.random.default_rng(61)
    row = rng.standard_normal(7)
    import itertools
    best = max(itertools.combinations(range(7), 3), key=lambda c: sum(row[i] for i in c))
    assert dsa_topk_ref(row[None, :], [7], 3)[0].tolist() == sorted(best)


def test_dsa_with_every_token_selected_is_dense_mla():
    from oracle import dsa_index_scores_ref, dsa_mla_decode_ref, dsa_topk_ref, mla_decode_ref
    rng = np.random.default_rng(62)
    B, H, Dc, Dr, T = 2, 3, 8, 4, 20
    qn, qp = rng.standard_normal((B, 1, H, Dc)), rng.standard_normal((B, 1, H, Dr))
    kv, pe = rng.standard_normal((B, T, Dc)), rng.standard_normal((B, T, Dr))
    lens = [20, 13]
    s = dsa_index_scores_ref(rng.standard_normal((B, 2, 5)), rng.standard_normal((B, 2)),
                             rng.standard_normal((B, T, 5)), lens)
    o, l = dsa_mla_decode_ref(qn, qp, kv, pe, dsa_topk_ref(s, lens, 64), 0.3)
    ro, rl = mla_decode_ref(qn, qp, kv, pe, lens, 0.3)
    assert np.allclose(o, ro, atol=1e-12) and np.allclose(l, rl, atol=1e-12)


def test_dsa_equals_dense_softmax_with_unselected_tokens_masked():
    """Attending only the selected tokens = the dense score row with -inf on the others."""
    from oracle import dsa_mla_decode_ref, two_pass_softmax_rows
    rng = np.random.default_rng(63)
    B, H, Dc, Dr, T = 1, 2, 8, 4, 30
    qn, qp = rng.standard_normal((B, 1, H, Dc)), rng.standard_normal((B, 1, H, Dr))
    kv, pe = rng.standard_normal((B, T, Dc)), rng.standard_normal((B, T, Dr))
    sel = np.array([2, 3, 11, 17, 29])
    o, l = dsa_mla_decode_ref(qn, qp, kv, pe, [sel], 0.25)
    for h in range(H):
        sc = (kv[0] @ qn[0, 0, h] + pe[0] @ qp[0, 0, h]) * 0.25
        masked = np.full(T, -np.inf)
        masked[sel] = sc[sel]
        p, lse = two_pass_softmax_rows(masked[None, :])
        assert np.allclose(o[0, 0, h], (p @ kv[0])[0], atol=1e-12) and abs(l[0, 0, h] - lse[0]) < 1e-12


# ------------------------------------------------------ RoPE scaling variants
def _interleave_halves(x):
    """(x[i], x[i + D/2]) -> positions (2i, 2i + 1)."""
    d = x.shape[-1]
    out = np.empty_like(x)
    out[..., 0::2] = x[..., :d // 2]
    out[..., 1::2] = x[..., d // 2:]
    return out


def test_half_split_rope_is_interleaved_rope_on_permuted_dims():
    from oracle import apply_rope
    rng = np.random.default_rng(70)
    x = rng.standard_normal((5, 16))
    half = apply_rope(x, 500.0, layout="half")
    inter = apply_rope(_interleave_halves(x), 500.0)
    assert np.allclose(_interleave_halves(half), inter, atol=1e-13)
    # and it is not the same function (a plausible mix-up)
    assert not np.allclose(half, apply_rope(x, 500.0), atol=1e-3)


def test_half_split_rope_closed_form_d4():
    """D = 4, half layout: pairs (0, 2) with theta_0 = 1 and (1, 3) with theta_1 = theta^-1/2."""
    from oracle import apply_rope
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    p, th = 3, 16.0
    y = apply_rope(x, th, positions=np.array([p]), layout="half")[0]
    a0, a1 = p * 1.0, p * th ** -0.5
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    assert np.allclose(y, want, atol=1e-14)


def test_frequency_scale_equals_scaled_positions():
    from oracle import apply_rope
    rng = np.random.default_rng(71)
    x = rng.standard_normal((6, 32))
    pos = np.arange(6) * 7
    a = apply_rope(x, 1e4, positions=4 * pos, freq_scale=0.25)
    b = apply_rope(x, 1e4, positions=pos)
    assert np.array_equal(a, b)  # 4p * (theta_i / 4) = p * theta_i exactly in binary


def test_prefill_half_split_equals_interleaved_on_permuted_q_k():
    from oracle import prefill_ref
    rng = np.random.default_rng(72)
    q, k, v = rng.standard_normal((1, 4, 40, 16)), rng.standard_normal((1, 2, 40, 16)), rng.standard_normal((1, 2, 40, 16))
    o1, l1 = prefill_ref(q, k, v, rope_theta=100.0, rope_layout="half", rope_freq_scale=0.5)
    o2, l2 = prefill_ref(_interleave_halves(q), _interleave_halves(k), v, rope_theta=100.0, rope_freq_scale=0.5)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_ntk_aware_and_length_scaled_bases():
    """NTK-aware: the lowest frequency is divided by the stretch, the highest (pair 0)
    stays 1, for several head dims and stretches. Length-aware base of the long-context
    page (section 2.4): theta at L = L0 or alpha = 0, linear in L / L0 at alpha = 1."""
    from oracle import length_scaled_theta_ref, ntk_aware_theta_ref
    for D in (64, 128, 192):
        for s, th in ((8.0, 1e4), (4.0, 5e5), (32.0, 1e6)):
            t2 = ntk_aware_theta_ref(th, s, D)
            lowest = lambda t: t ** (-2.0 * (D // 2 - 1) / D)  # noqa: E731
            assert abs(lowest(t2) - lowest(th) / s) < 1e-12 * lowest(th)
            assert t2 ** 0.0 == 1.0  # pair 0 rotates at frequency 1 whatever the base
        assert ntk_aware_theta_ref(1e4, 1.0, D) == 1e4
    assert length_scaled_theta_ref(1e4, 4096, 4096, 0.2) == 1e4
    assert length_scaled_theta_ref(1e4, 65536, 4096, 0.0) == 1e4
    assert length_scaled_theta_ref(1e4, 8192, 4096, 1.0) == 2e4
    assert abs(length_scaled_theta_ref(1e4, 16384, 4096, 0.5) - 2e4) < 1e-9


def test_chunk_prefill_half_split_equals_interleaved_on_permuted_dims():
    """The layouts differ by a fixed permutation of d: outputs agree, stored keys are permuted."""
    from oracle import chunk_prefill_ref
    rng = np.random.default_rng(73)
    B, Hq, Hkv, D, S_new = 2, 4, 2, 16, 5
    cache = [0, 21]
    q = rng.standard_normal((B, Hq, S_new, D))
    k = rng.standard_normal((B, Hkv, S_new, D))
    v = rng.standard_normal((B, Hkv, S_new, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, cache, S_new)
    kh, vh, oh, lh = chunk_prefill_ref(q, k, v, kp, vp, table, cache, rope_theta=50.0, rope_freq_scale=0.5,
                                       rope_layout="half", store=lambda x: x)
    ki, vi, oi, li = chunk_prefill_ref(_interleave_halves(q), _interleave_halves(k), v, _interleave_halves(kp), vp,
                                       table, cache, rope_theta=50.0, rope_freq_scale=0.5, store=lambda x: x)
    assert np.allclose(oh, oi, atol=1e-12) and np.allclose(lh, li, atol=1e-12)
    assert np.allclose(_interleave_halves(kh), ki, atol=1e-12)


def test_dsa_fp8_latent_equals_dsa_over_the_dequantised_cache():
    from oracle import dsa_mla_decode_fp8_ref, dsa_mla_decode_ref, e4m3_to_float
    rng = np.random.default_rng(74)
    B, H, Dc, Dr, T = 2, 3, 256, 8, 12
    codes = rng.integers(0, 256, size=(B, T, Dc), dtype=np.uint8) & 0xF7  # no NaN codes
    sc = rng.uniform(0.01, 3.0, size=(B, T, Dc // 128))
    pe = rng.standard_normal((B, T, Dr))
    qn, qp = rng.standard_normal((B, 1, H, Dc)), rng.standard_normal((B, 1, H, Dr))
    sel = [np.array([1, 4, 5, 11]), np.array([0, 2])]
    o, l = dsa_mla_decode_fp8_ref(qn, qp, codes, sc, pe, sel, 0.2)
    kv = e4m3_to_float(codes) * np.repeat(sc, 128, axis=2)
    ro, rl = dsa_mla_decode_ref(qn, qp, kv, pe, sel, 0.2)
    assert np.allclose(o, ro, atol=1e-12) and np.allclose(l, rl, atol=1e-12)
    # block b of the latent uses scale b: scaling one block's scale changes only that block's values
    sc2 = sc.copy()
    sc2[:, :, 1] *= 2.0
    o2, _ = dsa_mla_decode_fp8_ref(qn, qp, codes, sc2, pe, sel, 0.2)
    assert not np.allclose(o2, o)


def test_chunk_prefill_varlen_pins():
    """Per-sequence chunk lengths: (a) all lengths S_new is the uniform call; (b) each
    sequence equals that sequence alone with its own S_new (brute force per sequence);
    (c) a zero length appends nothing and leaves its rows at o = 0, lse = -inf;
    (d) appending n1 then n2 tokens gives the second chunk's rows of one n1 + n2 chunk
    (chunking does not change the attention)."""
    from oracle import chunk_prefill_ref
    rng = np.random.default_rng(75)
    B, Hq, Hkv, D, S_new = 3, 4, 2, 16, 9
    cache = [0, 20, 5]
    q = rng.standard_normal((B, Hq, S_new, D))
    k = rng.standard_normal((B, Hkv, S_new, D))
    v = rng.standard_normal((B, Hkv, S_new, D))
    kp, vp, table = _paged_setup(rng, B, Hkv, D, cache, S_new)
    ku, vu, ou, lu = chunk_prefill_ref(q, k, v, kp, vp, table, cache, rope_theta=30.0)
    kf, vf, of, lf = chunk_prefill_ref(q, k, v, kp, vp, table, cache, rope_theta=30.0, new_lens=[S_new] * B)
    assert np.array_equal(ou, of) and np.array_equal(lu, lf) and np.array_equal(ku, kf)
    lens = [4, 0, 9]
    kv_, vv_, o, l = chunk_prefill_ref(q, k, v, kp, vp, table, cache, rope_theta=30.0, new_lens=lens)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(o[b] == 0) and np.all(np.isneginf(l[b]))
            continue
        _, _, ob, lb = chunk_prefill_ref(q[b:b + 1, :, :n], k[b:b + 1, :, :n], v[b:b + 1, :, :n], kp, vp,
                                         table[b:b + 1], cache[b:b + 1], rope_theta=30.0)
        assert np.allclose(o[b, :, :n], ob[0], atol=1e-12) and np.allclose(l[b, :, :n], lb[0], atol=1e-12)
        assert np.all(o[b, :, n:] == 0) and np.all(np.isneginf(l[b, :, n:]))
    # sequence 1 appended nothing: its pages are untouched
    assert np.array_equal(kv_[table[1]], kp[table[1]])
    # two chunks (3 then 6 tokens) equal one chunk of 9 for the second chunk's rows
    b = 2
    qb, kb, vb = q[b:b + 1], k[b:b + 1], v[b:b + 1]
    k1, v1, _, _ = chunk_prefill_ref(qb, kb, vb, kp, vp, table[b:b + 1], [cache[b]], rope_theta=30.0, new_lens=[3])
    _, _, o2, l2 = chunk_prefill_ref(qb[:, :, 3:], kb[:, :, 3:], vb[:, :, 3:], k1, v1, table[b:b + 1], [cache[b] + 3],
                                     rope_theta=30.0)
    _, _, o9, l9 = chunk_prefill_ref(qb, kb, vb, kp, vp, table[b:b + 1], [cache[b]], rope_theta=30.0)
    assert np.allclose(o2[0], o9[0, :, 3:], atol=1e-12) and np.allclose(l2[0], l9[0, :, 3:], atol=1e-12)
