"""Plain float64 CPU oracle for exact causal GQA attention, paged decode and MLA decode.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it. It shares no code with the CUDA library.

Every function computes the plain definition of what the method reaches, in the
order the pages state it, with no blocking, fusion or reordering beyond what that
definition allows:

* "attention study note" (makinaruto.github.io, llm_learning/attention), section
  "传统分块计算过程" (the standard, unfused flow): the full score row S = Q K^T is
  materialised, softmax is taken over it, and O = P V. The oracle follows that
  flow with a two-pass softmax (max, then exp/sum).
* same page, section "online-softmax 分块计算原理": the running-max / running-sum
  recurrence. ``online_softmax_merge`` writes it out (with the maximum read as
  max(m_old, m_c); the page prints a minus sign there) together with the
  output-accumulator rescaling that the recurrence implies.
* same page, section "一些推导" under GQA: the worked 4-head, 2-group table maps
  Q1,Q2 to K1 and Q3,Q4 to K2, i.e. query head h reads kv head h // (Hq/Hkv).
* same page, section "Page Attention": keys and values live in fixed-size pages
  reached through a per-sequence table of physical page numbers.
* "From 32K to 256K: DeepSeek long-context" (tqpw.cn), section 2.1: RoPE with
  theta_i = base^(-2i/d) rotating adjacent (even, odd) pairs by pos * theta_i;
  section 2.5: the cos/sin cache of shape [max_len, head_dim/2, 2] built once
  from integer positions (no accumulated phase).
* "DeepSeek-V3 attention: einsum vs hand-optimised" (dksg.cn), absorbed MLA
  scores: scores = (q_nope . kv_cache^T + q_pe . pe_cache^T) * scale, and
  out = softmax(scores) . kv_cache.
* "attention study note", section "Lighting Indexer": index score of a token =
  sum over indexer heads j of w_j * ReLU(q_j . k_s); only the most relevant tokens
  are attended (DeepSeek sparse attention).
* "7 anti-patterns of DeepSeek attention optimisation" (lpnh.cn), section 3.3: the
  FP8 E4M3 format (largest value 448) with scale factors.

Readings taken where the pages are silent or garbled (all also listed in the
design notes): RoPE positions start at 0 for Q and K; the score scale multiplies
Q K^T before the softmax; LSE is the natural log of the sum of exp of the scaled
scores; decode and MLA inputs arrive already rotated and attend to every cached
token; a sequence of length 0 gives out = 0 and lse = -inf.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64
_ROW_BLOCK = 1024  # rows of the score matrix materialised at once (memory only)


# --------------------------------------------------------------------------- RoPE
def rope_cache(seq_len: int, head_dim: int, theta: float, freq_scale: float = 1.0) -> np.ndarray:
    """cos/sin cache [seq_len, head_dim/2, 2] in float64.

    Long-context page, section 2.5 (cache layout) and section 2.1 (theta_i =
    theta^(-2i/d)). Each angle is pos * theta_i computed directly from the
    integer position, never by accumulation. freq_scale multiplies every theta_i
    (section 2.2's frequency scaling; 1 = plain RoPE).
    """
    if head_dim % 2:
        raise ValueError("RoPE needs an even head dimension")
    i = np.arange(head_dim // 2, dtype=F64)
    inv_freq = F64(freq_scale) * np.power(F64(theta), -2.0 * i / head_dim)
    pos = np.arange(seq_len, dtype=F64)
    ang = pos[:, None] * inv_freq[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def ntk_aware_theta_ref(theta: float, scale: float, head_dim: int) -> float:
    """NTK-aware RoPE base for a context stretched by ``scale`` ("From 32K to 256K:
    DeepSeek long-context", section 2.2 names NTK-aware scaling; the rule is the published
    one): rescale the base so that the lowest rotary frequency theta^(-(D-2)/D) is divided
    by ``scale`` while the highest (pair 0, frequency 1) stays: theta' = theta * scale^(D/(D-2))."""
    return float(theta) * float(scale) ** (float(head_dim) / (head_dim - 2.0))


def length_scaled_theta_ref(theta: float, length: int, base_length: int, alpha: float) -> float:
    """Length-aware RoPE base of the same page, section 2.4: theta * (L / L0)^alpha."""
    return float(theta) * (float(length) / float(base_length)) ** float(alpha)


def _pair_slices(d: int, layout: str):
    """The two members of each rotated pair: adjacent (2i, 2i+1) ("interleaved", the
    long-context page's section 2.1) or the two halves (i, i + d/2) ("half", the
    concatenated-halves form of its section 2.4)."""
    if layout == "interleaved":
        return slice(0, None, 2), slice(1, None, 2)
    if layout == "half":
        return slice(0, d // 2), slice(d // 2, d)
    raise ValueError(f"unknown RoPE layout {layout!r}")


def apply_rope(x: np.ndarray, theta: float, positions: np.ndarray | None = None, freq_scale: float = 1.0,
               layout: str = "interleaved") -> np.ndarray:
    """Rotate the pairs of the last axis by pos * freq_scale * theta_i.

    Long-context page, section 2.1: [x0 cos - x1 sin, x0 sin + x1 cos] on the pair
    (x0, x1). ``x`` is [..., S, D]; positions default to 0..S-1.
    """
    x = np.asarray(x, dtype=F64)
    s, d = x.shape[-2], x.shape[-1]
    if positions is None:
        cs = rope_cache(s, d, theta, freq_scale)
    else:
        i = np.arange(d // 2, dtype=F64)
        inv_freq = F64(freq_scale) * np.power(F64(theta), -2.0 * i / d)
        ang = np.asarray(positions, dtype=F64)[:, None] * inv_freq[None, :]
        cs = np.stack([np.cos(ang), np.sin(ang)], axis=-1)
    cos, sin = cs[..., 0], cs[..., 1]
    a, b = _pair_slices(d, layout)
    x0 = x[..., a]
    x1 = x[..., b]
    out = np.empty_like(x)
    out[..., a] = x0 * cos - x1 * sin
    out[..., b] = x0 * sin + x1 * cos
    return out


# ----------------------------------------------------------------- softmax pieces
def two_pass_softmax_rows(scores: np.ndarray):
    """Return (P, lse) for score rows, two passes: row max, then exp and sum.

    Rows whose every entry is -inf (nothing to attend) give P = 0 and lse = -inf.
    """
    m = np.max(scores, axis=-1, keepdims=True)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(scores - m_safe)
    l = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
        lse = np.where(finite[..., 0], m_safe[..., 0] + np.log(np.where(l[..., 0] > 0, l[..., 0], 1.0)), -np.inf)
    return p, lse


def online_softmax_merge(blocks_scores, blocks_values):
    """Attention over a row of key blocks using the page's running-statistics recurrence.

    Attention study note, section "online-softmax 分块计算原理":
        m_new = max(m_old, m_c)
        l_new = l_old * exp(m_old - m_new) + l_c * exp(m_c - m_new)
    where m_c, l_c are the current block's max and sum of exp(s - m_c). The output
    accumulator is rescaled by the same factors (the page leaves that step
    implicit): acc_new = acc_old * exp(m_old - m_new) + (sum_j exp(s_j - m_c) v_j) * exp(m_c - m_new).
    Returns (o, lse) for one query row. Used only to pin the oracle.
    """
    m_old, l_old, acc = -np.inf, 0.0, None
    for s, v in zip(blocks_scores, blocks_values):
        s = np.asarray(s, dtype=F64)
        v = np.asarray(v, dtype=F64)
        m_c = float(np.max(s))
        e = np.exp(s - m_c)
        l_c = float(np.sum(e))
        acc_c = e @ v
        m_new = max(m_old, m_c)
        a_old = math.exp(m_old - m_new) if np.isfinite(m_old) else 0.0
        a_c = math.exp(m_c - m_new)
        l_old = l_old * a_old + l_c * a_c
        acc = acc_c * a_c if acc is None else acc * a_old + acc_c * a_c
        m_old = m_new
    return acc / l_old, m_old + math.log(l_old)


def lse_merge(partial_o, partial_lse):
    """Combine partial results of disjoint key sets: o_s (normalised) and lse_s.

    The same recurrence at block level: L = max_s lse_s, w_s = exp(lse_s - L),
    lse = L + ln(sum w_s), o = sum w_s o_s / sum w_s. Partials with lse = -inf
    (empty key sets) carry zero weight.
    """
    po = np.asarray(partial_o, dtype=F64)
    pl = np.asarray(partial_lse, dtype=F64)
    big = np.max(pl, axis=0)
    if not np.isfinite(big):
        return np.zeros(po.shape[1:]), -np.inf
    w = np.exp(pl - big)
    tot = np.sum(w)
    o = np.tensordot(w, po, axes=(0, 0)) / tot
    return o, big + math.log(tot)


# -------------------------------------------------------------------- prefill
def prefill_ref(q, k, v, causal: bool = True, rope_theta: float = 10000.0, scale: float | None = None,
                rows=None, rope_freq_scale: float = 1.0, rope_layout: str = "interleaved"):
    """Exact (causal) GQA/MQA/MHA attention with RoPE on Q and K.

    q: [B, Hq, S, D]; k, v: [B, Hkv, S, D] (any float dtype, upcast to float64).
    rope_theta <= 0 disables RoPE; rope_freq_scale and rope_layout as ``apply_rope``.
    scale defaults to 1/sqrt(D).
    rows: optional iterable of (b, h, i) triples; when given, only those output rows
    are computed and returned as (o [n, D], lse [n]). Otherwise returns full
    (o [B, Hq, S, D], lse [B, Hq, S]).

    Head map: kv head = h // (Hq // Hkv) (contiguous groups, attention study note,
    GQA worked table). Scores are materialised row block by row block, each row
    in full; mask j > i to -inf when causal; two-pass softmax; O = P V.
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    if rope_theta and rope_theta > 0:
        cs = rope_cache(S, D, rope_theta, rope_freq_scale)
        pa, pb = _pair_slices(D, rope_layout)

        def rot(x):
            out = np.empty_like(x)
            c, s_ = cs[..., 0], cs[..., 1]
            out[..., pa] = x[..., pa] * c - x[..., pb] * s_
            out[..., pb] = x[..., pa] * s_ + x[..., pb] * c
            return out
    else:
        def rot(x):
            return x

    if rows is not None:
        rows = list(rows)
        o = np.zeros((len(rows), D))
        lse = np.zeros(len(rows))
        cache_k = {}
        for n, (b, h, i) in enumerate(rows):
            kvh = h // G
            if (b, kvh) not in cache_k:
                cache_k[(b, kvh)] = rot(k[b, kvh])
            kr = cache_k[(b, kvh)]
            qi = q[b, h, i][None, :]
            qi_r = (rot_one(qi, i, D, rope_theta, rope_freq_scale, rope_layout) if (rope_theta and rope_theta > 0)
                    else qi)
            hi = i + 1 if causal else S
            s = scale * (qi_r @ kr[:hi].T)
            p, l_ = two_pass_softmax_rows(s)
            o[n] = (p @ v[b, kvh, :hi])[0]
            lse[n] = l_[0]
        return o, lse

    o = np.zeros((B, Hq, S, D))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for kvh in range(Hkv):
            kr = rot(k[b, kvh])
            vv = v[b, kvh]
            for h in range(kvh * G, (kvh + 1) * G):
                qr = rot(q[b, h])
                for r0 in range(0, S, _ROW_BLOCK):
                    r1 = min(S, r0 + _ROW_BLOCK)
                    s = scale * (qr[r0:r1] @ kr.T)
                    if causal:
                        ii = np.arange(r0, r1)[:, None]
                        jj = np.arange(S)[None, :]
                        s = np.where(jj > ii, -np.inf, s)
                    p, l_ = two_pass_softmax_rows(s)
                    o[b, h, r0:r1] = p @ vv
                    lse[b, h, r0:r1] = l_
    return o, lse


def rot_one(x, pos: int, D: int, theta: float, freq_scale: float = 1.0, layout: str = "interleaved"):
    """RoPE of row vector(s) x [n, D] at a single position ``pos``."""
    return apply_rope(x, theta, positions=np.full(x.shape[0], pos), freq_scale=freq_scale, layout=layout)


# --------------------------------------------------------------- paged decode
def gather_pages(pages, block_table_row, seq_len: int, page_size: int):
    """Logical token t of a sequence lives in physical page table[t // page_size],
    slot t % page_size (attention study note, section "Page Attention").
    pages: [num_pages, page_size, Hkv, D] -> [seq_len, Hkv, D]."""
    t = np.arange(seq_len)
    phys = np.asarray(block_table_row)[t // page_size]
    return np.asarray(pages)[phys, t % page_size]


def decode_paged_ref(q, k_pages, v_pages, block_table, seq_lens, scale: float | None = None,
                     page_size: int = 16, pairs=None):
    """One-token GQA decode over a paged KV cache.

    q: [B, Hq, D]; k_pages, v_pages: [num_pages, page_size, Hkv, D];
    block_table: [B, max_pages] int; seq_lens: [B] int.
    The query attends to every cached token t < seq_lens[b] (no mask, no RoPE:
    cached keys are already rotated). pairs: optional list of (b, h) to compute
    only those rows; returns (o [n, D], lse [n]). Otherwise (o [B, Hq, D], lse [B, Hq]).
    """
    q = np.asarray(q, dtype=F64)
    B, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    if pairs is None:
        pairs_l = [(b, h) for b in range(B) for h in range(Hq)]
    else:
        pairs_l = list(pairs)
    o = np.zeros((len(pairs_l), D))
    lse = np.zeros(len(pairs_l))
    cache = {}
    for n, (b, h) in enumerate(pairs_l):
        L = int(seq_lens[b])
        if L == 0:
            o[n] = 0.0
            lse[n] = -np.inf
            continue
        if b not in cache:
            kk = gather_pages(k_pages, block_table[b], L, page_size).astype(F64)
            vv = gather_pages(v_pages, block_table[b], L, page_size).astype(F64)
            cache = {b: (kk, vv)}
        kk, vv = cache[b]
        kvh = h // G
        s = scale * (kk[:, kvh, :] @ q[b, h])
        p, l_ = two_pass_softmax_rows(s[None, :])
        o[n] = (p @ vv[:, kvh, :])[0]
        lse[n] = l_[0]
    if pairs is None:
        return o.reshape(B, Hq, D), lse.reshape(B, Hq)
    return o, lse


# ------------------------------------------- chunked prefill into the paged cache
def to_bf16(x):
    """Round values to bfloat16 (round to nearest, ties to even) and return them as
    float64: the precision a bf16 KV cache stores."""
    x32 = np.asarray(x, dtype=np.float32)
    b = x32.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(F64)


def chunk_prefill_ref(q, k_new, v_new, k_pages, v_pages, block_table, cache_lens, rope_theta: float = 10000.0,
                      scale: float | None = None, page_size: int = 16, store=to_bf16, rope_freq_scale: float = 1.0,
                      rope_layout: str = "interleaved", new_lens=None):
    """Append a chunk of new tokens to a paged KV cache and attend over the whole cache.

    "From 32K to 256K: DeepSeek long-context", chapter 1 (key architecture path: a
    streaming KV cache for incremental processing, long sequences cut into chunks, a
    PagedAttention variant); "attention study note", section "Page Attention" (pages
    reached through a per-sequence block table).

    q: [B, Hq, S_new, D]; k_new, v_new: [B, Hkv, S_new, D], not rotated. New token i of
    sequence b sits at position cache_lens[b] + i. k_pages, v_pages: [num_pages,
    page_size, Hkv, D]; the first cache_lens[b] tokens of sequence b are already there
    (keys rotated). block_table: [B, max_pages].

    Steps: rotate the new keys at their positions and write them and the new values
    into their pages with ``store`` (the cache's precision, bf16); rotate the queries at
    the same positions (float64); query i attends the stored keys t <= cache_lens[b] + i
    (the causal mask aligned to the end of the cache), two-pass softmax, O = P V.
    rope_freq_scale and rope_layout as ``apply_rope`` (the cached keys are taken as
    rotated the same way).
    new_lens: optional [B] chunk lengths (0 <= new_lens[b] <= S_new, a batch of chunks of
    different lengths padded to S_new): sequence b appends and attends only its first
    new_lens[b] new tokens; its rows past them are o = 0, lse = -inf.
    Returns (k_pages', v_pages', o [B, Hq, S_new, D], lse [B, Hq, S_new]).
    """
    q = np.asarray(q, dtype=F64)
    k_new = np.asarray(k_new, dtype=F64)
    v_new = np.asarray(v_new, dtype=F64)
    kp = np.array(k_pages, dtype=F64)
    vp = np.array(v_pages, dtype=F64)
    B, Hq, S_new, D = q.shape
    Hkv = k_new.shape[1]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    use_rope = rope_theta and rope_theta > 0
    o = np.zeros((B, Hq, S_new, D))
    lse = np.full((B, Hq, S_new), -np.inf)
    for b in range(B):
        L = int(cache_lens[b])
        n = S_new if new_lens is None else int(new_lens[b])
        if n == 0:
            continue
        pos = L + np.arange(n)
        table = np.asarray(block_table[b])
        for kvh in range(Hkv):
            kr = (apply_rope(k_new[b, kvh, :n], rope_theta, positions=pos, freq_scale=rope_freq_scale,
                             layout=rope_layout) if use_rope else k_new[b, kvh, :n])
            kp[table[pos // page_size], pos % page_size, kvh] = store(kr)
            vp[table[pos // page_size], pos % page_size, kvh] = store(v_new[b, kvh, :n])
        kk = gather_pages(kp, table, L + n, page_size)
        vv = gather_pages(vp, table, L + n, page_size)
        for h in range(Hq):
            kvh = h // G
            qr = (apply_rope(q[b, h, :n], rope_theta, positions=pos, freq_scale=rope_freq_scale, layout=rope_layout)
                  if use_rope else q[b, h, :n])
            s = scale * (qr @ kk[:, kvh, :].T)
            jj = np.arange(L + n)[None, :]
            s = np.where(jj > pos[:, None], -np.inf, s)
            p, l_ = two_pass_softmax_rows(s)
            o[b, h, :n] = p @ vv[:, kvh, :]
            lse[b, h, :n] = l_
    return kp, vp, o, lse


# ------------------------------------------------------ FP8 (E4M3) paged decode
def e4m3_to_float(codes):
    """Value of FP8 E4M3 codes (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent 0 encodes subnormals m/8 * 2^-6; 0x7F and 0xFF are NaN, there is no
    infinity), as float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(F64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def decode_paged_fp8_ref(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale: float | None = None,
                         page_size: int = 16, pairs=None):
    """One-token GQA decode over an FP8 (E4M3) paged KV cache with one scale per
    (page, kv head): the cached key is e4m3(code) * k_scale[page, head] (likewise the
    value), then exactly ``decode_paged_ref`` on those values.
    k_codes, v_codes: [num_pages, page_size, Hkv, D] uint8; k_scale, v_scale: [num_pages, Hkv]."""
    # Only the pages of the sequences that are computed are dequantised (same values;
    # the block table is renumbered onto the compact page list).
    table = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    seqs = range(table.shape[0]) if pairs is None else sorted({b for b, _ in pairs})
    used = sorted({int(table[b, j]) for b in seqs for j in range((int(lens[b]) + page_size - 1) // page_size)})
    remap = {pg: i for i, pg in enumerate(used)}
    table2 = np.zeros_like(table)
    for b in seqs:
        for j in range((int(lens[b]) + page_size - 1) // page_size):
            table2[b, j] = remap[int(table[b, j])]
    idx = np.asarray(used, dtype=np.int64)
    kf = e4m3_to_float(np.asarray(k_codes)[idx]) * np.asarray(k_scale, dtype=F64)[idx][:, None, :, None]
    vf = e4m3_to_float(np.asarray(v_codes)[idx]) * np.asarray(v_scale, dtype=F64)[idx][:, None, :, None]
    if not used:
        kf = np.zeros((1,) + np.asarray(k_codes).shape[1:])
        vf = np.zeros_like(kf)
    return decode_paged_ref(q, kf, vf, table2, lens, scale=scale, page_size=page_size, pairs=pairs)


# ------------------------------------------------------------------ MLA decode
def mla_decode_ref(q_nope, q_pe, kv_cache, pe_cache, seq_lens, scale: float, pairs=None):
    """DeepSeek MLA absorbed decode (einsum vs hand-optimised page, absorbed form).

    q_nope [B, 1, H, Dc], q_pe [B, 1, H, Dr], kv_cache [B, T, Dc], pe_cache [B, T, Dr].
    scores[h, t] = (q_nope[h] . kv_cache[t] + q_pe[h] . pe_cache[t]) * scale for t < seq_lens[b];
    out[h] = softmax(scores[h]) . kv_cache (latent space). Two-pass softmax.
    pairs: optional list of (b, h). Returns (out [B,1,H,Dc], lse [B,1,H]) or
    (out [n, Dc], lse [n]).
    """
    B, _, H, Dc = q_nope.shape
    if pairs is None:
        pairs_l = [(b, h) for b in range(B) for h in range(H)]
    else:
        pairs_l = list(pairs)
    o = np.zeros((len(pairs_l), Dc))
    lse = np.zeros(len(pairs_l))
    cache = {}
    for n, (b, h) in enumerate(pairs_l):
        L = int(seq_lens[b])
        if L == 0:
            o[n] = 0.0
            lse[n] = -np.inf
            continue
        if b not in cache:
            kv = np.asarray(kv_cache[b, :L], dtype=F64)
            pe = np.asarray(pe_cache[b, :L], dtype=F64)
            cache = {b: (kv, pe)}
        kv, pe = cache[b]
        qn = np.asarray(q_nope[b, 0, h], dtype=F64)
        qp = np.asarray(q_pe[b, 0, h], dtype=F64)
        s = (kv @ qn + pe @ qp) * scale
        p, l_ = two_pass_softmax_rows(s[None, :])
        o[n] = (p @ kv)[0]
        lse[n] = l_[0]
    if pairs is None:
        return o.reshape(B, 1, H, Dc), lse.reshape(B, 1, H)
    return o, lse


def mla_naive_ref(x_q, c_kv, k_pe, w_uk, w_uv, q_pe, scale: float):
    """Naive (non-absorbed) MLA for one sequence, used only to pin the absorbed form.

    Attention study note, MLA derivation: K_h = C^KV W^K_up,h and V_h = C^KV W^V_up,h,
    with the decoupled rotary part concatenated (q = [q_h, q_pe,h], k = [K_h, k_pe],
    k_pe shared across heads). x_q: [H, dk] per-head query (content part);
    c_kv: [T, Dc]; k_pe: [T, Dr]; w_uk, w_uv: [H, Dc, dk]; q_pe: [H, Dr].
    Returns per-head outputs in value space [H, dk] and lse [H].
    """
    H = x_q.shape[0]
    outs, lses = [], []
    for h in range(H):
        K = np.concatenate([c_kv @ w_uk[h], k_pe], axis=1)
        V = c_kv @ w_uv[h]
        qh = np.concatenate([x_q[h], q_pe[h]])
        s = scale * (K @ qh)
        p, l_ = two_pass_softmax_rows(s[None, :])
        outs.append((p @ V)[0])
        lses.append(l_[0])
    return np.stack(outs), np.array(lses)


# ---------------------------------------------------------------------------
# DeepSeek sparse attention: lightning indexer, top-k selection, MLA over the
# selected tokens ("attention study note", section "Lighting Indexer").
# ---------------------------------------------------------------------------
def dsa_index_scores_ref(q_idx, w_idx, k_idx, seq_lens):
    """Lightning-indexer scores for one decode query per sequence.

    The page forms indexer queries q_j (one per indexer head j) and one indexer key
    k_s per token, and sums w_j * ReLU(q_j . k_s) over the heads into the token's
    index score:  I[b, s] = sum_j w[b, j] * max(q[b, j] . k[b, s], 0)  for s < seq_lens[b],
    and -inf for the slots past the sequence (never selected).
    q_idx [B, H_I, d_I], w_idx [B, H_I], k_idx [B, T, d_I]. Returns [B, T] float64."""
    q = np.asarray(q_idx, dtype=F64)
    w = np.asarray(w_idx, dtype=F64)
    B, T = k_idx.shape[0], k_idx.shape[1]
    out = np.full((B, T), -np.inf)
    for b in range(B):
        L = min(max(int(seq_lens[b]), 0), T)
        if L == 0:
            continue
        k = np.asarray(k_idx[b, :L], dtype=F64)
        dots = q[b] @ k.T  # [H_I, L]
        out[b, :L] = w[b] @ np.maximum(dots, 0.0)
    return out


def dsa_topk_ref(scores, seq_lens, top_k: int):
    """The tokens kept for attention: the min(top_k, L) cached tokens with the largest
    index scores. Ties are broken toward the smaller token index (a reading: the page
    does not say), so the set is unique. Returned per sequence in ascending token order."""
    res = []
    for b in range(scores.shape[0]):
        L = min(max(int(seq_lens[b]), 0), scores.shape[1])
        n = min(int(top_k), L)
        if n <= 0:
            res.append(np.zeros(0, dtype=np.int64))
            continue
        s = np.asarray(scores[b, :L], dtype=F64)
        order = np.lexsort((np.arange(L), -s))  # score descending, then index ascending
        res.append(np.sort(order[:n]))
    return res


def dsa_mla_decode_ref(q_nope, q_pe, kv_cache, pe_cache, indices, scale: float, pairs=None):
    """MLA absorbed decode restricted to the selected tokens: exactly ``mla_decode_ref``
    over the rows kv_cache[b, indices[b]] and pe_cache[b, indices[b]] (attention is
    invariant to the order of its keys, so the ascending order changes nothing)."""
    B = q_nope.shape[0]
    n = [len(ix) for ix in indices]
    t = max([1] + n)
    kv = np.zeros((B, t, kv_cache.shape[2]))
    pe = np.zeros((B, t, pe_cache.shape[2]))
    seqs = range(B) if pairs is None else sorted({b for b, _ in pairs})
    for b in seqs:
        ix = np.asarray(indices[b], dtype=np.int64)
        if len(ix):
            kv[b, :len(ix)] = np.asarray(kv_cache[b][ix], dtype=F64)
            pe[b, :len(ix)] = np.asarray(pe_cache[b][ix], dtype=F64)
    return mla_decode_ref(q_nope, q_pe, kv, pe, n, scale, pairs=pairs)


def dsa_mla_decode_fp8_ref(q_nope, q_pe, kv_codes, kv_scale, pe_cache, indices, scale: float, pairs=None,
                           block: int = 128):
    """Sparse MLA decode over an FP8 (E4M3) latent cache: the latent row of token t is
    e4m3(kv_codes[b, t, c]) * kv_scale[b, t, c // block] ("7 anti-patterns of DeepSeek
    attention optimisation", section 3.3: E4M3 with scale factors; one scale per token and
    128-wide latent block is a reading), the rotary cache stays bf16; then exactly
    ``dsa_mla_decode_ref`` over those values. Only the selected rows are dequantised."""
    B, Dc = kv_codes.shape[0], kv_codes.shape[2]
    n = [len(ix) for ix in indices]
    t = max([1] + n)
    kv = np.zeros((B, t, Dc))
    pe = np.zeros((B, t, pe_cache.shape[2]))
    seqs = range(B) if pairs is None else sorted({b for b, _ in pairs})
    for b in seqs:
        ix = np.asarray(indices[b], dtype=np.int64)
        if len(ix):
            codes = np.asarray(kv_codes[b][ix])
            sc = np.asarray(kv_scale[b][ix], dtype=F64)
            kv[b, :len(ix)] = e4m3_to_float(codes) * np.repeat(sc, block, axis=1)[:, :Dc]
            pe[b, :len(ix)] = np.asarray(pe_cache[b][ix], dtype=F64)
    return dsa_mla_decode_ref(q_nope, q_pe, kv, pe, [np.arange(m) for m in n], scale, pairs=pairs)
