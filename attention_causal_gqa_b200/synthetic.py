"""Seeded synthetic inputs shaped like the workloads on the pages.

This module only draws random numbers and lays them out (tensor shapes, page
permutation, block table); it contains none of the attention arithmetic. Both the
CUDA path and the CPU oracle consume what it returns.

Recipe (also stated in the design notes):
* values: i.i.d. N(0, 1) * std drawn in float32 by a seeded torch generator on the
  target device, then rounded to the storage dtype (bf16 round-to-nearest-even);
* integer structure (sequence lengths, page permutation): numpy PCG64 seeded from
  the same seed, drawn on the host so it does not depend on the device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_SIZE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "prefill" | "decode" | "mla" | "chunk" | "dsa"
    params: dict = field(default_factory=dict)


# The workloads, named by what they are.
WORKLOADS = {
    "mha_prefill_b1_h4_s256_d64_f32": Workload(
        "mha_prefill_b1_h4_s256_d64_f32", "prefill",
        dict(B=1, Hq=4, Hkv=4, S=256, D=64, dtype="f32", std=1.0, theta=1e4, scale=1.0 / 8.0)),
    "gqa_prefill_b2_hq32_hkv8_s4096_d128": Workload(
        "gqa_prefill_b2_hq32_hkv8_s4096_d128", "prefill",
        dict(B=2, Hq=32, Hkv=8, S=4096, D=128, dtype="bf16", std=1.0, theta=1e4, scale=1.0 / math.sqrt(128))),
    "gqa_prefill_b1_hq32_hkv8_s32768_d128": Workload(
        "gqa_prefill_b1_hq32_hkv8_s32768_d128", "prefill",
        dict(B=1, Hq=32, Hkv=8, S=32768, D=128, dtype="bf16", std=0.5, theta=1e6, scale=1.0 / math.sqrt(128))),
    "paged_decode_b64_hq32_hkv8_d128": Workload(
        "paged_decode_b64_hq32_hkv8_d128", "decode",
        dict(B=64, Hq=32, Hkv=8, D=128, lmin=1024, lmax=32768, std=1.0, scale=1.0 / math.sqrt(128))),
    "chunk_prefill_b8_hq32_hkv8_d128_n2048_cache4k_28k": Workload(
        "chunk_prefill_b8_hq32_hkv8_d128_n2048_cache4k_28k", "chunk",
        dict(B=8, Hq=32, Hkv=8, D=128, S_new=2048, lmin=4096, lmax=28672, std=1.0, theta=1e4,
             scale=1.0 / math.sqrt(128))),
    "mla_decode_b32_h128_dc512_dr64": Workload(
        "mla_decode_b32_h128_dc512_dr64", "mla",
        dict(B=32, H=128, Dc=512, Dr=64, lmin=4096, lmax=32768, std=1.0, scale=1.0 / math.sqrt(192))),
    # the MLA decode workload with a lightning indexer in front: 64 indexer heads of
    # width 128, the 2048 best-scoring cached tokens attended
    "dsa_mla_decode_b32_h128_dc512_dr64_hi64_di128_top2048": Workload(
        "dsa_mla_decode_b32_h128_dc512_dr64_hi64_di128_top2048", "dsa",
        dict(B=32, H=128, Dc=512, Dr=64, lmin=4096, lmax=32768, std=1.0, scale=1.0 / math.sqrt(192),
             HI=64, dI=128, top_k=2048)),
}

_TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, std, dtype, g, device):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(_TORCH_DT[dtype])


def prefill_inputs(B, Hq, Hkv, S, D, dtype="bf16", std=1.0, seed=0, device="cpu"):
    """q [B,Hq,S,D], k [B,Hkv,S,D], v [B,Hkv,S,D] (contiguous, BNHS order)."""
    g = _gen(seed, device)
    q = _randn((B, Hq, S, D), std, dtype, g, device)
    k = _randn((B, Hkv, S, D), std, dtype, g, device)
    v = _randn((B, Hkv, S, D), std, dtype, g, device)
    return q, k, v


def draw_lengths(B, lmin, lmax, seed):
    """Integer lengths uniform in [lmin, lmax] (inclusive), numpy PCG64."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lmin, lmax + 1, size=B).astype(np.int32)


def decode_inputs(B, Hq, Hkv, D, lmin=1024, lmax=32768, std=1.0, seed=0, device="cpu",
                  seq_lens=None, max_pages_per_seq=None, page_size=PAGE_SIZE, dtype="bf16",
                  extra_pages=0):
    """Paged KV cache for one-token decode.

    k_pages, v_pages: [num_pages, page_size, Hkv, D]; every slot is filled with
    random values, including the unused tail of each sequence's last page.
    block_table: [B, max_pages_per_seq] int32; logical page j of sequence b is at
    physical page block_table[b, j]; the physical order is a seeded random
    permutation; entries past the end of a sequence are -1.
    extra_pages adds unreferenced pages to the pool (their content is never read).
    """
    if seq_lens is None:
        seq_lens = draw_lengths(B, lmin, lmax, seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    npages = [int(math.ceil(int(L) / page_size)) for L in seq_lens]
    if max_pages_per_seq is None:
        max_pages_per_seq = max(1, int(math.ceil(lmax / page_size)), max(npages) if npages else 1)
    total = int(sum(npages)) + int(extra_pages)
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    perm = rng.permutation(max(total, 1)).astype(np.int32)
    table = np.full((B, max_pages_per_seq), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npages):
        table[b, :n] = perm[off:off + n]
        off += n
    g = _gen(seed, device)
    q = _randn((B, Hq, D), std, dtype, g, device)
    num_pages = max(total, 1)
    k_pages = _randn((num_pages, page_size, Hkv, D), std, dtype, g, device)
    v_pages = _randn((num_pages, page_size, Hkv, D), std, dtype, g, device)
    return dict(q=q, k_pages=k_pages, v_pages=v_pages,
                block_table=torch.from_numpy(table).to(device),
                seq_lens=torch.from_numpy(seq_lens).to(device),
                max_pages_per_seq=max_pages_per_seq, num_pages=num_pages, page_size=page_size)


def quantize_e4m3(x, page_axis=0, head_axis=2):
    """E4M3 codes of x [num_pages, page_size, Hkv, D] with one scale per (page, head) =
    absmax / 448 (torch's float8_e4m3fn conversion, round to nearest); returns (codes
    uint8, scales fp32 [num_pages, Hkv])."""
    xf = x.float()
    amax = xf.abs().amax(dim=(1, 3)).clamp(min=1e-12)
    sc = amax / 448.0
    codes = (xf / sc[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), sc.contiguous()


def quantize_e4m3_rows(x, block=128):
    """E4M3 codes of x [..., D] with one scale per row and `block`-wide column block =
    absmax / 448 (round to nearest); returns (codes uint8 [..., D], scales fp32 [..., D/block])."""
    xf = x.float()
    shp = xf.shape
    blk = xf.reshape(*shp[:-1], shp[-1] // block, block)
    sc = (blk.abs().amax(dim=-1) / 448.0).clamp(min=1e-12)
    codes = (blk / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(shp)
    return codes.contiguous(), sc.contiguous()


def dsa_inputs_fp8(B, H, Dc, Dr, HI, dI, lmin=4096, lmax=32768, std=1.0, seed=0, device="cpu", seq_lens=None,
                   T_max=None):
    """The DSA inputs of ``dsa_inputs`` with the latent cache quantised to E4M3 (one scale
    per token and 128-wide latent block): kv_codes [B,T,Dc] uint8, kv_scale [B,T,Dc/128] fp32;
    the rotary cache stays bf16."""
    d = dsa_inputs(B, H, Dc, Dr, HI, dI, lmin, lmax, std, seed, device, seq_lens, T_max)
    d["kv_codes"], d["kv_scale"] = quantize_e4m3_rows(d["kv_cache"])
    del d["kv_cache"]
    return d


def decode_inputs_fp8(B, Hq, Hkv, D, lmin=1024, lmax=32768, std=1.0, seed=0, device="cpu", seq_lens=None,
                      max_pages_per_seq=None, extra_pages=0):
    """The paged decode inputs of decode_inputs with K and V pages quantised to E4M3
    (one scale per page and kv head)."""
    d = decode_inputs(B, Hq, Hkv, D, lmin, lmax, std, seed, device, seq_lens, max_pages_per_seq,
                      extra_pages=extra_pages)
    d["k_pages"], d["k_scale"] = quantize_e4m3(d["k_pages"])
    d["v_pages"], d["v_scale"] = quantize_e4m3(d["v_pages"])
    return d


def mla_inputs(B, H, Dc, Dr, lmin=4096, lmax=32768, std=1.0, seed=0, device="cpu", seq_lens=None,
               T_max=None):
    """Absorbed-MLA decode inputs: q_nope [B,1,H,Dc], q_pe [B,1,H,Dr],
    kv_cache [B,T_max,Dc], pe_cache [B,T_max,Dr] (filled beyond each length too),
    seq_lens [B] int32."""
    if seq_lens is None:
        seq_lens = draw_lengths(B, lmin, lmax, seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    if T_max is None:
        T_max = max(int(lmax), int(seq_lens.max()) if len(seq_lens) else 1)
    g = _gen(seed, device)
    q_nope = _randn((B, 1, H, Dc), std, "bf16", g, device)
    q_pe = _randn((B, 1, H, Dr), std, "bf16", g, device)
    kv = _randn((B, T_max, Dc), std, "bf16", g, device)
    pe = _randn((B, T_max, Dr), std, "bf16", g, device)
    return dict(q_nope=q_nope, q_pe=q_pe, kv_cache=kv, pe_cache=pe,
                seq_lens=torch.from_numpy(seq_lens).to(device), T_max=T_max)


def dsa_inputs(B, H, Dc, Dr, HI, dI, lmin=4096, lmax=32768, std=1.0, seed=0, device="cpu", seq_lens=None,
               T_max=None):
    """The MLA decode inputs of ``mla_inputs`` (same seed, same tensors) plus the lightning
    indexer's inputs: q_idx [B,HI,dI] bf16 (one query per indexer head), w_idx [B,HI] fp32
    head weights drawn N(0, 1/HI), k_idx [B,T_max,dI] bf16 (one key per cached token,
    filled beyond each length too)."""
    d = mla_inputs(B, H, Dc, Dr, lmin, lmax, std, seed, device, seq_lens, T_max)
    g = _gen(seed + 104729, device)
    d["q_idx"] = _randn((B, HI, dI), std, "bf16", g, device)
    d["w_idx"] = _randn((B, HI), 1.0 / math.sqrt(HI), "f32", g, device)
    d["k_idx"] = _randn((B, d["T_max"], dI), std, "bf16", g, device)
    return d


def chunk_inputs(B, Hq, Hkv, D, S_new, lmin=4096, lmax=28672, std=1.0, seed=0, device="cpu", cache_lens=None,
                 page_size=PAGE_SIZE):
    """A chunk of S_new new tokens per sequence and a paged cache that already holds
    cache_lens[b] tokens (lengths uniform in [lmin, lmax] unless given). Pages for the
    cached prefix and the chunk are mapped in a seeded random physical order; every
    slot is filled with random values. q, k, v: [B, H, S_new, D] bf16 (not rotated)."""
    if cache_lens is None:
        cache_lens = draw_lengths(B, lmin, lmax, seed)
    cache_lens = np.asarray(cache_lens, dtype=np.int32)
    npages = [int(math.ceil((int(L) + S_new) / page_size)) for L in cache_lens]
    max_pages = max(npages)
    total = int(sum(npages))
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    perm = rng.permutation(total).astype(np.int32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npages):
        table[b, :n] = perm[off:off + n]
        off += n
    g = _gen(seed, device)
    q = _randn((B, Hq, S_new, D), std, "bf16", g, device)
    k = _randn((B, Hkv, S_new, D), std, "bf16", g, device)
    v = _randn((B, Hkv, S_new, D), std, "bf16", g, device)
    k_pages = _randn((total, page_size, Hkv, D), std, "bf16", g, device)
    v_pages = _randn((total, page_size, Hkv, D), std, "bf16", g, device)
    return dict(q=q, k=k, v=v, k_pages=k_pages, v_pages=v_pages, block_table=torch.from_numpy(table).to(device),
                cache_lens=torch.from_numpy(cache_lens).to(device), max_cache_len=int(cache_lens.max()))


def workload_inputs(name: str, seed: int = 20261202, device="cpu"):
    w = WORKLOADS[name]
    p = w.params
    if w.kind == "prefill":
        return prefill_inputs(p["B"], p["Hq"], p["Hkv"], p["S"], p["D"], p["dtype"], p["std"], seed, device)
    if w.kind == "decode":
        return decode_inputs(p["B"], p["Hq"], p["Hkv"], p["D"], p["lmin"], p["lmax"], p["std"], seed, device)
    if w.kind == "chunk":
        return chunk_inputs(p["B"], p["Hq"], p["Hkv"], p["D"], p["S_new"], p["lmin"], p["lmax"], p["std"], seed, device)
    if w.kind == "dsa":
        return dsa_inputs(p["B"], p["H"], p["Dc"], p["Dr"], p["HI"], p["dI"], p["lmin"], p["lmax"], p["std"], seed,
                          device)
    return mla_inputs(p["B"], p["H"], p["Dc"], p["Dr"], p["lmin"], p["lmax"], p["std"], seed, device)
