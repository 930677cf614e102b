"""Multi-GPU split of the hot path (one process per GPU).

Decode and MLA shard the KV sequence: every rank holds a contiguous slice of each
sequence's cache, attends the query over its slice with the single-GPU kernels, and
the ranks' partial results (outputs and LSEs) are all-gathered and combined by the
LSE merge (attn_lse_merge) — the block-level form of the online-softmax recurrence
("attention study note", section "online-softmax 分块计算原理"). Prefill needs no
exchange: its (batch, kv-head) units are independent and are dealt out in contiguous
ranges. The only collective is one all-gather of the partials per decode step; every
TMA load of the library reads this GPU's own memory into the issuing CTA, and no library
kernel ever reads another GPU's memory.

The partition functions are plain host code; ``split_and_merge`` runs any
(attend, merge) pair over a torch.distributed group, so the same orchestration serves
the CUDA path (``decode_sequence_parallel``, ``mla_sequence_parallel``) and host tests.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def unit_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Rank `rank`'s contiguous run of n_units: [floor(n r / W), floor(n (r + 1) / W))."""
    return n_units * rank // world, n_units * (rank + 1) // world


def kv_slice(seq_len: int, rank: int, world: int, unit: int) -> tuple[int, int]:
    """Rank `rank`'s tokens [start, start + length) of a sequence of seq_len tokens, cut
    in whole units of `unit` tokens (16-token pages for paged decode, any tile for MLA)."""
    n = (max(seq_len, 0) + unit - 1) // unit
    u0, u1 = unit_range(n, rank, world)
    start = u0 * unit
    return start, max(0, min(seq_len, u1 * unit) - start)


def local_block_table(block_table: torch.Tensor, seq_lens: torch.Tensor, rank: int, world: int,
                      page_size: int = 16) -> tuple[torch.Tensor, torch.Tensor]:
    """The paged-decode view of rank `rank`: row b lists the physical pages of its slice of
    sequence b (the rest -1), with the slice's length. Pages stay where they are, so a rank
    only ever reads pages of its own slice."""
    lens = [int(x) for x in seq_lens.tolist()]
    starts_lens = [kv_slice(L, rank, world, page_size) for L in lens]
    width = max(1, max((n + page_size - 1) // page_size for _, n in starts_lens))
    table = torch.full((len(lens), width), -1, dtype=torch.int32, device=block_table.device)
    for b, (s, n) in enumerate(starts_lens):
        p0, np_ = s // page_size, (n + page_size - 1) // page_size
        if np_:
            table[b, :np_] = block_table[b, p0:p0 + np_]
    return table, torch.tensor([n for _, n in starts_lens], dtype=torch.int32, device=seq_lens.device)


def prefill_units(B: int, Hkv: int, rank: int, world: int) -> list[tuple[int, int]]:
    """Rank `rank`'s (batch, kv head) units of a prefill, a contiguous range of the
    B * Hkv units (a unit covers the query heads of its kv head; no exchange needed)."""
    u0, u1 = unit_range(B * Hkv, rank, world)
    return [(u // Hkv, u % Hkv) for u in range(u0, u1)]


def gather_partials(out: torch.Tensor, lse: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """All-gathers every rank's partial output and LSE into [world, ...] tensors (in the
    memory of this rank's device)."""
    world = dist.get_world_size(group)
    o_parts = torch.empty((world, *out.shape), dtype=out.dtype, device=out.device)
    l_parts = torch.empty((world, *lse.shape), dtype=lse.dtype, device=lse.device)
    dist.all_gather(list(o_parts.unbind(0)), out.contiguous(), group=group)
    dist.all_gather(list(l_parts.unbind(0)), lse.contiguous(), group=group)
    return o_parts, l_parts


def split_and_merge(attend_local, merge, group=None):
    """attend_local() -> (out, lse) of this rank's slice; the partials of all ranks are
    gathered and merge(o_parts, lse_parts) -> (out, lse) combines them."""
    out, lse = attend_local()
    return merge(*gather_partials(out, lse, group))


def decode_sequence_parallel(q, k_pages, v_pages, block_table, seq_lens, scale=None, group=None):
    """Paged GQA decode with the KV sequence split across the ranks of `group`: rank r
    attends to its slice of every sequence (pages of the global block table) and the
    partials are merged on every rank. Returns (out [B,Hq,D] bf16, lse [B,Hq] fp32)."""
    from . import binding
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    table, lens = local_block_table(block_table, seq_lens, rank, world, k_pages.shape[1])
    return split_and_merge(
        lambda: binding.attn_decode_paged(q, k_pages, v_pages, table, lens, scale=scale),
        binding.lse_merge, group)


def mla_sequence_parallel(q_nope, q_pe, kv_local, pe_local, lens_local, scale, group=None):
    """MLA absorbed decode over a cache that is itself sharded: kv_local / pe_local hold
    this rank's slice of every sequence (rows [0, lens_local[b]), e.g. the slice of
    kv_slice(L, rank, world, unit)). Returns (out [B,1,H,Dc] bf16, lse [B,1,H] fp32)."""
    from . import binding
    return split_and_merge(lambda: binding.mla_decode(q_nope, q_pe, kv_local, pe_local, lens_local, scale),
                           binding.lse_merge, group)
