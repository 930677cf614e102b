"""Thin ctypes binding over libattn_b200.so (argument marshalling only).

Every step of the attention path runs in the CUDA library; this module only
allocates outputs / workspace through torch (device memory plumbing), passes
raw pointers and the current CUDA stream, and turns error codes into
exceptions. There is no CPU fallback: if the library is missing, importing
this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_DEVICE = 5
ATTN_DTYPE_F32 = 0
ATTN_DTYPE_BF16 = 1
ATTN_DEV_TIMEOUT = 1
ATTN_DEV_BAD_PAGE = 2
ATTN_DEV_BAD_LENGTH = 4
ATTN_DEV_RANGE = 8
ATTN_DEV_BAD_INDEX = 16

EXPORTED = (
    "attn_prefill_workspace_size", "attn_prefill", "attn_prefill_ex", "attn_prefill_chunk_ex",
    "attn_prefill_chunk_varlen",
    "attn_decode_paged_workspace_size", "attn_decode_paged",
    "attn_decode_paged_fp8_workspace_size", "mla_decode_workspace_size", "mla_decode",
    "dsa_index_topk_workspace_size", "dsa_index_topk", "dsa_mla_decode_workspace_size", "dsa_mla_decode",
    "dsa_mla_decode_fp8",
    "attn_last_error", "attn_read_status", "attn_selftest_wait_timeout", "attn_selftest_exp2",
    "attn_rope_ntk_theta", "attn_rope_length_scaled_theta", "attn_decode_paged_noalloc_status", "attn_lse_merge",
    "attn_profile_enable", "attn_profile_collect",
)


class AttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"attn_b200 error {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB):
        raise ImportError(f"CUDA library not built: {LIB} is missing (run attention_causal_gqa_b200.build)")
    lib = ctypes.CDLL(LIB)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_prefill_workspace_size.restype = sz
    lib.attn_prefill_workspace_size.argtypes = [i32] * 5
    lib.attn_prefill_ex.restype = i32
    lib.attn_prefill_ex.argtypes = [vp] * 5 + [i32] * 6 + [f32, f32, i32, f32, i32, vp, sz, vp]
    lib.attn_prefill.restype = i32
    lib.attn_prefill.argtypes = [vp] * 5 + [i32] * 6 + [f32, f32, i32, vp, sz, vp]
    lib.attn_decode_paged_workspace_size.restype = sz
    lib.attn_decode_paged_workspace_size.argtypes = [i32] * 5
    lib.attn_decode_paged.restype = i32
    lib.attn_decode_paged.argtypes = [vp] * 7 + [i32] * 7 + [f32, i32, vp, sz, vp]
    lib.attn_decode_paged_fp8.restype = i32
    lib.attn_decode_paged_fp8.argtypes = [vp] * 9 + [i32] * 7 + [f32, vp, sz, vp]
    lib.attn_prefill_chunk_workspace_size.restype = sz
    lib.attn_prefill_chunk_workspace_size.argtypes = [i32] * 5
    lib.attn_prefill_chunk.restype = i32
    lib.attn_prefill_chunk.argtypes = [vp] * 9 + [i32] * 9 + [f32, f32, vp, sz, vp]
    lib.attn_prefill_chunk_ex.restype = i32
    lib.attn_prefill_chunk_ex.argtypes = [vp] * 9 + [i32] * 9 + [f32, f32, i32, f32, vp, sz, vp]
    lib.attn_prefill_chunk_varlen.restype = i32
    lib.attn_prefill_chunk_varlen.argtypes = [vp] * 10 + [i32] * 9 + [f32, f32, i32, f32, vp, sz, vp]
    lib.attn_decode_paged_fp8_workspace_size.restype = sz
    lib.attn_decode_paged_fp8_workspace_size.argtypes = [i32] * 5
    lib.mla_decode_workspace_size.restype = sz
    lib.mla_decode_workspace_size.argtypes = [i32] * 5
    lib.mla_decode.restype = i32
    lib.mla_decode.argtypes = [vp] * 5 + [f32, vp, vp] + [i32] * 5 + [vp, sz, vp]
    lib.dsa_index_topk_workspace_size.restype = sz
    lib.dsa_index_topk_workspace_size.argtypes = [i32] * 5
    lib.dsa_index_topk.restype = i32
    lib.dsa_index_topk.argtypes = [vp] * 6 + [i32] * 5 + [vp, sz, vp]
    lib.dsa_mla_decode_workspace_size.restype = sz
    lib.dsa_mla_decode_workspace_size.argtypes = [i32] * 5
    lib.dsa_mla_decode.restype = i32
    lib.dsa_mla_decode.argtypes = [vp] * 6 + [i32, f32, vp, vp] + [i32] * 5 + [vp, sz, vp]
    lib.dsa_mla_decode_fp8.restype = i32
    lib.dsa_mla_decode_fp8.argtypes = [vp] * 7 + [i32, f32, vp, vp] + [i32] * 5 + [vp, sz, vp]
    lib.attn_last_error.restype = ctypes.c_char_p
    lib.attn_last_error.argtypes = []
    lib.attn_read_status.restype = i32
    lib.attn_read_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    lib.attn_lse_merge.restype = i32
    lib.attn_lse_merge.argtypes = [vp, vp, i32, ctypes.c_longlong, i32, vp, vp, vp]
    lib.attn_rope_ntk_theta.restype = ctypes.c_double
    lib.attn_rope_ntk_theta.argtypes = [ctypes.c_double, ctypes.c_double, i32]
    lib.attn_rope_length_scaled_theta.restype = ctypes.c_double
    lib.attn_rope_length_scaled_theta.argtypes = [ctypes.c_double, i32, i32, ctypes.c_double]
    lib.attn_selftest_exp2.restype = i32
    lib.attn_selftest_exp2.argtypes = [vp, vp, i32, vp]
    lib.attn_selftest_wait_timeout.restype = i32
    lib.attn_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_ulonglong, vp]
    lib.attn_profile_enable.restype = i32
    lib.attn_profile_enable.argtypes = [i32]
    lib.attn_profile_collect.restype = i32
    lib.attn_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i32)]
    return lib


lib = _load()


def _check(rc: int):
    if rc != ATTN_OK:
        raise AttnError(rc, lib.attn_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("attn_b200 takes CUDA tensors (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("attn_b200 takes contiguous tensors")


def _flags_or_raise(ws, stream, what: str) -> None:
    """Waits for the stream and raises AttnError when the call's device status word has
    flags (ATTN_DEV_*): an out-of-range operand, a bad page, a bad length or a timeout
    means the outputs are not valid."""
    flags = read_status(ws, stream)
    if flags:
        names = [n for bit, n in ((ATTN_DEV_TIMEOUT, "timeout"), (ATTN_DEV_BAD_PAGE, "bad page"),
                                  (ATTN_DEV_BAD_LENGTH, "bad length"), (ATTN_DEV_RANGE, "fp16 operand range"),
                                  (ATTN_DEV_BAD_INDEX, "bad index")) if flags & bit]
        raise AttnError(ATTN_ERR_DEVICE, f"{what}: device status flags {flags:#x} ({', '.join(names)})")


def _workspace(nbytes: int, device, workspace):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ prefill
def prefill_workspace_size(B, Hkv, S, D, dtype=torch.bfloat16) -> int:
    dt = ATTN_DTYPE_F32 if dtype == torch.float32 else ATTN_DTYPE_BF16
    return int(lib.attn_prefill_workspace_size(B, Hkv, S, D, dt))


ROPE_LAYOUTS = {"interleaved": 0, "half": 1}  # ATTN_ROPE_INTERLEAVED, ATTN_ROPE_HALF_SPLIT
ATTN_ROPE_BF16_OPERANDS = 4


def ntk_aware_theta(theta: float, scale: float, head_dim: int) -> float:
    """NTK-aware RoPE base for a context stretched by `scale` (computed by the library:
    attn_rope_ntk_theta)."""
    r = float(lib.attn_rope_ntk_theta(float(theta), float(scale), int(head_dim)))
    if not r > 0.0:
        raise AttnError(ATTN_ERR_INVALID_ARG, lib.attn_last_error().decode())
    return r


def length_scaled_theta(theta: float, length: int, base_length: int, alpha: float) -> float:
    """Length-aware RoPE base theta * (L / L0)^alpha (computed by the library:
    attn_rope_length_scaled_theta)."""
    r = float(lib.attn_rope_length_scaled_theta(float(theta), int(length), int(base_length), float(alpha)))
    if not r > 0.0:
        raise AttnError(ATTN_ERR_INVALID_ARG, lib.attn_last_error().decode())
    return r


def attn_prefill(q, k, v, causal=True, rope_theta=10000.0, scale=None, out=None, lse=None, workspace=None,
                 stream=None, rope_freq_scale=1.0, rope_layout="interleaved", check=False, bf16_operands=False):
    """Causal GQA prefill with RoPE. q [B,Hq,S,D], k/v [B,Hkv,S,D] (bf16 or fp32).
    rope_freq_scale multiplies every rotary frequency; rope_layout "interleaved" pairs
    (2i, 2i+1), "half" pairs (i, i + D/2). Returns (out [B,Hq,S,D] same dtype, lse [B,Hq,S] fp32).

    With RoPE on bf16 input the rotated q and k are fp16 tensor-core operands; a rotated
    value beyond 65504 sets ATTN_DEV_RANGE and makes the result invalid. check=True waits
    for the call, and when that flag is set re-runs it with bf16 operands
    (ATTN_ROPE_BF16_OPERANDS, valid for any bf16 input at 8x the operand rounding) before
    raising on any flag left; bf16_operands=True asks for that form directly."""
    _need_cuda(q, k, v)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    dt = ATTN_DTYPE_F32 if q.dtype == torch.float32 else ATTN_DTYPE_BF16
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    ws_bytes = prefill_workspace_size(B, Hkv, S, D, q.dtype)
    ws = _workspace(ws_bytes, q.device, workspace)
    if rope_layout not in ROPE_LAYOUTS:
        raise ValueError(f"rope_layout must be one of {sorted(ROPE_LAYOUTS)}")

    def run(bf16_ops):
        if float(rope_freq_scale) == 1.0 and rope_layout == "interleaved" and not bf16_ops:
            rc = lib.attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S, D,
                                  int(bool(causal)), float(rope_theta if rope_theta else 0.0), float(scale or 0.0), dt,
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
        else:
            layout = ROPE_LAYOUTS[rope_layout] | (ATTN_ROPE_BF16_OPERANDS if bf16_ops else 0)
            rc = lib.attn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S, D,
                                     int(bool(causal)), float(rope_theta if rope_theta else 0.0),
                                     float(rope_freq_scale), layout, float(scale or 0.0), dt, _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream))
        _check(rc)

    run(bf16_operands)
    if check:
        rope_bf16 = dt == ATTN_DTYPE_BF16 and bool(rope_theta) and rope_theta > 0
        if rope_bf16 and not bf16_operands and read_status(ws, stream) & ATTN_DEV_RANGE:
            run(True)
        _flags_or_raise(ws, stream, "attn_prefill")
    return out, lse


# ------------------------------------------------------------- paged decode
def decode_workspace_size(B, Hq, D, max_pages_per_seq, page_size=16) -> int:
    return int(lib.attn_decode_paged_workspace_size(B, Hq, D, max_pages_per_seq, page_size))


def decode_fp8_workspace_size(B, Hq, D, max_pages_per_seq, page_size=16) -> int:
    return int(lib.attn_decode_paged_fp8_workspace_size(B, Hq, D, max_pages_per_seq, page_size))


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale=None, out=None, lse=None, workspace=None,
                      stream=None, check=False):
    """Paged GQA decode. q [B,Hq,D] bf16, k/v_pages [P,16,Hkv,D] bf16, block_table [B,maxp] int32,
    seq_lens [B] int32. Returns (out [B,Hq,D] bf16, lse [B,Hq] fp32)."""
    _need_cuda(q, k_pages, v_pages, block_table, seq_lens)
    B, Hq, D = q.shape
    P, ps, Hkv, _ = k_pages.shape
    maxp = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws = _workspace(decode_workspace_size(B, Hq, D, maxp, ps), q.device, workspace)
    rc = lib.attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), _ptr(out),
                               _ptr(lse), B, Hq, Hkv, D, ps, maxp, P, float(scale or 0.0), ATTN_DTYPE_BF16, _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    if check:  # waits; raises on a bad page, a length beyond the table or a timeout
        _flags_or_raise(ws, stream, "attn_decode_paged")
    return out, lse


def attn_decode_paged_fp8(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, scale=None, out=None, lse=None,
                          workspace=None, stream=None, check=False):
    """Paged GQA decode over an FP8 E4M3 cache. q [B,Hq,D] bf16; k/v_pages [P,16,Hkv,D] uint8 codes;
    k/v_scale [P,Hkv] fp32; block_table [B,maxp] int32; seq_lens [B] int32.
    Returns (out [B,Hq,D] bf16, lse [B,Hq] fp32)."""
    _need_cuda(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens)
    B, Hq, D = q.shape
    P, ps, Hkv, _ = k_pages.shape
    maxp = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws = _workspace(decode_fp8_workspace_size(B, Hq, D, maxp, ps), q.device, workspace)
    rc = lib.attn_decode_paged_fp8(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale),
                                   _ptr(block_table), _ptr(seq_lens), _ptr(out), _ptr(lse), B, Hq, Hkv, D, ps, maxp,
                                   P, float(scale or 0.0), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    if check:  # waits; raises when q left the fp16 range (ATTN_DEV_RANGE) or on any other flag
        _flags_or_raise(ws, stream, "attn_decode_paged_fp8")
    return out, lse


# -------------------------------------------- chunked prefill into the paged cache
def prefill_chunk_workspace_size(B, Hkv, S_new, max_cache_len, D) -> int:
    return int(lib.attn_prefill_chunk_workspace_size(B, Hkv, S_new, max_cache_len, D))


def attn_prefill_chunk(q, k, v, k_pages, v_pages, block_table, cache_lens, max_cache_len, rope_theta=10000.0,
                       scale=None, out=None, lse=None, workspace=None, stream=None, rope_freq_scale=1.0,
                       rope_layout="interleaved", check=False, new_lens=None):
    """Append a chunk of new tokens to the paged KV cache and attend over the whole cache.
    q [B,Hq,S_new,D], k/v [B,Hkv,S_new,D] bf16 (not rotated); k/v_pages [P,16,Hkv,D] bf16, updated in
    place; block_table [B,maxp] int32; cache_lens [B] int32 (tokens already cached, each <= max_cache_len).
    new_lens [B] int32 (optional): chunks of different lengths padded to S_new; sequence b takes only its
    first new_lens[b] tokens and its rows past them come back as out = 0, lse = -inf.
    Returns (out [B,Hq,S_new,D] bf16, lse [B,Hq,S_new] fp32)."""
    _need_cuda(q, k, v, k_pages, v_pages, block_table, cache_lens)
    if new_lens is not None:
        _need_cuda(new_lens)
    B, Hq, S_new, D = q.shape
    Hkv = k.shape[1]
    P, ps, _, _ = k_pages.shape
    maxp = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S_new), dtype=torch.float32, device=q.device)
    ws = _workspace(prefill_chunk_workspace_size(B, Hkv, S_new, int(max_cache_len), D), q.device, workspace)
    if rope_layout not in ROPE_LAYOUTS:
        raise ValueError(f"rope_layout must be one of {sorted(ROPE_LAYOUTS)}")
    if new_lens is not None:
        rc = lib.attn_prefill_chunk_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                           _ptr(cache_lens), _ptr(new_lens), _ptr(out), _ptr(lse), B, Hq, Hkv, S_new,
                                           D, ps, maxp, P, int(max_cache_len), float(rope_theta if rope_theta else 0.0),
                                           float(rope_freq_scale), ROPE_LAYOUTS[rope_layout], float(scale or 0.0),
                                           _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    elif float(rope_freq_scale) == 1.0 and rope_layout == "interleaved":
        rc = lib.attn_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                    _ptr(cache_lens), _ptr(out), _ptr(lse), B, Hq, Hkv, S_new, D, ps, maxp, P,
                                    int(max_cache_len), float(rope_theta if rope_theta else 0.0), float(scale or 0.0),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    else:
        rc = lib.attn_prefill_chunk_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                       _ptr(cache_lens), _ptr(out), _ptr(lse), B, Hq, Hkv, S_new, D, ps, maxp, P,
                                       int(max_cache_len), float(rope_theta if rope_theta else 0.0),
                                       float(rope_freq_scale), ROPE_LAYOUTS[rope_layout], float(scale or 0.0),
                                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    if check:  # waits; raises when a rotated query or a cached key left the fp16 range, or on any other flag
        _flags_or_raise(ws, stream, "attn_prefill_chunk")
    return out, lse


# --------------------------------------------------------------- MLA decode
def mla_workspace_size(B, H, Dc, Dr, T_max) -> int:
    return int(lib.mla_decode_workspace_size(B, H, Dc, Dr, T_max))


def mla_decode(q_nope, q_pe, kv_cache, pe_cache, seq_lens, scale, out=None, lse=None, workspace=None,
               stream=None, check=False):
    """MLA absorbed decode. q_nope [B,1,H,Dc], q_pe [B,1,H,Dr], kv_cache [B,T,Dc], pe_cache [B,T,Dr] (bf16),
    seq_lens [B] int32. Returns (out [B,1,H,Dc] bf16, lse [B,1,H] fp32)."""
    _need_cuda(q_nope, q_pe, kv_cache, pe_cache, seq_lens)
    B, _, H, Dc = q_nope.shape
    Dr = q_pe.shape[-1]
    T = kv_cache.shape[1]
    if not scale or scale <= 0:
        raise ValueError("mla_decode needs an explicit positive scale (DeepSeek-V3 shapes: 1/sqrt(192))")
    if out is None:
        out = torch.empty_like(q_nope)
    if lse is None:
        lse = torch.empty((B, 1, H), dtype=torch.float32, device=q_nope.device)
    ws = _workspace(mla_workspace_size(B, H, Dc, Dr, T), q_nope.device, workspace)
    rc = lib.mla_decode(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(seq_lens), float(scale),
                        _ptr(out), _ptr(lse), B, H, Dc, Dr, T, _ptr(ws), ws.numel() * ws.element_size(),
                        _stream(stream))
    _check(rc)
    if check:  # waits; raises on a timeout flag
        _flags_or_raise(ws, stream, "mla_decode")
    return out, lse


def lse_merge(o_parts, lse_parts, out=None, lse=None, stream=None):
    """Combines partial results over disjoint key sets (e.g. gathered from the ranks of a
    sequence-parallel decode). o_parts [n, ..., D] bf16, lse_parts [n, ...] fp32 (same
    leading shape). Returns (out [..., D] bf16, lse [...] fp32)."""
    _need_cuda(o_parts, lse_parts)
    n, D = o_parts.shape[0], o_parts.shape[-1]
    if tuple(lse_parts.shape) != tuple(o_parts.shape[:-1]) or o_parts.dtype != torch.bfloat16:
        raise ValueError("o_parts [n, ..., D] bf16 and lse_parts [n, ...] fp32 with matching shapes")
    rows = lse_parts[0].numel()
    if out is None:
        out = torch.empty(o_parts.shape[1:], dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    _check(lib.attn_lse_merge(_ptr(o_parts), _ptr(lse_parts), n, rows, D, _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


# ------------------------------------------------- DeepSeek sparse attention
def dsa_index_topk(q_idx, w_idx, k_idx, seq_lens, top_k, scores=None, topk_idx=None, workspace=None, stream=None):
    """Lightning-indexer scores and top-k selection. q_idx [B,H_I,d_I] bf16, w_idx [B,H_I] fp32,
    k_idx [B,T,d_I] bf16, seq_lens [B] int32. Returns (scores [B,T] fp32, topk_idx [B,top_k] int32)."""
    _need_cuda(q_idx, w_idx, k_idx, seq_lens)
    B, HI, dI = q_idx.shape
    T = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((B, T), dtype=torch.float32, device=q_idx.device)
    if topk_idx is None:
        topk_idx = torch.empty((B, int(top_k)), dtype=torch.int32, device=q_idx.device)
    ws = _workspace(lib.dsa_index_topk_workspace_size(B, HI, dI, T, int(top_k)), q_idx.device, workspace)
    rc = lib.dsa_index_topk(_ptr(q_idx), _ptr(w_idx), _ptr(k_idx), _ptr(seq_lens), _ptr(scores), _ptr(topk_idx), B, HI,
                            dI, T, int(top_k), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    return scores, topk_idx


def dsa_mla_workspace_size(B, H, Dc, Dr, top_k) -> int:
    return int(lib.dsa_mla_decode_workspace_size(B, H, Dc, Dr, top_k))


def dsa_mla_decode(q_nope, q_pe, kv_cache, pe_cache, seq_lens, topk_idx, scale, out=None, lse=None, workspace=None,
                   stream=None):
    """MLA absorbed decode over the selected tokens topk_idx [B, top_k] int32 (from dsa_index_topk).
    Other tensors as mla_decode. Returns (out [B,1,H,Dc] bf16, lse [B,1,H] fp32)."""
    _need_cuda(q_nope, q_pe, kv_cache, pe_cache, seq_lens, topk_idx)
    B, _, H, Dc = q_nope.shape
    Dr = q_pe.shape[-1]
    T = kv_cache.shape[1]
    top_k = topk_idx.shape[1]
    if not scale or scale <= 0:
        raise ValueError("dsa_mla_decode needs an explicit positive scale")
    if out is None:
        out = torch.empty_like(q_nope)
    if lse is None:
        lse = torch.empty((B, 1, H), dtype=torch.float32, device=q_nope.device)
    ws = _workspace(dsa_mla_workspace_size(B, H, Dc, Dr, top_k), q_nope.device, workspace)
    rc = lib.dsa_mla_decode(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(seq_lens), _ptr(topk_idx),
                            top_k, float(scale), _ptr(out), _ptr(lse), B, H, Dc, Dr, T, _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    return out, lse


def dsa_mla_decode_fp8(q_nope, q_pe, kv_codes, kv_scale, pe_cache, seq_lens, topk_idx, scale, out=None, lse=None,
                       workspace=None, stream=None):
    """dsa_mla_decode over an E4M3 latent cache: kv_codes [B,T,512] uint8, kv_scale [B,T,4] fp32
    (one scale per token and 128-wide block), pe_cache [B,T,64] bf16. Returns (out, lse) as mla_decode."""
    _need_cuda(q_nope, q_pe, kv_codes, kv_scale, pe_cache, seq_lens, topk_idx)
    B, _, H, Dc = q_nope.shape
    Dr = q_pe.shape[-1]
    T = kv_codes.shape[1]
    top_k = topk_idx.shape[1]
    if not scale or scale <= 0:
        raise ValueError("dsa_mla_decode_fp8 needs an explicit positive scale")
    if out is None:
        out = torch.empty_like(q_nope)
    if lse is None:
        lse = torch.empty((B, 1, H), dtype=torch.float32, device=q_nope.device)
    ws = _workspace(dsa_mla_workspace_size(B, H, Dc, Dr, top_k), q_nope.device, workspace)
    rc = lib.dsa_mla_decode_fp8(_ptr(q_nope), _ptr(q_pe), _ptr(kv_codes), _ptr(kv_scale), _ptr(pe_cache),
                                _ptr(seq_lens), _ptr(topk_idx), top_k, float(scale), _ptr(out), _ptr(lse), B, H, Dc,
                                Dr, T, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc)
    return out, lse


# ------------------------------------------------------------------- status
def read_status(workspace, stream=None) -> int:
    flags = ctypes.c_int(0)
    rc = lib.attn_read_status(_ptr(workspace), ctypes.byref(flags), _stream(stream))
    if rc not in (ATTN_OK, ATTN_ERR_DEVICE):
        _check(rc)
    return flags.value


def selftest_exp2(z: torch.Tensor, stream=None) -> torch.Tensor:
    """2^z as the prefill softmax's FMA-pipe exponential computes it (z: CUDA fp32)."""
    assert z.is_cuda and z.dtype == torch.float32 and z.is_contiguous()
    y = torch.empty_like(z)
    _check(lib.attn_selftest_exp2(_ptr(z), _ptr(y), z.numel(), _stream(stream)))
    return y


def selftest_wait_timeout(timeout_ns: int, workspace=None, stream=None) -> int:
    ws = workspace if workspace is not None else torch.zeros(256, dtype=torch.uint8, device="cuda")
    _check(lib.attn_selftest_wait_timeout(_ptr(ws), ws.numel(), int(timeout_ns), _stream(stream)))
    return read_status(ws, stream)


# ------------------------------------------------------------ timing hook
def profile_enable(on: bool = True):
    _check(lib.attn_profile_enable(1 if on else 0))


def profile_collect():
    """(summed main-kernel milliseconds, number of recorded calls) since the last collect."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int(0)
    _check(lib.attn_profile_collect(ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value
