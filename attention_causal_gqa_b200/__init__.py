"""attention_causal_gqa_b200: exact causal GQA prefill, paged GQA decode and MLA
absorbed decode as hand-written sm_100a CUDA behind a C ABI (libattn_b200.so).

The public calls (attn_prefill, attn_prefill_chunk, attn_decode_paged, mla_decode, ...) live in
``binding`` and are loaded lazily, so ``synthetic`` can be imported without the
library; calling any of them without the built library raises.
"""
__all__ = ["attn_prefill", "attn_prefill_chunk", "attn_decode_paged", "attn_decode_paged_fp8", "mla_decode", "dsa_index_topk",
           "dsa_mla_decode", "dsa_mla_decode_fp8", "read_status", "selftest_wait_timeout"]


def __getattr__(name):
    if name in __all__ or name in ("prefill_workspace_size", "prefill_chunk_workspace_size", "decode_workspace_size",
                                   "decode_fp8_workspace_size",
                                   "mla_workspace_size", "dsa_mla_workspace_size", "AttnError", "lib"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
