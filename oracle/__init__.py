"""CPU float64 oracle: test infrastructure, not part of the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm
of ``bench.py`` may import this package. The CUDA library neither imports nor
links it, and it shares no code with the CUDA path.
"""
from .attention import (  # noqa: F401
    apply_rope,
    chunk_prefill_ref,
    decode_paged_fp8_ref,
    decode_paged_ref,
    dsa_index_scores_ref,
    dsa_mla_decode_fp8_ref,
    dsa_mla_decode_ref,
    dsa_topk_ref,
    e4m3_to_float,
    gather_pages,
    length_scaled_theta_ref,
    lse_merge,
    mla_decode_ref,
    mla_naive_ref,
    ntk_aware_theta_ref,
    online_softmax_merge,
    prefill_ref,
    rope_cache,
    to_bf16,
    two_pass_softmax_rows,
)
