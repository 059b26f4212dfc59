"""B200-native Qwen2-style grouped-query causal attention (GQA) with RoPE.

The computation lives in libgqa.so (hand-written sm_100a CUDA behind the C ABI of
include/gqa.h); this package is its thin Python binding.
"""
from ._lib import (  # noqa: F401
    GQAError, DEVERR_PAGE, DEVERR_SEQLEN, DEVERR_TIMEOUT, LIB_PATH, decode, decode_paged, last_error, load, prefill,
    out_proj, prefill_rotated, prefill_schedule, qkv_append, qkv_rope, release, set_decode_cache_rotated, set_decode_self_in_cache,
    set_rope_scaling, set_timing_events, strerror,
)
