"""Tile-routed mixed-precision causal attention for NVIDIA B200 (sm_100a).

Every query-key score tile of a causal prefill is routed to skip, INT4, INT8 or
BF16 score computation -- by two per-head diagonal-distance boundaries
(TriAttention) or by a packed bitmask with one bit per group of key tiles
(TileMix) -- and all paths update one online-softmax state.  The quantised K/V
are then reused as a compressed KV cache by a bandwidth-bound decode kernel.

The compute lives in the CUDA library ``libtra.so`` (C ABI: ``include/tra.h``);
``_lib`` marshals torch tensors into it and ``api`` wires the calls together.
"""
from ._lib import (  # noqa: F401
    TraError, Shape, Policy, QTiles, load, quantize_qkv_tiles, tile_lists_size,
    build_tile_lists, routed_attention_prefill, routed_attention_decode,
    decode_workspace_bytes, PREC_INT4, PREC_INT8, PREC_BF16, PREC_FP8, POLICY_BOUNDARY, POLICY_BITMASK,
    POLICY_MIXED, FMT_Q8F, FMT_K8F,
    LISTS_PREFILL, LISTS_DECODE_CACHE, FMT_Q8, FMT_Q4, FMT_K8, FMT_K4, FMT_V8, FMT_V4, FMT_Q4X, FMT_K4X,
    DEV_TIMEOUT, DEV_TAIL_FULL, DEV_BAD_LIST, tra_selftest_bounded_wait, boundary_tile_counts,
    allocate_boundaries, prefill_cost_model, fit_prefill_cost_model, Hybrid, hybrid_select_tokens, hybrid_attention_decode,
    hybrid_attention_prefill,
)
