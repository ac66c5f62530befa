"""Plans that wire the four ABI calls together with torch-owned buffers.

``PrefillPlan``: quantize_qkv_tiles -> build_tile_lists -> routed_attention_prefill.
``DecodePlan``:  build_tile_lists (decode-cache kind, once) -> routed_attention_decode
per step, over the K/V tiles a PrefillPlan (or quantize_qkv_tiles) produced.
``HybridDecodePlan``: hybrid_select_tokens (once, over the prefix) ->
hybrid_attention_decode per step (token-level hybrid: INT4 tiles plus bf16 selected
and recent tokens).
``HybridPrefillPlan``: quantize_qkv_tiles (K and V INT4 scales) ->
hybrid_select_tokens -> hybrid_attention_prefill.
Buffers are allocated once per plan; ``run``/``step`` only enqueue kernels.  The
decode workspace is zero-filled once (the decode's arrival counters need that, and
every step leaves them at zero).
"""
from __future__ import annotations

import math

import torch

from . import _lib as L


class PrefillPlan:
    def __init__(self, shape: L.Shape, policy: L.Policy, keep_v_cache: bool = False,
                 device="cuda"):
        self.shape, self.policy = shape, policy
        fm = L.FMT_Q8 | L.FMT_K8
        if policy.has_int4:
            fm |= L.FMT_Q4X | L.FMT_K4X     # INT4 codes in the tensor-core operand form
        if policy.has_fp8:
            fm |= L.FMT_Q8F | L.FMT_K8F     # FP8 E4M3 codes of the FP8 band
        if keep_v_cache:
            fm |= L.FMT_K4 | L.FMT_V8 | L.FMT_V4
        self.tiles = L.QTiles(shape, fm, device)
        rows, nnz = L.tile_lists_size(shape, policy, L.LISTS_PREFILL)
        self.rows, self.nnz = rows, nnz
        self.row_ptr = torch.zeros(rows + 1, dtype=torch.int32, device=device)
        self.entries = torch.zeros(max(nnz, 4), dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def quantize(self, q, k, v, stream=None):
        L.quantize_qkv_tiles(self.shape, q, k, v, self.tiles, stream)

    def lists(self, stream=None):
        L.build_tile_lists(self.shape, self.policy, L.LISTS_PREFILL, self.row_ptr, self.entries, stream)

    def attend(self, q, k, v, out, lse=None, scale=None, dump_coords=None, dump_out=None,
               stream=None):
        scale = 1.0 / math.sqrt(self.shape.d) if scale is None else scale
        L.routed_attention_prefill(self.shape, self.policy, q, k, v, self.tiles, self.row_ptr,
                                   self.entries, scale, out, lse, dump_coords, dump_out,
                                   self.status, stream)

    def run(self, q, k, v, out, lse=None, scale=None, stream=None):
        """One full prefill pass: quantise, build traversals, fused attention."""
        self.quantize(q, k, v, stream)
        self.lists(stream)
        self.attend(q, k, v, out, lse, scale, stream=stream)


class DecodePlan:
    def __init__(self, shape: L.Shape, policy: L.Policy, cache: L.QTiles, tail_cap: int,
                 device="cuda"):
        self.shape, self.policy, self.cache = shape, policy, cache
        rows, nnz = L.tile_lists_size(shape, policy, L.LISTS_DECODE_CACHE)
        self.row_ptr = torch.zeros(rows + 1, dtype=torch.int32, device=device)
        self.entries = torch.zeros(max(nnz, 4), dtype=torch.int32, device=device)
        self.nnz = nnz
        B, Hkv, d = shape.B, shape.Hkv, shape.d
        self.k_tail = torch.zeros((B, Hkv, tail_cap, d), dtype=torch.bfloat16, device=device)
        self.v_tail = torch.zeros_like(self.k_tail)
        self.tail_len = torch.zeros(B, dtype=torch.int32, device=device)
        nbytes = L.decode_workspace_bytes(B, shape.Hq, Hkv, d)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def build(self, stream=None):
        L.build_tile_lists(self.shape, self.policy, L.LISTS_DECODE_CACHE, self.row_ptr,
                           self.entries, stream)

    def step(self, q, k_new, v_new, out, scale=None, stream=None):
        scale = 1.0 / math.sqrt(self.shape.d) if scale is None else scale
        L.routed_attention_decode(self.shape, self.policy, q, k_new, v_new, self.cache,
                                  self.row_ptr, self.entries, self.k_tail, self.v_tail,
                                  self.tail_len, scale, out, self.workspace, self.status, stream)


class HybridDecodePlan:
    def __init__(self, shape: L.Shape, cache: L.QTiles, frac: float, window: int, tail_cap: int,
                 device="cuda"):
        self.shape, self.cache = shape, cache
        self.hy = L.Hybrid(shape, frac, window, device)
        B, Hkv, d = shape.B, shape.Hkv, shape.d
        self.k_tail = torch.zeros((B, Hkv, tail_cap, d), dtype=torch.bfloat16, device=device)
        self.v_tail = torch.zeros_like(self.k_tail)
        self.tail_len = torch.zeros(B, dtype=torch.int32, device=device)
        nbytes = L.decode_workspace_bytes(B, shape.Hq, Hkv, d)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def select(self, importance, k, v, stream=None):
        L.hybrid_select_tokens(self.shape, importance, self.hy.frac, k, v, self.hy, stream)

    def step(self, q, k_new, v_new, out, scale=None, stream=None):
        scale = 1.0 / math.sqrt(self.shape.d) if scale is None else scale
        L.hybrid_attention_decode(self.shape, self.hy, q, k_new, v_new, self.cache, self.k_tail,
                                  self.v_tail, self.tail_len, scale, out, self.workspace,
                                  self.status, stream)


class HybridPrefillPlan:
    """Causal prefill of the token-level hybrid: keys outside the query's window are read
    from their INT4 tile unless selected; the selection also serves a HybridDecodePlan."""

    def __init__(self, shape: L.Shape, frac: float, window: int, device="cuda"):
        self.shape = shape
        self.tiles = L.QTiles(shape, L.FMT_K4 | L.FMT_V4, device)
        self.hy = L.Hybrid(shape, frac, window, device)
        ntok = int(shape.cu_host[-1])
        self.k_mix = torch.zeros((max(ntok, 1), shape.Hkv, shape.d), dtype=torch.bfloat16,
                                 device=device)
        self.v_mix = torch.zeros_like(self.k_mix)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def prepare(self, k, v, importance, stream=None):
        """Quantise K and V (INT4 scales) and select the bf16 tokens."""
        L.quantize_qkv_tiles(self.shape, None, k, v, self.tiles, stream)
        L.hybrid_select_tokens(self.shape, importance, self.hy.frac, k, v, self.hy, stream)

    def attend(self, q, k, v, out, lse=None, scale=None, stream=None):
        scale = 1.0 / math.sqrt(self.shape.d) if scale is None else scale
        L.hybrid_attention_prefill(self.shape, self.hy, q, k, v, self.tiles, self.k_mix,
                                   self.v_mix, scale, out, lse, self.status, stream)

    def run(self, q, k, v, importance, out, lse=None, scale=None, stream=None):
        self.prepare(k, v, importance, stream)
        self.attend(q, k, v, out, lse, scale, stream)
