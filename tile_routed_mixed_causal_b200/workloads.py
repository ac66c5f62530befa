"""Seeded synthetic workloads (inputs only).

This module draws random inputs and routing policies and nothing else: it holds
none of the attention, quantisation or routing arithmetic, so both the CUDA
path and the CPU oracle can be fed from it without sharing any of the method.

Recipe (all configurations):
  * lengths (varlen only) are drawn first with ``numpy.random.default_rng(seed)``;
  * Q, K, V are fp32 N(0, 1) from ``torch.Generator(device).manual_seed(seed)``
    in the order Q, K, V, then rounded to bf16 (round-to-nearest-even);
  * "outlier" configurations pick, per head of Q and of K, 4 distinct channels
    (``torch.randperm`` on the same generator, Q heads first, then K heads) and
    scale them by 10 before rounding; V stays N(0, 1);
  * the routing policy is drawn with ``numpy.random.default_rng(seed + 1000)``;
  * decode steps draw q [B, Hq, d] and the new k, v [B, Hkv, d] per step from a
    generator seeded ``seed + 2000``.

The five named workloads follow the sizes of the pages' long-context setting
(32/8-head GQA with head_dim 128, 8K and 32K contexts, a batch of 16 decoding
over a 32K prefix) with synthetic values in place of model activations.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

TILE = 64


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    lengths: list
    seed: int
    outliers: bool
    mode: str                      # "boundary", "bitmask" or "mixed" (both)
    b1: Optional[np.ndarray] = None
    b2: Optional[np.ndarray] = None
    bitmask: Optional[np.ndarray] = None   # uint32 [Hq, ntiles, W]
    G: int = 1
    decode_steps: int = 0
    tail_cap: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    @property
    def ntok(self) -> int:
        return int(sum(self.lengths))

    @property
    def tiles_per_seq(self) -> list:
        return [(int(t) + TILE - 1) // TILE for t in self.lengths]

    @property
    def ntiles(self) -> int:
        return int(sum(self.tiles_per_seq))


def _tensors(w: Workload, device, need_q: bool = True):
    gen = torch.Generator(device=device).manual_seed(w.seed)
    out = {}
    shapes = {"q": (w.ntok, w.Hq, w.d), "k": (w.ntok, w.Hkv, w.d), "v": (w.ntok, w.Hkv, w.d)}
    for name in ("q", "k", "v"):
        if name == "q" and not need_q:
            # keep the generator stream identical whether or not Q is materialised
            n = w.ntok * w.Hq * w.d
            chunk = 1 << 26
            while n > 0:
                torch.randn(min(n, chunk), generator=gen, device=device)
                n -= chunk
            out[name] = None
            continue
        out[name] = torch.randn(shapes[name], generator=gen, device=device, dtype=torch.float32)
    if w.outliers:
        for name, H in (("q", w.Hq), ("k", w.Hkv)):
            for h in range(H):
                ch = torch.randperm(w.d, generator=gen, device=device)[:4]
                if out[name] is not None:
                    out[name][:, h, ch] *= 10.0
    return {k: (None if t is None else t.to(torch.bfloat16).contiguous()) for k, t in out.items()}


def make_inputs(w: Workload, device="cpu", need_q: bool = True):
    """Q, K, V bf16 tensors [ntok, H, d] on ``device`` (Q may be skipped)."""
    return _tensors(w, device, need_q)


def make_decode_inputs(w: Workload, device="cpu"):
    """Per-step decode inputs: q [S, B, Hq, d], k_new / v_new [S, B, Hkv, d] (bf16)."""
    gen = torch.Generator(device=device).manual_seed(w.seed + 2000)
    S = w.decode_steps
    q = torch.randn((S, w.B, w.Hq, w.d), generator=gen, device=device).to(torch.bfloat16)
    kn = torch.randn((S, w.B, w.Hkv, w.d), generator=gen, device=device).to(torch.bfloat16)
    vn = torch.randn((S, w.B, w.Hkv, w.d), generator=gen, device=device).to(torch.bfloat16)
    return q, kn, vn


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _bitmask_words(nt_max: int, G: int) -> int:
    groups = (nt_max + G - 1) // G
    return max(1, (groups + 31) // 32)


def _draw_bitmask(rng, Hq: int, ntiles: int, W: int, p_bf16: float) -> np.ndarray:
    bits = rng.random((Hq, ntiles, W * 32)) < p_bf16
    words = np.zeros((Hq, ntiles, W), np.uint32)
    for j in range(32):
        words |= (bits[:, :, j::32].astype(np.uint32) << np.uint32(j))
    return words


def tiny(seed: int = 0) -> Workload:
    """Batch 1, 2 heads (no GQA), 256 tokens, head_dim 64, (b1, b2) = (1, 3)."""
    w = Workload("tiny_causal_b1_h2_t256_d64", 1, 2, 2, 64, [256], seed, False, "boundary")
    w.b1 = np.array([1, 1], np.int32)
    w.b2 = np.array([3, 3], np.int32)
    return w


def llama8b_8k(seed: int = 1) -> Workload:
    """Llama-3-8B-shaped prefill: 32/8 heads, d 128, 8192 tokens, per-head boundaries."""
    w = Workload("llama3_8b_prefill_t8192_boundary", 1, 32, 8, 128, [8192], seed, True, "boundary")
    rng = np.random.default_rng(seed + 1000)
    w.b1 = rng.integers(1, 9, size=w.Hq).astype(np.int32)
    w.b2 = np.array([rng.integers(b, 65) for b in w.b1], np.int32)
    return w


def mixed_8k(seed: int = 5) -> Workload:
    """Both policies at once on the Llama-3-8B shape (32/8 heads, d 128, 8192 tokens):
    per-head boundaries as in llama8b_8k, then a G = 4 bitmask with 25% of bits set
    promoting kept tiles to BF16."""
    w = Workload("mixed_prefill_t8192_g4", 1, 32, 8, 128, [8192], seed, True, "mixed", G=4)
    rng = np.random.default_rng(seed + 1000)
    w.b1 = rng.integers(1, 9, size=w.Hq).astype(np.int32)
    w.b2 = np.array([rng.integers(b, 65) for b in w.b1], np.int32)
    W = _bitmask_words(w.ntiles, w.G)
    w.bitmask = _draw_bitmask(rng, w.Hq, w.ntiles, W, 0.25)
    return w


def bitmask_32k(seed: int = 2, T: int = 32768) -> Workload:
    """Bitmask mode: 32/8 heads, d 128, 32K tokens, G = 4, 25% of bits BF16."""
    w = Workload(f"bitmask_prefill_t{T}_g4", 1, 32, 8, 128, [T], seed, True, "bitmask", G=4)
    rng = np.random.default_rng(seed + 1000)
    W = _bitmask_words(w.ntiles, w.G)
    w.bitmask = _draw_bitmask(rng, w.Hq, w.ntiles, W, 0.25)
    return w


def varlen_8(seed: int = 3) -> Workload:
    """8 sequences, lengths U[1024, 16384], 28/4 heads, about half the causal tiles skipped."""
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(1024, 16385, size=8)]
    w = Workload("varlen_b8_h28_4_skip50", 8, 28, 4, 128, lengths, seed, True, "boundary")
    prng = np.random.default_rng(seed + 1000)
    nts = w.tiles_per_seq
    causal = sum(n * (n + 1) // 2 for n in nts)

    def kept(c):  # tiles within diagonal distance < c, summed over the batch
        return sum(sum(min(qt + 1, c) for qt in range(n)) for n in nts)

    lo, hi = 1, max(nts)
    while lo < hi:                   # smallest c whose kept share reaches one half
        mid = (lo + hi) // 2
        if kept(mid) * 2 >= causal:
            hi = mid
        else:
            lo = mid + 1
    c = lo
    w.b2 = np.array([prng.integers(max(2, c - 16), c + 17) for _ in range(w.Hq)], np.int32)
    w.b1 = np.array([prng.integers(1, b // 2 + 1) for b in w.b2], np.int32)
    w.notes["centre"] = c
    w.notes["kept_fraction"] = float(sum(kept(int(b)) for b in w.b2) / (w.Hq * causal))
    return w


def decode_32k(seed: int = 4, B: int = 16, T: int = 32768, steps: int = 64,
               literal: bool = False) -> Workload:
    """Decode over a compressed KV cache: batch 16, 32K prefix, 32/8 heads, 64 steps.

    ``literal`` uses (b1, b2) = (1, 3) for every head (a cache small enough to sit in
    L2); the default draws b1 ~ U{64..192}, b2 ~ U{b1+128..480} per head so the
    cache is HBM-sized.
    """
    name = f"decode_b{B}_t{T}_h32_8_steps{steps}" + ("_literal" if literal else "")
    w = Workload(name, B, 32, 8, 128, [T] * B, seed, True, "boundary",
                 decode_steps=steps, tail_cap=steps)
    rng = np.random.default_rng(seed + 1000)
    if literal:
        w.b1 = np.full(w.Hq, 1, np.int32)
        w.b2 = np.full(w.Hq, 3, np.int32)
    else:
        w.b1 = rng.integers(64, 193, size=w.Hq).astype(np.int32)
        w.b2 = np.array([rng.integers(b + 128, 481) for b in w.b1], np.int32)
    return w


def custom(name, lengths, Hq, Hkv, d, seed, mode, *, b1=None, b2=None, G=1,
           p_bf16=0.25, outliers=True, decode_steps=0, tail_cap=0) -> Workload:
    """Small ad-hoc workload for tests (ragged lengths, GQA, any policy; a mixed one
    draws its boundaries first, then its bitmask)."""
    w = Workload(name, len(lengths), Hq, Hkv, d, list(lengths), seed, outliers, mode,
                 decode_steps=decode_steps, tail_cap=tail_cap, G=G)
    rng = np.random.default_rng(seed + 1000)
    if mode in ("boundary", "mixed"):
        if b1 is None:
            w.b1 = rng.integers(1, 4, size=Hq).astype(np.int32)
            w.b2 = np.array([rng.integers(b, b + 5) for b in w.b1], np.int32)
        else:
            w.b1 = np.asarray(b1, np.int32)
            w.b2 = np.asarray(b2, np.int32)
    if mode in ("bitmask", "mixed"):
        W = _bitmask_words(max(w.tiles_per_seq), G)
        w.bitmask = _draw_bitmask(rng, Hq, w.ntiles, W, p_bf16)
    return w


def synthetic_boundary_errors(Hq: int, cands, nt: int, seed: int) -> np.ndarray:
    """Seeded synthetic calibration errors [Hq][len(cands)] for boundary pairs (b1, b2):
    a skip term that falls as b2 keeps more distant tiles and an INT4 term that grows with
    the INT4 band (b2 - b1) and falls as b1 keeps more tiles in INT8, each with per-head
    sensitivities.  Stands in for the normalised projected-output errors that an offline
    calibration of a real model would measure."""
    rng = np.random.default_rng(seed)
    a = np.exp(rng.uniform(np.log(0.05), np.log(2.0), Hq))      # skip sensitivity
    tau = rng.uniform(0.05, 0.5, Hq) * nt                        # reach of useful context
    c = np.exp(rng.uniform(np.log(0.01), np.log(0.5), Hq))      # INT4 sensitivity
    sig = rng.uniform(1.0, 16.0, Hq)
    err = np.zeros((Hq, len(cands)))
    for j, (b1, b2) in enumerate(cands):
        err[:, j] = (a * np.exp(-b2 / tau)
                     + c * (b2 - b1) / b2 * np.exp(-b1 / sig))
    return err


def hybrid_importance(w: "Workload", seed: int) -> np.ndarray:
    """Seeded synthetic importance [ntok, Hkv] of key positions for the token-level hybrid
    (heavy-tailed, so that a few positions stand out as vertical lines would)."""
    rng = np.random.default_rng(seed + 3000)
    return rng.pareto(1.5, size=(w.ntok, w.Hkv))


CONFIGS = {
    "tiny": tiny,
    "llama8b_8k": llama8b_8k,
    "bitmask_32k": bitmask_32k,
    "varlen": varlen_8,
    "decode_32k": decode_32k,
}
