"""CPU oracle for tile-routed mixed-precision causal attention.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its Python binding) never imports this package, and this package
never imports the product.  The arithmetic of the hot path lives in
``tra_oracle.c`` (plain C, fp64, IEEE fp32 for the quantiser), which this module
compiles with gcc and calls with numpy arrays; the boundary allocator's
enumeration and the token-level hybrid (HyQuant) are plain numpy / Python below,
fp64.

Sources (page titles): "TriAttention: Unified Sparse Mixed-Precision Attention
for Long-Context LLM Inference" (abstract), "TileMix: Tile-Centric
Mixed-Precision Attention for LLM Inference Acceleration" (abstract),
"HyQuant Uses Hybrid Precision to Compress LLM Attention" ("How HyQuant works").
Each C function cites the sentence it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tra_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

TILE = 64
INT4, INT8, BF16, FP8 = 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile tra_oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
            "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_int64
            D = ctypes.c_double
            lib.orc_set_threads.argtypes = [I]
            lib.orc_set_threads.restype = I
            lib.orc_num_tiles.argtypes = [P, I]
            lib.orc_num_tiles.restype = L
            lib.orc_quantize.argtypes = [P, P, I, I, I, P, P, P, P]
            lib.orc_quantize.restype = I
            lib.orc_e4m3_value.argtypes = [I]
            lib.orc_e4m3_value.restype = D
            lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
            lib.orc_e4m3_encode.restype = I
            lib.orc_quantize_f8.argtypes = [P, P, I, I, I, P, P]
            lib.orc_quantize_f8.restype = I
            lib.orc_lists_boundary.argtypes = [P, I, I, P, P, P, P, P]
            lib.orc_lists_boundary.restype = L
            lib.orc_lists_bitmask.argtypes = [P, I, I, P, I, I, P, P]
            lib.orc_lists_bitmask.restype = L
            lib.orc_lists_mixed.argtypes = [P, I, I, P, P, P, I, I, P, P]
            lib.orc_lists_mixed.restype = L
            lib.orc_lists_decode.argtypes = [P, I, I, I, I, P, P, P, P, P]
            lib.orc_lists_decode.restype = L
            lib.orc_int_tile.argtypes = [I, I, P, P, P, P, P]
            lib.orc_int_tile.restype = I
            lib.orc_prefill_rows.argtypes = [P, P, P, P, I, I, I, I,
                                             P, P, P, P, P, P, P, P,
                                             P, P, P, P,
                                             P, P, D, I, P, P, P]
            lib.orc_prefill_rows.restype = I
            lib.orc_decode_step.argtypes = [P, P, I, I, I, I,
                                            P, P, P, P, P, P, P, P,
                                            P, P, P, P, P, I, D, P]
            lib.orc_decode_step.restype = I
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> int:
    """Threads prefill_rows spreads its independent rows over (n < 1: every core);
    returns the count set.  Results do not depend on it."""
    return int(_load().orc_set_threads(int(n)))


def num_tiles(cu_seqlens) -> int:
    cu = _c(cu_seqlens, np.int32)
    return int(_load().orc_num_tiles(_p(cu), len(cu) - 1))


def quantize(x_bits, cu_seqlens, want8=True, want4=True):
    """Per-(head, 64-token tile) symmetric quantisation of one tensor.

    x_bits: uint16 bf16 bit patterns [ntok, H, d].  Returns (x8, x4, s8, s4)
    with x8 int8 [H, ntiles, 64, d], x4 uint8 [H, ntiles, 64, d/2] (two INT4
    codes per byte, even channel in the low nibble), s8/s4 float32 [H, ntiles].
    """
    x = _c(x_bits, np.uint16)
    cu = _c(cu_seqlens, np.int32)
    ntok, H, d = x.shape
    nt = num_tiles(cu)
    x8 = np.zeros((H, nt, TILE, d), np.int8) if want8 else None
    x4 = np.zeros((H, nt, TILE, d // 2), np.uint8) if want4 else None
    s8 = np.zeros((H, nt), np.float32) if want8 else None
    s4 = np.zeros((H, nt), np.float32) if want4 else None
    rc = _load().orc_quantize(_p(x), _p(cu), len(cu) - 1, H, d, _p(x8), _p(x4), _p(s8), _p(s4))
    if rc != 0:
        raise ValueError("oracle quantize failed")
    return x8, x4, s8, s4


def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 code (the format's definition)."""
    return float(_load().orc_e4m3_value(int(code)))


def e4m3_encode(r) -> int:
    """E4M3 code of the fp32 value r: round to nearest, ties to even, saturating at 448."""
    return int(_load().orc_e4m3_encode(float(np.float32(r))))


def quantize_f8(x_bits, cu_seqlens):
    """Per-(head, 64-token tile) FP8 E4M3 quantisation: (codes uint8 [H, ntiles, 64, d],
    scales float32 [H, ntiles]) with sf = fl32(amax / 448), code = E4M3(fl32(x / sf))."""
    x = _c(x_bits, np.uint16)
    cu = _c(cu_seqlens, np.int32)
    ntok, H, d = x.shape
    nt = num_tiles(cu)
    xf = np.zeros((H, nt, TILE, d), np.uint8)
    sf = np.zeros((H, nt), np.float32)
    if _load().orc_quantize_f8(_p(x), _p(cu), len(cu) - 1, H, d, _p(xf), _p(sf)) != 0:
        raise ValueError("oracle FP8 quantize failed")
    return xf, sf


def lists_boundary(cu_seqlens, b1, b2, b8=None):
    """Precision-grouped traversal rows (h, q-tile) from two diagonal boundaries, with an
    optional FP8 band [b1, b8) between the INT8 and INT4 regions."""
    cu = _c(cu_seqlens, np.int32)
    b1 = _c(b1, np.int32)
    b2 = _c(b2, np.int32)
    b8 = None if b8 is None else _c(b8, np.int32)
    lib = _load()
    B, Hq = len(cu) - 1, len(b1)
    nnz = lib.orc_lists_boundary(_p(cu), B, Hq, _p(b1), _p(b8), _p(b2), None, None)
    if nnz < 0:
        raise ValueError("invalid boundaries")
    row_ptr = np.zeros(Hq * num_tiles(cu) + 1, np.int32)
    entries = np.zeros(max(nnz, 1), np.uint32)
    lib.orc_lists_boundary(_p(cu), B, Hq, _p(b1), _p(b8), _p(b2), _p(row_ptr), _p(entries))
    return row_ptr, entries[:nnz]


def lists_bitmask(cu_seqlens, bitmask, G):
    """Traversal rows from a packed bitmask [Hq, ntiles, W] (1 -> BF16, 0 -> INT8)."""
    cu = _c(cu_seqlens, np.int32)
    bm = _c(bitmask, np.uint32)
    Hq, _, W = bm.shape
    lib = _load()
    B = len(cu) - 1
    nnz = lib.orc_lists_bitmask(_p(cu), B, Hq, _p(bm), G, W, None, None)
    if nnz < 0:
        raise ValueError("invalid bitmask policy")
    row_ptr = np.zeros(Hq * num_tiles(cu) + 1, np.int32)
    entries = np.zeros(max(nnz, 1), np.uint32)
    lib.orc_lists_bitmask(_p(cu), B, Hq, _p(bm), G, W, _p(row_ptr), _p(entries))
    return row_ptr, entries[:nnz]


def lists_mixed(cu_seqlens, b1, b2, bitmask, G):
    """Four-way rows: boundaries give skip / INT4 / INT8, a set bitmask bit of a
    kept tile's group promotes it to BF16 (a reading combining both pages)."""
    cu = _c(cu_seqlens, np.int32)
    b1 = _c(b1, np.int32)
    b2 = _c(b2, np.int32)
    bm = _c(bitmask, np.uint32)
    Hq, _, W = bm.shape
    lib = _load()
    B = len(cu) - 1
    nnz = lib.orc_lists_mixed(_p(cu), B, Hq, _p(b1), _p(b2), _p(bm), G, W, None, None)
    if nnz < 0:
        raise ValueError("invalid mixed policy")
    row_ptr = np.zeros(Hq * num_tiles(cu) + 1, np.int32)
    entries = np.zeros(max(nnz, 1), np.uint32)
    lib.orc_lists_mixed(_p(cu), B, Hq, _p(b1), _p(b2), _p(bm), G, W, _p(row_ptr), _p(entries))
    return row_ptr, entries[:nnz]


def lists_decode(cu_seqlens, Hq, Hkv, b1=None, b2=None, b8=None):
    """Decode-cache rows (b, kv-head); boundary mode if b1/b2 given (an FP8-band tile is
    cached as INT8), else all INT8."""
    cu = _c(cu_seqlens, np.int32)
    mode = 1 if b1 is None else 0
    b1a = _c(b1 if b1 is not None else np.zeros(Hq), np.int32)
    b2a = _c(b2 if b2 is not None else np.zeros(Hq), np.int32)
    b8a = None if b8 is None else _c(b8, np.int32)
    lib = _load()
    B = len(cu) - 1
    nnz = lib.orc_lists_decode(_p(cu), B, Hq, Hkv, mode, _p(b1a), _p(b8a), _p(b2a), None, None)
    if nnz < 0:
        raise ValueError("invalid decode policy")
    row_ptr = np.zeros(B * Hkv + 1, np.int32)
    entries = np.zeros(max(nnz, 1), np.uint32)
    lib.orc_lists_decode(_p(cu), B, Hq, Hkv, mode, _p(b1a), _p(b8a), _p(b2a), _p(row_ptr),
                         _p(entries))
    return row_ptr, entries[:nnz]


def int_tile(prec, q8t=None, q4t=None, k8t=None, k4t=None, d=None):
    """Raw int32 Q-code * K-code^T of one 64x64 tile (no masking)."""
    out = np.zeros((TILE, TILE), np.int32)
    if prec == INT8:
        q8t = _c(q8t, np.int8); k8t = _c(k8t, np.int8); d = q8t.shape[-1]
    else:
        q4t = _c(q4t, np.uint8); k4t = _c(k4t, np.uint8); d = 2 * q4t.shape[-1]
    rc = _load().orc_int_tile(prec, d, _p(q8t), _p(q4t), _p(k8t), _p(k4t), _p(out))
    if rc != 0:
        raise ValueError("bad precision")
    return out


class Quantised:
    """Oracle-side quantised tensors of one prefill (its own, never the GPU's)."""

    def __init__(self, q_bits, k_bits, v_bits, cu_seqlens, want_f8=False):
        none = (None, None, None, None)
        self.q8, self.q4, self.sq8, self.sq4 = (
            quantize(q_bits, cu_seqlens) if q_bits is not None else none)
        self.k8, self.k4, self.sk8, self.sk4 = (
            quantize(k_bits, cu_seqlens) if k_bits is not None else none)
        self.v8, self.v4, self.sv8, self.sv4 = (
            quantize(v_bits, cu_seqlens) if v_bits is not None else none)
        self.qf = self.sqf = self.kf = self.skf = None
        if want_f8 and q_bits is not None:
            self.qf, self.sqf = quantize_f8(q_bits, cu_seqlens)
        if want_f8 and k_bits is not None:
            self.kf, self.skf = quantize_f8(k_bits, cu_seqlens)


def prefill_rows(q_bits, k_bits, v_bits, cu_seqlens, qz: Quantised, row_ptr, entries,
                 rows, scale=None):
    """fp64 output [len(rows), 64, d] and lse [len(rows), 64] for traversal rows."""
    q = _c(q_bits, np.uint16); k = _c(k_bits, np.uint16); v = _c(v_bits, np.uint16)
    cu = _c(cu_seqlens, np.int32)
    _, Hq, d = q.shape
    Hkv = k.shape[1]
    rows = _c(rows, np.int64)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((len(rows), TILE, d), np.float64)
    lse = np.zeros((len(rows), TILE), np.float64)
    rp = _c(row_ptr, np.int32); en = _c(entries, np.uint32)
    rc = _load().orc_prefill_rows(
        _p(q), _p(k), _p(v), _p(cu), len(cu) - 1, Hq, Hkv, d,
        _p(qz.q8), _p(qz.q4), _p(qz.sq8), _p(qz.sq4),
        _p(qz.k8), _p(qz.k4), _p(qz.sk8), _p(qz.sk4),
        _p(qz.qf), _p(qz.sqf), _p(qz.kf), _p(qz.skf),
        _p(rp), _p(en), float(scale), len(rows), _p(rows), _p(out), _p(lse))
    if rc != 0:
        raise ValueError(f"oracle prefill failed ({rc})")
    return out, lse


def gather_rows(out_rows, cu_seqlens, rows, Hq):
    """Scatter per-row oracle output [nrows, 64, d] into token order for one head.

    Returns a dict {(h, token): vector} for the valid tokens of each row.
    """
    cu = np.asarray(cu_seqlens, np.int64)
    nt = [(int(cu[b + 1] - cu[b]) + TILE - 1) // TILE for b in range(len(cu) - 1)]
    off = np.concatenate([[0], np.cumsum(nt)])
    ntiles = int(off[-1])
    res = {}
    for i, row in enumerate(rows):
        h, gq = divmod(int(row), ntiles)
        b = int(np.searchsorted(off, gq, side="right") - 1)
        qt = gq - off[b]
        T = int(cu[b + 1] - cu[b])
        for r in range(TILE):
            t = qt * TILE + r
            if t < T:
                res[(h, int(cu[b]) + t)] = out_rows[i, r]
    return res


def decode_step(qd_bits, cu_seqlens, Hkv, cache: Quantised, row_ptr, entries,
                k_tail_bits, v_tail_bits, tail_len, scale=None):
    """fp64 decode output [B, Hq, d]; the tails already hold the new token."""
    qd = _c(qd_bits, np.uint16)
    cu = _c(cu_seqlens, np.int32)
    B, Hq, d = qd.shape
    kt = _c(k_tail_bits, np.uint16); vt = _c(v_tail_bits, np.uint16)
    cap = kt.shape[2]
    tl = _c(tail_len, np.int32)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((B, Hq, d), np.float64)
    rp = _c(row_ptr, np.int32); en = _c(entries, np.uint32)
    rc = _load().orc_decode_step(
        _p(qd), _p(cu), B, Hq, Hkv, d,
        _p(cache.k8), _p(cache.k4), _p(cache.sk8), _p(cache.sk4),
        _p(cache.v8), _p(cache.v4), _p(cache.sv8), _p(cache.sv4),
        _p(rp), _p(en), _p(kt), _p(vt), _p(tl), cap, float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle decode failed")
    return out


def allocate_boundaries(err, cost, budget):
    """Model-wide boundary allocation by enumeration (TriAttention abstract: an allocator
    selects each head's boundaries to minimise calibration error under a shared
    computation budget).  err / cost [heads][candidates]; every combination of one
    candidate per head is tried, the least total error with total cost <= budget wins
    (ties: the lexicographically smallest choice).  Small cases only: the work is
    candidates ** heads.  Returns (choice, total_err, total_cost), or None when nothing
    fits the budget."""
    import itertools
    err = np.asarray(err, np.float64)
    cost = np.asarray(cost, np.int64)
    H, C = err.shape
    best = None
    for pick in itertools.product(range(C), repeat=H):
        c = sum(int(cost[h, pick[h]]) for h in range(H))
        if c > budget:
            continue
        e = sum(float(err[h, pick[h]]) for h in range(H))
        if best is None or e < best[1]:
            best = (list(pick), e, c)
    return best


# --------------------------------------------------------------- token-level hybrid
# HyQuant ("The observation behind the method"; "How HyQuant works"): a small set of
# important key positions and a recent window keep high precision, the rest of the
# context is quantised.  Readings: per (sequence, KV head) the ceil(frac * T) most
# important prefix tokens and every key within `window` positions of the query stay
# bf16; the other keys and values use their tile's INT4 codes times the tile scale;
# queries stay bf16.  Plain numpy in fp64.

def _f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _int4_values(x4, s4, cu, H):
    """Dequantised INT4 codes [ntok, H, d] in token order (fp64)."""
    cu = _c(cu, np.int32)
    nib = np.stack([x4 & 0xF, x4 >> 4], -1).reshape(*x4.shape[:-1], -1).astype(np.int64)
    codes = np.where(nib >= 8, nib - 16, nib).astype(np.float64)      # [H, nt, 64, d]
    ntok = int(cu[-1])
    out = np.zeros((ntok, H, codes.shape[-1]), np.float64)
    gt = 0
    for b in range(len(cu) - 1):
        L = int(cu[b + 1] - cu[b])
        for t in range((L + TILE - 1) // TILE):
            n = min(TILE, L - t * TILE)
            for h in range(H):
                out[cu[b] + t * TILE: cu[b] + t * TILE + n, h] = codes[h, gt, :n] * np.float64(s4[h, gt])
            gt += 1
    return out


def hybrid_select(importance, cu_seqlens, frac=0.05):
    """bool [ntok, Hkv]: per sequence and KV head, the ceil(frac * T) tokens of largest
    importance (ties: the earlier position)."""
    imp = np.asarray(importance, np.float64)
    cu = _c(cu_seqlens, np.int32)
    sel = np.zeros(imp.shape, bool)
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        n = int(np.ceil(frac * (e - s)))
        for h in range(imp.shape[1]):
            order = sorted(range(s, e), key=lambda j: (-imp[j, h], j))
            sel[order[:n], h] = True
    return sel


def hybrid_prefill(q_bits, k_bits, v_bits, cu_seqlens, kv: Quantised, selected, window,
                   scale=None, rows=None, with_lse=False):
    """fp64 output [ntok, Hq, d]: causal attention in which query i reads key j <= i (same
    sequence) at bf16 when j is selected or i - j < window, else from its INT4 tile.
    rows: optional global query-token indices; only those rows are computed (the others
    stay zero), each exactly as in the full computation.  with_lse: also return lse
    [Hq, ntok], the natural log of the row's sum of exp of the scaled scores."""
    q = _f64(q_bits); k = _f64(k_bits); v = _f64(v_bits)
    cu = _c(cu_seqlens, np.int32)
    ntok, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    k4 = _int4_values(kv.k4, kv.sk4, cu, Hkv)
    v4 = _int4_values(kv.v4, kv.sv4, cu, Hkv)
    want = np.ones(ntok, bool)
    if rows is not None:
        want = np.zeros(ntok, bool)
        want[np.asarray(rows, np.int64)] = True
    out = np.zeros((ntok, Hq, d), np.float64)
    lse = np.zeros((Hq, ntok), np.float64)
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        T = e - s
        ii = np.nonzero(want[s:e])[0]
        if T == 0 or len(ii) == 0:
            continue
        i = ii[:, None]
        j = np.arange(T)[None, :]
        causal = j <= i
        for h in range(Hq):
            kh = h // g
            hi = selected[s:e, kh][None, :] | (i - j < window)
            s_hi = q[s + ii, h] @ k[s:e, kh].T
            s_lo = q[s + ii, h] @ k4[s:e, kh].T
            sc = np.where(hi, s_hi, s_lo) * scale
            sc = np.where(causal, sc, -np.inf)
            mx = sc.max(axis=1, keepdims=True)
            p = np.exp(sc - mx)
            tot = p.sum(axis=1, keepdims=True)
            lse[h, s + ii] = (mx + np.log(tot))[:, 0]
            p /= tot
            out[s + ii, h] = (p * hi) @ v[s:e, kh] + (p * ~hi) @ v4[s:e, kh]
    return (out, lse) if with_lse else out


def hybrid_decode_step(qd_bits, k_bits, v_bits, cu_seqlens, kv: Quantised, selected, window,
                       k_tail_bits, v_tail_bits, tail_len, scale=None):
    """fp64 output [B, Hq, d] of one decode step: the query, at position T_b + tail_len_b - 1,
    reads every prefix token (bf16 when selected or within `window` positions of it, else
    from its INT4 tile) and the bf16 tail tokens [0, tail_len_b), which hold the new one."""
    qd = _f64(qd_bits); k = _f64(k_bits); v = _f64(v_bits)
    kt = _f64(k_tail_bits); vt = _f64(v_tail_bits)
    cu = _c(cu_seqlens, np.int32)
    B, Hq, d = qd.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    k4 = _int4_values(kv.k4, kv.sk4, cu, Hkv)
    v4 = _int4_values(kv.v4, kv.sv4, cu, Hkv)
    out = np.zeros((B, Hq, d), np.float64)
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        tl = int(tail_len[b])
        pos = (e - s) + tl - 1
        j = np.arange(e - s)
        for h in range(Hq):
            kh = h // g
            hi = selected[s:e, kh] | (pos - j < window)
            kp = np.where(hi[:, None], k[s:e, kh], k4[s:e, kh])
            vp = np.where(hi[:, None], v[s:e, kh], v4[s:e, kh])
            keys = np.concatenate([kp, kt[b, kh, :tl]])
            vals = np.concatenate([vp, vt[b, kh, :tl]])
            sc = keys @ qd[b, h] * scale
            p = np.exp(sc - sc.max())
            out[b, h] = p @ vals / p.sum()
    return out
