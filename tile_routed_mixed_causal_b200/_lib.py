"""ctypes binding of ``libtra.so`` (the C ABI in ``include/tra.h``).

Argument marshalling only: every step of the path runs in the CUDA library.
torch supplies device memory and the current stream.  There is no fallback:
if ``libtra.so`` is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtra.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "tra.h")

TILE = 64
PREC_INT4, PREC_INT8, PREC_BF16, PREC_FP8 = 1, 2, 3, 4
POLICY_BOUNDARY, POLICY_BITMASK, POLICY_MIXED = 0, 1, 2
LISTS_PREFILL, LISTS_DECODE_CACHE = 0, 1
FMT_Q8, FMT_Q4, FMT_K8, FMT_K4, FMT_V8, FMT_V4 = 0x1, 0x2, 0x4, 0x8, 0x10, 0x20
FMT_Q4X, FMT_K4X = 0x40, 0x80
FMT_Q8F, FMT_K8F = 0x100, 0x200
DEV_TIMEOUT, DEV_TAIL_FULL, DEV_BAD_LIST = 0x1, 0x2, 0x4
STATUS = {0: "TRA_OK", 1: "TRA_ERR_INVALID", 2: "TRA_ERR_UNSUPPORTED", 3: "TRA_ERR_BUFFER",
          4: "TRA_ERR_CUDA", 5: "TRA_ERR_TIMEOUT"}


class TraError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("cu_seqlens_dev", ctypes.c_void_p),
                ("cu_seqlens_host", ctypes.c_void_p)]


class _Policy(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("b1", ctypes.c_void_p), ("b2", ctypes.c_void_p),
                ("bitmask_dev", ctypes.c_void_p), ("G", ctypes.c_int32), ("W", ctypes.c_int32),
                ("b8", ctypes.c_void_p)]


class _Hybrid(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("cap", ctypes.c_int32)] + \
               [(n, ctypes.c_void_p) for n in
                ("sel_count", "sel_pos", "sel_mask", "k_sel", "v_sel", "k_win", "v_win")]


class _QTiles(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q8", "q4", "k8", "k4", "v8", "v4", "sq8", "sq4", "sk8", "sk4", "sv8", "sv4")] + \
               [("formats", ctypes.c_uint32), ("q4x", ctypes.c_void_p), ("k4x", ctypes.c_void_p),
                ("q8f", ctypes.c_void_p), ("k8f", ctypes.c_void_p), ("sqf", ctypes.c_void_p),
                ("skf", ctypes.c_void_p)]


_lib = None


def load():
    """Load libtra.so; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m tile_routed_mixed_causal_b200.build` "
            "(the CUDA library is the only implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    sig = {
        "tra_last_error": ([], ctypes.c_char_p),
        "tra_version": ([], ctypes.c_char_p),
        "tra_num_tiles": ([P], I64),
        "tra_qtiles_bytes": ([P, ctypes.c_uint32], SZ),
        "quantize_qkv_tiles": ([P, P, P, P, P, P], I32),
        "tra_tile_lists_size": ([P, P, I32, P, P], I32),
        "build_tile_lists": ([P, P, I32, P, I64, P, I64, P], I32),
        "routed_attention_prefill": ([P, P, P, P, P, P, P, P, F, P, P, P, I32, P, P, P], I32),
        "tra_decode_workspace_bytes": ([I32, I32, I32, I32], SZ),
        "routed_attention_decode": ([P, P, P, P, P, P, P, P, P, P, P, I32, F, P, P, SZ, P, P], I32),
        "routed_attention_decode_noalloc": ([P, P, P, P, P, P, P, P, P, P, P, I32, F, P, P, P], I32),
        "tra_selftest_bounded_wait": ([P, I64, P], I32),
        "tra_boundary_tile_counts": ([P, I32, I32, P, P], I32),
        "tra_allocate_boundaries": ([I32, I32, P, P, I64, P, P, P], I32),
        "tra_hybrid_capacity": ([P, ctypes.c_double], I32),
        "tra_prefill_cost_model": ([P, P, P, ctypes.c_double, ctypes.c_double, I32, P, P], I32),
        "hybrid_select_tokens": ([P, P, ctypes.c_double, P, P, P, P], I32),
        "hybrid_attention_decode": ([P, P, P, P, P, P, P, P, P, I32, F, P, P, SZ, P, P], I32),
        "hybrid_attention_prefill": ([P, P, P, P, P, P, P, P, F, P, P, P, P], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def header_functions():
    """Names of the functions include/tra.h declares (TRA_API ... name()."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"TRA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def _check(status: int):
    if status != 0:
        raise TraError(status, load().tra_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return ctypes.c_void_p(t.data_ptr())
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(ctypes.c_void_p)
    return ctypes.c_void_p(int(t))


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


class Shape:
    """Batch geometry: B sequences (cu_seqlens), Hq/Hkv heads, head dim d."""

    def __init__(self, cu_seqlens, Hq: int, Hkv: int, d: int, device="cuda"):
        self.cu_host = np.ascontiguousarray(np.asarray(cu_seqlens, np.int32))
        self.cu_dev = torch.as_tensor(self.cu_host).to(device) if device is not None else None
        self.B = len(self.cu_host) - 1
        self.Hq, self.Hkv, self.d = Hq, Hkv, d
        self._c = _Shape(self.B, Hq, Hkv, d,
                         self.cu_dev.data_ptr() if self.cu_dev is not None else 16,
                         self.cu_host.ctypes.data)

    @property
    def c(self):
        return ctypes.byref(self._c)

    @property
    def ntok(self) -> int:
        return int(self.cu_host[-1])

    @property
    def ntiles(self) -> int:
        n = load().tra_num_tiles(self.c)
        if n < 0:
            raise TraError(1, load().tra_last_error().decode())
        return int(n)


class Policy:
    """Boundary policy (host b1/b2 per head, optionally an FP8 band [b1, b8)), bitmask
    policy (device words, G), or both at once (mixed: boundaries decide skip / INT4 /
    INT8, a set bit BF16)."""

    def __init__(self, mode, b1=None, b2=None, bitmask=None, G=1, b8=None):
        self.mode = mode
        self.b1 = None if b1 is None else np.ascontiguousarray(np.asarray(b1, np.int32))
        self.b2 = None if b2 is None else np.ascontiguousarray(np.asarray(b2, np.int32))
        self.b8 = None if b8 is None else np.ascontiguousarray(np.asarray(b8, np.int32))
        self.bitmask = bitmask
        self.G = int(G)
        self.W = int(bitmask.shape[-1]) if bitmask is not None else 0
        self._c = _Policy(mode,
                          self.b1.ctypes.data if self.b1 is not None else None,
                          self.b2.ctypes.data if self.b2 is not None else None,
                          bitmask.data_ptr() if isinstance(bitmask, torch.Tensor) else None,
                          self.G, self.W,
                          self.b8.ctypes.data if self.b8 is not None else None)

    @classmethod
    def boundary(cls, b1, b2, b8=None):
        return cls(POLICY_BOUNDARY, b1=b1, b2=b2, b8=b8)

    @classmethod
    def from_bitmask(cls, bitmask: torch.Tensor, G: int):
        return cls(POLICY_BITMASK, bitmask=bitmask, G=G)

    @classmethod
    def mixed(cls, b1, b2, bitmask: torch.Tensor, G: int):
        return cls(POLICY_MIXED, b1=b1, b2=b2, bitmask=bitmask, G=G)

    @property
    def c(self):
        return ctypes.byref(self._c)

    @property
    def has_int4(self) -> bool:
        lo = self.b8 if self.b8 is not None else self.b1
        return self.mode != POLICY_BITMASK and bool(np.any(self.b2 > lo))

    @property
    def has_fp8(self) -> bool:
        return self.mode == POLICY_BOUNDARY and self.b8 is not None and bool(np.any(self.b8 > self.b1))


class QTiles:
    """Quantised tile buffers (torch-allocated device memory) for the requested formats."""

    def __init__(self, shape: Shape, formats: int, device="cuda"):
        nt, d = shape.ntiles, shape.d
        self.formats = formats
        spec = {"q": shape.Hq, "k": shape.Hkv, "v": shape.Hkv}
        self.t = {}
        for i, (name, H) in enumerate(spec.items()):
            if formats & (FMT_Q8 << (2 * i)):
                self.t[name + "8"] = torch.zeros((H, nt, TILE, d), dtype=torch.int8, device=device)
                self.t["s" + name + "8"] = torch.zeros((H, nt), dtype=torch.float32, device=device)
            if formats & (FMT_Q4 << (2 * i)):
                self.t[name + "4"] = torch.zeros((H, nt, TILE, d // 2), dtype=torch.uint8, device=device)
            x4 = {"q": FMT_Q4X, "k": FMT_K4X}.get(name, 0)
            if formats & x4:
                self.t[name + "4x"] = torch.zeros((H, nt, TILE, d), dtype=torch.int8, device=device)
            if formats & ((FMT_Q4 << (2 * i)) | x4):
                self.t["s" + name + "4"] = torch.zeros((H, nt), dtype=torch.float32, device=device)
            if formats & {"q": FMT_Q8F, "k": FMT_K8F}.get(name, 0):
                self.t[name + "8f"] = torch.zeros((H, nt, TILE, d), dtype=torch.uint8, device=device)
                self.t["s" + name + "f"] = torch.zeros((H, nt), dtype=torch.float32, device=device)
        ptr = lambda n: self.t[n].data_ptr() if n in self.t else None
        self._c = _QTiles(*[ptr(n) for n in ("q8", "q4", "k8", "k4", "v8", "v4",
                                             "sq8", "sq4", "sk8", "sk4", "sv8", "sv4")],
                          formats, ptr("q4x"), ptr("k4x"), ptr("q8f"), ptr("k8f"), ptr("sqf"),
                          ptr("skf"))

    def __getitem__(self, k):
        return self.t[k]

    @property
    def c(self):
        return ctypes.byref(self._c)


# ---------------------------------------------------------------- ABI calls (same names)
def quantize_qkv_tiles(shape: Shape, q, k, v, out: QTiles, stream=None):
    _check(load().quantize_qkv_tiles(shape.c, _ptr(q), _ptr(k), _ptr(v), out.c, _stream(stream)))


def tile_lists_size(shape: Shape, policy: Policy, kind: int = LISTS_PREFILL):
    rows, nnz = ctypes.c_int64(), ctypes.c_int64()
    _check(load().tra_tile_lists_size(shape.c, policy.c, kind, ctypes.byref(rows), ctypes.byref(nnz)))
    return rows.value, nnz.value


def build_tile_lists(shape: Shape, policy: Policy, kind: int, row_ptr, entries, stream=None):
    _check(load().build_tile_lists(shape.c, policy.c, kind, _ptr(row_ptr), row_ptr.numel(),
                                   _ptr(entries), entries.numel(), _stream(stream)))


def routed_attention_prefill(shape: Shape, policy: Policy, q, k, v, tiles: QTiles, row_ptr,
                             entries, softmax_scale, out, lse=None, dump_coords=None,
                             dump_out=None, status=None, stream=None):
    n_dump = 0 if dump_coords is None else int(dump_coords.shape[0])
    _check(load().routed_attention_prefill(
        shape.c, policy.c, _ptr(q), _ptr(k), _ptr(v), tiles.c, _ptr(row_ptr), _ptr(entries),
        float(softmax_scale), _ptr(out), _ptr(lse), _ptr(dump_coords), n_dump, _ptr(dump_out),
        _ptr(status), _stream(stream)))


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int) -> int:
    return int(load().tra_decode_workspace_bytes(B, Hq, Hkv, d))


def routed_attention_decode(shape: Shape, policy: Policy, q, k_new, v_new, cache: QTiles, row_ptr,
                            entries, k_tail, v_tail, tail_len, softmax_scale, out, workspace,
                            status, stream=None):
    _check(load().routed_attention_decode(
        shape.c, policy.c, _ptr(q), _ptr(k_new), _ptr(v_new), cache.c, _ptr(row_ptr),
        _ptr(entries), _ptr(k_tail), _ptr(v_tail), _ptr(tail_len), int(k_tail.shape[2]),
        float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def routed_attention_decode_noalloc(shape: Shape, policy: Policy, q, k_new, v_new, cache: QTiles,
                                    row_ptr, entries, k_tail, v_tail, tail_len, softmax_scale, out,
                                    status, stream=None):
    """Decode step without a caller workspace (the library's fixed scratch array is used)."""
    _check(load().routed_attention_decode_noalloc(
        shape.c, policy.c, _ptr(q), _ptr(k_new), _ptr(v_new), cache.c, _ptr(row_ptr),
        _ptr(entries), _ptr(k_tail), _ptr(v_tail), _ptr(tail_len), int(k_tail.shape[2]),
        float(softmax_scale), _ptr(out), _ptr(status), _stream(stream)))


def tra_selftest_bounded_wait(status, limit_ns: int, stream=None):
    """Diagnostic: a kernel whose mbarrier wait never completes must give up after
    limit_ns and OR DEV_TIMEOUT into the device int32 `status` (see include/tra.h)."""
    _check(load().tra_selftest_bounded_wait(_ptr(status), int(limit_ns), _stream(stream)))


class Hybrid:
    """Device arrays of the token-level hybrid's high-precision side (torch-allocated):
    per (sequence, KV head) the ceil(frac * T) selected positions, their tile masks and
    bf16 K / V rows, and the bf16 K / V of the last `window` prefix tokens."""

    def __init__(self, shape: Shape, frac: float, window: int, device="cuda"):
        cap = int(load().tra_hybrid_capacity(shape.c, float(frac)))
        if cap < 0:
            raise TraError(1, "invalid shape or frac")
        B, Hkv, d, nt = shape.B, shape.Hkv, shape.d, shape.ntiles
        self.frac, self.window, self.cap = float(frac), int(window), cap
        c1, w1 = max(cap, 1), max(window, 1)
        self.sel_count = torch.zeros(B, dtype=torch.int32, device=device)
        self.sel_pos = torch.zeros((B, Hkv, c1), dtype=torch.int32, device=device)
        self.sel_mask = torch.zeros((Hkv, max(nt, 1)), dtype=torch.int64, device=device)
        self.k_sel = torch.zeros((B, Hkv, c1, d), dtype=torch.bfloat16, device=device)
        self.v_sel = torch.zeros_like(self.k_sel)
        self.k_win = torch.zeros((B, Hkv, w1, d), dtype=torch.bfloat16, device=device)
        self.v_win = torch.zeros_like(self.k_win)
        self._c = _Hybrid(self.window, cap, *[getattr(self, n).data_ptr() for n in
                                             ("sel_count", "sel_pos", "sel_mask", "k_sel", "v_sel",
                                              "k_win", "v_win")])

    @property
    def c(self):
        return ctypes.byref(self._c)


def hybrid_select_tokens(shape: Shape, importance, frac: float, k, v, hy: Hybrid, stream=None):
    _check(load().hybrid_select_tokens(shape.c, _ptr(importance), float(frac), _ptr(k), _ptr(v),
                                       hy.c, _stream(stream)))


def hybrid_attention_decode(shape: Shape, hy: Hybrid, q, k_new, v_new, cache: QTiles, k_tail,
                            v_tail, tail_len, softmax_scale, out, workspace, status, stream=None):
    _check(load().hybrid_attention_decode(
        shape.c, hy.c, _ptr(q), _ptr(k_new), _ptr(v_new), cache.c, _ptr(k_tail), _ptr(v_tail),
        _ptr(tail_len), int(k_tail.shape[2]), float(softmax_scale), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))


def hybrid_attention_prefill(shape: Shape, hy: Hybrid, q, k, v, kv: QTiles, k_mix, v_mix,
                             softmax_scale, out, lse, status, stream=None):
    _check(load().hybrid_attention_prefill(
        shape.c, hy.c, _ptr(q), _ptr(k), _ptr(v), kv.c, _ptr(k_mix), _ptr(v_mix),
        float(softmax_scale), _ptr(out), _ptr(lse) if lse is not None else None, _ptr(status),
        _stream(stream)))


def boundary_tile_counts(shape: Shape, b1: int, b2: int):
    """(INT8 tiles, INT4 tiles) of one head's boundary pair over the batch."""
    n8, n4 = ctypes.c_int64(), ctypes.c_int64()
    _check(load().tra_boundary_tile_counts(shape.c, int(b1), int(b2), ctypes.byref(n8),
                                           ctypes.byref(n4)))
    return n8.value, n4.value


def prefill_cost_model(shape: Shape, b1, b2, dual_weight: float = 1.25, solo: float = 1.0,
                       n_sm: int = 148):
    """(makespan in entry units, total entries) of the prefill under boundaries b1 / b2
    (host arrays [Hq]); see tra_prefill_cost_model in include/tra.h."""
    b1 = np.ascontiguousarray(np.asarray(b1, np.int32))
    b2 = np.ascontiguousarray(np.asarray(b2, np.int32))
    ms, ne = ctypes.c_double(), ctypes.c_double()
    _check(load().tra_prefill_cost_model(shape.c, _ptr(b1), _ptr(b2), float(dual_weight),
                                         float(solo), int(n_sm), ctypes.byref(ms), ctypes.byref(ne)))
    return ms.value, ne.value


def fit_prefill_cost_model(shape: Shape, policies, times_ms, dual_weight: float = 1.25,
                           n_sm: int = 148):
    """Fit (entry_time_ms, fixed_ms, solo) of tra_prefill_cost_model to measured kernel times of
    boundary policies [(b1, b2), ...]: least squares in the two linear constants for each
    solo on a grid over (0, 1], keeping the best.  Host arithmetic only."""
    best = None
    y = np.asarray(times_ms, np.float64)
    for solo in np.linspace(0.3, 1.0, 36):
        X = np.array([[prefill_cost_model(shape, b1, b2, dual_weight, solo, n_sm)[0], 1.0]
                      for b1, b2 in policies])
        coef, *_ = np.linalg.lstsq(X, y, rcond=None)
        res = float(np.sum((X @ coef - y) ** 2))
        if best is None or res < best[0]:
            best = (res, float(coef[0]), float(coef[1]), float(solo))
    return best[1], best[2], best[3]


def allocate_boundaries(err, cost, budget: int):
    """One candidate per head minimising the total error with total cost <= budget.
    err float64 [heads][candidates], cost int64 (same shape).  Returns (choice int32
    [heads], total error, total cost)."""
    err = np.ascontiguousarray(np.asarray(err, np.float64))
    cost = np.ascontiguousarray(np.asarray(cost, np.int64))
    H, C = err.shape
    assert cost.shape == (H, C)
    choice = np.zeros(H, np.int32)
    te, tc = ctypes.c_double(), ctypes.c_int64()
    _check(load().tra_allocate_boundaries(H, C, _ptr(err), _ptr(cost), int(budget), _ptr(choice),
                                          ctypes.byref(te), ctypes.byref(tc)))
    return choice, te.value, tc.value
