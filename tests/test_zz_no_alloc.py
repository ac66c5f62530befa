"""routed_attention_decode_noalloc: the decode step for callers that cannot
allocate device memory (plugins handed only input/output buffers, or loops that
reserved all device memory up front).  It runs the same kernel as the regular
entry point, whose scratch comes from a caller workspace, so on the same inputs
the two must agree bit for bit; both are also checked against the oracle.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test before it.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import tile_routed_mixed_causal_b200 as tra
from tile_routed_mixed_causal_b200 import _lib as L
from tile_routed_mixed_causal_b200 import api
from tile_routed_mixed_causal_b200 import build as tra_build
from tile_routed_mixed_causal_b200 import workloads as wl

MAX_TOL, MEAN_TOL = 1e-2, 1e-3   # the tolerance of the GPU parity tests


def _assert_close(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    a = np.abs(ref)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8), 0.0)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert float(np.max(err - half_ulp)) <= MAX_TOL and float(np.mean(err)) <= MEAN_TOL


class _Run:
    """One decode problem with two sets of tails: one stepped by the regular entry point
    (caller workspace), one by the no-allocation entry point; plus oracle tails."""

    def __init__(self, w):
        self.w = w
        t = wl.make_inputs(w, "cpu")
        self.kb, self.vb = wl.bf16_bits(t["k"]), wl.bf16_bits(t["v"])
        self.shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
        self.pol = tra.Policy.boundary(w.b1, w.b2)
        self.cache = tra.QTiles(self.shape, tra.FMT_K8 | tra.FMT_K4 | tra.FMT_V8 | tra.FMT_V4)
        tra.quantize_qkv_tiles(self.shape, None, t["k"].cuda(), t["v"].cuda(), self.cache)
        self.ref_plan = api.DecodePlan(self.shape, self.pol, self.cache, w.tail_cap)
        self.na_plan = api.DecodePlan(self.shape, self.pol, self.cache, w.tail_cap)
        self.ref_plan.build()
        self.na_plan.build()
        self.qs, self.kn, self.vn = (x.cuda() for x in wl.make_decode_inputs(w, "cpu"))
        self.scale = 1.0 / math.sqrt(w.d)
        self.ocache = oracle.Quantised(None, self.kb, self.vb, w.cu_seqlens)
        self.orp, self.oen = oracle.lists_decode(w.cu_seqlens, w.Hq, w.Hkv, w.b1, w.b2)
        self.kt = np.zeros((w.B, w.Hkv, w.tail_cap, w.d), np.uint16)
        self.vt = np.zeros_like(self.kt)

    def step(self, i):
        w = self.w
        out_ref = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
        out_na = torch.full_like(out_ref, float("nan"))
        self.ref_plan.step(self.qs[i], self.kn[i], self.vn[i], out_ref, self.scale)
        p = self.na_plan
        L.routed_attention_decode_noalloc(
            self.shape, self.pol, self.qs[i], self.kn[i], self.vn[i], self.cache, p.row_ptr,
            p.entries, p.k_tail, p.v_tail, p.tail_len, self.scale, out_na, p.status)
        torch.cuda.synchronize()
        # same kernel, same inputs: identical bits
        assert torch.equal(out_na.view(torch.int16), out_ref.view(torch.int16)), (w.name, i)
        self.kt[:, :, i] = wl.bf16_bits(self.kn[i])
        self.vt[:, :, i] = wl.bf16_bits(self.vn[i])
        ref = oracle.decode_step(wl.bf16_bits(self.qs[i]), w.cu_seqlens, w.Hkv, self.ocache,
                                 self.orp, self.oen, self.kt, self.vt,
                                 np.full(w.B, i + 1, np.int32))
        _assert_close(out_na.float().cpu().numpy(), ref)

    def check_state(self, steps):
        assert int(self.ref_plan.status.item()) == 0 and int(self.na_plan.status.item()) == 0
        assert np.array_equal(self.na_plan.tail_len.cpu().numpy(), np.full(self.w.B, steps))
        assert torch.equal(self.na_plan.tail_len, self.ref_plan.tail_len)
        assert torch.equal(self.na_plan.k_tail, self.ref_plan.k_tail)
        assert torch.equal(self.na_plan.v_tail, self.ref_plan.v_tail)


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_entry_point():
    """Two calls in a row of one shape, then a call of another (B, Hkv) shape between two
    more calls of the first: the shared array's counters must come back to zero and every
    output must match the regular entry point bit for bit (and the oracle)."""
    a = _Run(wl.custom("noalloc_a", [64 * 12 + 5, 64 * 7], 8, 2, 128, 61, "boundary",
                       b1=[1, 2, 3, 1, 4, 1, 2, 2], b2=[3, 2, 9, 5, 4, 12, 6, 2],
                       decode_steps=3, tail_cap=4))
    b = _Run(wl.custom("noalloc_b", [64 * 3 + 9, 64 * 5, 64 * 2 + 1], 4, 4, 64, 62, "boundary",
                       b1=[1, 2, 1, 3], b2=[2, 4, 5, 3], decode_steps=1, tail_cap=2))
    a.step(0)
    a.step(1)          # two calls in a row
    b.step(0)          # another shape in between
    a.step(2)
    a.check_state(3)
    b.check_state(1)


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    """Host-side size checks: no device work is attempted when the scratch is too small
    or when the arrival counters would leave the fixed counter area."""
    tra_build.build()
    lib = L.load()
    pol_args = ([1] * 32, [2] * 32)
    fake = ctypes.c_void_p(1 << 20)
    # 512 sequences x 32 heads: more than 4 MiB of partials
    cu = np.array([0, 64 * 4] + [64 * 4 * (i + 2) for i in range(511)], np.int32)
    shape = L.Shape(cu, 32, 8, 128, device=None)
    assert lib.tra_decode_workspace_bytes(512, 32, 8, 128) > 4 << 20
    pol = L.Policy.boundary(*pol_args)
    st = lib.routed_attention_decode_noalloc(shape.c, pol.c, *([fake] * 9), 4, 0.1, fake, fake,
                                             None)
    assert st == 2
    assert b"fixed" in lib.tra_last_error()
    # 8193 single-token sequences, Hq = Hkv = 1: small scratch, but B * (Hkv + 1) > 16384
    B = 8193
    cu = np.arange(B + 1, dtype=np.int32)
    shape = L.Shape(cu, 1, 1, 64, device=None)
    assert lib.tra_decode_workspace_bytes(B, 1, 1, 64) <= 4 << 20
    pol = L.Policy.boundary([1], [2])
    st = lib.routed_attention_decode_noalloc(shape.c, pol.c, *([fake] * 9), 4, 0.1, fake, fake,
                                             None)
    assert st == 2
    assert b"arrival counters" in lib.tra_last_error()
