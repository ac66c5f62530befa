"""routed_attention_decode_noalloc: the decode step for callers that cannot
allocate device memory (plugins handed only input/output buffers, or loops that
reserved all device memory up front).  It must give the results of the regular
entry point, which takes a caller workspace, without any workspace argument.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test before it.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

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


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_entry_point():
    w = wl.custom("noalloc", [64 * 12 + 5, 64 * 7], 8, 2, 128, 61, "boundary",
                  b1=[1, 2, 3, 1, 4, 1, 2, 2], b2=[3, 2, 9, 5, 4, 12, 6, 2],
                  decode_steps=2, tail_cap=4)
    t = wl.make_inputs(w, "cpu")
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
    pol = tra.Policy.boundary(w.b1, w.b2)
    cache = tra.QTiles(shape, tra.FMT_K8 | tra.FMT_K4 | tra.FMT_V8 | tra.FMT_V4)
    tra.quantize_qkv_tiles(shape, None, t["k"].cuda(), t["v"].cuda(), cache)
    ref_plan = api.DecodePlan(shape, pol, cache, w.tail_cap)    # caller workspace
    na_plan = api.DecodePlan(shape, pol, cache, w.tail_cap)     # its workspace stays unused
    ref_plan.build()
    na_plan.build()
    qs, kn, vn = (x.cuda() for x in wl.make_decode_inputs(w, "cpu"))
    scale = 1.0 / math.sqrt(w.d)
    out_ref = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    out_na = torch.full_like(out_ref, float("nan"))
    for step in range(2):                                     # two calls in a row
        ref_plan.step(qs[step], kn[step], vn[step], out_ref, scale)
        L.routed_attention_decode_noalloc(
            shape, pol, qs[step], kn[step], vn[step], cache, na_plan.row_ptr, na_plan.entries,
            na_plan.k_tail, na_plan.v_tail, na_plan.tail_len, scale, out_na, na_plan.status)
        torch.cuda.synchronize()
        _assert_close(out_na.float().cpu().numpy(), out_ref.float().cpu().numpy())
    assert int(ref_plan.status.item()) == 0 and int(na_plan.status.item()) == 0
    assert torch.equal(na_plan.tail_len, ref_plan.tail_len)
    assert torch.equal(na_plan.k_tail, ref_plan.k_tail)
    assert torch.equal(na_plan.v_tail, ref_plan.v_tail)


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    """Host-side size check: no device work is attempted when the scratch is too small."""
    tra_build.build()
    lib = L.load()
    cu = np.array([0, 64 * 4] + [64 * 4 * (i + 2) for i in range(511)], np.int32)
    shape = L.Shape(cu, 32, 8, 128, device=None)             # 512 sequences x 32 heads
    assert lib.tra_decode_workspace_bytes(512, 32, 8, 128) > 4 << 20
    pol = L.Policy.boundary([1] * 32, [2] * 32)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.routed_attention_decode_noalloc(shape.c, pol.c, *([fake] * 9), 4, 0.1, fake, fake,
                                             None)
    assert st == 2
    assert b"fixed" in lib.tra_last_error()
