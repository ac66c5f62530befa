"""GPU parity of the token-level hybrid (HyQuant Uses Hybrid Precision to Compress LLM
Attention, "How HyQuant works"): token selection bit-exact against the oracle's
selection, decode steps within the output tolerance of the other GPU parity tests.

Selection: per (sequence, KV head) the ceil(frac * T) positions of largest importance,
ties to the earlier position; importance is handed to both sides in fp32.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import tile_routed_mixed_causal_b200 as tra
from tile_routed_mixed_causal_b200 import api
from tile_routed_mixed_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL = 1e-2, 1e-3


def _assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    a = np.abs(ref)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8), 0.0)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    excess, mean = float(np.max(err - half_ulp)), float(np.mean(err))
    assert excess <= MAX_TOL and mean <= MEAN_TOL, f"{what}: excess {excess:.3e} mean {mean:.3e}"


def _importance(w, seed, ties=False):
    imp = wl.hybrid_importance(w, seed).astype(np.float32)
    if ties:  # equal scores (ties go to the earlier position), signed zeros, exact repeats
        imp[3:9, 0] = imp[:, 0].max()
        imp[20:40, -1] = 0.0
        imp[25, -1] = -0.0
        imp[60:70] = imp[50:60]
    return imp


class HybridCase:
    def __init__(self, w, frac, window, seed, gen_device="cpu", ties=False):
        self.w, self.frac, self.window = w, frac, window
        t = wl.make_inputs(w, gen_device, need_q=False)
        self.k, self.v = t["k"].cuda(), t["v"].cuda()
        self.kb, self.vb = wl.bf16_bits(t["k"]), wl.bf16_bits(t["v"])
        self.shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
        self.imp = _importance(w, seed, ties)
        self.cache = tra.QTiles(self.shape, tra.FMT_K4 | tra.FMT_V4)
        tra.quantize_qkv_tiles(self.shape, None, self.k, self.v, self.cache)
        self.plan = api.HybridDecodePlan(self.shape, self.cache, frac, window, w.tail_cap)
        self.plan.select(torch.from_numpy(self.imp).cuda(), self.k, self.v)
        torch.cuda.synchronize()
        self.sel = oracle.hybrid_select(self.imp.astype(np.float64), w.cu_seqlens, frac)


SMALL = [
    (wl.custom("hy_varlen_gqa4", [64 * 9 + 17, 64 * 3, 1, 200], 8, 2, 128, 81, "boundary",
               decode_steps=3, tail_cap=4), 0.05, 128),
    (wl.custom("hy_d64_win16", [700, 65], 4, 4, 64, 82, "boundary", decode_steps=2, tail_cap=3),
     0.2, 16),
    (wl.custom("hy_nowin_all", [300], 4, 1, 128, 83, "boundary", decode_steps=2, tail_cap=2),
     1.0, 0),
    (wl.custom("hy_none", [500, 130], 8, 2, 128, 84, "boundary", decode_steps=2, tail_cap=2),
     0.0, 40),
]


@pytest.mark.parametrize("w,frac,window", SMALL, ids=lambda x: getattr(x, "name", str(x)))
def test_hybrid_select_bit_exact(w, frac, window):
    c = HybridCase(w, frac, window, seed=5, ties=w.ntok > 80)
    hy = c.plan.hy
    cu = w.cu_seqlens
    nts = w.tiles_per_seq
    off = np.concatenate([[0], np.cumsum(nts)])
    counts = hy.sel_count.cpu().numpy()
    pos = hy.sel_pos.cpu().numpy()
    mask = hy.sel_mask.cpu().numpy().view(np.uint64)
    ksel, vsel = wl.bf16_bits(hy.k_sel), wl.bf16_bits(hy.v_sel)
    kwin = wl.bf16_bits(hy.k_win)
    for b in range(w.B):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        T = s1 - s0
        n = int(np.ceil(frac * T))
        assert counts[b] == n
        for h in range(w.Hkv):
            ref = np.nonzero(c.sel[s0:s1, h])[0]
            assert np.array_equal(pos[b, h, :n], ref), (b, h)
            bits = np.zeros(nts[b] * 64, bool)
            bits[ref] = True
            for kt in range(nts[b]):
                word = int(mask[h, off[b] + kt])
                assert word == sum(1 << i for i in range(64) if bits[kt * 64 + i]), (b, h, kt)
            assert np.array_equal(ksel[b, h, :n], c.kb[s0 + ref, h])
            assert np.array_equal(vsel[b, h, :n], c.vb[s0 + ref, h])
            for x in range(window):
                j = T - window + x
                want = c.kb[s0 + j, h] if j >= 0 else np.zeros(w.d, np.uint16)
                assert np.array_equal(kwin[b, h, x], want)


@pytest.mark.parametrize("w,frac,window", SMALL, ids=lambda x: getattr(x, "name", str(x)))
def test_hybrid_decode_matches_oracle(w, frac, window):
    c = HybridCase(w, frac, window, seed=6)
    qs, kn, vn = (x.cuda() for x in wl.make_decode_inputs(w, "cpu"))
    cu = w.cu_seqlens
    kv = oracle.Quantised(None, c.kb, c.vb, cu)
    kt = np.zeros((w.B, w.Hkv, w.tail_cap, w.d), np.uint16)
    vt = np.zeros_like(kt)
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    for step in range(w.decode_steps):
        c.plan.step(qs[step], kn[step], vn[step], out)
        torch.cuda.synchronize()
        kt[:, :, step] = wl.bf16_bits(kn[step])
        vt[:, :, step] = wl.bf16_bits(vn[step])
        ref = oracle.hybrid_decode_step(wl.bf16_bits(qs[step]), c.kb, c.vb, cu, kv, c.sel, window,
                                        kt, vt, np.full(w.B, step + 1, np.int32))
        _assert_close(out.float().cpu().numpy(), ref, f"{w.name} step {step}")
    assert int(c.plan.status.item()) == 0
    assert np.array_equal(c.plan.tail_len.cpu().numpy(), np.full(w.B, w.decode_steps))


def test_hybrid_decode_full_size_sampled():
    """Batch 16 over a 32K prefix (32/8 heads, d 128), 5% selected, 128-token window, 64
    steps as benchmarked; sampled sequences and steps against the oracle."""
    w = wl.decode_32k()
    c = HybridCase(w, 0.05, 128, seed=7, gen_device="cuda")
    qs, kn, vn = wl.make_decode_inputs(w, "cuda")
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    check = {0, 40, 63}
    outs = {}
    for step in range(w.decode_steps):
        c.plan.step(qs[step], kn[step], vn[step], out)
        if step in check:
            outs[step] = out.float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(c.plan.status.item()) == 0
    T = w.lengths[0]
    for b in (0, 11):
        cu1 = np.array([0, T], np.int32)
        kb, vb = c.kb[b * T:(b + 1) * T], c.vb[b * T:(b + 1) * T]
        kv = oracle.Quantised(None, kb, vb, cu1)
        sel = c.sel[b * T:(b + 1) * T]
        for step in sorted(check):
            kt = np.ascontiguousarray(wl.bf16_bits(kn[:step + 1, b]).transpose(1, 0, 2)[None])
            vt = np.ascontiguousarray(wl.bf16_bits(vn[:step + 1, b]).transpose(1, 0, 2)[None])
            ref = oracle.hybrid_decode_step(wl.bf16_bits(qs[step, b:b + 1]), kb, vb, cu1, kv, sel,
                                            128, kt, vt, np.array([step + 1], np.int32))
            _assert_close(outs[step][b], ref[0], f"hybrid b={b} step={step}")
