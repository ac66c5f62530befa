"""GPU parity of the token-level hybrid (HyQuant Uses Hybrid Precision to Compress LLM
Attention, "How HyQuant works"): token selection and the prefill's mixed operands
bit-exact against the oracle's selection and codes, prefill rows and decode steps within
the output tolerance of the other GPU parity tests.

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
    def __init__(self, w, frac, window, seed, gen_device="cpu", ties=False, need_q=False):
        self.w, self.frac, self.window = w, frac, window
        t = wl.make_inputs(w, gen_device, need_q=need_q)
        self.q = t["q"].cuda() if need_q else None
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


# --------------------------------------------------------------------------- prefill
LSE_TOL = 2.0 ** -8


def _codes4(x4):
    """[H][nt][64][d/2] packed INT4 (even channel in the low nibble) -> int codes [H][nt][64][d]."""
    x4 = np.asarray(x4, np.uint8)
    lo = (x4 & 0xF).astype(np.int16)
    hi = (x4 >> 4).astype(np.int16)
    out = np.empty(x4.shape[:-1] + (2 * x4.shape[-1],), np.int16)
    out[..., 0::2] = np.where(lo > 7, lo - 16, lo)
    out[..., 1::2] = np.where(hi > 7, hi - 16, hi)
    return out


def _tiles_to_tokens(codes, cu):
    """[H][ntiles][64][d] -> [ntok][H][d] (rows past a sequence's end dropped)."""
    rows = []
    t0 = 0
    for b in range(len(cu) - 1):
        T = int(cu[b + 1] - cu[b])
        nt = (T + 63) // 64
        rows.append(codes[:, t0:t0 + nt].reshape(codes.shape[0], nt * 64, -1)[:, :T])
        t0 += nt
    return np.concatenate(rows, axis=1).transpose(1, 0, 2)


def _bf16_of_ints(c):
    return (np.asarray(c, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _run_hybrid_prefill(c, with_lse=True):
    w = c.w
    k_mix = torch.zeros((w.ntok, w.Hkv, w.d), dtype=torch.bfloat16, device="cuda")
    v_mix = torch.zeros_like(k_mix)
    out = torch.full((w.ntok, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.Hq, w.ntok), dtype=torch.float32, device="cuda") if with_lse else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tra.hybrid_attention_prefill(c.shape, c.plan.hy, c.q, c.k, c.v, c.cache, k_mix, v_mix,
                                 1.0 / math.sqrt(w.d), out, lse, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return k_mix, v_mix, out, lse


HSMALL = SMALL + [
    (wl.custom("hy_win100", [64 * 7 + 5, 129], 8, 2, 128, 85, "boundary"), 0.05, 100),
    (wl.custom("hy_win300_d64", [900, 3], 4, 2, 64, 86, "boundary"), 0.1, 300),
    (wl.custom("hy_win64_g8", [64 * 6], 8, 1, 128, 87, "boundary"), 0.05, 64),
    # rows of one warp that meet their first keys in different entries (window edges)
    (wl.custom("hy_win200", [64 * 7 + 5, 129], 8, 2, 128, 85, "boundary"), 0.05, 200),
    (wl.custom("hy_win1", [64 * 5 + 9, 70], 4, 2, 128, 88, "boundary"), 0.0, 1),
]


@pytest.mark.parametrize("w,frac,window", HSMALL, ids=lambda x: getattr(x, "name", str(x)))
def test_hybrid_prefill_matches_oracle(w, frac, window):
    """Every row against the oracle (selection from the oracle, which the selection test
    shows is the GPU's), and the mixed operands bit for bit: a selected token's bf16
    row, else its INT4 codes from the oracle's quantiser as bf16 integers."""
    c = HybridCase(w, frac, window, seed=9, need_q=True)
    k_mix, v_mix, out, lse = _run_hybrid_prefill(c)
    cu = w.cu_seqlens
    kv = oracle.Quantised(None, c.kb, c.vb, cu)
    sel = c.sel[:, :, None]
    want_k = np.where(sel, c.kb, _bf16_of_ints(_tiles_to_tokens(_codes4(kv.k4), cu)))
    want_v = np.where(sel, c.vb, _bf16_of_ints(_tiles_to_tokens(_codes4(kv.v4), cu)))
    assert np.array_equal(wl.bf16_bits(k_mix), want_k)
    assert np.array_equal(wl.bf16_bits(v_mix), want_v)
    ref, ref_lse = oracle.hybrid_prefill(wl.bf16_bits(c.q), c.kb, c.vb, cu, kv, c.sel, window,
                                         with_lse=True)
    _assert_close(out.float().cpu().numpy(), ref, w.name)
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) <= LSE_TOL


def test_hybrid_prefill_plan_end_to_end():
    """HybridPrefillPlan (quantise K/V, select, attend) equals the calls made one by one."""
    w, frac, window = HSMALL[0]
    c = HybridCase(w, frac, window, seed=9, need_q=True)
    _, _, out_ref, _ = _run_hybrid_prefill(c, with_lse=False)
    plan = api.HybridPrefillPlan(c.shape, frac, window)
    out = torch.zeros_like(out_ref)
    plan.run(c.q, c.k, c.v, torch.from_numpy(c.imp).cuda(), out)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


def test_hybrid_prefill_full_size_sampled():
    """32K context, 32/8 heads, d 128, 5% selected, 128-token window (the benchmarked
    hybrid prefill): sampled rows around tile and window edges against the oracle."""
    w = wl.bitmask_32k()
    c = HybridCase(w, 0.05, 128, seed=10, gen_device="cuda", need_q=True)
    _, _, out, lse = _run_hybrid_prefill(c)
    rows = np.array([0, 1, 63, 64, 127, 128, 129, 191, 192, 255, 1000, 4095, 4096, 16383,
                     20000, 32766, 32767])
    kv = oracle.Quantised(None, c.kb, c.vb, w.cu_seqlens)
    ref, ref_lse = oracle.hybrid_prefill(wl.bf16_bits(c.q), c.kb, c.vb, w.cu_seqlens, kv, c.sel,
                                         128, rows=rows, with_lse=True)
    _assert_close(out.float().cpu().numpy()[rows], ref[rows], "hybrid prefill 32K")
    assert np.max(np.abs(lse.cpu().numpy()[:, rows] - ref_lse[:, rows])) <= LSE_TOL
