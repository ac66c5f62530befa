"""GPU parity of the FP8 (E4M3) middle band of a boundary policy: b1 <= dist < b8 scores on
FP8 codes (a third boundary between the INT8 and INT4 regions; the pages have no FP8 tier).

Codes, scales and traversal lists bit-exact against the oracle; prefill outputs within the
output tolerance of the other GPU parity tests (same helpers); the decode cache keeps a band
tile as INT8; FP8 tiles (fp32 accumulators) are not part of the integer dump.
"""
import numpy as np
import pytest
import torch

import oracle
import tile_routed_mixed_causal_b200 as tra
from tile_routed_mixed_causal_b200 import api
from tile_routed_mixed_causal_b200 import workloads as wl

from test_gpu_parity import _compare_rows, _sampled_rows, to_np_u32

pytestmark = pytest.mark.gpu


class F8Case:
    def __init__(self, w, b8, gen_device="cpu"):
        self.w, self.b8 = w, np.asarray(b8, np.int32)
        t = wl.make_inputs(w, gen_device)
        self.q, self.k, self.v = (t[n].cuda() for n in ("q", "k", "v"))
        self.qb, self.kb, self.vb = (wl.bf16_bits(t[n]) for n in ("q", "k", "v"))
        self.shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
        self.policy = tra.Policy.boundary(w.b1, w.b2, b8=self.b8)

    def oracle_lists(self):
        return oracle.lists_boundary(self.w.cu_seqlens, self.w.b1, self.w.b2, b8=self.b8)


CASES = [
    (wl.custom("f8_d64_ragged", [130, 64, 1, 200, 577], 4, 2, 64, 71, "boundary",
               b1=[1, 2, 1, 3], b2=[4, 6, 4, 9]), [3, 2, 4, 5]),
    (wl.custom("f8_d128_gqa4", [2049, 640], 8, 2, 128, 72, "boundary",
               b1=[1, 2, 3, 4, 1, 1, 2, 8], b2=[3, 5, 9, 30, 1, 20, 4, 8]),
     [2, 5, 9, 4, 1, 9, 3, 8]),
    # every off-diagonal tile FP8, no INT4 region
    (wl.custom("f8_d128_all", [1000], 2, 2, 128, 73, "boundary", b1=[1, 1], b2=[16, 16]),
     [16, 16]),
]


def _run(c, with_lse=True):
    plan = api.PrefillPlan(c.shape, c.policy)
    out = torch.zeros_like(c.q)
    lse = torch.zeros((c.w.Hq, c.w.ntok), dtype=torch.float32, device="cuda") if with_lse else None
    plan.run(c.q, c.k, c.v, out, lse)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    return plan, out, lse


@pytest.mark.parametrize("w,b8", CASES, ids=lambda x: getattr(x, "name", ""))
def test_fp8_codes_scales_and_lists_bit_exact(w, b8):
    c = F8Case(w, b8)
    qt = tra.QTiles(c.shape, tra.FMT_Q8F | tra.FMT_K8F)
    tra.quantize_qkv_tiles(c.shape, c.q, c.k, None, qt)
    torch.cuda.synchronize()
    for name, bits in (("q", c.qb), ("k", c.kb)):
        codes, scales = oracle.quantize_f8(bits, w.cu_seqlens)
        assert np.array_equal(qt[name + "8f"].cpu().numpy(), codes), name
        assert np.array_equal(qt["s" + name + "f"].cpu().numpy().view(np.uint32),
                              scales.view(np.uint32)), name
    plan = api.PrefillPlan(c.shape, c.policy)
    plan.lists()
    dp = api.DecodePlan(c.shape, c.policy, None, 4)
    dp.build()
    torch.cuda.synchronize()
    rp, en = c.oracle_lists()
    assert np.array_equal(plan.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(plan.entries)[:plan.nnz], en)
    drp, den = oracle.lists_decode(w.cu_seqlens, w.Hq, w.Hkv, w.b1, w.b2, b8=c.b8)
    assert np.array_equal(dp.row_ptr.cpu().numpy(), drp)
    assert np.array_equal(to_np_u32(dp.entries)[:dp.nnz], den)


@pytest.mark.parametrize("w,b8", CASES, ids=lambda x: getattr(x, "name", ""))
def test_fp8_prefill_matches_oracle(w, b8):
    c = F8Case(w, b8)
    plan, out, lse = _run(c)
    rp, en = c.oracle_lists()
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens, want_f8=True)
    rows = np.arange(len(rp) - 1)
    ref, ref_lse = oracle.prefill_rows(c.qb, c.kb, c.vb, w.cu_seqlens, qz, rp, en, rows)
    _compare_rows(c, rows, ref, ref_lse, out, lse, w.name)


def test_fp8_band_equal_b1_is_the_boundary_prefill():
    """b8 = b1 (an empty band) runs the plain boundary kernel: output bit-identical."""
    w, _ = CASES[1]
    c = F8Case(w, w.b1)
    _, out_band, _ = _run(c, with_lse=False)
    plain = api.PrefillPlan(c.shape, tra.Policy.boundary(w.b1, w.b2))
    out = torch.zeros_like(c.q)
    plain.run(c.q, c.k, c.v, out)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out_band.view(torch.int16))


def test_fp8_tiles_are_not_dumped():
    """The integer dump covers INT8 / INT4 tiles; an FP8 tile's slot is left as it was."""
    w, b8 = CASES[2]
    c = F8Case(w, b8)
    plan = api.PrefillPlan(c.shape, c.policy)
    plan.quantize(c.q, c.k, c.v)
    plan.lists()
    dc = torch.tensor([[0, 0, 5, 3], [0, 0, 5, 5]], dtype=torch.int32, device="cuda")  # FP8, INT8
    dump = torch.full((2, 64, 64), -7, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(c.q)
    plan.attend(c.q, c.k, c.v, out, dump_coords=dc, dump_out=dump)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    d = dump.cpu().numpy()
    assert (d[0] == -7).all()
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens)
    assert np.array_equal(d[1], oracle.int_tile(oracle.INT8, q8t=qz.q8[0, 5], k8t=qz.k8[0, 5]))


def test_fp8_full_size_sampled():
    """The Llama-3-8B-shaped 8K workload with an FP8 band halfway between each head's b1
    and b2 (the benchmarked FP8 record): sampled rows, lists and codes in full."""
    w = wl.llama8b_8k()
    b8 = (w.b1 + w.b2) // 2
    c = F8Case(w, b8, gen_device="cuda")
    plan, out, lse = _run(c)
    rp, en = c.oracle_lists()
    assert np.array_equal(plan.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(plan.entries)[:plan.nnz], en)
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens, want_f8=True)
    assert np.array_equal(plan.tiles["q8f"].cpu().numpy(), qz.qf)
    assert np.array_equal(plan.tiles["k8f"].cpu().numpy(), qz.kf)
    rows = _sampled_rows(w, [0, 13, 31], lambda nt: [0, 1, 7, 64, nt - 2, nt - 1])
    ref, ref_lse = oracle.prefill_rows(c.qb, c.kb, c.vb, w.cu_seqlens, qz, rp, en, rows)
    _compare_rows(c, rows, ref, ref_lse, out, lse, "llama8b_8k fp8 band")
