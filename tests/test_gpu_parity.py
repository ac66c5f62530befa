"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle.

Integer work (codes, scales, traversal lists, integer QK accumulators) must be
bit-exact.  Floating outputs must satisfy, element by element,
    max(|o_gpu - o_ref| - ulp_bf16(o_ref) / 2) <= 1e-2   and   mean |o_gpu - o_ref| <= 1e-3,
i.e. a 1e-2 max / 1e-3 mean budget on top of the unavoidable rounding of the
bf16 output.
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


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    excess = float(np.max(err - half_ulp_bf16(ref)))
    mean = float(np.mean(err))
    assert excess <= MAX_TOL and mean <= MEAN_TOL, \
        f"{what}: max excess {excess:.3e} (raw max {err.max():.3e}), mean {mean:.3e}"
    return float(err.max()), mean


def to_np_u32(t):
    return t.cpu().numpy().view(np.uint32)


def v4_rowmajor(x):
    """The V4 cache is stored in the decode kernel's fragment order: in every 16-byte
    group m of a row, byte 2g + e holds the row-major byte 16m + 8e + g.  Undo that
    (an index permutation only) so that the codes compare with the oracle's."""
    nb = x.shape[-1]
    src = np.empty(nb, np.int64)
    for m in range(nb // 16):
        for e in range(2):
            for g in range(8):
                src[16 * m + 8 * e + g] = 16 * m + 2 * g + e
    return x[..., src]


class Case:
    """A workload materialised on the GPU plus its host copies for the oracle."""

    def __init__(self, w: wl.Workload, gen_device="cpu"):
        self.w = w
        t = wl.make_inputs(w, gen_device)
        self.q, self.k, self.v = (t[n].cuda() for n in ("q", "k", "v"))
        self.qb, self.kb, self.vb = (wl.bf16_bits(t[n]) for n in ("q", "k", "v"))
        self.shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
        if w.mode == "boundary":
            self.policy = tra.Policy.boundary(w.b1, w.b2)
        elif w.mode == "mixed":
            self.bitmask = torch.from_numpy(w.bitmask.view(np.int32)).cuda()
            self.policy = tra.Policy.mixed(w.b1, w.b2, self.bitmask, w.G)
        else:
            self.bitmask = torch.from_numpy(w.bitmask.view(np.int32)).cuda()
            self.policy = tra.Policy.from_bitmask(self.bitmask, w.G)

    def oracle_lists(self):
        if self.w.mode == "boundary":
            return oracle.lists_boundary(self.w.cu_seqlens, self.w.b1, self.w.b2)
        if self.w.mode == "mixed":
            return oracle.lists_mixed(self.w.cu_seqlens, self.w.b1, self.w.b2, self.w.bitmask,
                                      self.w.G)
        return oracle.lists_bitmask(self.w.cu_seqlens, self.w.bitmask, self.w.G)


SMALL = [
    wl.tiny(),
    wl.custom("b_d64_gqa_ragged", [130, 64, 1, 200, 577], 4, 2, 64, 31, "boundary"),
    wl.custom("b_d128_local", [1000], 2, 2, 128, 32, "boundary", b1=[1, 1], b2=[1, 1]),
    wl.custom("b_d128_all8", [700, 300], 2, 1, 128, 33, "boundary", b1=[12, 3], b2=[12, 9]),
    wl.custom("b_d128_gqa4", [2049, 640], 8, 2, 128, 34, "boundary",
              b1=[1, 2, 3, 4, 1, 1, 2, 8], b2=[3, 2, 9, 30, 1, 20, 4, 8]),
    wl.custom("m_d128_g1", [900, 65, 300], 8, 2, 128, 35, "bitmask", G=1, p_bf16=0.3),
    wl.custom("m_d64_g3", [1500], 2, 2, 64, 36, "bitmask", G=3, p_bf16=0.5),
    wl.custom("m_d128_allbf16", [513], 4, 4, 128, 37, "bitmask", G=2, p_bf16=1.0),
    wl.custom("m_d128_all8", [777], 4, 2, 128, 38, "bitmask", G=4, p_bf16=0.0),
    # four-way: boundaries (skip / INT4 / INT8) with a bitmask promoting kept tiles to BF16
    wl.custom("x_d128_gqa4", [1500, 300, 64], 8, 2, 128, 60, "mixed",
              b1=[1, 2, 3, 1, 4, 1, 2, 8], b2=[3, 5, 9, 30, 4, 1, 20, 8], G=2, p_bf16=0.3),
    wl.custom("x_d64_ragged", [900, 65, 1], 4, 4, 64, 61, "mixed", G=3, p_bf16=0.5),
]


def _run_prefill(c: Case, with_lse=True):
    plan = api.PrefillPlan(c.shape, c.policy)
    out = torch.zeros_like(c.q)
    lse = torch.zeros((c.w.Hq, c.w.ntok), dtype=torch.float32, device="cuda") if with_lse else None
    plan.run(c.q, c.k, c.v, out, lse)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    return plan, out, lse


# ---------------------------------------------------------------- quantiser
@pytest.mark.parametrize("w", SMALL[:5], ids=lambda w: w.name)
def test_quantize_bit_exact(w):
    c = Case(w)
    qt = tra.QTiles(c.shape, 0xFF)
    tra.quantize_qkv_tiles(c.shape, c.q, c.k, c.v, qt)
    torch.cuda.synchronize()
    for name, bits in (("q", c.qb), ("k", c.kb), ("v", c.vb)):
        x8, x4, s8, s4 = oracle.quantize(bits, w.cu_seqlens)
        if name != "v":  # INT4 codes in the int8 operand form: 16 x the signed code
            nib = np.stack([x4 & 0xF, x4 >> 4], -1).reshape(*x4.shape[:-1], -1).astype(np.int16)
            codes = np.where(nib >= 8, nib - 16, nib)
            assert np.array_equal(qt[name + "4x"].cpu().numpy().astype(np.int16), 16 * codes), name + "4x"
        got8 = qt[name + "8"].cpu().numpy()
        if name == "v":  # V8 is stored offset-binary: code + 128
            got8 = (got8.view(np.uint8) ^ 0x80).view(np.int8)
        assert np.array_equal(got8, x8), name + "8"
        got4 = qt[name + "4"].cpu().numpy()
        assert np.array_equal(v4_rowmajor(got4) if name == "v" else got4, x4), name + "4"
        assert np.array_equal(qt["s" + name + "8"].cpu().numpy().view(np.uint32), s8.view(np.uint32))
        assert np.array_equal(qt["s" + name + "4"].cpu().numpy().view(np.uint32), s4.view(np.uint32))


def test_quantize_edge_values():
    """Zero tiles, ties, tiny and huge magnitudes, a partial tile."""
    w = wl.custom("edge", [64, 70, 3], 2, 2, 128, 40, "boundary")
    c = Case(w)
    x = c.q.float()
    x[0:64, 0] = 0.0                                     # all-zero tile
    x[64:128, 1] = torch.linspace(-7, 7, 64 * 128, device="cuda").view(64, 128)
    x[128:134, 0] *= 1e-30                               # denormal-range products
    x[134:137, 1] *= 3e4
    q = x.to(torch.bfloat16)
    qt = tra.QTiles(c.shape, tra.FMT_Q8 | tra.FMT_Q4)
    tra.quantize_qkv_tiles(c.shape, q, None, None, qt)
    torch.cuda.synchronize()
    x8, x4, s8, s4 = oracle.quantize(wl.bf16_bits(q), w.cu_seqlens)
    assert np.array_equal(qt["q8"].cpu().numpy(), x8)
    assert np.array_equal(qt["q4"].cpu().numpy(), x4)
    assert np.array_equal(qt["sq8"].cpu().numpy(), s8)
    assert np.array_equal(qt["sq4"].cpu().numpy(), s4)


# ---------------------------------------------------------------- traversal lists
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_lists_bit_exact(w):
    c = Case(w)
    plan = api.PrefillPlan(c.shape, c.policy)
    plan.lists()
    torch.cuda.synchronize()
    rp, en = c.oracle_lists()
    assert np.array_equal(plan.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(plan.entries)[:plan.nnz], en)
    # decode caches follow the boundaries; a bitmask-only policy caches every tile in INT8
    dp = api.DecodePlan(c.shape, c.policy, None, 4)
    dp.build()
    torch.cuda.synchronize()
    if w.mode in ("boundary", "mixed"):
        rp, en = oracle.lists_decode(w.cu_seqlens, w.Hq, w.Hkv, w.b1, w.b2)
    else:
        rp, en = oracle.lists_decode(w.cu_seqlens, w.Hq, w.Hkv)
    assert np.array_equal(dp.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(dp.entries)[:dp.nnz], en)


# ---------------------------------------------------------------- prefill
def _oracle_full(c: Case):
    rp, en = c.oracle_lists()
    qz = oracle.Quantised(c.qb, c.kb, None, c.w.cu_seqlens)
    rows = np.arange(len(rp) - 1)
    out, lse = oracle.prefill_rows(c.qb, c.kb, c.vb, c.w.cu_seqlens, qz, rp, en, rows)
    return qz, rows, out, lse


def _compare_rows(c: Case, rows, ref_out, ref_lse, gpu_out, gpu_lse, what):
    w = c.w
    cu = np.asarray(w.cu_seqlens, np.int64)
    nts = [(int(cu[b + 1] - cu[b]) + 63) // 64 for b in range(w.B)]
    off = np.concatenate([[0], np.cumsum(nts)])
    got, ref, gl, rl = [], [], [], []
    go = gpu_out.float().cpu().numpy()
    glse = gpu_lse.cpu().numpy() if gpu_lse is not None else None
    for i, row in enumerate(rows):
        h, gq = divmod(int(row), int(off[-1]))
        b = int(np.searchsorted(off, gq, side="right") - 1)
        qt = gq - off[b]
        T = int(cu[b + 1] - cu[b])
        n = min(64, T - qt * 64)
        toks = cu[b] + qt * 64 + np.arange(n)
        got.append(go[toks, h])
        ref.append(ref_out[i, :n])
        if glse is not None:
            gl.append(glse[h, toks])
            rl.append(ref_lse[i, :n])
    res = assert_close(np.concatenate(got), np.concatenate(ref), what)
    if glse is not None:
        # l is summed from the bf16-rounded P the MMA consumes (relative error <= 2^-9 per
        # term), so log(l) may differ from the exact fp64 value by up to about 2^-9.
        assert np.max(np.abs(np.concatenate(gl) - np.concatenate(rl))) < 2.0 ** -8, what + " lse"
    return res


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_prefill_matches_oracle(w):
    c = Case(w)
    plan, out, lse = _run_prefill(c)
    _, rows, ref, ref_lse = _oracle_full(c)
    _compare_rows(c, rows, ref, ref_lse, out, lse, w.name)


def test_prefill_integer_accumulator_dump():
    """Every INT8/INT4 tile of the tiny configuration: raw int32 Q-code K-code^T, bit-exact."""
    w = wl.tiny()
    c = Case(w)
    plan = api.PrefillPlan(c.shape, c.policy)
    plan.quantize(c.q, c.k, c.v)
    plan.lists()
    rp, en = c.oracle_lists()
    coords = []
    for h in range(w.Hq):
        for qt in range(4):
            row = h * 4 + qt
            for e in en[rp[row]:rp[row + 1]]:
                coords.append((0, h, qt, int(e & 0x0FFFFFFF), int(e >> 28)))
    dc = torch.tensor([x[:4] for x in coords], dtype=torch.int32, device="cuda")
    dump = torch.full((len(coords), 64, 64), -7, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(c.q)
    plan.attend(c.q, c.k, c.v, out, dump_coords=dc, dump_out=dump)
    torch.cuda.synchronize()
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens)
    for i, (_, h, qt, kt, prec) in enumerate(coords):
        if prec == oracle.INT8:
            ref = oracle.int_tile(prec, q8t=qz.q8[h, qt], k8t=qz.k8[h, kt])
        else:
            ref = oracle.int_tile(prec, q4t=qz.q4[h, qt], k4t=qz.k4[h, kt])
        assert np.array_equal(dump[i].cpu().numpy(), ref), (h, qt, kt, prec)


def _dump_coords(c: Case, rows_hq, per_prec=6, limit=64):
    """Dump coordinates (b, h, qt, kt) for integer tiles of the oracle's lists at the given
    (h, b, qt) rows: up to per_prec INT8 and per_prec INT4 entries per row (first, last and
    evenly spread between), at most `limit` in all."""
    w = c.w
    rp, en = c.oracle_lists()
    off = np.concatenate([[0], np.cumsum(w.tiles_per_seq)])
    coords = []
    for h, b, qt in rows_hq:
        row = h * int(off[-1]) + int(off[b]) + qt
        ent = en[rp[row]:rp[row + 1]]
        for prec in (oracle.INT8, oracle.INT4):
            sel = ent[(ent >> 28) == prec]
            if len(sel) == 0:
                continue
            idx = np.unique(np.linspace(0, len(sel) - 1, min(per_prec, len(sel))).astype(int))
            for i in idx:
                coords.append((b, h, qt, int(sel[i] & 0x0FFFFFFF), prec))
    return coords[:limit]


def _check_dump(c: Case, coords, gen_device="cpu"):
    """Run the prefill with an integer dump of `coords`; every dumped tile must equal the
    oracle's own int32 Q-code x K-code^T product bit for bit."""
    w = c.w
    plan = api.PrefillPlan(c.shape, c.policy)
    plan.quantize(c.q, c.k, c.v)
    plan.lists()
    dc = torch.tensor([x[:4] for x in coords], dtype=torch.int32, device="cuda")
    dump = torch.full((len(coords), 64, 64), -7, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(c.q)
    plan.attend(c.q, c.k, c.v, out, dump_coords=dc, dump_out=dump)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens)
    off = np.concatenate([[0], np.cumsum(w.tiles_per_seq)])
    got = dump.cpu().numpy()
    for i, (b, h, qt, kt, prec) in enumerate(coords):
        gq, gk = int(off[b]) + qt, int(off[b]) + kt
        kvh = h // (w.Hq // w.Hkv)
        if prec == oracle.INT8:
            ref = oracle.int_tile(prec, q8t=qz.q8[h, gq], k8t=qz.k8[kvh, gk])
        else:
            ref = oracle.int_tile(prec, q4t=qz.q4[h, gq], k4t=qz.k4[kvh, gk])
        # rows past the sequence end hold no query: the kernel writes only valid rows
        n = min(64, w.lengths[b] - qt * 64)
        assert np.array_equal(got[i, :n], ref[:n]), (b, h, qt, kt, prec)
    return out


DUMP_FULL = {
    # d = 128 at full size: INT8 and INT4 tiles (128-byte swizzle, INT4 as 16 x code)
    "llama8b_8k": (wl.llama8b_8k, [(0, 0, 127), (13, 0, 64), (31, 0, 9), (7, 0, 126)]),
    "bitmask_32k": (wl.bitmask_32k, [(0, 0, 511), (17, 0, 300), (31, 0, 3)]),
    "mixed_8k": (wl.mixed_8k, [(0, 0, 127), (21, 0, 70), (31, 0, 5), (9, 0, 100)]),
    "varlen": (wl.varlen_8, [(0, 0, 20), (27, 3, 5), (13, 7, 0)]),
}


@pytest.mark.parametrize("name", list(DUMP_FULL))
def test_prefill_integer_dump_full_size(name):
    """Bit-exact int32 accumulators of sampled INT8 / INT4 tiles at full size (d = 128) under
    boundary, bitmask and mixed policies, in the launch configuration the benchmark uses."""
    make, rows = DUMP_FULL[name]
    w = make()
    c = Case(w, gen_device="cuda")
    rows = [(h, b, min(qt, w.tiles_per_seq[b] - 1)) for h, b, qt in rows]
    coords = _dump_coords(c, rows)
    assert any(x[4] == oracle.INT8 for x in coords)
    if w.mode != "bitmask":
        assert any(x[4] == oracle.INT4 for x in coords)
    _check_dump(c, coords)


@pytest.mark.parametrize("w", [x for x in SMALL if x.d == 128 and x.mode != "bitmask"] +
                         [SMALL[6]], ids=lambda w: w.name)
def test_prefill_integer_dump_small(w):
    """Every integer tile of a few rows of the small d = 128 (and a d = 64 bitmask) cases."""
    c = Case(w)
    rows = []
    for h in range(min(w.Hq, 4)):
        for b, nt in enumerate(w.tiles_per_seq):
            rows.append((h, b, nt - 1))
    coords = _dump_coords(c, rows, per_prec=3)
    if coords:
        _check_dump(c, coords)


def _sampled_rows(w, heads, qtiles_per_seq):
    nts = w.tiles_per_seq
    off = np.concatenate([[0], np.cumsum(nts)])
    rows = []
    for h in heads:
        for b, nt in enumerate(nts):
            for qt in qtiles_per_seq(nt):
                rows.append(h * off[-1] + off[b] + qt)
    return np.array(rows, np.int64)


FULL = {
    "llama8b_8k": (wl.llama8b_8k, [0, 13, 31], lambda nt: [0, 1, 7, 64, nt - 2, nt - 1]),
    "bitmask_32k": (wl.bitmask_32k, [0, 17, 31], lambda nt: [0, 3, 255, nt - 1]),
    "varlen": (wl.varlen_8, [0, 27], lambda nt: [0, nt // 2, nt - 1]),
    "mixed_8k": (wl.mixed_8k, [0, 21, 31], lambda nt: [0, 2, 64, nt - 1]),
}


@pytest.mark.parametrize("name", list(FULL))
def test_prefill_full_size_sampled(name):
    """Full-size configurations, same launch as the benchmark, sampled rows vs the oracle."""
    make, heads, qts = FULL[name]
    w = make()
    c = Case(w, gen_device="cuda")
    plan, out, lse = _run_prefill(c)
    rows = _sampled_rows(w, heads, qts)
    rp, en = c.oracle_lists()
    # traversal lists are checked in full at this size too
    assert np.array_equal(plan.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(plan.entries)[:plan.nnz], en)
    qz = oracle.Quantised(c.qb, c.kb, None, w.cu_seqlens)
    assert np.array_equal(plan.tiles["q8"].cpu().numpy(), qz.q8)
    assert np.array_equal(plan.tiles["k8"].cpu().numpy(), qz.k8)
    ref, ref_lse = oracle.prefill_rows(c.qb, c.kb, c.vb, w.cu_seqlens, qz, rp, en, rows)
    _compare_rows(c, rows, ref, ref_lse, out, lse, name)


# ---------------------------------------------------------------- decode
def _decode_case(w, gen_device="cpu"):
    c = Case(w, gen_device)
    fm = tra.FMT_K8 | tra.FMT_K4 | tra.FMT_V8 | tra.FMT_V4
    cache = tra.QTiles(c.shape, fm)
    tra.quantize_qkv_tiles(c.shape, None, c.k, c.v, cache)
    dp = api.DecodePlan(c.shape, c.policy, cache, w.tail_cap)
    dp.build()
    qs, kn, vn = wl.make_decode_inputs(w, gen_device)
    return c, cache, dp, qs.cuda(), kn.cuda(), vn.cuda()


DEC = [
    wl.custom("dec_small", [64 * 6 + 10, 64 * 3, 1], 4, 2, 64, 50, "boundary",
              b1=[1, 2, 1, 1], b2=[2, 4, 3, 1], decode_steps=5, tail_cap=8),
    wl.custom("dec_d128_g4", [64 * 40, 64 * 33 + 17], 8, 2, 128, 51, "boundary",
              b1=[3, 1, 9, 2, 1, 1, 4, 2], b2=[20, 5, 9, 30, 1, 2, 4, 16], decode_steps=4,
              tail_cap=70),
    wl.custom("dec_d128_mha", [64 * 20], 2, 2, 128, 52, "boundary", b1=[1, 2], b2=[1, 2],
              decode_steps=3, tail_cap=3),
]


@pytest.mark.parametrize("w", DEC, ids=lambda w: w.name)
def test_decode_matches_oracle(w):
    c, cache, dp, qs, kn, vn = _decode_case(w)
    cu = w.cu_seqlens
    ocache = oracle.Quantised(None, c.kb, c.vb, cu)
    rp, en = oracle.lists_decode(cu, w.Hq, w.Hkv, w.b1, w.b2)
    kt = np.zeros((w.B, w.Hkv, w.tail_cap, w.d), np.uint16)
    vt = np.zeros_like(kt)
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    for step in range(w.decode_steps):
        dp.step(qs[step], kn[step], vn[step], out)
        torch.cuda.synchronize()
        kt[:, :, step] = wl.bf16_bits(kn[step])
        vt[:, :, step] = wl.bf16_bits(vn[step])
        ref = oracle.decode_step(wl.bf16_bits(qs[step]), cu, w.Hkv, ocache, rp, en, kt, vt,
                                 np.full(w.B, step + 1, np.int32))
        assert_close(out.float().cpu().numpy(), ref, f"{w.name} step {step}")
    assert int(dp.status.item()) == 0
    assert np.array_equal(dp.tail_len.cpu().numpy(), np.full(w.B, w.decode_steps))
    assert np.array_equal(wl.bf16_bits(dp.k_tail[:, :, :w.decode_steps]), kt[:, :, :w.decode_steps])


def _decode_vs_oracle(w, c, dp, qs, kn, vn, steps, cu_lists=None):
    """Run `steps` decode steps and compare each with the oracle (full batch)."""
    cu = w.cu_seqlens
    ocache = oracle.Quantised(None, c.kb, c.vb, cu)
    if w.mode == "bitmask":
        rp, en = oracle.lists_decode(cu, w.Hq, w.Hkv)
    else:
        rp, en = oracle.lists_decode(cu, w.Hq, w.Hkv, w.b1, w.b2)
    assert np.array_equal(dp.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(to_np_u32(dp.entries)[:dp.nnz], en)
    kt = np.zeros((w.B, w.Hkv, w.tail_cap, w.d), np.uint16)
    vt = np.zeros_like(kt)
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    for step in range(steps):
        dp.step(qs[step], kn[step], vn[step], out)
        torch.cuda.synchronize()
        kt[:, :, step] = wl.bf16_bits(kn[step])
        vt[:, :, step] = wl.bf16_bits(vn[step])
        ref = oracle.decode_step(wl.bf16_bits(qs[step]), cu, w.Hkv, ocache, rp, en, kt, vt,
                                 np.full(w.B, step + 1, np.int32))
        assert_close(out.float().cpu().numpy(), ref, f"{w.name} step {step}")
    assert int(dp.status.item()) == 0


def test_decode_after_bitmask_prefill():
    """TileMix's INT8 K/V cache: a bitmask-policy prefill quantises K/V; its decode-cache
    lists hold every tile in INT8 (no b1/b2); decode steps over that cache vs the oracle."""
    w = wl.custom("bm_prefill_decode", [64 * 21 + 7, 64 * 9, 64 * 4], 8, 2, 128, 70, "bitmask",
                  G=4, p_bf16=0.25, decode_steps=3, tail_cap=5)
    c = Case(w)
    plan = api.PrefillPlan(c.shape, c.policy, keep_v_cache=True)
    out = torch.zeros_like(c.q)
    plan.run(c.q, c.k, c.v, out)
    dp = api.DecodePlan(c.shape, c.policy, plan.tiles, w.tail_cap)
    dp.build()
    qs, kn, vn = (x.cuda() for x in wl.make_decode_inputs(w, "cpu"))
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    _decode_vs_oracle(w, c, dp, qs, kn, vn, w.decode_steps)


@pytest.mark.parametrize("where", ["every_head", "one_group"])
def test_decode_query_high_dynamic_range(where):
    """Queries whose channels span far more than 2^7 within a head: per head one channel
    x 1e3 (or x 30) and several x 1e-3.  The decode must still follow the bf16 query
    within the output tolerance.  one_group: only the heads of (sequence 0, KV head 0)
    get such a query, so that one step mixes groups of small and large queries."""
    w = wl.custom("dec_hdr", [64 * 40, 64 * 33 + 17], 8, 2, 128, 71, "boundary",
                  b1=[3, 1, 9, 2, 1, 1, 4, 2], b2=[20, 5, 9, 30, 1, 2, 4, 16], decode_steps=3,
                  tail_cap=4)
    c, cache, dp, qs, kn, vn = _decode_case(w)
    g = torch.Generator().manual_seed(123)
    q = qs.float().cpu()
    grp = w.Hq // w.Hkv
    for h in range(w.Hq):
        ch = torch.randperm(w.d, generator=g)[:7]
        bs = slice(None) if where == "every_head" else slice(0, 1)
        if where == "one_group" and h >= grp:
            continue
        q[:, bs, h, ch[0]] *= 1e3 if h % 2 == 0 else 30.0
        q[:, bs, h, ch[1:]] *= 1e-3
    qs = q.to(torch.bfloat16).cuda()
    _decode_vs_oracle(w, c, dp, qs, kn, vn, w.decode_steps)
    assert np.array_equal(dp.tail_len.cpu().numpy(), np.full(w.B, w.decode_steps))


def test_decode_workspace_shared_across_shapes():
    """The decode's arrival counters sit at a fixed place of the workspace and every call
    leaves them at zero, so one zero-filled workspace serves two shapes in turn: steps of
    both, interleaved on it, match steps on separate workspaces bit for bit."""
    runs = {}
    for w in DEC[:2]:
        own = _decode_case(w)
        shared = _decode_case(w)
        runs[w.name] = (w, own, shared)
    nbytes = max(r[2][2].workspace.numel() for r in runs.values())
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for _, (_, _, sh) in runs.items():
        sh[2].workspace = ws
    steps = min(w.decode_steps for w, _, _ in runs.values())
    for step in range(steps):
        for name, (w, own, sh) in runs.items():
            outs = []
            for c, cache, dp, qs, kn, vn in (own, sh):
                out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
                dp.step(qs[step], kn[step], vn[step], out)
                outs.append(out)
            torch.cuda.synchronize()
            assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), (name, step)
    for _, (_, own, sh) in runs.items():
        assert int(own[2].status.item()) == 0 and int(sh[2].status.item()) == 0
    assert int(ws[:4 * 16384].count_nonzero().item()) == 0   # counters back at zero


def test_decode_tail_full_sets_status():
    w = wl.custom("dec_full", [128], 2, 1, 64, 53, "boundary", b1=[1, 1], b2=[2, 2],
                  decode_steps=2, tail_cap=1)
    c, cache, dp, qs, kn, vn = _decode_case(w)
    out = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda")
    dp.step(qs[0], kn[0], vn[0], out)
    torch.cuda.synchronize()
    first = out.clone()
    assert int(dp.status.item()) == 0 and int(dp.tail_len.item()) == 1
    dp.step(qs[1], kn[1], vn[1], out)
    torch.cuda.synchronize()
    assert int(dp.status.item()) & tra.DEV_TAIL_FULL
    assert int(dp.tail_len.item()) == 1
    assert torch.equal(out, first)


@pytest.mark.parametrize("literal", [False, True], ids=["headline", "literal_1_3"])
def test_decode_full_size_sampled(literal):
    """Batch 16 over a 32K prefix, 64 steps as benchmarked; sampled sequences vs the oracle.
    literal: the cache of the (b1, b2) = (1, 3) rule for every head (INT8 tile 511, INT4
    tiles 509-510 of each sequence); headline: the per-head HBM-sized cache."""
    w = wl.decode_32k(literal=literal)
    c, cache, dp, qs, kn, vn = _decode_case(w, gen_device="cuda")
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    check_steps = {0, 31, 63}
    sample_b = [0, 9, 15]
    outs = {}
    for step in range(w.decode_steps):
        dp.step(qs[step], kn[step], vn[step], out)
        if step in check_steps:
            outs[step] = out.float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(dp.status.item()) == 0
    T = w.lengths[0]
    for b in sample_b:
        cu1 = np.array([0, T], np.int32)
        kb = wl.bf16_bits(c.k[b * T:(b + 1) * T])
        vb = wl.bf16_bits(c.v[b * T:(b + 1) * T])
        ocache = oracle.Quantised(None, kb, vb, cu1)
        rp, en = oracle.lists_decode(cu1, w.Hq, w.Hkv, w.b1, w.b2)
        for step in sorted(check_steps):
            kt = wl.bf16_bits(kn[:step + 1, b]).transpose(1, 0, 2)[None]
            vt = wl.bf16_bits(vn[:step + 1, b]).transpose(1, 0, 2)[None]
            ref = oracle.decode_step(wl.bf16_bits(qs[step, b:b + 1]), cu1, w.Hkv, ocache, rp, en,
                                     np.ascontiguousarray(kt), np.ascontiguousarray(vt),
                                     np.array([step + 1], np.int32))
            assert_close(outs[step][b], ref[0], f"decode b={b} step={step}")
