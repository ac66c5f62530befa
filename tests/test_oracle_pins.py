"""Pins for the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or mathematics fix:
hand-worked quantisation examples, closed-form list counts, textbook dense
causal softmax attention (the all-BF16 policy), block-local attention
(b1 = b2 = 1), dense attention over dequantised INT8 scores (b1 = b2 >= tiles),
a per-(query, key) brute force of the routing rule, and probability rows that
sum to one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from tile_routed_mixed_causal_b200 import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden")
T = 64


def bits_of(x: np.ndarray) -> np.ndarray:
    return wl.bf16_bits(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def val_of(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def read_golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([c.strip() for c in line.split("|")])
    return rows


# --------------------------------------------------------------------------- quantiser
@pytest.mark.parametrize("row", read_golden("quant_examples.txt"))
def test_quant_hand_examples(row):
    fmt, vals, codes, scale = row
    vals = [float(x) for x in vals.split()]
    codes = [int(x) for x in codes.split()]
    d = 64
    x = np.zeros((T, 1, d), np.float32)
    x[0, 0, :len(vals)] = vals
    x8, x4, s8, s4 = oracle.quantize(bits_of(x), [0, T])
    if fmt == "int8":
        got = x8[0, 0, 0, :len(vals)].tolist()
        s = s8[0, 0]
    else:
        c = x4[0, 0, 0]
        nib = np.stack([c & 0xF, c >> 4], -1).reshape(-1).astype(np.int32)
        got = np.where(nib >= 8, nib - 16, nib)[:len(vals)].tolist()
        s = s4[0, 0]
    assert got == codes
    if scale != "-":
        assert s == np.float32(float(scale))


@pytest.mark.parametrize("row", read_golden("int4_packing.txt"))
def test_int4_packing(row):
    pair, byte = row
    ce, co = [int(x) for x in pair.split()]
    d = 64
    x = np.zeros((T, 1, d), np.float32)
    x[0, 0, 0], x[0, 0, 1] = ce, co
    x[1, 0, 0] = 7.0          # amax 7 -> INT4 scale exactly 1
    _, x4, _, s4 = oracle.quantize(bits_of(x), [0, T])
    assert s4[0, 0] == 1.0
    assert x4[0, 0, 0, 0] == int(byte, 16)


def test_quant_invariants_random():
    """Scale = fl32(amax/qmax); |code| <= qmax; amax maps to +-qmax; |x/s - code| <= 1/2;
    padded rows and all-zero tiles give code 0; scales are per (head, tile)."""
    rng = np.random.default_rng(7)
    lengths = [100, 64, 1, 130]
    ntok, H, d = sum(lengths), 3, 64
    x = rng.standard_normal((ntok, H, d)).astype(np.float32) * rng.uniform(0.01, 50, size=(1, H, 1))
    x[100:164, 1, :] = 0.0       # an all-zero tile (sequence 1, head 1)
    bits = bits_of(x)
    xv = val_of(bits)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    x8, x4, s8, s4 = oracle.quantize(bits, cu)
    nt = oracle.num_tiles(cu)
    assert nt == sum((L + 63) // 64 for L in lengths)
    gt = 0
    for b, L in enumerate(lengths):
        for t in range((L + 63) // 64):
            for h in range(H):
                rows = xv[cu[b] + t * 64: cu[b] + min(L, t * 64 + 64), h, :]
                amax = np.float32(np.abs(rows).max())
                assert s8[h, gt] == np.float32(amax / np.float32(127.0))
                assert s4[h, gt] == np.float32(amax / np.float32(7.0))
                n = rows.shape[0]
                c8 = x8[h, gt, :n].astype(np.int64)
                nib = np.stack([x4[h, gt, :n] & 0xF, x4[h, gt, :n] >> 4], -1).reshape(n, d).astype(np.int64)
                c4 = np.where(nib >= 8, nib - 16, nib)
                assert np.all(np.abs(c8) <= 127) and np.all(np.abs(c4) <= 7)
                assert np.all(x8[h, gt, n:] == 0) and np.all(x4[h, gt, n:] == 0)
                if amax == 0:
                    assert np.all(c8 == 0) and np.all(c4 == 0)
                    continue
                assert np.abs(c8).max() == 127 and np.abs(c4).max() == 7
                r8 = rows.astype(np.float32) / s8[h, gt]
                r4 = rows.astype(np.float32) / s4[h, gt]
                assert np.all(np.abs(r8 - c8) <= 0.5 + 1e-6)
                assert np.all(np.abs(r4 - c4) <= 0.5 + 1e-6)
            gt += 1


# --------------------------------------------------------------------------- traversal lists
def _decode_entries(e):
    return (e >> 28).astype(np.int64), (e & 0x0FFFFFFF).astype(np.int64)


@pytest.mark.parametrize("lengths,b1,b2", [
    ([256], [1, 1], [3, 3]),
    ([1000, 1, 64, 65, 700], [1, 2, 3, 1], [1, 5, 3, 40]),
])
def test_lists_boundary_closed_form(lengths, b1, b2):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    rp, en = oracle.lists_boundary(cu, b1, b2)
    prec, kt = _decode_entries(en)
    nts = [(L + 63) // 64 for L in lengths]
    row = 0
    nnz = 0
    for h in range(len(b1)):
        for nt in nts:
            for qt in range(nt):
                n = min(qt + 1, b2[h])
                n8 = min(qt + 1, b1[h])
                s, e = rp[row], rp[row + 1]
                assert e - s == n
                # INT4 block first: the n - n8 tiles qt-b2+1 .. qt-b1, ascending
                assert list(prec[s:s + n - n8]) == [1] * (n - n8)
                assert list(kt[s:s + n - n8]) == list(range(qt - n + 1, qt - n8 + 1))
                # then INT8: qt-n8+1 .. qt ascending; the diagonal is last
                assert list(prec[s + n - n8:e]) == [2] * n8
                assert list(kt[s + n - n8:e]) == list(range(qt - n8 + 1, qt + 1))
                nnz += n
                row += 1
    assert rp[-1] == nnz == len(en)


def test_lists_bitmask_closed_form():
    lengths = [64 * 37, 5, 64 * 9 + 3]
    G = 3
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    nts = [(L + 63) // 64 for L in lengths]
    Hq = 2
    rng = np.random.default_rng(3)
    W = 1
    bm = rng.integers(0, 2**32, size=(Hq, sum(nts), W), dtype=np.uint64).astype(np.uint32)
    rp, en = oracle.lists_bitmask(cu, bm, G)
    prec, kt = _decode_entries(en)
    row = 0
    for h in range(Hq):
        gt = 0
        for nt in nts:
            for qt in range(nt):
                word = int(bm[h, gt + qt, 0])
                hi = [j for j in range(qt + 1) if (word >> (j // G)) & 1]
                lo = [j for j in range(qt + 1) if not (word >> (j // G)) & 1]
                s, e = rp[row], rp[row + 1]
                assert e - s == qt + 1              # dense connectivity: no skips
                assert list(kt[s:e]) == lo + hi
                assert list(prec[s:e]) == [2] * len(lo) + [3] * len(hi)
                row += 1
            gt += nt


def _mixed_case(seed=5):
    lengths = [64 * 30 + 7, 64, 64 * 11]
    G = 2
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    nts = [(L + 63) // 64 for L in lengths]
    b1 = [1, 3, 2, 5]
    b2 = [4, 3, 9, 40]
    rng = np.random.default_rng(seed)
    bm = rng.integers(0, 2**32, size=(len(b1), sum(nts), 1), dtype=np.uint64).astype(np.uint32)
    return lengths, nts, cu, b1, b2, bm, G


def test_lists_mixed_closed_form():
    """Four-way rows: kept tiles min(qt+1, b2) as in the boundary rule, each promoted to
    BF16 when its group's bit is set; INT4 block, then INT8, then BF16, each ascending."""
    lengths, nts, cu, b1, b2, bm, G = _mixed_case()
    rp, en = oracle.lists_mixed(cu, b1, b2, bm, G)
    prec, kt = _decode_entries(en)
    row = 0
    for h in range(len(b1)):
        gt = 0
        for nt in nts:
            for qt in range(nt):
                word = int(bm[h, gt + qt, 0])
                kept = range(max(0, qt - b2[h] + 1), qt + 1)
                hi = [j for j in kept if (word >> (j // G)) & 1]
                t4 = [j for j in kept if not (word >> (j // G)) & 1 and qt - j >= b1[h]]
                t8 = [j for j in kept if not (word >> (j // G)) & 1 and qt - j < b1[h]]
                s, e = rp[row], rp[row + 1]
                assert e - s == min(qt + 1, b2[h])
                assert list(kt[s:e]) == t4 + t8 + hi
                assert list(prec[s:e]) == [1] * len(t4) + [2] * len(t8) + [3] * len(hi)
                row += 1
            gt += nt
    assert rp[-1] == len(en)


def test_lists_mixed_reduces_to_each_policy():
    """No bit set: the boundary policy's lists.  b1 = b2 >= every tile count (nothing
    skipped, no INT4): the bitmask policy's lists."""
    lengths, nts, cu, b1, b2, bm, G = _mixed_case(seed=6)
    zero = np.zeros_like(bm)
    rp_m, en_m = oracle.lists_mixed(cu, b1, b2, zero, G)
    rp_b, en_b = oracle.lists_boundary(cu, b1, b2)
    assert np.array_equal(rp_m, rp_b) and np.array_equal(en_m, en_b)
    big = [max(nts)] * len(b1)
    rp_m, en_m = oracle.lists_mixed(cu, big, big, bm, G)
    rp_k, en_k = oracle.lists_bitmask(cu, bm, G)
    assert np.array_equal(rp_m, rp_k) and np.array_equal(en_m, en_k)


def test_lists_decode_closed_form():
    lengths = [64 * 20, 64 * 7 + 5]
    Hq, Hkv = 4, 2
    b1 = [2, 5, 1, 1]
    b2 = [3, 9, 1, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    rp, en = oracle.lists_decode(cu, Hq, Hkv, b1, b2)
    prec, kt = _decode_entries(en)
    row = 0
    for L in lengths:
        nt = (L + 63) // 64
        for kvh in range(Hkv):
            hs = range(kvh * 2, kvh * 2 + 2)
            B1 = max(b1[h] for h in hs)
            B2 = max(b2[h] for h in hs)
            n8 = min(nt, B1)
            n = min(nt, B2)
            s, e = rp[row], rp[row + 1]
            assert e - s == n
            assert list(kt[s:e]) == list(range(nt - n, nt - n8)) + list(range(nt - n8, nt))
            assert list(prec[s:e]) == [1] * (n - n8) + [2] * n8
            row += 1
    # bitmask mode: every prefill tile is cached as INT8
    rp, en = oracle.lists_decode(cu, Hq, Hkv)
    assert rp[-1] == Hkv * sum((L + 63) // 64 for L in lengths)
    assert np.all((en >> 28) == 2)


def test_policy_storage_independent_of_length():
    """Two int32 boundaries per head: 8 * Hq bytes at every context length."""
    sizes = set()
    for T in (256, 8192, 32768, 131072):
        w = wl.custom("p", [T], 32, 8, 128, 0, "boundary", b1=np.ones(32), b2=np.full(32, 3))
        sizes.add(w.b1.nbytes + w.b2.nbytes)
    assert sizes == {8 * 32}


# --------------------------------------------------------------------------- integer tiles
def test_int_tile_matches_integer_matmul():
    rng = np.random.default_rng(11)
    for d in (64, 128):
        q8 = rng.integers(-127, 128, size=(T, d)).astype(np.int8)
        k8 = rng.integers(-127, 128, size=(T, d)).astype(np.int8)
        ref = q8.astype(np.int64) @ k8.astype(np.int64).T
        assert np.array_equal(oracle.int_tile(oracle.INT8, q8t=q8, k8t=k8), ref)
        q4c = rng.integers(-7, 8, size=(T, d))
        k4c = rng.integers(-7, 8, size=(T, d))
        pack = lambda c: ((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8)
        ref4 = q4c.astype(np.int64) @ k4c.astype(np.int64).T
        assert np.array_equal(oracle.int_tile(oracle.INT4, q4t=pack(q4c), k4t=pack(k4c)), ref4)


# --------------------------------------------------------------------------- prefill
def _dense_causal(qv, kv, vv, cu, Hq, Hkv, scores_fn=None):
    """Textbook causal softmax attention per sequence and head, fp64."""
    d = qv.shape[-1]
    out = np.zeros_like(qv)
    grp = Hq // Hkv
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        L = s1 - s0
        for h in range(Hq):
            if scores_fn is None:
                S = qv[s0:s1, h] @ kv[s0:s1, h // grp].T / np.sqrt(d)
            else:
                S = scores_fn(b, h)
            mask = np.tril(np.ones((L, L), bool))
            S = np.where(mask, S, -np.inf)
            P = np.exp(S - S.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            out[s0:s1, h] = P @ vv[s0:s1, h // grp]
    return out


def _run_oracle_all_rows(w: wl.Workload, q, k, v, cu):
    qz = oracle.Quantised(q, k, None, cu)
    if w.mode == "boundary":
        rp, en = oracle.lists_boundary(cu, w.b1, w.b2)
    else:
        rp, en = oracle.lists_bitmask(cu, w.bitmask, w.G)
    rows = np.arange(len(rp) - 1)
    out, lse = oracle.prefill_rows(q, k, v, cu, qz, rp, en, rows)
    res = oracle.gather_rows(out, cu, rows, w.Hq)
    full = np.zeros((cu[-1], w.Hq, q.shape[-1]))
    for (h, t), vec in res.items():
        full[t, h] = vec
    return full, qz, lse


def _inputs(w):
    t = wl.make_inputs(w, "cpu")
    return tuple(wl.bf16_bits(t[n]) for n in ("q", "k", "v"))


def _dequant_tokens(codes8, s8, cu, d, H):
    """Token-major dequantised values [ntok, H, d] from tile-major INT8 codes."""
    ntok = cu[-1]
    out = np.zeros((ntok, H, d))
    gt = 0
    for b in range(len(cu) - 1):
        L = cu[b + 1] - cu[b]
        for t in range((L + 63) // 64):
            n = min(64, L - t * 64)
            for h in range(H):
                out[cu[b] + t * 64: cu[b] + t * 64 + n, h] = codes8[h, gt, :n].astype(np.float64) * s8[h, gt]
            gt += 1
    return out


def _unpack4(x4):
    nib = np.stack([x4 & 0xF, x4 >> 4], -1).reshape(*x4.shape[:-1], -1).astype(np.int64)
    return np.where(nib >= 8, nib - 16, nib)


def test_prefill_all_bf16_is_dense_attention():
    """All-BF16 bitmask == textbook dense causal attention (GQA, varlen, ragged)."""
    w = wl.custom("allbf16", [130, 64, 1, 200], 4, 2, 64, 5, "bitmask", G=2, p_bf16=1.0)
    q, k, v = _inputs(w)
    cu = w.cu_seqlens
    got, _, lse = _run_oracle_all_rows(w, q, k, v, cu)
    ref = _dense_causal(val_of(q), val_of(k), val_of(v), cu, w.Hq, w.Hkv)
    assert np.max(np.abs(got - ref)) < 1e-12
    # lse against scipy's logsumexp of the masked textbook scores
    from scipy.special import logsumexp
    qv, kv = val_of(q), val_of(k)
    grp = w.Hq // w.Hkv
    ref_lse = np.zeros((cu[-1], w.Hq))
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        L = s1 - s0
        for h in range(w.Hq):
            S = qv[s0:s1, h] @ kv[s0:s1, h // grp].T / np.sqrt(q.shape[-1])
            S = np.where(np.tril(np.ones((L, L), bool)), S, -np.inf)
            ref_lse[s0:s1, h] = logsumexp(S, axis=1)
    assert np.max(np.abs(_lse_tokens(lse, cu, w.Hq) - ref_lse)) < 1e-10


def test_prefill_block_local():
    """b1 = b2 = 1: each query sees only its own tile's causal keys, INT8 scores."""
    w = wl.custom("local", [200, 64], 2, 1, 64, 6, "boundary", b1=[1, 1], b2=[1, 1])
    q, k, v = _inputs(w)
    cu = w.cu_seqlens
    got, qz, _ = _run_oracle_all_rows(w, q, k, v, cu)
    qd = _dequant_tokens(qz.q8, qz.sq8, cu, 64, w.Hq)
    kd = _dequant_tokens(qz.k8, qz.sk8, cu, 64, w.Hkv)
    vv = val_of(v)
    ref = np.zeros_like(got)
    for b in range(len(cu) - 1):
        for t0 in range(cu[b], cu[b + 1], 64):
            t1 = min(t0 + 64, cu[b + 1])
            L = t1 - t0
            for h in range(w.Hq):
                S = qd[t0:t1, h] @ kd[t0:t1, 0].T / 8.0
                S = np.where(np.tril(np.ones((L, L), bool)), S, -np.inf)
                P = np.exp(S - S.max(1, keepdims=True))
                P /= P.sum(1, keepdims=True)
                ref[t0:t1, h] = P @ vv[t0:t1, 0]
    assert np.max(np.abs(got - ref)) < 1e-12


def test_prefill_all_int8_is_dense_over_dequantised_scores():
    """b1 = b2 >= tiles: every causal tile in INT8, none skipped."""
    w = wl.custom("int8", [300, 90], 2, 2, 64, 8, "boundary", b1=[5, 9], b2=[5, 9])
    q, k, v = _inputs(w)
    cu = w.cu_seqlens
    got, qz, _ = _run_oracle_all_rows(w, q, k, v, cu)
    qd = _dequant_tokens(qz.q8, qz.sq8, cu, 64, w.Hq)
    kd = _dequant_tokens(qz.k8, qz.sk8, cu, 64, w.Hkv)
    ref = _dense_causal(qd, kd, val_of(v), cu, w.Hq, w.Hkv)
    assert np.max(np.abs(got - ref)) < 1e-12


def _brute_force_prefill(w, q, k, v, qz, with_lse=False):
    """Per (query, key) pair: pick the precision by the boundary/bitmask rule directly.
    With with_lse, also the natural-log logsumexp of each query's scaled scores
    [ntok, Hq], written out as log(sum(exp(s))) with a shift for range only."""
    cu = w.cu_seqlens
    d = q.shape[-1]
    grp = w.Hq // w.Hkv
    qv, kvv, vv = val_of(q), val_of(k), val_of(v)
    q8 = _dequant_tokens(qz.q8, qz.sq8, cu, d, w.Hq)
    k8 = _dequant_tokens(qz.k8, qz.sk8, cu, d, w.Hkv)
    q4 = _dequant_tokens(_unpack4(qz.q4), qz.sq4, cu, d, w.Hq) if qz.q4 is not None else None
    k4 = _dequant_tokens(_unpack4(qz.k4), qz.sk4, cu, d, w.Hkv) if qz.k4 is not None else None
    out = np.zeros((cu[-1], w.Hq, d))
    lse = np.zeros((cu[-1], w.Hq))
    gt0 = 0
    for b in range(len(cu) - 1):
        L = cu[b + 1] - cu[b]
        for h in range(w.Hq):
            kvh = h // grp
            for i in range(L):
                s = []
                keys = []
                for j in range(i + 1):
                    qt, kt = i // 64, j // 64
                    if w.mode == "boundary":
                        dist = qt - kt
                        if dist < w.b1[h]:
                            sc = q8[cu[b] + i, h] @ k8[cu[b] + j, kvh]
                        elif dist < w.b2[h]:
                            sc = q4[cu[b] + i, h] @ k4[cu[b] + j, kvh]
                        else:
                            continue
                    else:
                        g = kt // w.G
                        bit = (int(w.bitmask[h, gt0 + qt, g // 32]) >> (g % 32)) & 1
                        if bit:
                            sc = qv[cu[b] + i, h] @ kvv[cu[b] + j, kvh]
                        else:
                            sc = q8[cu[b] + i, h] @ k8[cu[b] + j, kvh]
                    s.append(sc / np.sqrt(d))
                    keys.append(j)
                s = np.array(s)
                shift = s[0]                      # any finite shift; the first key's score
                lse[cu[b] + i, h] = shift + np.log(np.sum(np.exp(s - shift)))
                p = np.exp(s - s.max())
                p /= p.sum()
                out[cu[b] + i, h] = p @ vv[cu[b] + np.array(keys), kvh]
        gt0 += (L + 63) // 64
    return (out, lse) if with_lse else out


def _lse_tokens(lse_rows, cu, Hq):
    """Oracle lse [rows, 64] (rows h-major over global q-tiles) -> [ntok, Hq]."""
    cu = np.asarray(cu, np.int64)
    nts = [(int(cu[b + 1] - cu[b]) + 63) // 64 for b in range(len(cu) - 1)]
    ntiles = sum(nts)
    out = np.full((int(cu[-1]), Hq), np.nan)
    for h in range(Hq):
        g = 0
        for b, nt in enumerate(nts):
            T = int(cu[b + 1] - cu[b])
            for qt in range(nt):
                n = min(64, T - qt * 64)
                out[cu[b] + qt * 64: cu[b] + qt * 64 + n, h] = lse_rows[h * ntiles + g, :n]
                g += 1
    return out


def test_prefill_brute_force_tiny_config():
    """The tiny configuration (1 x 2 heads x 256 tokens, (b1, b2) = (1, 3)), brute force."""
    w = wl.tiny()
    q, k, v = _inputs(w)
    got, qz, lse = _run_oracle_all_rows(w, q, k, v, w.cu_seqlens)
    ref, ref_lse = _brute_force_prefill(w, q, k, v, qz, with_lse=True)
    assert np.max(np.abs(got - ref)) < 1e-12
    # lse: natural log of the sum of exp over the kept, scaled scores of each query
    assert np.max(np.abs(_lse_tokens(lse, w.cu_seqlens, w.Hq) - ref_lse)) < 1e-10


def test_prefill_brute_force_bitmask_gqa_varlen():
    w = wl.custom("bm", [190, 70], 4, 2, 64, 12, "bitmask", G=2, p_bf16=0.4)
    q, k, v = _inputs(w)
    got, qz, lse = _run_oracle_all_rows(w, q, k, v, w.cu_seqlens)
    ref, ref_lse = _brute_force_prefill(w, q, k, v, qz, with_lse=True)
    assert np.max(np.abs(got - ref)) < 1e-12
    assert np.max(np.abs(_lse_tokens(lse, w.cu_seqlens, w.Hq) - ref_lse)) < 1e-10


def test_prefill_rows_sum_to_one():
    """With V = 1 everywhere every output equals 1: each probability row sums to 1."""
    w = wl.custom("ones", [333], 2, 1, 64, 13, "boundary", b1=[1, 2], b2=[2, 4])
    q, k, _ = _inputs(w)
    ones = bits_of(np.ones((333, 1, 64), np.float32))
    got, _, lse = _run_oracle_all_rows(w, q, k, ones, w.cu_seqlens)
    assert np.max(np.abs(got - 1.0)) < 1e-12
    assert np.all(np.isfinite(lse))


# --------------------------------------------------------------------------- decode
def test_decode_matches_naive_dense_softmax():
    lengths = [64 * 6 + 10, 64 * 3]
    w = wl.custom("dec", lengths, 4, 2, 64, 21, "boundary", b1=[1, 2, 1, 1], b2=[2, 4, 3, 1],
                  decode_steps=3, tail_cap=4)
    t = wl.make_inputs(w, "cpu")
    k, v = wl.bf16_bits(t["k"]), wl.bf16_bits(t["v"])
    cu = w.cu_seqlens
    cache = oracle.Quantised(None, k, v, cu)
    rp, en = oracle.lists_decode(cu, w.Hq, w.Hkv, w.b1, w.b2)
    qs, kn, vn = (wl.bf16_bits(x) for x in wl.make_decode_inputs(w, "cpu"))
    B, cap, d = len(lengths), 4, 64
    kt = np.zeros((B, w.Hkv, cap, d), np.uint16)
    vt = np.zeros((B, w.Hkv, cap, d), np.uint16)
    for step in range(3):
        kt[:, :, step] = kn[step]
        vt[:, :, step] = vn[step]
        tl = np.full(B, step + 1, np.int32)
        got = oracle.decode_step(qs[step], cu, w.Hkv, cache, rp, en, kt, vt, tl)
        # naive: dequantise every kept token, append the tail, dense softmax
        for b in range(B):
            L = lengths[b]
            nt = (L + 63) // 64
            for h in range(w.Hq):
                kvh = h // 2
                keys, vals = [], []
                for kt_ in range(nt):
                    dist = nt - 1 - kt_
                    hs = (kvh * 2, kvh * 2 + 1)
                    p8 = any(dist < w.b1[x] for x in hs)
                    p4 = any(dist < w.b2[x] for x in hs)
                    if not p4:
                        continue
                    gt = sum((x + 63) // 64 for x in lengths[:b]) + kt_
                    n = min(64, L - kt_ * 64)
                    if p8:
                        kk = cache.k8[kvh, gt, :n] * np.float64(cache.sk8[kvh, gt])
                        vv = cache.v8[kvh, gt, :n] * np.float64(cache.sv8[kvh, gt])
                    else:
                        kk = _unpack4(cache.k4[kvh, gt, :n]) * np.float64(cache.sk4[kvh, gt])
                        vv = _unpack4(cache.v4[kvh, gt, :n]) * np.float64(cache.sv4[kvh, gt])
                    keys.append(kk)
                    vals.append(vv)
                keys.append(val_of(kt[b, kvh, :step + 1]))
                vals.append(val_of(vt[b, kvh, :step + 1]))
                K = np.concatenate(keys)
                V = np.concatenate(vals)
                s = K @ val_of(qs[step, b, h]) / 8.0
                p = np.exp(s - s.max())
                p /= p.sum()
                assert np.max(np.abs(got[b, h] - p @ V)) < 1e-12


# --------------------------------------------------------------------------- token-level hybrid
def _hybrid_case():
    w = wl.custom("hybrid", [300, 64, 1, 200], 4, 2, 64, 71, "boundary")
    q, k, v = _inputs(w)
    cu = w.cu_seqlens
    kv = oracle.Quantised(None, k, v, cu)
    return w, q, k, v, cu, kv


def test_hybrid_select_top_fraction():
    """ceil(frac * T) positions per sequence and KV head, none less important than any
    position left out (ties to the earlier position)."""
    w, q, k, v, cu, kv = _hybrid_case()
    imp = wl.hybrid_importance(w, 3)
    imp[5, 0] = imp[6, 0] = imp[:300, 0].max() + 1.0        # a tie at the top
    sel = oracle.hybrid_select(imp, cu, 0.05)
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        for h in range(w.Hkv):
            n = int(np.ceil(0.05 * (e - s)))
            assert int(sel[s:e, h].sum()) == n
            if 0 < n < e - s:
                assert imp[s:e, h][sel[s:e, h]].min() >= imp[s:e, h][~sel[s:e, h]].max()
    assert sel[5, 0] and sel[6, 0]


def test_hybrid_prefill_reduces_to_dense_attention():
    """Everything kept in bf16 (all selected, or a window covering every key) is textbook
    causal attention; nothing kept is textbook attention over the INT4-dequantised K and V."""
    w, q, k, v, cu, kv = _hybrid_case()
    qv, kvv, vv = val_of(q), val_of(k), val_of(v)
    dense = _dense_causal(qv, kvv, vv, cu, w.Hq, w.Hkv)
    every = np.ones((w.ntok, w.Hkv), bool)
    none = np.zeros((w.ntok, w.Hkv), bool)
    assert np.max(np.abs(oracle.hybrid_prefill(q, k, v, cu, kv, every, 0) - dense)) < 1e-12
    assert np.max(np.abs(oracle.hybrid_prefill(q, k, v, cu, kv, none, 10**6) - dense)) < 1e-12
    k4 = _dequant_tokens(_unpack4(kv.k4), kv.sk4, cu, w.d, w.Hkv)
    v4 = _dequant_tokens(_unpack4(kv.v4), kv.sv4, cu, w.d, w.Hkv)
    low = _dense_causal(qv, k4, v4, cu, w.Hq, w.Hkv)
    assert np.max(np.abs(oracle.hybrid_prefill(q, k, v, cu, kv, none, 0) - low)) < 1e-12


def test_hybrid_prefill_mixes_per_key_and_rows_sum_to_one():
    """A key's precision depends only on its selection and its distance to the query: with
    V = 1 every output is a convex combination of 1 (bf16 keys) and 7 fl32(1/7) (the same
    value read from INT4), so the weights sum to one; changing the precision of one
    unselected, distant key moves only the rows that read it from INT4."""
    w, q, k, v, cu, kv = _hybrid_case()
    sel = oracle.hybrid_select(wl.hybrid_importance(w, 4), cu, 0.05)
    ones = np.full_like(v, 0x3F80)                            # bf16 1.0
    kv1 = oracle.Quantised(None, k, ones, cu)
    out = oracle.hybrid_prefill(q, k, ones, cu, kv1, sel, 16)
    lo4 = 7.0 * np.float64(np.float32(1.0) / np.float32(7.0))
    assert out.min() >= min(1.0, lo4) - 1e-12 and out.max() <= max(1.0, lo4) + 1e-12
    assert np.max(np.abs(out - 1.0)) > 0.0                    # some rows did read INT4
    base = oracle.hybrid_prefill(q, k, v, cu, kv, sel, 16)
    j = int(np.flatnonzero(~sel[:300, 0])[0])                 # an unselected key of sequence 0
    sel2 = sel.copy()
    sel2[j, 0] = True
    moved = oracle.hybrid_prefill(q, k, v, cu, kv, sel2, 16)
    diff = np.abs(moved - base).max(axis=2)                   # [ntok, Hq]
    heads = [h for h in range(w.Hq) if h // (w.Hq // w.Hkv) == 0]
    for i in range(w.ntok):
        reads_lo = 0 <= i - j < 300 - j and i - j >= 16 and i < 300
        for h in range(w.Hq):
            if not (reads_lo and h in heads):
                assert diff[i, h] == 0.0
    assert diff[j + 16:300, heads].max() > 0.0


def test_hybrid_prefill_row_subset_and_lse():
    """A row subset is the same rows of the full computation; with every key in bf16 the
    lse is scipy's logsumexp of the row's scaled causal scores, and nothing-in-bf16 moves
    it only through the INT4 keys."""
    from scipy.special import logsumexp
    w, q, k, v, cu, kv = _hybrid_case()
    sel = oracle.hybrid_select(wl.hybrid_importance(w, 8), cu, 0.05)
    full, lse_full = oracle.hybrid_prefill(q, k, v, cu, kv, sel, 16, with_lse=True)
    rows = np.array([0, 63, 64, 299, 300, 364, 365, 400, w.ntok - 1])
    part, lse_part = oracle.hybrid_prefill(q, k, v, cu, kv, sel, 16, rows=rows, with_lse=True)
    assert np.max(np.abs(part[rows] - full[rows])) < 1e-13
    assert np.max(np.abs(lse_part[:, rows] - lse_full[:, rows])) < 1e-13
    rest = np.setdiff1d(np.arange(w.ntok), rows)
    assert not part[rest].any() and not lse_part[:, rest].any()
    every = np.ones((w.ntok, w.Hkv), bool)
    _, lse = oracle.hybrid_prefill(q, k, v, cu, kv, every, 0, with_lse=True)
    qv, kvv = val_of(q), val_of(k)
    g = w.Hq // w.Hkv
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        for i in range(s, e, 7):
            for h in range(w.Hq):
                sc = kvv[s:i + 1, h // g] @ qv[i, h] / np.sqrt(w.d)
                assert abs(lse[h, i] - logsumexp(sc)) < 1e-12


def test_hybrid_decode_reduces_to_dense_softmax():
    """One decode step: all prefix keys in bf16 gives the textbook softmax over the prefix
    plus the tail; none gives it over the INT4-dequantised prefix plus the tail."""
    w, q, k, v, cu, kv = _hybrid_case()
    B, Hq, Hkv, d = w.B, w.Hq, w.Hkv, w.d
    rng = np.random.default_rng(9)
    qd = wl.bf16_bits(torch.from_numpy(rng.standard_normal((B, Hq, d)).astype(np.float32)).bfloat16())
    cap, tl = 4, np.array([1, 3, 2, 4], np.int32)
    kt = wl.bf16_bits(torch.from_numpy(rng.standard_normal((B, Hkv, cap, d)).astype(np.float32)).bfloat16())
    vt = wl.bf16_bits(torch.from_numpy(rng.standard_normal((B, Hkv, cap, d)).astype(np.float32)).bfloat16())
    every = np.ones((w.ntok, Hkv), bool)
    none = np.zeros((w.ntok, Hkv), bool)
    k4 = _dequant_tokens(_unpack4(kv.k4), kv.sk4, cu, d, Hkv)
    v4 = _dequant_tokens(_unpack4(kv.v4), kv.sv4, cu, d, Hkv)
    for sel, kk, vv_ in ((every, val_of(k), val_of(v)), (none, k4, v4)):
        got = oracle.hybrid_decode_step(qd, k, v, cu, kv, sel, 0, kt, vt, tl)
        for b in range(B):
            for h in range(Hq):
                kh = h // (Hq // Hkv)
                keys = np.concatenate([kk[cu[b]:cu[b + 1], kh], val_of(kt[b, kh, :tl[b]])])
                vals = np.concatenate([vv_[cu[b]:cu[b + 1], kh], val_of(vt[b, kh, :tl[b]])])
                sc = keys @ val_of(qd[b, h]) / np.sqrt(d)
                p = np.exp(sc - sc.max())
                assert np.max(np.abs(got[b, h] - p @ vals / p.sum())) < 1e-12


# --------------------------------------------------------------------------- FP8 middle band
def _torch_e4m3(codes) -> np.ndarray:
    """Values of E4M3 codes decoded by torch's float8_e4m3fn (an implementation of the
    format independent of the oracle)."""
    c = torch.from_numpy(np.asarray(codes, np.uint8).copy())
    return c.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_values_match_the_format():
    """Every finite code decodes as torch does; spot values of the format (largest finite
    448, smallest normal 2^-6, smallest subnormal 2^-9, 1.0, 1.875, -1.0)."""
    codes = [c for c in range(256) if c & 0x7F != 0x7F]
    ours = np.array([oracle.e4m3_value(c) for c in codes])
    assert np.array_equal(ours, _torch_e4m3(codes))
    for c, v in ((0x7E, 448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x38, 1.0), (0x3F, 1.875),
                 (0xB8, -1.0), (0x00, 0.0)):
        assert oracle.e4m3_value(c) == v


def test_e4m3_encode_round_to_nearest_even_and_saturation():
    """Round to the nearest finite E4M3 value (torch's conversion agrees on every value in
    range, midpoints included: ties to the even code), saturate beyond 448, keep the sign
    of zero; every code's own value encodes back to it."""
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 3.0,
        np.exp2(rng.uniform(-14, 8.8, 2000)) * rng.choice([-1, 1], 2000)]).astype(np.float32)
    finite = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = ((finite[:-1] + finite[1:]) / 2).astype(np.float32)     # exact in fp32
    vals = np.concatenate([vals, mids, -mids]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    ours = np.array([oracle.e4m3_encode(x) for x in vals], np.uint8)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    for c in range(0x7F):
        assert oracle.e4m3_encode(finite[c]) == c
        assert oracle.e4m3_encode(-finite[c]) == 0x80 | c
    assert oracle.e4m3_encode(500.0) == 0x7E and oracle.e4m3_encode(-1e9) == 0xFE
    assert oracle.e4m3_encode(464.0) == 0x7E                        # past the last midpoint
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(-1e-9) == 0x80


def test_quantize_f8_invariants():
    """sf = fl32(amax / 448); the tile's largest magnitude maps to +-448; every code is the
    nearest E4M3 value to fl32(x / sf); zero tiles give sf = 0 and codes 0; rows past the
    sequence end are 0."""
    w = wl.custom("f8q", [130, 64, 1], 2, 2, 64, 21, "boundary")
    q, _, _ = _inputs(w)
    q[64:128, 1] = 0                                                 # an all-zero tile of head 1
    cu = w.cu_seqlens
    xf, sf = oracle.quantize_f8(q, cu)
    x = val_of(q).astype(np.float32)
    gt = 0
    for b in range(len(cu) - 1):
        L = cu[b + 1] - cu[b]
        for t in range((L + 63) // 64):
            n = min(64, L - t * 64)
            for h in range(w.Hq):
                tile = x[cu[b] + t * 64: cu[b] + t * 64 + n, h]
                amax = np.float32(np.abs(tile).max())
                assert sf[h, gt] == np.float32(amax / np.float32(448.0))
                codes = xf[h, gt, :n]
                assert not xf[h, gt, n:].any()
                if amax == 0:
                    assert not codes.any()
                    continue
                r = (tile / sf[h, gt]).astype(np.float32)
                assert np.all(np.abs(r) <= np.float32(448.0) * (1 + 2 ** -20))
                ref = torch.from_numpy(np.clip(r, -448, 448)).to(torch.float8_e4m3fn)
                assert np.array_equal(codes, ref.view(torch.uint8).numpy())
                peak = codes.reshape(-1)[np.abs(tile).reshape(-1).argmax()]
                assert peak & 0x7F == 0x7E
            gt += 1


def test_lists_fp8_band_closed_form():
    """With the band [b1, b8): per row qt, FP8 tiles are min(qt+1, b8) - min(qt+1, b1), listed
    after the INT8 group with precision code 4; b8 = b1 gives the two-boundary lists exactly;
    the decode cache keeps a band tile as INT8, i.e. equals the cache of b1 := b8."""
    cu = np.array([0, 700, 700 + 190], np.int32)
    b1 = np.array([1, 3, 2, 5])
    b8 = np.array([4, 3, 9, 5])
    b2 = np.array([6, 7, 9, 11])
    rp, en = oracle.lists_boundary(cu, b1, b2, b8=b8)
    rp0, en0 = oracle.lists_boundary(cu, b1, b2)
    rpe, ene = oracle.lists_boundary(cu, b1, b2, b8=b1)
    assert np.array_equal(rp0, rpe) and np.array_equal(en0, ene)
    nts = [(int(cu[i + 1] - cu[i]) + 63) // 64 for i in range(len(cu) - 1)]
    row = 0
    for h in range(len(b1)):
        for nt in nts:
            for qt in range(nt):
                e = en[rp[row]:rp[row + 1]]
                prec, kt = e >> 28, e & 0x0FFFFFFF
                n8 = min(qt + 1, b1[h])
                nf = min(qt + 1, b8[h]) - n8
                n4 = min(qt + 1, b2[h]) - n8 - nf
                assert (prec == oracle.INT8).sum() == n8 and (prec == oracle.FP8).sum() == nf
                assert (prec == oracle.INT4).sum() == n4
                assert list(prec) == sorted(prec, key=lambda p: [1, 2, 3, 4].index(p))
                for p, k in zip(prec, kt):
                    dist = qt - k
                    want = 2 if dist < b1[h] else 4 if dist < b8[h] else 1
                    assert p == want
                row += 1
    drp, den = oracle.lists_decode(cu, 4, 2, b1, b2, b8=b8)
    drp1, den1 = oracle.lists_decode(cu, 4, 2, b8, b2)
    assert np.array_equal(drp, drp1) and np.array_equal(den, den1)


def test_prefill_fp8_band_brute_force():
    """Every query/key pair through the routing rule with the band, scores from the codes
    (FP8 codes decoded by torch, INT8 and INT4 codes as integers) times the two scales,
    fp64 softmax and P V with bf16 V: the oracle's prefill agrees to 1e-12; b8 = b1
    reproduces the two-boundary prefill."""
    w = wl.custom("f8p", [200, 64, 1], 4, 2, 64, 23, "boundary", b1=[1, 2, 1, 3], b2=[4, 4, 2, 4])
    b8 = np.array([3, 2, 2, 4])
    q, k, v = _inputs(w)
    cu = w.cu_seqlens
    qz = oracle.Quantised(q, k, None, cu, want_f8=True)
    rp, en = oracle.lists_boundary(cu, w.b1, w.b2, b8=b8)
    rows = np.arange(len(rp) - 1)
    out, lse = oracle.prefill_rows(q, k, v, cu, qz, rp, en, rows)
    got = oracle.gather_rows(out, cu, rows, w.Hq)
    d, grp = w.d, w.Hq // w.Hkv
    vv = val_of(v)

    def tok(codes, b, t):          # tile-major [H][nt][64][..] -> (global tile, row)
        off = sum((cu[i + 1] - cu[i] + 63) // 64 for i in range(b))
        return off + t // 64, t % 64

    qf = _torch_e4m3(qz.qf.reshape(-1)).reshape(qz.qf.shape)
    kf = _torch_e4m3(qz.kf.reshape(-1)).reshape(qz.kf.shape)
    q4, k4 = _unpack4(qz.q4), _unpack4(qz.k4)
    for b in range(len(cu) - 1):
        T = cu[b + 1] - cu[b]
        for h in range(w.Hq):
            kh = h // grp
            for i in range(T):
                gq, rq = tok(None, b, i)
                sc, vals = [], []
                for j in range(i + 1):
                    gk, rk = tok(None, b, j)
                    dist = i // 64 - j // 64
                    if dist < w.b1[h]:
                        s = float(qz.q8[h, gq, rq].astype(np.int64) @ qz.k8[kh, gk, rk].astype(np.int64))
                        s *= float(qz.sq8[h, gq]) * float(qz.sk8[kh, gk])
                    elif dist < b8[h]:
                        s = float(qf[h, gq, rq] @ kf[kh, gk, rk]) * float(qz.sqf[h, gq]) * float(qz.skf[kh, gk])
                    elif dist < w.b2[h]:
                        s = float(q4[h, gq, rq] @ k4[kh, gk, rk]) * float(qz.sq4[h, gq]) * float(qz.sk4[kh, gk])
                    else:
                        continue
                    sc.append(s / np.sqrt(d))
                    vals.append(vv[cu[b] + j, kh])
                sc = np.array(sc)
                p = np.exp(sc - sc.max())
                ref = (p / p.sum()) @ np.array(vals)
                assert np.max(np.abs(got[(h, cu[b] + i)] - ref)) < 1e-12
    rp0, en0 = oracle.lists_boundary(cu, w.b1, w.b2)
    out0, _ = oracle.prefill_rows(q, k, v, cu, qz, rp0, en0, rows)
    rpe, ene = oracle.lists_boundary(cu, w.b1, w.b2, b8=w.b1)
    oute, _ = oracle.prefill_rows(q, k, v, cu, qz, rpe, ene, rows)
    assert np.array_equal(out0, oute)
