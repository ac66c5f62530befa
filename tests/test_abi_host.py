"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/tra.h declares, validates arguments before any launch,
and its closed-form sizes agree with the oracle's enumerated lists."""
import ctypes

import numpy as np
import pytest

import oracle
from tile_routed_mixed_causal_b200 import _lib as L
from tile_routed_mixed_causal_b200 import build as tra_build
from tile_routed_mixed_causal_b200 import workloads as wl


@pytest.fixture(scope="module")
def lib():
    tra_build.build()
    return L.load()


def test_exports_every_declared_function(lib):
    names = L.header_functions()
    assert {"quantize_qkv_tiles", "build_tile_lists", "routed_attention_prefill",
            "routed_attention_decode"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert b"sm_100a" in lib.tra_version()


def _shape(lengths, Hq=4, Hkv=2, d=128):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return L.Shape(cu, Hq, Hkv, d, device=None)


FAKE = ctypes.c_void_p(1 << 20)   # aligned non-null stand-in; validation fails before any use


def _status(fn, *args):
    return fn(*args)


@pytest.mark.parametrize("Hq,Hkv,d,lengths,code", [
    (4, 3, 128, [64], L.TraError),
    (4, 2, 96, [64], L.TraError),
    (4, 2, 128, [], L.TraError),
])
def test_shape_validation(lib, Hq, Hkv, d, lengths, code):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = L.Shape(cu, Hq, Hkv, d, device=None)
    assert lib.tra_num_tiles(s.c) == -1


def test_shape_errors_have_codes(lib):
    s = L.Shape(np.array([0, 64], np.int32), 4, 2, 96, device=None)
    pol = L.Policy.boundary([1] * 4, [2] * 4)
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, pol)
    assert e.value.status == 2          # unsupported head dim
    s = L.Shape(np.array([0, 64, 32], np.int32), 4, 2, 128, device=None)
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, pol)
    assert e.value.status == 1 and "non-decreasing" in str(e.value)
    s = L.Shape(np.array([5, 64], np.int32), 4, 2, 128, device=None)
    with pytest.raises(L.TraError):
        L.tile_lists_size(s, pol)


@pytest.mark.parametrize("b1,b2", [([0, 1, 1, 1], [1, 1, 1, 1]), ([2, 1, 1, 1], [1, 1, 1, 1])])
def test_boundary_policy_validation(lib, b1, b2):
    s = _shape([300])
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, L.Policy.boundary(b1, b2))
    assert e.value.status == 1


def test_bitmask_policy_validation(lib):
    s = _shape([64 * 200])
    pol = L.Policy(L.POLICY_BITMASK, G=0)
    pol._c.W = 1
    with pytest.raises(L.TraError):
        L.tile_lists_size(s, pol)
    pol = L.Policy(L.POLICY_BITMASK, G=2)
    pol._c.W = 1                        # 200 tiles / G=2 = 100 groups > 32 bits
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, pol)
    assert "words" in str(e.value)
    pol._c.W = 4
    assert L.tile_lists_size(s, pol) == (4 * 200, 4 * 200 * 201 // 2)


@pytest.mark.parametrize("lengths,b1,b2", [
    ([256], [1, 1], [3, 3]),
    ([1000, 1, 64, 0, 700], [1, 2, 3, 1], [1, 5, 3, 40]),
])
def test_list_sizes_match_oracle(lib, lengths, b1, b2):
    Hq = len(b1)
    s = _shape(lengths, Hq=Hq, Hkv=Hq // 2 if Hq % 2 == 0 else Hq)
    pol = L.Policy.boundary(b1, b2)
    rows, nnz = L.tile_lists_size(s, pol, L.LISTS_PREFILL)
    rp, en = oracle.lists_boundary(s.cu_host, b1, b2)
    assert rows == len(rp) - 1 and nnz == len(en)
    rows, nnz = L.tile_lists_size(s, pol, L.LISTS_DECODE_CACHE)
    rp, en = oracle.lists_decode(s.cu_host, s.Hq, s.Hkv, b1, b2)
    assert rows == len(rp) - 1 and nnz == len(en)


def test_buffer_and_argument_errors(lib):
    s = _shape([300])
    pol = L.Policy.boundary([1] * 4, [2] * 4)
    st = lib.build_tile_lists(s.c, pol.c, L.LISTS_PREFILL, FAKE, 3, FAKE, 10**6, None)
    assert st == 3 and b"row_ptr" in lib.tra_last_error()
    st = lib.build_tile_lists(s.c, pol.c, L.LISTS_PREFILL, FAKE, 10**6, FAKE, 2, None)
    assert st == 3
    st = lib.build_tile_lists(s.c, pol.c, 7, FAKE, 10**6, FAKE, 10**6, None)
    assert st == 1
    # prefill: missing pointers, misalignment, INT4 tiles required, bad scale, dump limit
    qt = L._QTiles(*([None] * 12), L.FMT_Q8 | L.FMT_K8)
    args = [s.c, pol.c, FAKE, FAKE, FAKE, ctypes.byref(qt), FAKE, FAKE, 0.1, FAKE, None, None, 0,
            None, FAKE, None]
    qt.q8 = qt.k8 = qt.sq8 = qt.sk8 = 1 << 20
    assert lib.routed_attention_prefill(*args) == 1
    assert b"Q4" in lib.tra_last_error()
    a2 = list(args)
    a2[2] = ctypes.c_void_p((1 << 20) + 2)
    assert lib.routed_attention_prefill(*a2) == 1
    assert b"aligned" in lib.tra_last_error()
    pol8 = L.Policy.boundary([2] * 4, [2] * 4)
    a3 = list(args)
    a3[1] = pol8.c
    a3[8] = -1.0
    assert lib.routed_attention_prefill(*a3) == 1
    a3[8] = 0.1
    a3[12] = 1000
    assert lib.routed_attention_prefill(*a3) == 1
    a3[12] = 0
    a3[14] = None
    assert lib.routed_attention_prefill(*a3) == 1


def test_decode_validation(lib):
    s = _shape([640], Hq=32, Hkv=2)
    pol = L.Policy.boundary([1] * 32, [1] * 32)
    cache = L._QTiles(*([None] * 12), L.FMT_K8 | L.FMT_V8)
    cache.k8 = cache.v8 = cache.sk8 = cache.sv8 = 1 << 20
    args = [s.c, pol.c] + [FAKE] * 3 + [ctypes.byref(cache)] + [FAKE] * 5 + [4, 0.1, FAKE, FAKE,
                                                                             1 << 30, FAKE, None]
    assert lib.routed_attention_decode(*args) == 2          # group of 16 > 8
    s = _shape([640], Hq=8, Hkv=2)
    args[0] = s.c
    need = lib.tra_decode_workspace_bytes(1, 8, 2, 128)
    assert need > 0
    args[15] = need - 1
    assert lib.routed_attention_decode(*args) == 3
    args[15] = need
    args[11] = 0
    assert lib.routed_attention_decode(*args) == 1         # tail_cap
    args[11] = 4
    pol4 = L.Policy.boundary([1] * 8, [2] * 8)
    args[1] = pol4.c
    assert lib.routed_attention_decode(*args) == 1
    assert b"K4" in lib.tra_last_error()


def test_qtiles_bytes(lib):
    s = _shape([100, 64], Hq=4, Hkv=2, d=64)
    nt = 3
    assert lib.tra_num_tiles(s.c) == nt
    assert lib.tra_qtiles_bytes(s.c, L.FMT_Q8) == 4 * nt * 64 * 64 + 256
    assert lib.tra_qtiles_bytes(s.c, L.FMT_K4) == 2 * nt * 64 * 32 + 256


def test_workload_shapes():
    w = wl.varlen_8()
    assert 0.45 <= w.notes["kept_fraction"] <= 0.55
    assert np.all(w.b1 >= 1) and np.all(w.b2 >= w.b1)
    w = wl.bitmask_32k()
    assert w.bitmask.shape == (32, 512, 4)
    frac = np.mean(np.unpackbits(w.bitmask.view(np.uint8)))
    assert 0.24 < frac < 0.26


def test_selftest_argument_errors(lib):
    """The bounded-wait self-test rejects a missing status word and limits outside
    [1 us, 1 s] on the host, before anything is launched."""
    assert lib.tra_selftest_bounded_wait(None, 10**6, None) == 1
    assert b"status" in lib.tra_last_error()
    assert lib.tra_selftest_bounded_wait(FAKE, 999, None) == 1
    assert lib.tra_selftest_bounded_wait(FAKE, 10**9 + 1, None) == 1
    assert b"limit_ns" in lib.tra_last_error()


def test_mixed_policy_sizes_and_validation(lib):
    """A mixed policy keeps the boundary rule's tile counts (the bitmask only changes
    precisions), its decode caches follow the boundaries, and both halves of the
    policy are validated."""
    import torch
    lengths = [64 * 40 + 3, 65, 64 * 9]
    b1, b2 = [1, 2, 1, 3], [4, 2, 9, 40]
    s = _shape(lengths, Hq=4, Hkv=2)
    nt = sum((L_ + 63) // 64 for L_ in lengths)
    rng = np.random.default_rng(11)
    bm = torch.from_numpy(rng.integers(0, 2**31, size=(4, nt, 1), dtype=np.int64).astype(np.int32))
    pol = L.Policy.mixed(b1, b2, bm, 2)
    assert pol.has_int4
    rows, nnz = L.tile_lists_size(s, pol, L.LISTS_PREFILL)
    rp, en = oracle.lists_mixed(s.cu_host, b1, b2, bm.numpy().view(np.uint32), 2)
    assert rows == len(rp) - 1 and nnz == len(en)
    rows, nnz = L.tile_lists_size(s, pol, L.LISTS_DECODE_CACHE)
    rp, en = oracle.lists_decode(s.cu_host, 4, 2, b1, b2)
    assert rows == len(rp) - 1 and nnz == len(en)
    with pytest.raises(L.TraError):                      # boundary half: b2 < b1
        L.tile_lists_size(s, L.Policy.mixed([2, 1, 1, 1], [1, 1, 1, 1], bm, 2))
    with pytest.raises(L.TraError):                      # bitmask half: G < 1
        L.tile_lists_size(s, L.Policy.mixed(b1, b2, bm, 0))
    bad = L.Policy.mixed(b1, b2, bm, 1)
    bad._c.W = 1                                         # 41 tiles / G=1 > 32 bits
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, bad)
    assert "words" in str(e.value)
    odd = L.Policy.mixed(b1, b2, bm, 2)
    odd._c.mode = 7
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, odd)
    assert "unknown policy mode" in str(e.value)


def test_mixed_policy_needs_its_bitmask(lib):
    """build_tile_lists rejects a mixed policy without device bitmask words, on the host."""
    s = _shape([300], Hq=4, Hkv=2)
    pol = L.Policy(L.POLICY_MIXED, b1=[1, 1, 1, 1], b2=[3, 3, 3, 3], G=2)
    pol._c.W = 1
    rows, nnz = L.tile_lists_size(s, pol, L.LISTS_PREFILL)
    st = lib.build_tile_lists(s.c, pol.c, L.LISTS_PREFILL, FAKE, rows + 1, FAKE, nnz, None)
    assert st == 1 and b"bitmask" in lib.tra_last_error()


def test_hybrid_capacity_and_validation(lib):
    """Token-level hybrid: the selected-token capacity is max_b ceil(frac * T_b) (in double,
    as the oracle computes it); bad fractions, windows and short capacities are rejected
    before any launch."""
    lengths = [300, 64, 1, 257]
    s = _shape(lengths)
    for frac in (0.0, 0.05, 0.2, 1.0, 1.0 / 3.0):
        want = max(min(T, int(np.ceil(frac * T))) for T in lengths)
        assert lib.tra_hybrid_capacity(s.c, frac) == want
    assert lib.tra_hybrid_capacity(s.c, -0.1) == -1
    assert lib.tra_hybrid_capacity(s.c, 1.5) == -1
    cap = lib.tra_hybrid_capacity(s.c, 0.05)
    hy = L._Hybrid(128, cap, *([1 << 20] * 7))
    hy.cap = cap - 1            # (only calls that validation rejects: nothing is launched)
    st = lib.hybrid_select_tokens(s.c, FAKE, ctypes.c_double(0.05), FAKE, FAKE, ctypes.byref(hy), None)
    assert st == 3 and b"cap" in lib.tra_last_error()
    hy.cap, hy.window = cap, -1
    st = lib.hybrid_select_tokens(s.c, FAKE, ctypes.c_double(0.05), FAKE, FAKE, ctypes.byref(hy), None)
    assert st == 1 and b"window" in lib.tra_last_error()
    hy.window = 128
    st = lib.hybrid_select_tokens(s.c, FAKE, ctypes.c_double(1.5), FAKE, FAKE, ctypes.byref(hy), None)
    assert st == 1 and b"frac" in lib.tra_last_error()
    # decode: K4 / V4 cache tiles are required
    qt = L._QTiles(*([None] * 12), L.FMT_K8 | L.FMT_V8)
    args = [s.c, ctypes.byref(hy), FAKE, FAKE, FAKE, ctypes.byref(qt), FAKE, FAKE, FAKE, 4, 0.1,
            FAKE, FAKE, 1 << 30, FAKE, None]
    assert lib.hybrid_attention_decode(*args) == 1 and b"K4" in lib.tra_last_error()


def test_fp8_band_validation_and_sizes(lib):
    """b8 must lie in [b1, b2]; only boundary policies take it; an FP8 band relabels kept
    tiles, so list sizes equal the oracle's (with and without a band); the prefill asks for
    the FP8 tiles before any launch; Q8F / K8F sizes."""
    s = _shape([1000, 64, 1], Hq=4, Hkv=2)
    b1, b2 = [1, 2, 3, 1], [4, 5, 9, 40]
    for bad in ([0, 2, 3, 1], [5, 2, 3, 1]):          # below b1, above b2
        with pytest.raises(L.TraError) as e:
            L.tile_lists_size(s, L.Policy.boundary(b1, b2, b8=bad))
        assert e.value.status == 1
    b8 = [3, 2, 9, 20]
    pol = L.Policy.boundary(b1, b2, b8=b8)
    assert pol.has_fp8 and pol.has_int4
    assert not L.Policy.boundary(b1, b2, b8=b1).has_fp8
    assert not L.Policy.boundary([1, 1], [4, 4], b8=[4, 4]).has_int4
    for kind, ref in ((L.LISTS_PREFILL, oracle.lists_boundary(s.cu_host, b1, b2, b8=b8)),
                      (L.LISTS_DECODE_CACHE, oracle.lists_decode(s.cu_host, 4, 2, b1, b2, b8=b8))):
        rows, nnz = L.tile_lists_size(s, pol, kind)
        assert rows == len(ref[0]) - 1 and nnz == len(ref[1])
    mixed = L.Policy(L.POLICY_MIXED, b1=b1, b2=b2, G=1, b8=b8)
    mixed._c.W = 1
    with pytest.raises(L.TraError) as e:
        L.tile_lists_size(s, mixed)
    assert e.value.status == 2
    qt = L._QTiles()
    qt.formats = L.FMT_Q8 | L.FMT_K8 | L.FMT_Q4X | L.FMT_K4X
    for f in ("q8", "k8", "sq8", "sk8", "q4x", "k4x", "sq4", "sk4"):
        setattr(qt, f, FAKE.value)
    st = lib.routed_attention_prefill(s.c, pol.c, FAKE, FAKE, FAKE, ctypes.byref(qt), FAKE, FAKE,
                                      ctypes.c_float(0.1), FAKE, None, None, 0, None, FAKE, None)
    assert st == 1 and b"Q8F" in lib.tra_last_error()
    nt = lib.tra_num_tiles(s.c)
    assert lib.tra_qtiles_bytes(s.c, L.FMT_Q8F) == 4 * nt * 64 * 128 + ((4 * nt * 4 + 255) // 256) * 256
