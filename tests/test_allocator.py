"""Complete-tile cost counts and the model-wide boundary allocator (host only, no GPU).

TriAttention (abstract): candidate boundary pairs are weighed by projected-output
errors and complete-tile execution costs, and a model-wide allocator picks each
head's pair to minimise the calibration error under a shared computation budget.
The library's dynamic programme is checked against the oracle's enumeration of every
combination; the tile counts against the oracle's enumerated traversal lists.
"""
import numpy as np
import pytest

import oracle
from tile_routed_mixed_causal_b200 import _lib as L
from tile_routed_mixed_causal_b200 import build as tra_build


@pytest.fixture(scope="module")
def lib():
    tra_build.build()
    return L.load()


def _shape(lengths, Hq=2, Hkv=1):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return L.Shape(cu, Hq, Hkv, 128, device=None)


@pytest.mark.parametrize("lengths", [[256], [1000, 1, 64, 0, 700], [64 * 130 + 5]])
@pytest.mark.parametrize("b1,b2", [(1, 1), (1, 3), (2, 9), (7, 7), (4, 200)])
def test_tile_counts_match_enumerated_lists(lib, lengths, b1, b2):
    s = _shape(lengths, Hq=1, Hkv=1)
    n8, n4 = L.boundary_tile_counts(s, b1, b2)
    _, en = oracle.lists_boundary(s.cu_host, [b1], [b2])
    prec = en >> 28
    assert n8 == int(np.sum(prec == L.PREC_INT8))
    assert n4 == int(np.sum(prec == L.PREC_INT4))


def test_tile_counts_validation(lib):
    s = _shape([300])
    for b1, b2 in ((0, 1), (3, 2)):
        with pytest.raises(L.TraError):
            L.boundary_tile_counts(s, b1, b2)


@pytest.mark.parametrize("seed", range(8))
def test_allocator_matches_enumeration(lib, seed):
    rng = np.random.default_rng(seed)
    H, C = int(rng.integers(2, 6)), int(rng.integers(1, 6))
    err = rng.random((H, C))
    cost = rng.integers(0, 12, size=(H, C))
    lo, hi = int(cost.min(axis=1).sum()), int(cost.max(axis=1).sum())
    for budget in sorted({lo, (lo + hi) // 2, hi, lo + 1}):
        ref = oracle.allocate_boundaries(err, cost, budget)
        choice, te, tc = L.allocate_boundaries(err, cost, budget)
        assert ref is not None
        assert list(choice) == ref[0]            # random errors: the optimum is unique
        assert te == pytest.approx(ref[1], rel=0, abs=1e-12)
        assert tc == ref[2] <= budget


def test_allocator_extremes(lib):
    rng = np.random.default_rng(42)
    H, C = 6, 9
    err = rng.random((H, C))
    cost = rng.integers(1, 50, size=(H, C))
    # an unlimited budget takes every head's least error
    choice, te, _ = L.allocate_boundaries(err, cost, int(cost.sum()))
    assert list(choice) == list(err.argmin(axis=1))
    assert te == pytest.approx(err.min(axis=1).sum(), abs=1e-12)
    # the least possible budget forces every head's cheapest candidate (least error
    # among equally cheap ones)
    budget = int(cost.min(axis=1).sum())
    choice, _, tc = L.allocate_boundaries(err, cost, budget)
    assert tc == budget
    for h in range(H):
        cheapest = np.flatnonzero(cost[h] == cost[h].min())
        assert choice[h] == cheapest[np.argmin(err[h, cheapest])]
    # below that nothing fits
    with pytest.raises(L.TraError):
        L.allocate_boundaries(err, cost, budget - 1)


def test_allocator_validation(lib):
    err = np.zeros((2, 3))
    cost = np.ones((2, 3), np.int64)
    with pytest.raises(L.TraError):
        L.allocate_boundaries(err, cost, -1)
    bad = err.copy()
    bad[1, 2] = np.nan
    with pytest.raises(L.TraError):
        L.allocate_boundaries(bad, cost, 10)
    neg = cost.copy()
    neg[0, 0] = -1
    with pytest.raises(L.TraError):
        L.allocate_boundaries(err, neg, 10)
    with pytest.raises(L.TraError) as e:                       # table too large
        L.allocate_boundaries(err, cost, 1 << 27)
    assert e.value.status == 2


def test_prefill_cost_model_counts_entries_of_the_oracle_lists():
    """The cost model's entries are the k-tiles either q-tile of a unit lists (from the
    oracle's traversal lists), duals those the two q-tiles give different precisions; with
    one SM the makespan is the sum over CTAs (two units each) of the heavier unit's work."""
    import oracle
    from tile_routed_mixed_causal_b200 import _lib as L
    lengths = [300, 64, 1, 700]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Hq, Hkv = 4, 2
    b1 = np.array([1, 2, 3, 1], np.int32)
    b2 = np.array([4, 2, 9, 6], np.int32)
    shape = L.Shape(cu, Hq, Hkv, 64, device=None)
    rp, en = oracle.lists_boundary(cu, b1, b2)
    nts = [(int(x) + 63) // 64 for x in lengths]
    off = np.concatenate([[0], np.cumsum(nts)])
    ntiles = int(off[-1])
    jmax = (max(nts) + 1) // 2
    dw = 1.5

    def row(h, b, qt):
        if qt >= nts[b]:
            return {}
        r = h * ntiles + off[b] + qt
        return {int(e & 0x0FFFFFFF): int(e >> 28) for e in en[rp[r]:rp[r + 1]]}

    def unit(uid):
        h, b, j = uid % Hq, (uid // Hq) % len(lengths), jmax - 1 - uid // (Hq * len(lengths))
        r0, r1 = row(h, b, 2 * j), row(h, b, 2 * j + 1)
        kts = set(r0) | set(r1)
        w = sum(dw if (kt in r0 and kt in r1 and r0[kt] != r1[kt]) else 1.0 for kt in kts)
        return w, len(kts)

    units = jmax * len(lengths) * Hq
    total = sum(unit(u)[1] for u in range(units))
    serial = sum(max(unit(2 * c)[0], unit(2 * c + 1)[0] if 2 * c + 1 < units else 0.0)
                 for c in range((units + 1) // 2))
    ms, ne = L.prefill_cost_model(shape, b1, b2, dual_weight=dw, solo=1.0, n_sm=1)
    assert ne == total and abs(ms - serial) < 1e-9
    ms_many, _ = L.prefill_cost_model(shape, b1, b2, dual_weight=dw, solo=1.0, n_sm=1000)
    assert ms_many == max(max(unit(2 * c)[0], unit(2 * c + 1)[0] if 2 * c + 1 < units else 0.0)
                          for c in range((units + 1) // 2))
    # a CTA's lighter unit ends first; the rest of the heavier one runs `solo` times as long
    solo = 0.6
    ms_solo, _ = L.prefill_cost_model(shape, b1, b2, dual_weight=dw, solo=solo, n_sm=1)

    def cta(c):
        w0 = unit(2 * c)[0]
        w1 = unit(2 * c + 1)[0] if 2 * c + 1 < units else 0.0
        return min(w0, w1) + solo * abs(w0 - w1)
    assert abs(ms_solo - sum(cta(c) for c in range((units + 1) // 2))) < 1e-9
