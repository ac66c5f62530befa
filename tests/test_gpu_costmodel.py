"""Complete-tile cost model on the GPU (TriAttention abstract: candidate boundary pairs
are weighed by complete-tile execution costs; an allocator selects each head's pair
under a shared budget).

The library's model (tra_prefill_cost_model) turns a boundary policy into a makespan in
entry units -- each (head, q-tile pair) unit's entries, two units per CTA (the heavier
one's tail running alone), CTAs placed on the SMs as the block scheduler does.  Three
constants (time per entry, fixed cost, solo factor) are fitted from three policies
measured on the Llama-3-8B prefill shape; the model must then predict the kernel time of
policies it was not fitted on within 10%: the shape's own per-head boundaries and the
allocator's choice for a synthetic error table.
"""
import numpy as np
import pytest
import torch

import tile_routed_mixed_causal_b200 as tra
from tile_routed_mixed_causal_b200 import api
from tile_routed_mixed_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _kernel_ms(shape, q, k, v, out, b1, b2, reps=20):
    plan = api.PrefillPlan(shape, tra.Policy.boundary(b1, b2))
    plan.run(q, k, v, out)
    for _ in range(3):
        plan.attend(q, k, v, out)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(reps):
        a.record()
        plan.attend(q, k, v, out)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    assert int(plan.status.item()) == 0
    return float(np.median(times))


def test_cost_model_predicts_unfitted_policies():
    w = wl.llama8b_8k()
    t = wl.make_inputs(w, "cuda")
    q, k, v = t["q"], t["k"], t["v"]
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
    out = torch.empty_like(q)
    H, nt = w.Hq, w.tiles_per_seq[0]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # fitted on: two uniform policies and one that pairs a long and a short unit in every CTA
    alt = [nt if h % 2 == 0 else nt // 8 for h in range(H)]
    fit = {"int8_all": ([nt] * H, [nt] * H), "int8_half": ([nt // 2] * H, [nt // 2] * H),
           "int8_alternating": (alt, alt)}
    times = [_kernel_ms(shape, q, k, v, out, b1, b2) for b1, b2 in fit.values()]
    per_entry, fixed, solo = tra.fit_prefill_cost_model(shape, list(fit.values()), times, n_sm=sms)
    assert per_entry > 0
    # the allocator's choice for a seeded synthetic error table at half the all-INT8 cost
    cands = [(b1, b2) for b1 in [1 << i for i in range(8) if (1 << i) <= nt]
             for b2 in [b1 << j for j in range(8) if (b1 << j) <= nt]]
    cost = np.zeros((H, len(cands)), np.int64)
    for c, (b1, b2) in enumerate(cands):
        n8, n4 = tra.boundary_tile_counts(shape, b1, b2)
        cost[:, c] = n8 + n4
    err = wl.synthetic_boundary_errors(H, cands, nt, 7)
    budget = int(0.5 * cost[:, [cands.index((nt, nt))]].sum())
    choice, _, _ = tra.allocate_boundaries(err, cost, budget)
    alloc = ([cands[c][0] for c in choice], [cands[c][1] for c in choice])
    for name, (b1, b2) in {"llama_per_head": (w.b1, w.b2), "allocated": alloc}.items():
        ms, _ = tra.prefill_cost_model(shape, b1, b2, solo=solo, n_sm=sms)
        predicted = per_entry * ms + fixed
        measured = _kernel_ms(shape, q, k, v, out, b1, b2)
        assert abs(predicted / measured - 1.0) < 0.10, (name, predicted, measured)
