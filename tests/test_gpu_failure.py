"""GPU failure detection without a GPU fault.

Every pipeline wait in the kernels is bounded: on expiry (or when another role
has already flagged an error) a role gives up, lets its own copies and MMAs in
flight complete, the CTA frees its TMEM and the kernel ORs a bit into a device
status word that the host reads.  These tests make that path run on purpose
with inputs that cannot fault, and then check that the CUDA context is still
usable:

* an mbarrier that nothing ever arrives on, waited on with a 1 ms limit, must
  end with TRA_DEV_TIMEOUT;
* traversal lists built for a boundary policy with an INT4 region, handed to
  the fused prefill under a policy without one (so no INT4 tiles are bound),
  must end with TRA_DEV_BAD_LIST rather than read a missing operand;
* a list entry whose key tile lies past its work unit's last causal tile must
  end with TRA_DEV_BAD_LIST: no copy is issued for it and no per-tile scale is
  read at its index (the prefill's own range check, so the input cannot fault).
"""
import math

import numpy as np
import pytest
import torch

import tile_routed_mixed_causal_b200 as tra
from tile_routed_mixed_causal_b200 import _lib as L
from tile_routed_mixed_causal_b200 import api
from tile_routed_mixed_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _prefill_case():
    w = wl.custom("fail_b_d128", [1000, 300], 4, 2, 128, 51, "boundary",
                  b1=[1, 2, 1, 3], b2=[4, 6, 2, 9])
    t = wl.make_inputs(w, "cpu")
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d)
    return w, shape, q, k, v


def _good_prefill(shape, policy, q, k, v):
    plan = api.PrefillPlan(shape, policy)
    out = torch.zeros_like(q)
    plan.run(q, k, v, out)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    return plan, out


def test_bounded_wait_reports_timeout_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tra.tra_selftest_bounded_wait(status, 1_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == tra.DEV_TIMEOUT
    # the context is intact: a full prefill still runs and reports no error
    w, shape, q, k, v = _prefill_case()
    _good_prefill(shape, tra.Policy.boundary(w.b1, w.b2), q, k, v)


def test_prefill_int4_list_without_int4_tiles_reports_bad_list():
    w, shape, q, k, v = _prefill_case()
    pol4 = tra.Policy.boundary(w.b1, w.b2)
    assert pol4.has_int4
    plan, out_ref = _good_prefill(shape, pol4, q, k, v)
    # same b1 everywhere, b2 = b1: no INT4 region, so no INT4 tiles are bound,
    # yet the lists still hold INT4 entries
    pol_no4 = tra.Policy.boundary(w.b1, w.b1)
    assert not pol_no4.has_int4
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_bad = torch.zeros_like(q)
    L.routed_attention_prefill(shape, pol_no4, q, k, v, plan.tiles, plan.row_ptr, plan.entries,
                               1.0 / math.sqrt(w.d), out_bad, None, status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & tra.DEV_BAD_LIST, f"status {st:#x}"
    assert not st & tra.DEV_TIMEOUT, f"status {st:#x}: the error path itself timed out"
    # the context is intact and the kernel deterministic: the correct call again
    # reproduces the first output bit for bit
    plan.status.zero_()
    out2 = torch.zeros_like(q)
    plan.attend(q, k, v, out2)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    assert torch.equal(out2.view(torch.int16), out_ref.view(torch.int16))


def test_prefill_out_of_range_key_tile_reports_bad_list():
    w, shape, q, k, v = _prefill_case()
    pol = tra.Policy.boundary(w.b1, w.b2)
    plan, out_ref = _good_prefill(shape, pol, q, k, v)
    # one entry of a row gets a key tile far past every sequence (precision kept)
    bad = plan.entries.clone()
    e = plan.nnz // 2
    word = int(bad[e].item()) & 0xFFFFFFFF
    bad[e] = np.int64((word & 0xF0000000) | 0x0FFFFF00).astype(np.int32).item()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_bad = torch.zeros_like(q)
    L.routed_attention_prefill(shape, pol, q, k, v, plan.tiles, plan.row_ptr, bad,
                               1.0 / math.sqrt(w.d), out_bad, None, status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & tra.DEV_BAD_LIST, f"status {st:#x}"
    assert not st & tra.DEV_TIMEOUT, f"status {st:#x}: the error path itself timed out"
    # the context is intact: the unmodified lists reproduce the first output bit for bit
    plan.status.zero_()
    out2 = torch.zeros_like(q)
    plan.attend(q, k, v, out2)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    assert torch.equal(out2.view(torch.int16), out_ref.view(torch.int16))
