#!/usr/bin/env python
"""Benchmark of the tile-routed mixed-precision causal attention path on B200.

One step = one whole prefill pass over the 32K bitmask workload (B=1, 32 query
/ 8 KV heads, head_dim 128, 32768 tokens, G=4, 25% of routing bits BF16):
quantize_qkv_tiles -> build_tile_lists -> routed_attention_prefill, inputs
resident in HBM.  The headline value is algorithmic tile operations per second
(complete 64x64 tiles, QK and PV both counted, INT8 and BF16 alike) in TOPS.

The same run also measures:
  * e2e      -- the same metric with pinned-host inputs copied in and the
                output copied back inside the timed region;
  * roofline -- the fused prefill kernel's own time (CUDA events on its stream)
                against the tile-mix-weighted tensor peak;
  * decode   -- the compressed-KV-cache decode (batch 16, 32K prefix, 32/8
                heads, 64 steps) in GB/s of algorithmic cache traffic;
  * cpu_baseline -- the CPU oracle on a bounded sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run; every rank runs an independent
replica (the method has no cross-GPU exchange) and rank 0 prints one JSON line.

Reduced lines (--only): "prefill" times one prefill workload (--workload
bitmask_32k | llama8b_8k | varlen_8 | mixed_8k | llama8b_8k_fp8, the last with an
FP8 band halfway between each head's b1 and b2), "decode" the decode alone,
"allocate" fits the complete-tile cost model and runs the boundary allocator on
synthetic error tables, then times the allocated policy; "hybrid" times the
token-level hybrid decode and prefill.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed prefill attn TOPS + tensor-pipe % at 32K; decode KV-cache GB/s"
UNIT = "TOPS"
TILE_OPS_PER_GEMM = 2 * 64 * 64  # x d: one 64x64 score tile (or P*V tile) multiply-add count x 2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-passes", type=int, default=5)
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-configuration prefill records and the allocator record")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the end-to-end leg (0: the same K as --steps)")
    ap.add_argument("--only", choices=["prefill", "decode", "allocate", "hybrid"], default=None,
                    help="run one part only (used for profiler captures); prints a reduced line. "
                         "allocate: measured complete-tile cost model + boundary allocator demo")
    ap.add_argument("--workload", choices=["bitmask_32k", "llama8b_8k", "varlen_8", "mixed_8k",
                                           "llama8b_8k_fp8"],
                    default="bitmask_32k",
                    help="prefill workload for --only prefill (the full bench line always uses "
                         "bitmask_32k)")
    return ap.parse_args()


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of
# each dominant kernel, keyed by the SHA-256 prefix of the kernel source that was captured; a
# source that has changed since reports null.
PROFILED_TRAFFIC = {
    # key: (source file, its sha256[:16] when captured, dram__bytes_read.sum + dram__bytes_write.sum
    # of one launch in the ncu capture); reported only while the source is unchanged
    "prefill_bitmask": ("prefill.cu", "94cee9f264c2ed5f", 2_862_144_000),
    "prefill_hybrid": ("prefill.cu", "94cee9f264c2ed5f", 2_239_947_776),
    "decode": ("decode.cu", "1fedbc1ad6951867", 666_226_944),
}


def profiled_traffic(key):
    import hashlib
    src, want, nbytes = PROFILED_TRAFFIC[key]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tile_routed_mixed_causal_b200",
                        "csrc", src)
    try:
        with open(path, "rb") as f:
            have = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return nbytes if have == want else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk["bf16_tflops"], pk["hbm_gbs"], "measured"
    return 1590.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ----------------------------------------------------------------------------- prefill
def prefill_setup(device, workload="bitmask_32k"):
    import tile_routed_mixed_causal_b200 as tra
    from tile_routed_mixed_causal_b200 import api
    from tile_routed_mixed_causal_b200 import workloads as wl

    fp8 = workload.endswith("_fp8")  # the same workload with an FP8 band between b1 and b2
    w = getattr(wl, workload[:-4] if fp8 else workload)()
    t = wl.make_inputs(w, device)
    q, k, v = t["q"], t["k"], t["v"]
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d, device=device)
    if w.mode == "bitmask":
        bitmask = torch.from_numpy(w.bitmask.view(np.int32)).to(device)
        pol = tra.Policy.from_bitmask(bitmask, w.G)
    elif w.mode == "mixed":
        bitmask = torch.from_numpy(w.bitmask.view(np.int32)).to(device)
        pol = tra.Policy.mixed(w.b1, w.b2, bitmask, w.G)
    else:
        bitmask = torch.zeros(1, dtype=torch.int32, device=device)
        pol = tra.Policy.boundary(w.b1, w.b2, b8=(w.b1 + w.b2) // 2 if fp8 else None)
    plan = api.PrefillPlan(shape, pol, device=device)
    out = torch.empty_like(q)
    plan.lists()
    torch.cuda.synchronize()
    prec = (plan.entries[:plan.nnz].cpu().numpy().view(np.uint32) >> 28)
    n16 = int(np.sum(prec == tra.PREC_BF16))
    n8 = int(np.sum(prec == tra.PREC_INT8))
    n4 = int(np.sum(prec == tra.PREC_INT4))
    nf = int(np.sum(prec == tra.PREC_FP8))
    name = w.name + ("_fp8band" if fp8 else "")
    return dict(w=w, name=name, q=q, k=k, v=v, shape=shape, bitmask=bitmask, pol=pol, plan=plan,
                out=out, tiles=plan.nnz, n16=n16, n8=n8, n4=n4, nf=nf)


def prefill_ops(S):
    per = TILE_OPS_PER_GEMM * S["w"].d
    return 2 * S["tiles"] * per   # QK + PV per kept tile


def roofline_time(S, bf16_tflops):
    """Tile-mix-weighted tensor roofline: INT8/INT4/FP8 QK at 2x the bf16 rate (the nominal
    4.5 / 2.25 PFLOP/s ratio of the int8 and fp8 kinds), BF16 QK and all P*V at the bf16
    rate."""
    per = TILE_OPS_PER_GEMM * S["w"].d
    bf = bf16_tflops * 1e12
    return ((S["n8"] + S["n4"] + S["nf"]) * per / (2 * bf) + S["n16"] * per / bf
            + S["tiles"] * per / bf)


def run_prefill_bench(S, steps, warmup, stream):
    plan, q, k, v, out = S["plan"], S["q"], S["k"], S["v"], S["out"]
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            plan.run(q, k, v, out, stream=stream)
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(steps):
            ev[i][0].record(stream)
            plan.quantize(q, k, v, stream=stream)
            plan.lists(stream=stream)
            ev[i][1].record(stream)
            plan.attend(q, k, v, out, stream=stream)
            ev[i][2].record(stream)
        end.record(stream)
        stream.synchronize()
    total_ms = start.elapsed_time(end)
    attn_ms = [a.elapsed_time(b) for _, a, b in ev]
    prep_ms = [a.elapsed_time(b) for a, b, _ in ev]
    return total_ms, attn_ms, prep_ms


def run_prefill_e2e(S, steps, stream):
    """Same path with pinned-host inputs copied in and the output copied out every step.
    Copies run on their own streams and are double-buffered: step i+1's input copy overlaps
    step i's kernels and step i-1's output copy; the timed region spans the first input
    copy to the last output copy."""
    plan = S["plan"]
    hq = S["q"].cpu().pin_memory()
    hk = S["k"].cpu().pin_memory()
    hv = S["v"].cpu().pin_memory()
    hbm = S["bitmask"].cpu().pin_memory()
    hout = [torch.empty(S["out"].shape, dtype=S["out"].dtype).pin_memory() for _ in range(2)]
    sets = [dict(q=torch.empty_like(S["q"]), k=torch.empty_like(S["k"]), v=torch.empty_like(S["v"]),
                 out=torch.empty_like(S["out"])) for _ in range(2)]
    dbm = S["bitmask"]
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + hbm.numel() * 4
    d2h = hout[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(stream.device), torch.cuda.Stream(stream.device)
    ev = lambda: torch.cuda.Event()

    def run(nsteps):
        loaded = [None, None]      # set i: its inputs are in
        computed = [None, None]    # set i: its kernels are done (its inputs free again)
        drained = [ev(), ev()]     # set i: its output copy is done (its output free again)
        for e in drained:
            e.record(s_out)
        for i in range(nsteps):
            b = i % 2
            st = sets[b]
            # the input copy waits only for the set's previous kernels, so it overlaps the
            # previous output copy (the other direction) as well as the other set's kernels
            if computed[b] is not None:
                s_in.wait_event(computed[b])
            with torch.cuda.stream(s_in):
                st["q"].copy_(hq, non_blocking=True)
                st["k"].copy_(hk, non_blocking=True)
                st["v"].copy_(hv, non_blocking=True)
                if i == 0:
                    dbm.copy_(hbm, non_blocking=True)
            loaded[b] = ev()
            loaded[b].record(s_in)
            stream.wait_event(loaded[b])
            stream.wait_event(drained[b])  # the set's output buffer has been copied out
            plan.run(st["q"], st["k"], st["v"], st["out"], stream=stream)
            computed[b] = ev()
            computed[b].record(stream)
            s_out.wait_event(computed[b])
            with torch.cuda.stream(s_out):
                hout[b].copy_(st["out"], non_blocking=True)
            drained[b] = ev()
            drained[b].record(s_out)

    run(2)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    stream.wait_event(start)
    s_out.wait_event(start)
    run(steps)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    end.record(s_out)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps, h2d, d2h


def quantize_bench(S, stream, reps=20):
    """quantize_qkv_tiles alone on the workload (its formats): ms and GB/s of algorithmic
    bytes (bf16 inputs read once, codes and scales written once)."""
    plan, q, k, v = S["plan"], S["q"], S["k"], S["v"]
    w = S["w"]
    nt = w.ntiles
    tiles = plan.tiles
    fm = tiles.formats
    bytes_ = 0
    for bit8, bit4, H, x in ((0x1, 0x2, w.Hq, q), (0x4, 0x8, w.Hkv, k), (0x10, 0x20, w.Hkv, v)):
        if fm & (bit8 | bit4):
            bytes_ += x.numel() * 2
            if fm & bit8:
                bytes_ += H * nt * 64 * w.d + H * nt * 4
            if fm & bit4:
                bytes_ += H * nt * 64 * w.d // 2 + H * nt * 4
    with torch.cuda.stream(stream):
        for _ in range(3):
            plan.quantize(q, k, v, stream=stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            plan.quantize(q, k, v, stream=stream)
        b.record(stream)
        stream.synchronize()
    ms = a.elapsed_time(b) / reps
    return {"ms": round(ms, 4), "bytes": int(bytes_), "GB/s": round(bytes_ / (ms * 1e-3) / 1e9, 1)}


def workload_records(device, stream, bf16_tflops,
                     names=("llama8b_8k", "varlen_8", "mixed_8k", "llama8b_8k_fp8"),
                     steps=10, warmup=3):
    """The other prefill configurations: kernel time, TOPS and tile-mix roofline fraction."""
    recs = {}
    for name in names:
        S = prefill_setup(device, name)
        total_ms, attn_ms, prep_ms = run_prefill_bench(S, steps, warmup, stream)
        ops = prefill_ops(S)
        kern = statistics.median(attn_ms)
        t_roof = roofline_time(S, bf16_tflops)
        recs[name] = {"workload": S["name"], "prefill_kernel_ms": round(kern, 4),
                      "ms_per_step": round(total_ms / steps, 4),
                      "kernel_TOPS": round(ops / (kern * 1e-3) / 1e12, 2),
                      "roofline_frac": round(t_roof / (kern * 1e-3), 4),
                      "tiles": S["tiles"], "bf16_tiles": S["n16"], "int8_tiles": S["n8"],
                      "int4_tiles": S["n4"], "fp8_tiles": S["nf"],
                      "prep_ms": round(statistics.median(prep_ms), 4)}
        del S
        torch.cuda.empty_cache()
    return recs


# ----------------------------------------------------------------------------- allocator
def allocate_bench(device, stream, budget_frac=0.5, units=4096, seed=7):
    """Complete-tile cost model and model-wide boundary allocation on the Llama-3-8B
    prefill shape (TriAttention abstract: candidate pairs weighed by calibration errors
    and complete-tile execution costs, an allocator choosing each head's pair under a
    shared budget).  Per-tile INT8 and INT4 times and a fixed term are fitted from three
    uniform policies; the errors are a seeded synthetic table (no model here); the budget
    is budget_frac of the all-INT8 cost.  The allocated policy's predicted kernel time is
    then compared with its measured time."""
    import math
    import tile_routed_mixed_causal_b200 as tra
    from tile_routed_mixed_causal_b200 import api
    from tile_routed_mixed_causal_b200 import workloads as wl

    w = wl.llama8b_8k()
    t = wl.make_inputs(w, device)
    q, k, v = t["q"], t["k"], t["v"]
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d, device=device)
    nt = w.tiles_per_seq[0]
    out = torch.empty_like(q)

    def kernel_ms(b1, b2, reps=20):
        plan = api.PrefillPlan(shape, tra.Policy.boundary(b1, b2), device=device)
        with torch.cuda.stream(stream):
            plan.run(q, k, v, out, stream=stream)
            for _ in range(3):
                plan.attend(q, k, v, out, stream=stream)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                plan.attend(q, k, v, out, stream=stream)
            b.record(stream)
            stream.synchronize()
        assert int(plan.status.item()) == 0
        return a.elapsed_time(b) / reps

    def counts(b1, b2):
        n8 = n4 = 0
        for h in range(w.Hq):
            c8, c4 = tra.boundary_tile_counts(shape, b1[h], b2[h])
            n8, n4 = n8 + c8, n4 + c4
        return n8, n4

    H = w.Hq
    full = [nt] * H
    half = [nt // 2] * H
    pol = {"int8_all": (full, full), "int8_half": (half, half), "int4_all": ([1] * H, full)}
    meas = {name: kernel_ms(*bb) for name, bb in pol.items()}
    cnt = {name: counts(*bb) for name, bb in pol.items()}
    w8 = (meas["int8_all"] - meas["int8_half"]) / (cnt["int8_all"][0] - cnt["int8_half"][0])
    t0 = meas["int8_all"] - cnt["int8_all"][0] * w8
    w4 = (meas["int4_all"] - t0 - cnt["int4_all"][0] * w8) / cnt["int4_all"][1]
    # a per-tile time fitted from noisy (e.g. profiled, serialised) launches can come out
    # at or below zero: the costs the allocator takes must stay positive
    w8 = max(w8, 1e-9)
    w4 = max(w4, 0.0)

    # candidates: b1 in powers of two, b2 in b1 x powers of two, up to nt
    cands = [(b1, b2) for b1 in [1 << i for i in range(8) if (1 << i) <= nt]
             for b2 in [b1 << j for j in range(8) if (b1 << j) <= nt]]
    C = len(cands)
    cost_ms = np.zeros((H, C))
    for c, (b1, b2) in enumerate(cands):
        n8, n4 = tra.boundary_tile_counts(shape, b1, b2)
        cost_ms[:, c] = n8 * w8 + n4 * w4
    quantum = cnt["int8_all"][0] * w8 / units          # all-INT8 cost = `units` units
    cost = np.ceil(cost_ms / quantum).astype(np.int64)
    err = wl.synthetic_boundary_errors(H, cands, nt, seed)
    budget = int(budget_frac * units)
    t_a = time.perf_counter()
    choice, total_err, total_units = tra.allocate_boundaries(err, cost, budget)
    alloc_ms = (time.perf_counter() - t_a) * 1e3
    # best single pair for every head within the same budget
    uni = [c for c in range(C) if cost[:, c].sum() <= budget]
    uni_c = min(uni, key=lambda c: err[:, c].sum())
    b1 = [cands[c][0] for c in choice]
    b2 = [cands[c][1] for c in choice]
    predicted = t0 + float(sum(cost_ms[h, choice[h]] for h in range(H)))
    measured = kernel_ms(b1, b2)
    # the library's scheduling-aware model: per-entry time and fixed cost fitted on the
    # same three uniform policies, evaluated on the allocated policy
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    alt = [nt if h % 2 == 0 else nt // 8 for h in range(H)]
    fitpol = [pol["int8_all"], pol["int8_half"], (alt, alt)]
    fit_ms = [meas["int8_all"], meas["int8_half"], kernel_ms(alt, alt)]
    per_entry, fixed, solo = tra.fit_prefill_cost_model(shape, fitpol, fit_ms, n_sm=sms)
    model_pred = per_entry * tra.prefill_cost_model(shape, b1, b2, solo=solo, n_sm=sms)[0] + fixed
    return {
        "makespan_model": {"per_entry_us": per_entry * 1e3, "fixed_ms": fixed, "solo": solo,
                           "predicted_kernel_ms": model_pred,
                           "predicted_over_measured": model_pred / measured},
        "shape": w.name, "tile_ms_model": {"int8_per_tile_ns": w8 * 1e6, "int4_per_tile_ns": w4 * 1e6,
                                           "fixed_ms": t0},
        "fit_points_ms": meas, "candidates_per_head": C, "budget_frac_of_all_int8": budget_frac,
        "budget_units": budget, "allocator_ms": alloc_ms, "total_err": total_err,
        "uniform_best_err": float(err[:, uni_c].sum()), "uniform_best_pair": list(cands[uni_c]),
        "used_units": int(total_units), "predicted_kernel_ms": predicted,
        "measured_kernel_ms": measured, "predicted_over_measured": predicted / measured,
        "b1": b1, "b2": b2,
    }


# ----------------------------------------------------------------------------- decode
def decode_bench(device, passes, stream, hbm_gbs):
    import tile_routed_mixed_causal_b200 as tra
    from tile_routed_mixed_causal_b200 import api
    from tile_routed_mixed_causal_b200 import workloads as wl

    w = wl.decode_32k()
    t = wl.make_inputs(w, device, need_q=False)
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d, device=device)
    pol = tra.Policy.boundary(w.b1, w.b2)
    cache = tra.QTiles(shape, tra.FMT_K8 | tra.FMT_K4 | tra.FMT_V8 | tra.FMT_V4, device)
    tra.quantize_qkv_tiles(shape, None, t["k"], t["v"], cache)
    del t
    dp = api.DecodePlan(shape, pol, cache, w.tail_cap, device)
    dp.build()
    qs, kn, vn = wl.make_decode_inputs(w, device)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=device)
    torch.cuda.synchronize()
    # algorithmic bytes: kept K/V codes + their scales once per GQA group, the bf16 tail,
    # the new token (read and appended), q and the output
    prec = dp.entries[:dp.nnz].cpu().numpy().view(np.uint32) >> 28
    n8 = int(np.sum(prec == tra.PREC_INT8))
    n4 = int(np.sum(prec == tra.PREC_INT4))
    d = w.d
    cache_bytes = n8 * (2 * 64 * d + 8) + n4 * (2 * 64 * d // 2 + 8)
    fixed = w.B * w.Hq * d * 2 * 2 + w.B * w.Hkv * d * 2 * 4
    steps = w.decode_steps
    tail_bytes = sum(w.B * w.Hkv * s * d * 2 * 2 for s in range(steps))
    pass_bytes = steps * (cache_bytes + fixed) + tail_bytes
    times = []
    with torch.cuda.stream(stream):
        for it in range(passes + 1):
            dp.tail_len.zero_()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for s in range(steps):
                dp.step(qs[s], kn[s], vn[s], out, stream=stream)
            s1.record(stream)
            stream.synchronize()
            if it > 0:
                times.append(s0.elapsed_time(s1))
    assert int(dp.status.item()) == 0, "decode reported a device error"
    ms = statistics.median(times)
    gbs = pass_bytes / (ms * 1e-3) / 1e9
    return {
        "metric": "decode KV-cache GB/s",
        "value": round(gbs, 1),
        "unit": "GB/s",
        "workload": w.name + f" (b1~U[64,192], b2~U[b1+128,480]; {n8} INT8 + {n4} INT4 cached tiles)",
        "ms_per_token_step": round(ms / steps, 4),
        "passes": len(times), "pass_ms": [round(t, 3) for t in times], "stat": "median of passes",
        "bytes_per_step": int(pass_bytes / steps),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
                     "frac": round(gbs / hbm_gbs, 4), "traffic": profiled_traffic("decode"),
                     "kernel": "decode_split_kernel (one ABI call: the two- and three-limb launches, each group in one)"},
        "gpu_launches_per_step": 2,
    }


# ----------------------------------------------------------------------------- hybrid decode
def hybrid_bench(device, passes, stream, hbm_gbs, frac=0.05, window=128):
    """Token-level hybrid decode (HyQuant, "How HyQuant works") on the decode workload:
    every prefix tile streamed in INT4 with the 5% selected and the in-window keys read
    from a bf16 side cache; 64 steps.  GB/s of algorithmic bytes."""
    import tile_routed_mixed_causal_b200 as tra
    from tile_routed_mixed_causal_b200 import api
    from tile_routed_mixed_causal_b200 import workloads as wl

    w = wl.decode_32k()
    t = wl.make_inputs(w, device, need_q=False)
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d, device=device)
    cache = tra.QTiles(shape, tra.FMT_K4 | tra.FMT_V4, device)
    tra.quantize_qkv_tiles(shape, None, t["k"], t["v"], cache)
    imp = torch.from_numpy(wl.hybrid_importance(w, 7).astype(np.float32)).to(device)
    hp = api.HybridDecodePlan(shape, cache, frac, window, w.tail_cap, device)
    torch.cuda.synchronize()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s0.record(stream)
        hp.select(imp, t["k"], t["v"], stream=stream)
        s1.record(stream)
    stream.synchronize()
    select_ms = s0.elapsed_time(s1)
    del t
    qs, kn, vn = wl.make_decode_inputs(w, device)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=device)
    d, nt = w.d, w.tiles_per_seq[0]
    nsel = int(np.ceil(frac * w.lengths[0]))
    steps = w.decode_steps
    int4_bytes = w.B * w.Hkv * nt * (2 * 64 * d // 2 + 8 + 8)   # codes, scales, key mask
    fixed = w.B * w.Hq * d * 2 * 2 + w.B * w.Hkv * d * 2 * 4      # q, out, new token
    pass_bytes = 0
    for s in range(steps):
        in_win = sum(1 for x in range(window) if (w.lengths[0] + s) - (w.lengths[0] - window + x) < window)
        hi_rows = nsel + in_win                                    # upper bound: overlaps counted twice
        pass_bytes += int4_bytes + fixed + w.B * w.Hkv * (hi_rows + s + 1) * d * 2 * 2
    times = []
    with torch.cuda.stream(stream):
        for it in range(passes + 1):
            hp.tail_len.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for s in range(steps):
                hp.step(qs[s], kn[s], vn[s], out, stream=stream)
            b.record(stream)
            stream.synchronize()
            if it > 0:
                times.append(a.elapsed_time(b))
    assert int(hp.status.item()) == 0, "hybrid decode reported a device error"
    ms = statistics.median(times)
    gbs = pass_bytes / (ms * 1e-3) / 1e9
    return {"metric": "hybrid decode KV-cache GB/s", "value": round(gbs, 1), "unit": "GB/s",
            "workload": w.name + f" (token-level hybrid: every tile INT4, {nsel} selected + "
                                 f"{window}-token window bf16 per sequence and KV head)",
            "ms_per_token_step": round(ms / steps, 4), "bytes_per_step": int(pass_bytes / steps),
            "select_ms": round(select_ms, 4), "stat": "median of passes",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
                         "frac": round(gbs / hbm_gbs, 4)}}


def hybrid_prefill_bench(device, stream, bf16_tflops, frac=0.05, window=128, reps=10):
    """Token-level hybrid prefill (HyQuant, "How HyQuant works": prefill support) on the
    32K, 32/8-head, d 128 shape: every causal key tile on the tensor cores in bf16, keys
    outside the 128-token window read from their INT4 codes unless among the 5% selected.
    Times one hybrid_attention_prefill call (mixed-operand build + attention) with inputs
    larger than L2; roofline: dense causal QK + PV ops at the measured bf16 rate."""
    import tile_routed_mixed_causal_b200 as tra
    from tile_routed_mixed_causal_b200 import api
    from tile_routed_mixed_causal_b200 import workloads as wl

    w = wl.bitmask_32k()
    t = wl.make_inputs(w, device)
    shape = tra.Shape(w.cu_seqlens, w.Hq, w.Hkv, w.d, device=device)
    plan = api.HybridPrefillPlan(shape, frac, window, device)
    imp = torch.from_numpy(wl.hybrid_importance(w, 7).astype(np.float32)).to(device)
    out = torch.empty_like(t["q"])
    with torch.cuda.stream(stream):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        plan.prepare(t["k"], t["v"], imp, stream=stream)
        b.record(stream)
        times = []
        for it in range(reps + 3):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            plan.attend(t["q"], t["k"], t["v"], out, stream=stream)
            e1.record(stream)
            stream.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
    assert int(plan.status.item()) == 0, "hybrid prefill reported a device error"
    prep_ms = a.elapsed_time(b)
    ms = statistics.median(times)
    tiles = sum(n * (n + 1) // 2 for n in w.tiles_per_seq) * w.Hq
    ops = tiles * 2 * (2 * 64 * 64 * w.d)
    t_roof = ops / (bf16_tflops * 1e12)
    achieved = ops / (ms * 1e-3) / 1e12
    return {"metric": "hybrid prefill TOPS", "value": round(achieved, 1), "unit": "TOPS",
            "workload": f"hybrid_prefill_t{w.lengths[0]}_h{w.Hq}_{w.Hkv}_d{w.d} ({frac:.0%} "
                        f"selected, {window}-token window bf16, other keys INT4)",
            "ms": round(ms, 4), "prep_ms": round(prep_ms, 4), "causal_tiles": tiles,
            "stat": "median of calls",
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": bf16_tflops,
                         "unit": "TFLOP/s", "frac": round(t_roof / (ms * 1e-3), 4),
                         "traffic": profiled_traffic("prefill_hybrid"),
                         "kernel": "hybrid_mix_kernel + prefill_kernel<128, hybrid> (one ABI call)"}}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, q, k, v, qtiles, head=0):
    """Run the oracle on rows (head, q-tile) of the prefill workload; returns (ops, seconds).

    Quantisation and traversal build are included and restricted to the sampled head
    (they are per-(head, tile) independent); the sample's work is its kept tiles."""
    import oracle
    from tile_routed_mixed_causal_b200 import workloads as wl

    grp = w.Hq // w.Hkv
    qh = wl.bf16_bits(q[:, head:head + 1])
    kh = wl.bf16_bits(k[:, head // grp:head // grp + 1])
    vh = wl.bf16_bits(v[:, head // grp:head // grp + 1])
    bm = w.bitmask[head:head + 1]
    t0 = time.perf_counter()
    qz = oracle.Quantised(qh, kh, None, w.cu_seqlens)
    rp, en = oracle.lists_bitmask(w.cu_seqlens, bm, w.G)
    rows = np.array(qtiles, np.int64)
    oracle.prefill_rows(qh, kh, vh, w.cu_seqlens, qz, rp, en, rows)
    dt = time.perf_counter() - t0
    tiles = int(sum(rp[r + 1] - rp[r] for r in rows))
    return 2 * tiles * TILE_OPS_PER_GEMM * w.d, dt, tiles


def cpu_baseline(S, budget_s=10.0):
    """The oracle as it stands on a bounded sample of the 32K workload's q-tile rows of head 0:
    first single-threaded, then with its rows spread over every host core."""
    import oracle
    w = S["w"]
    nt = w.ntiles
    order = [nt - 1, 3 * nt // 4, nt // 2, nt // 4]
    order += [int(x) for x in np.random.default_rng(7).permutation(nt) if int(x) not in order]
    res = {}
    cores = os.cpu_count() or 1
    for label, threads in (("single", 1), ("all", cores)):
        oracle.set_threads(threads)
        rows = []
        ops = secs = tiles = 0
        pos = 0
        while secs <= budget_s and pos < len(order):
            batch = order[pos:pos + threads]
            pos += len(batch)
            o, s_, t = oracle_sample(w, S["q"], S["k"], S["v"], batch)
            rows += batch
            ops += o
            secs += s_
            tiles += t
        res[label] = {"value": round(ops / secs / 1e12, 8), "cores": threads, "rows": len(rows),
                      "tiles": tiles, "seconds": round(secs, 2)}
    oracle.set_threads(1)
    a = res["all"]
    return {"value": a["value"], "unit": UNIT, "cores": a["cores"], "kind": "oracle",
            "single_thread": res["single"],
            "sample": f"head 0 q-tile rows of the 32K bitmask workload (first {order[:4]}, then a "
                      f"seeded permutation): all {a['cores']} host cores took {a['rows']} rows "
                      f"({a['tiles']} kept tiles) in {a['seconds']} s, one core took "
                      f"{res['single']['rows']} rows ({res['single']['tiles']} tiles) in "
                      f"{res['single']['seconds']} s; quantisation + traversal + fp64 attention"}


# ----------------------------------------------------------------------------- main
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host float over all ranks (every rank gets it); device tensor under NCCL,
    host tensor under gloo."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, units_per_rank, ms):
    """Whole-job throughput in units per second x 1e-12 (TOPS for ops): every rank processes
    units_per_rank in ms, the slowest rank's time being the job's."""
    return world * units_per_rank / (ms * 1e-3) / 1e12


def reference_arm(args, world, rank):
    """The CPU oracle as it stands, one bounded sample per step, rank 0 only."""
    if rank != 0:
        return
    from tile_routed_mixed_causal_b200 import workloads as wl
    import oracle
    w = wl.bitmask_32k()
    t = wl.make_inputs(w, "cpu")
    nt = w.ntiles
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    cycle = [nt // 4, nt // 3, nt // 2, nt // 5]
    rows_of = lambda i: [(cycle[i % len(cycle)] + 7 * j) % nt for j in range(cores)]
    for i in range(args.warmup):
        oracle_sample(w, t["q"], t["k"], t["v"], rows_of(i))
    ops = secs = tiles = 0
    for i in range(args.steps):
        o, s, tl = oracle_sample(w, t["q"], t["k"], t["v"], rows_of(i))
        ops += o
        secs += s
        tiles += tl
    value = ops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 8), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": 1, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
                   "seq_len": w.lengths[0], "G": w.G, "bf16_bit_fraction": 0.25},
        "cpu_baseline": {"value": round(value, 8), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{cores} q-tile rows of head 0 per step, one per core "
                                   f"({tiles} kept tiles over {args.steps} steps), quantisation + "
                                   f"traversal + fp64 attention"},
        "e2e": {"value": round(value, 8), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        # host-only: no process group; ranks other than 0 exit without work
        reference_arm(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args)
    import tile_routed_mixed_causal_b200 as tra
    tra.load()
    device = torch.device("cuda", local if world > 1 else 0)
    bf16_tflops, hbm_gbs, peak_src = load_peaks()
    stream = torch.cuda.Stream(device)
    if args.only == "decode":
        if rank == 0:
            print(json.dumps({"only": "decode", **decode_bench(device, args.decode_passes, stream,
                                                              hbm_gbs)}), flush=True)
        return
    if args.only == "hybrid":
        if rank == 0:
            print(json.dumps({"only": "hybrid", **hybrid_bench(device, args.decode_passes, stream,
                                                              hbm_gbs)}), flush=True)
            torch.cuda.empty_cache()
            print(json.dumps({"only": "hybrid_prefill",
                              **hybrid_prefill_bench(device, stream, bf16_tflops)}), flush=True)
        return
    if args.only == "allocate":
        if rank == 0:
            print(json.dumps({"only": "allocate", **allocate_bench(device, stream)}), flush=True)
        return
    if args.only == "prefill":
        S = prefill_setup(device, args.workload)
        total_ms, attn_ms, _ = run_prefill_bench(S, args.steps, args.warmup, stream)
        if rank == 0:
            ops = prefill_ops(S)
            kern = sum(attn_ms) / len(attn_ms)
            t_roof = roofline_time(S, bf16_tflops)
            print(json.dumps({"only": "prefill", "workload": S["name"],
                              "ms_per_step": total_ms / args.steps, "prefill_kernel_ms": kern,
                              "TOPS": ops / (total_ms / args.steps * 1e-3) / 1e12,
                              "kernel_TOPS": ops / (kern * 1e-3) / 1e12,
                              "roofline_frac": t_roof / (kern * 1e-3),
                              "tiles": S["tiles"], "bf16_tiles": S["n16"], "int8_tiles": S["n8"],
                              "int4_tiles": S["n4"], "fp8_tiles": S["nf"]}), flush=True)
        return
    S = prefill_setup(device)
    ops = prefill_ops(S)

    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    total_ms, attn_ms, prep_ms = run_prefill_bench(S, args.steps, args.warmup, stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    value = whole_job_value(world, ops, ms_step)

    attn_avg = sum(attn_ms) / len(attn_ms)
    prep_avg = sum(prep_ms) / len(prep_ms)
    t_roof = roofline_time(S, bf16_tflops)
    achieved = ops / (attn_avg * 1e-3) / 1e12
    peak_eff = ops / t_roof / 1e12

    e2e_steps = args.e2e_steps if args.e2e_steps > 0 else args.steps
    e2e_ms, h2d, d2h = run_prefill_e2e(S, e2e_steps, stream)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_value = whole_job_value(world, ops, e2e_ms)
    quant = quantize_bench(S, stream)
    quant["frac_of_hbm"] = round(quant["GB/s"] / hbm_gbs, 4)

    dec = None
    if not args.no_decode:
        S.pop("plan", None)
        torch.cuda.empty_cache()
        dec = decode_bench(device, args.decode_passes, stream, hbm_gbs)
        if world > 1:  # whole-job GB/s over the slowest rank's step time
            ms_dec = max_over_ranks(dec["ms_per_token_step"], world)
            gbs = whole_job_value(world, dec["bytes_per_step"], ms_dec) * 1e3
            dec.update(value=round(gbs, 1), ms_per_token_step=round(ms_dec, 4))
            dec["roofline"].update(achieved=round(gbs / world, 1),
                                   frac=round(gbs / world / hbm_gbs, 4))

    recs = alloc = hyb = hyp = None
    if not args.no_decode:
        torch.cuda.empty_cache()
        hyb = hybrid_bench(device, args.decode_passes, stream, hbm_gbs)
    if not args.no_workloads:
        torch.cuda.empty_cache()
        hyp = hybrid_prefill_bench(device, stream, bf16_tflops)
    if not args.no_workloads:
        base_S = S.pop("plan", None)
        del base_S
        torch.cuda.empty_cache()
        recs = workload_records(device, stream, bf16_tflops)
        alloc = allocate_bench(device, stream)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(S)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "i8+bf16 (fp32 accumulate/softmax)",
            "data": "synthetic",
            "config": {
                "workload": S["w"].name, "B": 1, "Hq": S["w"].Hq, "Hkv": S["w"].Hkv,
                "d": S["w"].d, "seq_len": S["w"].lengths[0], "G": S["w"].G,
                "bf16_bit_fraction": 0.25, "kept_tiles": S["tiles"], "bf16_tiles": S["n16"],
                "int8_tiles": S["n8"], "ops_per_step": ops,
                "step": "quantize_qkv_tiles + build_tile_lists + routed_attention_prefill",
                "l2": "inputs 0.40 GB bf16 > 126 MB L2; no flush",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "prep_ms": round(prep_avg, 4), "prefill_kernel_ms": round(attn_avg, 4),
            },
            "roofline": {
                "bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak_eff, 2),
                "unit": "TFLOP/s", "frac": round(achieved / peak_eff, 4),
                "traffic": profiled_traffic("prefill_bitmask"),
                "kernel": "prefill_kernel<128, bitmask>",
                "peak_basis": f"tile-mix weighted: bf16 {bf16_tflops} TF/s ({peak_src}, burst), "
                              f"int8 = 2x bf16 (nominal ratio)",
            },
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                    "copies": "pinned host buffers, copy-in and copy-out streams double-buffered "
                              "against the compute stream; the timed region runs from the first "
                              "step's copy-in to the last step's copy-out"},
            "gpu_launches": 3 * args.steps,
            "clocks": clk,
        }
        line["quantize"] = quant
        if dec is not None:
            line["decode"] = dec
        if recs is not None:
            line["workloads"] = recs
        if alloc is not None:
            line["allocate"] = alloc
        if hyb is not None:
            line["hybrid_decode"] = hyb
        if hyp is not None:
            line["hybrid_prefill"] = hyp
        if base is not None:
            line["cpu_baseline"] = base
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
