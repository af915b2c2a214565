#!/usr/bin/env python
"""Benchmark of the gated delta-rule layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--part all|prefill|decode|proj] [--decode-steps S] [--decode-slots]
                    [--no-cpu-baseline]

A step of the default workload is one pass of the prefill path of one layer
over B=1, T=4096 tokens: causal conv4+SiLU over the 10240 q|k|v channels ->
chunk-64 gated delta rule (16 key / 48 value heads, dim 128) -> gated RMSNorm.
The decode path (B=64 sequences, one token each, 1000 consecutive steps) is
measured in the same run and reported under "decode", and again in its
slot-indexed form (64 rows on a pool of 128 cached states) under
"decode_slots".  Inputs are seeded
synthetic tensors (gdr_inputs) with the layer's shapes; there are no weights.

`--part prefill` / `--part decode` / `--part proj` run one path alone (the
projections: `gdr_linear` beside cuBLAS) for profiling; the default `all` is the
benchmark.

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank runs its own
replica of the workload (the path has no cross-GPU exchange) and the value is
the sum over ranks divided by the max time over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gdr_inputs as GI  # noqa: E402

METRIC_PREFILL = "GDR prefill tokens/s/layer"
METRIC_DECODE = "GDR decode steps/s at B=64"
L2_BYTES = 126 * 1024 * 1024

# algorithmic HBM bytes per token of each kernel (bf16 tensors, fp32 states)
CX = 2 * GI.HK * GI.DK + GI.HV * GI.DV                  # 10240 conv channels
B_CONV = CX * 2 * 2                                      # x read + y write
B_CORE = (2 * GI.HK * GI.DK + GI.HV * GI.DV) * 2 + 2 * GI.HV * 2 + GI.HV * GI.DV * 2   # q,k,v,a,b + o
B_NORM = 3 * GI.HV * GI.DV * 2                           # o, z read + y write
B_FUSED = CX * 2 + 2 * GI.HV * 2 + 2 * GI.HV * GI.DV * 2 # x, a, b, z read + y write
STATE_BYTES = GI.HV * GI.DK * GI.DV * 4                  # one sequence's fp32 state

# DRAM bytes (read + written) per launch from one ncu capture of the current kernels:
# prefill = prep + state chain on full_T4096 (283.9 + 327.8 MB), decode = one B=64 step
# (a replayed launch, partly served from L2), and the same step in the slot-indexed form
TRAFFIC_PREFILL = 611_689_472
TRAFFIC_DECODE = 355_618_304
TRAFFIC_DECODE_SLOTS = 354_019_840


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def to_dev(torch, bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


class PrefillRunner:
    """conv -> chunk prefill -> gated RMSNorm over FullInputs, all on the device."""

    def __init__(self, torch, G, inp, device):
        self.torch, self.G, self.inp = torch, G, inp
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
        self.x = to_dev(torch, inp.x, device)
        self.w = to_dev(torch, inp.conv_w, device)
        self.a = to_dev(torch, inp.a, device)
        self.b = to_dev(torch, inp.b, device)
        self.z = to_dev(torch, inp.z, device).reshape(inp.T, inp.hv, 128)
        self.A_log, self.dt_bias = f(inp.A_log), f(inp.dt_bias)
        self.cu_host = inp.cu_seqlens
        self.cu = torch.from_numpy(inp.cu_seqlens.astype(np.int32)).to(device)
        self.h0 = f(inp.h0) if inp.h0 is not None else None
        T, hk, hv = inp.T, inp.hk, inp.hv
        self.conv_y = torch.empty((T, CX), dtype=torch.bfloat16, device=device)
        self.q = self.conv_y[:, : hk * 128]
        self.o = torch.empty((T, hv, 128), dtype=torch.bfloat16, device=device)
        self.y = torch.empty((T, hv, 128), dtype=torch.bfloat16, device=device)
        self.hT = torch.empty((inp.n_seqs, hv, 128, 128), dtype=torch.float32, device=device)
        self.ws = G.prefill_workspace(inp.cu_seqlens, hv, device)

    def step(self, prefill_events=None):
        torch, G, inp = self.torch, self.G, self.inp
        T, hk, hv = inp.T, inp.hk, inp.hv
        G.causal_conv(self.x, self.w, self.cu, self.cu_host, None, None, self.conv_y)
        y = self.conv_y
        # q, k, v are token-strided views of the [T, q|k|v] conv output, read in place
        q = y[:, : hk * 128].view(T, hk, 128)
        k = y[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
        v = y[:, 2 * hk * 128:].view(T, hv, 128)
        if prefill_events:
            prefill_events[0].record()
        G.chunk_prefill(q, k, v, self.a, self.b, self.A_log, self.dt_bias, self.cu, self.cu_host,
                        h0=self.h0, hT=self.hT, o=self.o, scale=inp.scale, workspace=self.ws)
        if prefill_events:
            prefill_events[1].record()
        G.gated_rmsnorm(self.o, self.z, None, inp.eps, self.y)


def max_over_ranks(torch, values, device):
    """Per-rank timings -> their maximum over the ranks (every rank receives it)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def bench_ours(args, rank, world, device):
    import torch
    import gated_delta_rule_63_b200 as G
    G.lib()
    torch.cuda.set_device(device)
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    inp = GI.workload_full_T4096()
    T = inp.T
    run = PrefillRunner(torch, G, inp, device)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else 0) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))                     # evict L2 between timed steps
            ev[i][0].record()
            run.step()
            ev[i][1].record()
        torch.cuda.synchronize()
        # the prefill call alone, for its roofline: a second pass with events around it (an
        # event between two kernels keeps the second from starting early, so these events
        # stay out of the step timing above)
        for i in range(args.steps):
            flush.fill_(float(i))
            run.step(pev[i])
        torch.cuda.synchronize()
        # decode: B=64, 1000 consecutive steps, state updated in place
        dec_res = bench_decode(torch, G, device, args, steps=args.decode_steps) if args.part == "all" else None
        slot_res = (bench_decode(torch, G, device, args, steps=args.decode_steps, slots=True)
                    if args.part == "all" else None)
        other = bench_long_and_varlen(torch, G, device) if args.part == "all" else None
        mixed = bench_mixed(torch, G, device, args) if args.part == "all" else None
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    pre_ms = [a.elapsed_time(b) for a, b in pev]
    ms = sum(step_ms) / len(step_ms)
    pms = sum(pre_ms) / len(pre_ms)
    if world > 1:
        ms, pms = max_over_ranks(torch, [ms, pms], device)
    value = job_rate(world, T, ms)

    # end to end through the C ABI with host buffers (pinned), copies inside
    e2e = bench_e2e(torch, G, inp, device, args) if args.part == "all" else None
    # the projections last: dense GEMMs run the GPU at its power cap, which would slow what follows
    proj = bench_projections(torch, G, device, flush) if args.part == "all" else None

    prefill_bytes = T * B_CORE + inp.n_seqs * STATE_BYTES
    achieved = prefill_bytes / (pms * 1e-3) / 1e9
    res = {
        "metric": METRIC_PREFILL, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in/out, fp32 state",
        "data": "synthetic (seeded gdr_inputs, no weights)",
        "config": {"workload": "full_T4096: B=1 T=4096 conv4+SiLU -> chunk-64 GDR -> gated RMSNorm, "
                               "hk=16 hv=48 d=128", "global_batch": world, "seq_len": T,
                   "parallelism": f"replicas x{world}", "l2": "flushed between timed steps (252 MB write)",
                   "fused": False},
        "roofline": {"kernel": "gdr_chunk_prefill", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                     "peak_kind": peak_kind, "traffic": TRAFFIC_PREFILL if TRAFFIC_PREFILL else None,
                     "algorithmic_bytes_per_launch": prefill_bytes, "ms_per_launch": pms},
        "step_roofline": {"bytes_per_token_unfused": B_CONV + B_CORE + B_NORM,
                          "bytes_per_token_fused": B_FUSED,
                          "frac_of_fused_hbm_roofline": (T * B_FUSED + STATE_BYTES) / (ms * 1e-3) / 1e9 / hbm_peak},
        "decode": dec_res,
        "decode_slots": slot_res,
        "long_context": other["long_context"] if other else None,
        "varlen8": other["varlen8"] if other else None,
        "mixed_serving": mixed,
        "projections": proj,
        "e2e": e2e,
        # conv, prep, chain, norm per step, in the step pass and the prefill-timing pass
        "gpu_launches": 8 * args.steps + sum(r["launches"] for r in (dec_res, slot_res, other, mixed, proj) if r),
        "clocks": clk.summary(),
    }
    return res


_DECODE = {}


def decode_workload(steps):
    """The decode_B64 workload (fresh seeded x, a, b for every step), drawn once per run."""
    if steps not in _DECODE:
        _DECODE.clear()
        _DECODE[steps] = GI.workload_decode_B64(steps=steps)
    return _DECODE[steps]


def bench_decode(torch, G, device, args, steps=1000, slots=False):
    """B=64 decode, `steps` consecutive steps, each on its own seeded x, a, b (the decode_B64
    workload).  slots=True runs the slot-indexed form on a pool of 128 entries (the 64 rows
    name a seeded random half of them)."""
    hbm_peak, _, _ = measured_peaks()
    dec = decode_workload(steps)
    xs = to_dev(torch, dec.x, device)
    as_ = to_dev(torch, dec.a, device)
    bs = to_dev(torch, dec.b, device)
    cw = to_dev(torch, dec.conv_w, device)
    cs = to_dev(torch, dec.conv_state, device)
    st = torch.from_numpy(dec.state).to(device)
    Al = torch.from_numpy(dec.A_log).to(device)
    db = torch.from_numpy(dec.dt_bias).to(device)
    o = torch.empty((64, dec.hv, 128), dtype=torch.bfloat16, device=device)
    kernel = "gdr_decode_step"
    if slots:
        kernel = "gdr_decode_step_slots"
        n_slots = 128
        slot = torch.from_numpy(GI.make_slot_table(7, 64, n_slots)).to(device)
        idx = slot.long()
        st_pool = torch.zeros((n_slots,) + tuple(st.shape[1:]), dtype=st.dtype, device=device)
        cs_pool = torch.zeros((n_slots,) + tuple(cs.shape[1:]), dtype=cs.dtype, device=device)
        st_pool[idx] = st
        cs_pool[idx] = cs
        warm = (st_pool.clone(), cs_pool.clone())

        def step(s, pools=(st_pool, cs_pool)):
            G.decode_step_slots(xs[s], cw, pools[1], as_[s], bs[s], Al, db, pools[0], slot, o)
    else:
        warm = (st.clone(), cs.clone())

        def step(s, pools=(st, cs)):
            G.decode_step(xs[s], cw, pools[1], as_[s], bs[s], Al, db, pools[0], o)
    for s in range(max(3, args.warmup)):      # warm-up on copies of the states
        step(s % steps, warm)
    torch.cuda.synchronize()
    del warm
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(steps):
        step(s)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    bytes_step = 64 * STATE_BYTES * 2
    achieved = bytes_step / (ms * 1e-3) / 1e9
    res = {"metric": METRIC_DECODE, "value": 1e3 / ms, "unit": "steps/s", "ms_per_step": ms,
           "steps": steps, "launches": steps,
           "inputs": "fresh seeded x, a, b for every step (decode_B64 workload)",
           "roofline": {"kernel": kernel, "bound": "hbm", "achieved": achieved,
                        "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                        "algorithmic_bytes_per_launch": bytes_step,
                        "traffic": TRAFFIC_DECODE_SLOTS if slots else TRAFFIC_DECODE}}
    if slots:
        res["config"] = {"workload": "decode_B64 on a pool of 128 cached states (rows name a seeded "
                                     "random 64 of them)"}
    return res


def bench_mixed(torch, G, device, args, steps=20):
    """A mixed serving step on one pool of 128 cached states (mixed_serving workload): 4 new
    requests of U{256..4096} tokens prefilled into free entries (gdr_chunk_prefill_slots, from
    zero), then one decode token for the 64 running rows from theirs (gdr_decode_step_slots,
    fresh decode_B64 inputs each step).  Events on the launching stream around each call; the
    pool (403 MB) and the step's inputs exceed L2."""
    hbm_peak, _, _ = measured_peaks()
    mix = GI.workload_mixed_serving()
    inp = mix.prefill
    dec = decode_workload(args.decode_steps)
    hv, d = GI.HV, GI.DK
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    q, k, v = to_dev(torch, inp.q, device), to_dev(torch, inp.k, device), to_dev(torch, inp.v, device)
    a, b = to_dev(torch, inp.a, device), to_dev(torch, inp.b, device)
    Al, db = f32(inp.A_log), f32(inp.dt_bias)
    cu_host = inp.cu_seqlens
    cu = torch.from_numpy(cu_host).to(device)
    T = inp.T
    o = torch.empty((T, hv, d), dtype=torch.bfloat16, device=device)
    ws = G.prefill_workspace(cu_host, hv, device, has_final_state=False)
    new_slot = torch.from_numpy(mix.new_slot).to(device)
    dslot = torch.from_numpy(mix.decode_slot).to(device)
    st_pool = torch.zeros((mix.n_slots, hv, d, d), dtype=torch.float32, device=device)
    st_pool[dslot.long()] = torch.from_numpy(dec.state).to(device)
    cs_pool = torch.zeros((mix.n_slots,) + tuple(dec.conv_state.shape[1:]), dtype=torch.bfloat16, device=device)
    cs_pool[dslot.long()] = to_dev(torch, dec.conv_state, device)
    xs, as_, bs = to_dev(torch, dec.x, device), to_dev(torch, dec.a, device), to_dev(torch, dec.b, device)
    cw = to_dev(torch, dec.conv_w, device)
    dAl, ddb = f32(dec.A_log), f32(dec.dt_bias)
    od = torch.empty((len(mix.decode_slot), hv, d), dtype=torch.bfloat16, device=device)
    n_dec = xs.shape[0]

    def prefill():
        G.chunk_prefill_slots(q, k, v, a, b, Al, db, cu, cu_host, st_pool, new_slot, init_from_pool=False,
                              o=o, workspace=ws)

    def decode(s):
        G.decode_step_slots(xs[s % n_dec], cw, cs_pool, as_[s % n_dec], bs[s % n_dec], dAl, ddb, st_pool,
                            dslot, o=od)

    for s in range(3):
        prefill()
        decode(s)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for s in range(steps):
        ev[s][0].record()
        prefill()
        ev[s][1].record()
        decode(3 + s)
        ev[s][2].record()
    torch.cuda.synchronize()
    pre = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    dms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    step = statistics.median(e[0].elapsed_time(e[2]) for e in ev)
    n_new, rows = len(mix.new_slot), len(mix.decode_slot)
    pbytes = T * B_CORE + n_new * STATE_BYTES          # from zero: the entries are only written
    dbytes = rows * STATE_BYTES * 2
    launches = 2 * n_windows(G, cu_host, hv, ws, False)[0] + 1
    return {"workload": f"mixed_serving: {n_new} new requests, lengths {[int(x) for x in np.diff(cu_host)]}, "
                        f"prefilled into free entries of a {mix.n_slots}-entry pool; {rows} running rows "
                        "decode one token from theirs (decode_B64 inputs)",
            "metric": "tokens/s (prompt + decoded tokens per mixed step)",
            "value": (T + rows) / (step * 1e-3), "unit": "tokens/s", "ms_per_step": step,
            "prefill_slots": {"ms": pre, "tokens_per_s": T / (pre * 1e-3),
                              "roofline": {"kernel": "gdr_chunk_prefill_slots", "bound": "hbm",
                                           "achieved": pbytes / (pre * 1e-3) / 1e9, "peak": hbm_peak,
                                           "unit": "GB/s", "frac": pbytes / (pre * 1e-3) / 1e9 / hbm_peak,
                                           "algorithmic_bytes_per_launch": pbytes}},
            "decode_slots": {"ms": dms,
                             "roofline": {"kernel": "gdr_decode_step_slots", "bound": "hbm",
                                          "achieved": dbytes / (dms * 1e-3) / 1e9, "peak": hbm_peak,
                                          "unit": "GB/s", "frac": dbytes / (dms * 1e-3) / 1e9 / hbm_peak}},
            "steps": steps, "launches": (3 + steps) * launches}


def bench_projections(torch, G, device, flush, reps=10):
    """The layer's two projections at T = 4096 (in: 4096 x 5120 -> 16 480 outputs, q|k|v, z, a,
    b; out: 4096 x 6144 -> 5120) on their seeded inputs: gdr_linear and, beside it, torch.matmul
    (cuBLAS) on the same tensors; CUDA events on the launching stream, L2 flushed before each
    call, median of `reps` after 3 untimed calls."""
    _, tc_peak, _ = measured_peaks()
    out = {}
    for name, (x, w) in (("in_proj", GI.workload_in_proj_T4096()), ("out_proj", GI.workload_out_proj_T4096())):
        xd, wd = to_dev(torch, x, device), to_dev(torch, w, device)
        M, K = x.shape
        N = w.shape[0]
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        y2 = torch.empty_like(y)
        wt = wd.t()

        def timed(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            ts = []
            for i in range(reps):
                flush.fill_(float(i))
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            return statistics.median(ts)
        ms = timed(lambda: G.linear(xd, wd, y))
        ms_cublas = timed(lambda: torch.matmul(xd, wt, out=y2))
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[name] = {"shape": {"M": M, "N": N, "K": K}, "ms": ms, "tflops": tf,
                     "roofline": {"kernel": "gdr_linear", "bound": "tensor", "achieved": tf, "peak": tc_peak,
                                  "unit": "TFLOP/s", "frac": tf / tc_peak},
                     "cublas_ms": ms_cublas, "cublas_tflops": 2.0 * M * N * K / (ms_cublas * 1e-3) / 1e12}
        del xd, wd, y, y2, wt
    out["launches"] = 2 * (3 + reps)
    return out


def n_windows(G, cu_host, hv, ws, has_final_state=True):
    """Chunk windows (each a prep and a chain launch) of one prefill call on workspace `ws`, and
    whether the call pipelines them (the library's own schedule query)."""
    return G.prefill_schedule(cu_host, hv, ws.numel(), has_final_state)


def bench_long_and_varlen(torch, G, device, reps=3):
    """The two other prefill workloads on their seeded inputs, timed with CUDA events on the
    launching stream (median of `reps` calls after one untimed call; inputs are far larger
    than L2): long_context = the recurrence alone over B=1, T=262144 (core_T262144);
    varlen8 = conv -> prefill -> gated norm over 8 packed sequences of U{1024..32768} tokens
    with initial states (full_varlen8)."""
    hbm_peak, _, _ = measured_peaks()
    out = {}
    hk, hv, d = GI.HK, GI.HV, GI.DK

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    inp = GI.workload_core_T262144()
    T = inp.T
    q, k, v = to_dev(torch, inp.q, device), to_dev(torch, inp.k, device), to_dev(torch, inp.v, device)
    a, b = to_dev(torch, inp.a, device), to_dev(torch, inp.b, device)
    Al, db = f32(inp.A_log), f32(inp.dt_bias)
    cu_host = inp.cu_seqlens
    cu = torch.from_numpy(cu_host).to(device)
    o = torch.empty((T, hv, d), dtype=torch.bfloat16, device=device)
    hT = torch.empty((1, hv, d, d), dtype=torch.float32, device=device)
    ws = G.prefill_workspace(cu_host, hv, device)
    windows, pipelined = n_windows(G, cu_host, hv, ws)
    launches = 2 * windows
    ms = timed(lambda: G.chunk_prefill(q, k, v, a, b, Al, db, cu, cu_host, hT=hT, o=o, workspace=ws))
    byts = T * B_CORE + STATE_BYTES
    out["long_context"] = {
        "workload": "core_T262144: B=1 T=262144, recurrence alone, zero initial state, final state out",
        "metric": METRIC_PREFILL, "value": T / (ms * 1e-3), "unit": "tokens/s", "ms": ms,
        "algorithmic_bytes": byts, "launches_per_call": launches,
        "schedule": {"windows": windows, "pipelined": pipelined, "workspace_bytes": int(ws.numel())},
        "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": byts / (ms * 1e-3) / 1e9 / hbm_peak}}
    del q, k, v, a, b, o, hT, ws, inp

    inp = GI.workload_full_varlen8()
    T, N = inp.T, inp.n_seqs
    run = PrefillRunner(torch, G, inp, device)
    launches8 = 2 + 2 * n_windows(G, inp.cu_seqlens, hv, run.ws)[0]
    ms = timed(run.step)
    fused = T * B_FUSED + 2 * N * STATE_BYTES
    unfused = T * (B_CONV + B_CORE + B_NORM) + 2 * N * STATE_BYTES
    out["varlen8"] = {
        "workload": "full_varlen8: 8 packed sequences, lengths U{1024..32768} (seed 4), initial states, "
                    "conv4+SiLU -> chunk-64 GDR -> gated RMSNorm",
        "lengths": [int(x) for x in np.diff(inp.cu_seqlens)],
        "metric": METRIC_PREFILL, "value": T / (ms * 1e-3), "unit": "tokens/s", "ms": ms,
        "algorithmic_bytes_fused": fused, "algorithmic_bytes_unfused": unfused, "launches_per_call": launches8,
        "roofline": {"bound": "hbm", "achieved": fused / (ms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": fused / (ms * 1e-3) / 1e9 / hbm_peak,
                     "frac_of_unfused_bytes": unfused / (ms * 1e-3) / 1e9 / hbm_peak}}
    out["launches"] = (1 + reps) * (launches + launches8)
    return out


def bench_e2e(torch, G, inp, device, args):
    """Same prefill step through the C ABI from pinned host buffers, copies included.

    Consecutive steps are pipelined the way a server would run them: the host-to-device
    copies of step i+1 run while step i computes and while its result is copied back (two
    device buffer sets, one stream for each copy direction and one for the kernels)."""
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
    hx, ha, hb, hz = pin(inp.x), pin(inp.a), pin(inp.b), pin(inp.z)
    runs = [PrefillRunner(torch, G, inp, device) for _ in range(2)]
    hys = [torch.empty(runs[0].y.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hTs = [torch.empty(runs[0].hT.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    out_done = [None, None]

    def one(i):
        k = i % 2
        run = runs[k]
        with torch.cuda.stream(s_in):
            if out_done[k] is not None:   # this buffer set's previous step is complete
                s_in.wait_event(out_done[k])
            run.x.view(torch.int16).copy_(hx, non_blocking=True)
            run.a.view(torch.int16).copy_(ha, non_blocking=True)
            run.b.view(torch.int16).copy_(hb, non_blocking=True)
            run.z.view(torch.int16).view(-1).copy_(hz.view(-1), non_blocking=True)
            in_done = torch.cuda.Event()
            in_done.record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(in_done)
            run.step()
            run_done = torch.cuda.Event()
            run_done.record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(run_done)
            hys[k].copy_(run.y, non_blocking=True)
            hTs[k].copy_(run.hT, non_blocking=True)
            out_done[k] = torch.cuda.Event()
            out_done[k].record(s_out)

    for i in range(max(1, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        one(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    h2d = (inp.x.nbytes + inp.a.nbytes + inp.b.nbytes + inp.z.nbytes)
    d2h = hys[0].numel() * 2 + hTs[0].numel() * 4
    return {"value": inp.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# --sweep: the same kernels over other sizes (one JSON line each); inputs drawn
# on the device with torch's generator from the workload distributions
# ---------------------------------------------------------------------------
def _dev_inputs(torch, device, seed, T, n_seqs, full):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    hk, hv, d = GI.HK, GI.HV, GI.DK
    rn = lambda *shape: torch.randn(shape, device=device, generator=g)
    out = {}
    if full:
        out["x"] = rn(T, CX).to(torch.bfloat16)
        out["w"] = (rn(CX, 4) * 0.5).to(torch.bfloat16)
        out["z"] = rn(T, hv, d).to(torch.bfloat16)
    else:
        unit = lambda x: (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        out["q"], out["k"] = unit(rn(T, hk, d)), unit(rn(T, hk, d))
        out["v"] = rn(T, hv, d).to(torch.bfloat16)
    out["a"], out["b"] = rn(T, hv).to(torch.bfloat16), rn(T, hv).to(torch.bfloat16)
    A = torch.empty(hv, device=device, dtype=torch.float64).uniform_(1.0, 16.0, generator=g)
    dt = torch.empty(hv, device=device, dtype=torch.float64).uniform_(1e-3, 0.1, generator=g)
    out["A_log"], out["dt_bias"] = torch.log(A).float(), torch.log(torch.expm1(dt)).float()
    out["h0"] = (rn(n_seqs, hv, d, d) * 0.02) if full else None
    return out


def _time_ms(torch, fn, flush, reps=5):
    fn()
    torch.cuda.synchronize()
    ts = []
    for i in range(reps):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def bench_sweep(torch, G, device):
    hbm_peak, _, _ = measured_peaks()
    hk, hv, d = GI.HK, GI.HV, GI.DK
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    lines = []
    # recurrence alone, one sequence (config 3 is T = 262144)
    for T in (1024, 4096, 16384, 65536, 262144):
        x = _dev_inputs(torch, device, 3, T, 1, full=False)
        cu_host = np.array([0, T], dtype=np.int32)
        cu = torch.from_numpy(cu_host).to(device)
        o = torch.empty((T, hv, d), dtype=torch.bfloat16, device=device)
        hT = torch.empty((1, hv, d, d), dtype=torch.float32, device=device)
        ws = G.prefill_workspace(cu_host, hv, device)
        run = lambda: G.chunk_prefill(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"], cu,
                                      cu_host, hT=hT, o=o, workspace=ws)
        ms = _time_ms(torch, run, flush)
        byts = T * B_CORE + STATE_BYTES
        lines.append({"sweep": "prefill recurrence, B=1", "T": T, "tokens_per_s": T / (ms * 1e-3), "ms": ms,
                      "hbm_frac": byts / (ms * 1e-3) / 1e9 / hbm_peak})
        del x, o, hT, ws
    # full path over 8 packed sequences with an initial state (config 4)
    lengths = GI.varlen8_lengths(4)
    cu_host = GI.cu_seqlens_from_lengths(lengths)
    T, N = int(cu_host[-1]), len(lengths)
    x = _dev_inputs(torch, device, 4, T, N, full=True)
    cu = torch.from_numpy(cu_host).to(device)
    conv_y = torch.empty((T, CX), dtype=torch.bfloat16, device=device)
    o = torch.empty((T, hv, d), dtype=torch.bfloat16, device=device)
    y = torch.empty((T, hv, d), dtype=torch.bfloat16, device=device)
    hT = torch.empty((N, hv, d, d), dtype=torch.float32, device=device)
    ws = G.prefill_workspace(cu_host, hv, device)

    def full_step():
        G.causal_conv(x["x"], x["w"], cu, cu_host, None, None, conv_y)
        q = conv_y[:, : hk * d].view(T, hk, d)
        k = conv_y[:, hk * d: 2 * hk * d].view(T, hk, d)
        v = conv_y[:, 2 * hk * d:].view(T, hv, d)
        G.chunk_prefill(q, k, v, x["a"], x["b"], x["A_log"], x["dt_bias"], cu, cu_host, h0=x["h0"], hT=hT, o=o,
                        workspace=ws)
        G.gated_rmsnorm(o, x["z"], None, 1e-6, y)
    ms = _time_ms(torch, full_step, flush)
    byts = T * B_FUSED + 2 * N * STATE_BYTES
    lines.append({"sweep": "full path, 8 packed sequences U{1024..32768}, h0", "T": T,
                  "lengths": [int(v) for v in lengths], "tokens_per_s": T / (ms * 1e-3), "ms": ms,
                  "frac_of_fused_hbm_roofline": byts / (ms * 1e-3) / 1e9 / hbm_peak})
    del x, conv_y, o, y, hT, ws
    # decode over batch sizes
    for B in (1, 8, 64, 256):
        dec = GI.make_decode_inputs(2, B, 1)
        xs, as_, bs = to_dev(torch, dec.x, device)[0], to_dev(torch, dec.a, device)[0], to_dev(torch, dec.b, device)[0]
        cw, cs = to_dev(torch, dec.conv_w, device), to_dev(torch, dec.conv_state, device)
        st = torch.from_numpy(dec.state).to(device)
        Al, db = torch.from_numpy(dec.A_log).to(device), torch.from_numpy(dec.dt_bias).to(device)
        od = torch.empty((B, hv, d), dtype=torch.bfloat16, device=device)
        step = lambda: G.decode_step(xs, cw, cs, as_, bs, Al, db, st, od)
        for _ in range(5):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(200):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 200
        lines.append({"sweep": "decode", "B": B, "steps_per_s": 1e3 / ms, "ms": ms,
                      "hbm_frac": B * STATE_BYTES * 2 / (ms * 1e-3) / 1e9 / hbm_peak})
    return lines


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle as it stands, on the host cores
# ---------------------------------------------------------------------------
def oracle_step(O, inp):
    return O.full_path(inp)


def cpu_baseline(inp=None):
    from oracle import oracle as O
    inp = inp or GI.workload_full_T4096()
    t0 = time.perf_counter()
    oracle_step(O, inp)
    dt = time.perf_counter() - t0
    # the core_T128 workload (recurrence alone, 48 heads) on one thread, for scale
    small = GI.workload_core_T128()
    t1 = time.perf_counter()
    O.core_path(small, nthreads=1)
    dt1 = time.perf_counter() - t1
    return {"value": inp.T / dt, "unit": "tokens/s", "cores": O.default_threads(), "kind": "oracle",
            "sample": f"one full_T4096 step (all 48 heads, T={inp.T}), fp64 stepwise, "
                      f"{dt:.2f} s wall",
            "one_thread_core_T128": {"value": small.T / dt1, "unit": "tokens/s", "cores": 1,
                                     "sample": f"core_T128 recurrence, all 48 heads, {dt1:.2f} s wall"}}


def bench_reference(args, rank, world):
    """The oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    from oracle import oracle as O
    inp = GI.workload_full_T4096()
    for _ in range(min(args.warmup, 1)):
        oracle_step(O, inp)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(O, inp)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    v = inp.T / (ms * 1e-3)
    return {"impl": "reference", "metric": METRIC_PREFILL, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded gdr_inputs, no weights)",
            "config": {"workload": "full_T4096: B=1 T=4096 conv4+SiLU -> chunk-64 GDR -> gated RMSNorm, "
                                   "hk=16 hv=48 d=128", "global_batch": 1, "seq_len": inp.T,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": O.default_threads(),
                             "kind": "oracle", "sample": "full_T4096 step, every head, fp64 stepwise"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--part", choices=["all", "prefill", "decode", "proj"], default="all")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--decode-slots", action="store_true",
                    help="with --part decode: the slot-indexed form on a pool of 128 cached states")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the bench line: the kernels over other sizes, one JSON line each")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = bench_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    if args.sweep:
        torch.cuda.set_device(device)
        import gated_delta_rule_63_b200 as G
        G.lib()
        for line in bench_sweep(torch, G, device):
            if rank == 0:
                print(json.dumps(line), flush=True)
        return
    if args.part == "proj":
        torch.cuda.set_device(device)
        import gated_delta_rule_63_b200 as G
        G.lib()
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
        res = bench_projections(torch, G, device, flush, reps=max(3, args.steps))
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if args.part == "decode":
        torch.cuda.set_device(device)
        import gated_delta_rule_63_b200 as G
        G.lib()
        res = bench_decode(torch, G, device, args, steps=args.decode_steps, slots=args.decode_slots)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res = bench_ours(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline()
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
