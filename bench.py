"""Benchmark of the Based attention path on B200.

One step = one pass of the prefill hot path over one batch of the
360M-layer-shape workload (B=8, L=2048, d_model=1024): causal Taylor linear
attention over 16 heads (d=16 -> 273 features, d_v=64) with state export, plus
sliding-window-64 softmax attention over 16 heads of d_head=64.  The metric is
tokens/s (B*L per step).  The same run also measures the recurrent decode step
(B=128 sequences x 16 + 16 heads, 273x64 fp32 states, 64-slot rings) and
reports it under "decode".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torchrun; each rank runs an independent replica (the
path has no exchange step), and value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "Based attn prefill tokens/s (L=2048) & decode tokens/s; % of roofline"
UNIT = "tokens/s"
PREFILL = "layer_360m"
DECODE = "decode_b128"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# replicas: one independent copy of the workload per rank, no data exchange
# ---------------------------------------------------------------------------

FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 74.4: CUDA-core fp32 peak of a B200


def max_over_ranks(ms: float, dev, world: int) -> float:
    """The slowest rank's time (every rank gets the same answer)."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: float, ms: float, world: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (ms / 1e3)


# ---------------------------------------------------------------------------
# DRAM traffic per launch from the committed ncu captures (profiles/traffic.json),
# reported only while the headers that define the kernel's code are unchanged
# since the capture
# ---------------------------------------------------------------------------

_KERNEL_SOURCES = {"linattn_prefill": "linattn_tc.cuh", "window_attn": "window_tc.cuh",
                   "decode_step": "decode.cuh"}


def measured_traffic(kernel):
    import hashlib
    csrc = os.path.join(ROOT, "linear_attention_lm_b200", "csrc")
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f)[kernel]
        h = hashlib.sha256()
        for name in (_KERNEL_SOURCES[kernel], "umma.cuh", "common.cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != entry["sources_sha256"]:
            return None
        return int(entry["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# algorithmic bytes / flops (per launch)
# ---------------------------------------------------------------------------

def linattn_bytes(w):
    """q, k (d), v, out (d_v) in the input dtype per token-head, + exported states."""
    es = 4 if w.dtype == "f32" else 2
    per_tok = (2 * w.d + 2 * w.dv) * es
    return w.B * w.H * w.L * per_tok + w.B * w.H * 273 * (w.dv + 1) * 4


def window_bytes(w):
    es = 4 if w.dtype == "f32" else 2
    return w.B * w.Hw * w.L * 4 * w.dh * es


def decode_bytes(w):
    es = 2 if w.dtype == "bf16" else 4
    lin = w.B * w.H * (2 * 273 * (w.dv + 1) * 4 + (2 * w.d + 2 * w.dv) * es)
    win = w.B * w.Hw * (2 * w.window * w.dh * es + 2 * w.dh * es + 4 * w.dh * es)
    return lin + win


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def mark(self, which):
        setattr(self, which, time.time())

    def summary(self):
        """Median SM clock and active throttle reasons over the samples taken
        inside [t_start, t_stop]; if the window was shorter than the sampling
        period, the samples nearest to it."""
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        t0, t1 = getattr(self, "t_start", None), getattr(self, "t_stop", None)
        inside = [r for r in rows if t0 is not None and t0 <= r[0] <= t1]
        sel = inside
        if not sel and rows and t0 is not None:
            mid = 0.5 * (t0 + t1)
            sel = sorted(rows, key=lambda r: abs(r[0] - mid))[:2]
        reasons = set()
        for r in sel:
            for n, val in zip(names, r[3]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median([r[1] for r in sel]) if sel else None,
                "sm_max_mhz": sel[0][2] if sel else None, "reasons": sorted(reasons),
                "samples_in_window": len(inside)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, dev):
    import linear_attention_lm_b200 as lab
    from linear_attention_lm_b200 import build as lab_build
    from linear_attention_lm_b200.inputs import WORKLOADS, decode_step_inputs, prefill_inputs

    if rank == 0:
        lab_build.build()
    if world > 1:
        torch.distributed.barrier()
    lab.load_library()
    peaks = load_peaks()
    w = WORKLOADS[PREFILL]
    # rotate input sets so that consecutive steps never find their data in L2
    set_bytes = linattn_bytes(w) + window_bytes(w)
    n_sets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(n_sets):
        x = prefill_inputs(w, device=dev) if i == 0 else {k: t.clone() for k, t in sets[0][0].items()}
        outs = {"y": torch.empty_like(x["v"]), "yw": torch.empty_like(x["wq"]),
                "S": torch.empty((w.B, w.H, 273, w.dv), dtype=torch.float32, device=dev),
                "z": torch.empty((w.B, w.H, 273), dtype=torch.float32, device=dev)}
        sets.append((x, outs))
    ws_bytes = lab.based_linattn_workspace_bytes(w.B, w.H, w.L, w.d, w.dv, lab.BASED_BF16)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

    def step(i, ev=None):
        x, o = sets[i % n_sets]
        if ev is not None:
            ev[0].record()
        lab.based_linattn_fwd(x["q"], x["k"], x["v"], o["y"], w.eps, o["S"], o["z"],
                              workspace=ws[:ws_bytes] if ws_bytes else None)
        if ev is not None:
            ev[1].record()
        lab.based_window_attn_fwd(x["wq"], x["wk"], x["wv"], o["yw"], w.window)
        if ev is not None:
            ev[2].record()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.3)  # let the sampler start
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        clk.mark("t_start")
        start.record()
        for i in range(args.steps):
            step(i, evs[i])
        stop.record()
        torch.cuda.synchronize()
        clk.mark("t_stop")
        if world > 1:
            torch.distributed.barrier()
    elapsed_ms = start.elapsed_time(stop)
    t_lin = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_win = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    assert lab.based_get_device_error() == 0
    elapsed_max = max_over_ranks(elapsed_ms, dev, world)
    value = replica_rate(w.B * w.L * args.steps, elapsed_max, world)

    # roofline of the dominant kernel (both are HBM-bound by algorithmic bytes)
    kern = {"linattn_prefill": (linattn_bytes(w), t_lin), "window_attn": (window_bytes(w), t_win)}
    dom = max(kern, key=lambda k: kern[k][1])
    b, t_ms = kern[dom]
    achieved = b / (t_ms / 1e3) / 1e9
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": measured_traffic(dom),
                "algorithmic_bytes": int(b), "peak_source": peaks["source"],
                "per_kernel_ms": {k: round(v[1], 5) for k, v in kern.items()},
                "per_kernel_frac": {k: round(v[0] / (v[1] / 1e3) / 1e9 / peaks["hbm_gbs"], 4)
                                    for k, v in kern.items()}}

    e2e = run_e2e(args, w, lab, dev, world, sets[0][0])
    decode = run_decode(args, lab, dev, world, peaks)
    try:
        projections = run_projections(args, lab, dev, world, peaks)
    except Exception as exc:  # reported in the JSON line, never hidden
        projections = {"error": f"{type(exc).__name__}: {exc}"}
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_max / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{PREFILL}: B=8 L=2048 d_model=1024; linear attn 16 heads "
                               f"d=16->273 d_v=64 (+state export); window-64 attn 16 heads d_h=64",
                   "global_batch": w.B * world, "seq_len": w.L,
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs larger than L2: {n_sets} rotating input sets of "
                         f"{set_bytes / 1e6:.0f} MB"},
        "roofline": roofline,
        "e2e": e2e,
        "decode": decode,
        "projections": projections,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def run_e2e(args, w, lab, dev, world, x):
    """Same metric through the public API from pinned host buffers: every step
    copies its inputs host->device, runs both kernels, and copies both outputs
    device->host.  Steps are pipelined the way a caller would run them: the
    inputs of step i+1 travel (copy stream) while step i computes (compute
    stream) and the outputs of step i-1 come back (a third stream), with two
    device buffer sets; PCIe carries both directions at once."""
    n = max(2, min(args.steps, 30))
    host_in = {k: t.to("cpu").pin_memory() for k, t in x.items()}
    host_out = [{"y": torch.empty(x["v"].shape, dtype=x["v"].dtype).pin_memory(),
                 "yw": torch.empty(x["wq"].shape, dtype=x["wq"].dtype).pin_memory()}
                for _ in range(2)]
    dev_in = [{k: torch.empty_like(t, device=dev) for k, t in x.items()} for _ in range(2)]
    dev_out = [(torch.empty_like(dev_in[0]["v"]), torch.empty_like(dev_in[0]["wq"]))
               for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_run[b])  # step i-2 no longer reads dev_in[b]
            for k in dev_in[b]:
                dev_in[b][k].copy_(host_in[k], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            if i >= 2:
                s_run.wait_event(ev_out[b])  # step i-2's outputs have left dev_out[b]
            y, yw = dev_out[b]
            lab.based_linattn_fwd(dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["v"], y, w.eps,
                                  stream=s_run)
            lab.based_window_attn_fwd(dev_in[b]["wq"], dev_in[b]["wk"], dev_in[b]["wv"], yw,
                                      w.window, stream=s_run)
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            host_out[b]["y"].copy_(dev_out[b][0], non_blocking=True)
            host_out[b]["yw"].copy_(dev_out[b][1], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(n):
        step(i)
    end.record(s_out)  # the last device->host copy waits on everything before it
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, dev, world)
    return {"value": round(world * w.B * w.L * n / (ms / 1e3), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n,
            "pipelined": "h2d(i+1) | kernels(i) | d2h(i-1) on three streams"}


def run_projections(args, lab, dev, world, peaks):
    """The rows next to the hot path, each on layer_360m's shapes (synthetic):
    the six per-head input projections of one linear-attention and one window
    layer (x [8, 2048, 1024] bf16; q, k: 16 heads of 16; v and the window's q,
    k, v: 16 heads of 64), one BaseConv block (D = 1024, 3 taps), and the
    linear attention's backward.  Four rotating x buffers (128 MB) keep L2 cold
    for the projections."""
    B, L, dm, H = 8, 2048, 1024, 16
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    xs = [torch.randn(B, L, dm, device=dev, generator=g).to(torch.bfloat16) for _ in range(4)]
    heads = [16, 16, 64, 64, 64, 64]
    ws = [(torch.randn(H * D, dm, device=dev, generator=g) * 0.02).to(torch.bfloat16) for D in heads]
    ys = [torch.empty(B, H, L, D, device=dev, dtype=torch.bfloat16) for D in heads]
    wb = (torch.randn(dm, dm, device=dev, generator=g) * 0.03).to(torch.bfloat16)
    bias = torch.randn(dm, device=dev, generator=g) * 0.1
    taps = torch.randn(dm, 3, device=dev, generator=g) * 0.5
    yb = torch.empty(B, L, dm, device=dev, dtype=torch.bfloat16)
    n = max(10, min(args.steps, 200))

    def timed(fn, n_iter):
        for i in range(max(3, args.warmup)):
            fn(i)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for i in range(n_iter):
            fn(i)
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / n_iter
        ms = max_over_ranks(ms, dev, world)
        return ms

    def proj_step(i):
        x = xs[i % 4]
        for w, y in zip(ws, ys):
            lab.based_proj_heads_fwd(x, w, y)

    def conv_step(i):
        lab.based_baseconv_fwd(xs[i % 4], wb, bias, taps, yb)

    # backward of the linear attention, layer_360m shape, CUDA cores (fp32 FMA)
    qb = (torch.randn(B, H, L, 16, device=dev, generator=g) * 0.25).to(torch.bfloat16)
    kb = (torch.randn(B, H, L, 16, device=dev, generator=g) * 0.25).to(torch.bfloat16)
    vb = torch.randn(B, H, L, 64, device=dev, generator=g).to(torch.bfloat16)
    dyb = torch.randn(B, H, L, 64, device=dev, generator=g).to(torch.bfloat16)
    gq, gk = torch.empty(B, H, L, 16, device=dev), torch.empty(B, H, L, 16, device=dev)
    gv = torch.empty(B, H, L, 64, device=dev)
    wsb = torch.empty(lab.based_linattn_bwd_workspace_bytes(B, H, L, 64), dtype=torch.uint8,
                      device=dev)

    def bwd_step(i):
        lab.based_linattn_bwd(qb, kb, vb, dyb, gq, gk, gv, 1e-6, workspace=wsb)

    out = {}
    peak = peaks["bf16_tflops"]
    for name, fn, flops, launches, what in (
            ("proj", proj_step, 2.0 * B * L * dm * H * sum(heads), len(heads),
             "six per-head projections of x [8, 2048, 1024]: q, k 16x16; v 16x64; window q, k, v 16x64"),
            ("baseconv", conv_step, 2.0 * B * L * dm * dm, 1,
             "BaseConv block, x [8, 2048, 1024], dense 1024x1024 + bias, 3 causal taps"),
            ("linattn_bwd", bwd_step, 480.0 * B * H * L * (L + 1) / 2, 2,
             "gradient of the linear attention, B=8 H=16 L=2048 d=16 d_v=64 (quadratic form, "
             "480 flop per (t, s) pair)")):
        ms = timed(fn, 10 if name == "linattn_bwd" else n)
        tf = flops / (ms / 1e3) / 1e12
        if name == "linattn_bwd":
            # CUDA-core fp32 FMA peak: 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz
            kern, bound, pk, src = "linattn_bwd", "alu", FP32_FMA_TFLOPS, "unit counts x max clock"
        else:
            kern, bound, pk, src = "proj_tc", "tensor", peak, peaks["source"]
        out[name] = {"workload": what, "ms_per_step": round(ms, 5), "launches_per_step": launches,
                     "tokens_per_s": round(world * B * L / (ms / 1e3), 1),
                     "roofline": {"kernel": kern, "bound": bound, "achieved": round(tf, 2),
                                  "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                                  "traffic": None, "peak_source": src}}
    assert lab.based_get_device_error() == 0
    return out


def run_decode(args, lab, dev, world, peaks):
    """Recurrent decode: prefill 512 tokens (state export + ring fill), then
    time decode steps; two independent batches alternate so the 176 MB of
    state + ring per batch is never resident in L2 from the previous step."""
    from linear_attention_lm_b200.inputs import WORKLOADS, decode_step_inputs, prefill_inputs
    w = WORKLOADS[DECODE]
    groups = []
    for gi in range(2):
        x = prefill_inputs(w, device=dev)
        _, S, z = lab.linattn(x["q"], x["k"], x["v"], w.eps, return_state=True)
        kr, vr = lab.window_ring_fill(x["wk"], x["wv"], w.window)
        groups.append((S, z, kr, vr))
        del x
    step_in = [decode_step_inputs(w, s, device=dev) for s in range(8)]
    out = torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    wout = torch.empty((w.B, w.Hw, w.dh), dtype=torch.bfloat16, device=dev)
    n = max(8, min(args.steps, 512))

    def one(i):
        S, z, kr, vr = groups[i % 2]
        d = step_in[i % len(step_in)]
        lab.based_decode_step(d["q"], d["k"], d["v"], S, z, out, d["wq"], d["wk"], d["wv"], kr,
                              vr, wout, pos=w.L + i // 2, window=w.window, eps=w.eps)

    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(n):
        one(i)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    ms = max_over_ranks(ms, dev, world)
    b = decode_bytes(w)
    ach = b / (ms / 1e3) / 1e9
    return {"value": round(world * w.B / (ms / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 5), "steps": n, "batch": w.B, "heads": w.H,
            "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": round(ach, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach / peaks["hbm_gbs"], 4),
                         "traffic": measured_traffic("decode_step"),
                         "algorithmic_bytes": int(b)}}


# ---------------------------------------------------------------------------
# CPU baselines (the fp64 oracle, as it stands)
# ---------------------------------------------------------------------------

def _oracle_step_sample(w, n_lin, n_win, n_tok, threads):
    """Run the oracle on n_lin linear-attention and n_win window sequences of
    the workload, each truncated to its first n_tok tokens; returns seconds."""
    import oracle
    from linear_attention_lm_b200.inputs import prefill_inputs, to_f64
    x = prefill_inputs(w.with_(B=1), device="cpu")
    q, k, v = (to_f64(x[n])[0, :, :n_tok] for n in ("q", "k", "v"))
    wq, wk, wv = (to_f64(x[n])[0, :, :n_tok] for n in ("wq", "wk", "wv"))
    reps_l = int(np.ceil(n_lin / w.H))
    reps_w = int(np.ceil(n_win / w.Hw))
    ql, kl, vl = (np.concatenate([a] * reps_l)[:n_lin] for a in (q, k, v))
    qw, kw, vw = (np.concatenate([a] * reps_w)[:n_win] for a in (wq, wk, wv))
    oracle.build()
    t0 = time.perf_counter()
    oracle.linattn_recurrent(ql, kl, vl, w.eps, threads=threads)
    oracle.window_attn(qw, kw, vw, w.window, threads=threads)
    return time.perf_counter() - t0


def cpu_baseline(w):
    threads = os.cpu_count() or 1
    n_seq = w.B * w.H  # one whole step of the workload
    sec = _oracle_step_sample(w, n_seq, n_seq, w.L, threads)
    tok_per_s = (n_seq * w.L / w.H) / sec  # tokens through all 16 + 16 heads
    return {"value": round(tok_per_s, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n_seq} linear-attention + {n_seq} window sequences of L={w.L} "
                      f"(fp64 recurrent form and direct window softmax), "
                      f"= {n_seq / w.H:.2f} batch rows of the {PREFILL} step"}


def run_reference(args, rank, world):
    """The fp64 oracle on host cores as the reference arm: each step is one
    linear-attention + one window sequence of the workload, truncated to a
    token count that keeps the whole run within a few minutes."""
    from linear_attention_lm_b200.inputs import WORKLOADS
    w = WORKLOADS[PREFILL]
    threads = 1
    budget_s = 150.0
    n_tok = w.L
    probe = _oracle_step_sample(w, 1, 1, 256, threads)
    per_tok = probe / 256
    n_tok = int(max(32, min(w.L, budget_s / max(1, args.steps + args.warmup) / per_tok)))
    for _ in range(args.warmup):
        _oracle_step_sample(w, 1, 1, n_tok, threads)
    t = 0.0
    for _ in range(args.steps):
        t += _oracle_step_sample(w, 1, 1, n_tok, threads)
    # one step pushes n_tok tokens through one head of each layer type; a token
    # of the workload needs 16 + 16 heads
    value = args.steps * n_tok / w.H / t
    sample = (f"per step: 1 linear-attention + 1 window sequence of the {PREFILL} workload, "
              f"first {n_tok} tokens; tokens/s counts a token once all 16+16 heads are done")
    return {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{PREFILL}: B=8 L=2048 d_model=1024; linear attn 16 heads "
                                   f"d=16->273 d_v=64; window-64 attn 16 heads d_h=64",
                       "global_batch": w.B, "seq_len": w.L, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        line = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
