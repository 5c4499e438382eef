"""Benchmark of the Based attention path on B200.

One step = one pass of the prefill hot path over one batch of the
360M-layer-shape workload (B=8, L=2048, d_model=1024): causal Taylor linear
attention over 16 heads (d=16 -> 273 features, d_v=64) with state export, plus
sliding-window-64 softmax attention over 16 heads of d_head=64.  The metric is
tokens/s (B*L per step).  The same run measures every other workload of the
path on one GPU and reports each under "workloads": the fp32 check (B=1, H=2,
L=256), the 1.3B layer shape (d_v = d_head = 128), the 16K-token prefill
(B=1, 128 chunks carried through one state), and the recurrent decode step
(B=128 sequences x 16 + 16 heads, 273x64 fp32 states, 64-slot rings).  Each
carries its kernels' device times, the roofline fraction of each kernel and
the fp64 oracle's time on the host cores for the same workload.

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
OTHER_PREFILL = ("tiny_fp32", "layer_1b3", "long_16k")
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

_KERNEL_SOURCES = {"linattn_prefill": ("linattn_tc.cuh",),
                   "window_attn": ("window_tcp.cuh", "window_softmax.cuh"),
                   "decode_step": ("decode.cuh",)}


def measured_traffic(kernel, workload):
    """DRAM bytes of one launch from the ncu capture of this kernel on this
    workload, or None (no capture of it, or the code changed since)."""
    import hashlib
    csrc = os.path.join(ROOT, "linear_attention_lm_b200", "csrc")
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f)[kernel]
        if entry["workload"] != workload:
            return None
        h = hashlib.sha256()
        for name in (*_KERNEL_SOURCES[kernel], "umma.cuh", "common.cuh"):
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

def linattn_bytes(w, state=True):
    """q, k (d), v, out (d_v) in the input dtype per token-head, + exported states."""
    es = 4 if w.dtype == "f32" else 2
    per_tok = (2 * w.d + 2 * w.dv) * es
    return w.B * w.H * w.L * per_tok + (w.B * w.H * 273 * (w.dv + 1) * 4 if state else 0)


def linattn_flops(w):
    """Minimum FLOPs of the recurrent form with the full 273 features: per
    token-head the state update and the read-out of the numerator (2 F d_v
    each) and of the denominator (2 F each), and the feature maps of q and k."""
    F = 273
    return w.B * w.H * w.L * (4.0 * F * w.dv + 4.0 * F + 2 * 2.0 * F)


def window_bytes(w):
    es = 4 if w.dtype == "f32" else 2
    return w.B * w.Hw * w.L * 4 * w.dh * es


def decode_bytes(w):
    es = 2 if w.dtype == "bf16" else 4
    lin = w.B * w.H * (2 * 273 * (w.dv + 1) * 4 + (2 * w.d + 2 * w.dv) * es)
    win = w.B * w.Hw * (2 * w.window * w.dh * es + 2 * w.dh * es + 4 * w.dh * es)
    return lin + win


def hbm_roofline(kernel, nbytes, ms, peaks, extra=None, workload=None):
    ach = nbytes / (ms / 1e3) / 1e9
    r = {"kernel": kernel, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
         "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
         "traffic": measured_traffic(kernel, workload) if kernel in _KERNEL_SOURCES else None,
         "algorithmic_bytes": int(nbytes), "ms": round(ms, 5), "peak_source": peaks["source"]}
    if extra:
        r.update(extra)
    return r


def tensor_side(w, ms, peaks):
    """The linear-attention prefill against the bf16 tensor-core peak, by its
    minimum (algorithmic) FLOPs."""
    tf = linattn_flops(w) / (ms / 1e3) / 1e12
    return {"flops_min": linattn_flops(w), "tflops_min": round(tf, 1),
            "frac_of_bf16_peak_min_flops": round(tf / peaks["bf16_tflops"], 4)}


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


class ClockWarmer:
    """Keeps the GPU busy for a while right before a timed region, so that the
    SM clock has left its idle level when timing starts (a short timed region
    straight after an idle period would otherwise run partly at a low clock).
    The work is plain writes over a buffer larger than L2, so it also leaves
    L2 holding none of the timed kernels' data."""

    def __init__(self, dev):
        self.buf = torch.empty(64 << 20, dtype=torch.float32, device=dev)  # 256 MB

    def __call__(self, ms: float = 150.0):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        spent, i = 0.0, 0
        while spent < ms:
            for _ in range(8):
                self.buf.fill_(float(i))
                i += 1
            e.record()
            e.synchronize()
            spent = s.elapsed_time(e)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def prefill_config(w, world):
    """The `config` object of a prefill step (shared with the reference arm)."""
    return {"workload": f"{w.name}: B={w.B} L={w.L}" +
                        (f" d_model={w.d_model}" if w.d_model else "") +
                        f"; linear attn {w.H} heads d={w.d}->273 d_v={w.dv} (+state export); "
                        f"window-{w.window} attn {w.Hw} heads d_h={w.dh}; {w.dtype}",
            "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2: input sets rotate between steps (GPU arm)"}


def make_sets(w, dev, min_sets=2):
    """Rotating input/output sets, enough that consecutive steps never find
    their data in L2."""
    from linear_attention_lm_b200.inputs import prefill_inputs
    set_bytes = linattn_bytes(w) + window_bytes(w)
    n_sets = max(min_sets, int(np.ceil(3 * L2_BYTES / set_bytes)))
    n_sets = min(n_sets, 64)
    sets = []
    base = prefill_inputs(w, device=dev)
    for i in range(n_sets):
        x = base if i == 0 else {k: t.clone() for k, t in base.items()}
        outs = {"y": torch.empty_like(x["v"]), "yw": torch.empty_like(x["wq"]),
                "S": torch.empty((w.B, w.H, 273, w.dv), dtype=torch.float32, device=dev),
                "z": torch.empty((w.B, w.H, 273), dtype=torch.float32, device=dev)}
        sets.append((x, outs))
    return sets, set_bytes


def time_prefill(lab, w, sets, steps, warmup, warm, dev, world):
    """Time `steps` prefill steps (linear attention with state export, then
    window attention); returns (total ms, linear ms and window ms per launch
    from event pairs inside the step, launches per step, the same two per-launch
    times with each kernel launched back to back on its own)."""
    ws_bytes = lab.based_linattn_workspace_bytes(w.B, w.H, w.L, w.d, w.dv,
                                                 lab.BASED_BF16 if w.dtype == "bf16" else lab.BASED_F32)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    n_sets = len(sets)

    def lin(i):
        x, o = sets[i % n_sets]
        lab.based_linattn_fwd(x["q"], x["k"], x["v"], o["y"], w.eps, o["S"], o["z"],
                              workspace=ws[:ws_bytes] if ws_bytes else None)

    def win(i):
        x, o = sets[i % n_sets]
        lab.based_window_attn_fwd(x["wq"], x["wk"], x["wv"], o["yw"], w.window)

    def step(i, ev=None):
        if ev is not None:
            ev[0].record()
        lin(i)
        if ev is not None:
            ev[1].record()
        win(i)
        if ev is not None:
            ev[2].record()

    def replayed(body, before=None, after=None):
        # body() captured once as a CUDA graph on a side stream, replayed once
        # untimed (the first launch uploads the graph) and once between the
        # optional events
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            body()
        graph.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        if before is not None:
            before.record()
        graph.replay()
        if after is not None:
            after.record()
        torch.cuda.synchronize()
        del graph

    def chained(fn):
        # K launches of one kernel back to back, each a dependent launch of the
        # previous one as inside the step; one event pair around all of them
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        replayed(lambda: [fn(i) for i in range(steps)], a, b)
        return a.elapsed_time(b) / steps

    warm()
    for i in range(warmup):
        step(i)
    # event-record nodes inside a graph (the per-kernel pass) need external events
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
           for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the step time: the K steps captured once as a CUDA graph (the same C-ABI
    # calls, nothing between the kernels, each kernel a programmatic dependent
    # launch of the previous one, so its set-up overlaps the previous one) and
    # replayed once, so that the host's cost per call does not pace short steps
    replayed(lambda: [step(i) for i in range(steps)], start, stop)
    # the per-kernel times: the same K steps again, replayed the same way, with
    # an event pair around each kernel (an event between two kernels ends their
    # launch overlap, so each time includes its kernel's launch latency); and,
    # for context, each kernel's K launches back to back on their own
    # (launches overlapped, but each kernel's output write-back now competes
    # with its next launch)
    replayed(lambda: [step(i, evs[i]) for i in range(steps)])
    t_lin = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    t_win = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    t_lin_chain = chained(lin)
    t_win_chain = chained(win)
    # the split path adds a state-only pass, and with more than two segments a
    # running sum over their partials (160 x 80 fp32 per 64-column slice)
    n_part = ws_bytes // (w.B * w.H * (w.dv // 64) * 160 * 80 * 4) if ws_bytes else 0
    launches = 2 + (1 if n_part >= 1 else 0) + (1 if n_part >= 2 else 0)
    return start.elapsed_time(stop), t_lin, t_win, launches, t_lin_chain, t_win_chain


def run_ours(args, rank, world, dev):
    import linear_attention_lm_b200 as lab
    from linear_attention_lm_b200 import build as lab_build
    from linear_attention_lm_b200.inputs import WORKLOADS

    if rank == 0:
        lab_build.build()
    if world > 1:
        torch.distributed.barrier()
    lab.load_library()
    peaks = load_peaks()
    warm = ClockWarmer(dev)
    w = WORKLOADS[PREFILL]
    sets, set_bytes = make_sets(w, dev)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.2)  # let the sampler start
        # the clock record covers the conditioning burn right before the timed
        # steps as well: a timed region of a few ms holds at most one sample
        clk.mark("t_start")
        warm()
        elapsed_ms, t_lin, t_win, launches, t_lin_p, t_win_p = time_prefill(
            lab, w, sets, args.steps, args.warmup, lambda: warm(30.0), dev, world)
        clk.mark("t_stop")
    assert lab.based_get_device_error() == 0
    elapsed_max = max_over_ranks(elapsed_ms, dev, world)
    value = replica_rate(w.B * w.L * args.steps, elapsed_max, world)

    # roofline of the dominant kernel (both are HBM-bound by algorithmic bytes)
    kern = {"linattn_prefill": (linattn_bytes(w), t_lin), "window_attn": (window_bytes(w), t_win)}
    dom = max(kern, key=lambda k: kern[k][1])
    b, t_ms = kern[dom]
    roofline = hbm_roofline(dom, b, t_ms, peaks, workload=w.name)
    chain = {"linattn_prefill": t_lin_p, "window_attn": t_win_p}
    roofline["per_kernel_ms"] = {k: round(v[1], 5) for k, v in kern.items()}
    roofline["per_kernel_timing"] = (
        "CUDA event pairs around each kernel, over a second pass of the same K steps right "
        "after the timed one (each pair includes its kernel's launch latency, which the "
        "step itself overlaps with the previous kernel); per_kernel_ms_chained: each "
        "kernel's K launches back to back on their own, on the same inputs")
    roofline["per_kernel_frac"] = {k: round(v[0] / (v[1] / 1e3) / 1e9 / peaks["hbm_gbs"], 4)
                                   for k, v in kern.items()}
    roofline["per_kernel_ms_chained"] = {k: round(v, 5) for k, v in chain.items()}
    roofline["per_kernel_frac_chained"] = {
        k: round(kern[k][0] / (v / 1e3) / 1e9 / peaks["hbm_gbs"], 4) for k, v in chain.items()}
    roofline["linattn_prefill_tensor"] = tensor_side(w, t_lin, peaks)
    del sets

    workloads = {PREFILL: {"tokens_per_s": round(value, 1),
                           "ms_per_step": round(elapsed_max / args.steps, 5),
                           "kernels": {"linattn_prefill": hbm_roofline(
                               "linattn_prefill", linattn_bytes(w), t_lin, peaks,
                               tensor_side(w, t_lin, peaks), workload=w.name),
                               "window_attn": hbm_roofline("window_attn", window_bytes(w),
                                                           t_win, peaks, workload=w.name)}}}
    for name in OTHER_PREFILL:
        workloads[name] = run_other_prefill(args, lab, WORKLOADS[name], dev, world, peaks, warm)
    decode = run_decode(args, lab, dev, world, peaks, warm)
    workloads[DECODE] = decode
    e2e = run_e2e(args, w, lab, dev, world, warm)
    try:
        projections = run_projections(args, lab, dev, world, peaks, warm)
    except Exception as exc:  # reported in the JSON line, never hidden
        projections = {"error": f"{type(exc).__name__}: {exc}"}
    clocks = clk.summary()
    clocks["window"] = "150 ms clock-conditioning burn + warm-up + timed steps"
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_max / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": prefill_config(w, world),
        "roofline": roofline,
        "e2e": e2e,
        "decode": {k: decode[k] for k in ("value", "unit", "ms_per_step", "steps", "roofline")},
        "workloads": workloads,
        "projections": projections,
        "gpu_launches": launches * args.steps,
        "step_timing": "CUDA events around one replay of a CUDA graph of the K steps, captured "
                       "from the same C-ABI calls; per-kernel times from event pairs around each "
                       "kernel in a second graph of the same steps",
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
        for name in OTHER_PREFILL:
            workloads[name]["cpu_baseline"] = cpu_baseline(WORKLOADS[name])
        workloads[PREFILL]["cpu_baseline"] = line["cpu_baseline"]
        workloads[DECODE]["cpu_baseline"] = cpu_baseline_decode(WORKLOADS[DECODE])
    return line


def run_other_prefill(args, lab, w, dev, world, peaks, warm):
    """One of the other prefill workloads: K1 (with state export) and K2 timed
    per kernel over rotating input sets; tokens/s = B L / (K1 + K2)."""
    sets, _ = make_sets(w, dev)
    n = max(10, min(args.steps, 200))
    total_ms, t_lin, t_win, launches, t_lin_p, t_win_p = time_prefill(lab, w, sets, n, args.warmup,
                                                                        warm, dev, world)
    assert lab.based_get_device_error() == 0
    del sets
    ms = max_over_ranks(total_ms / n, dev, world)
    lin = hbm_roofline("linattn_prefill", linattn_bytes(w), t_lin, peaks,
                       tensor_side(w, t_lin, peaks) if w.dtype == "bf16" else None,
                       workload=w.name)
    win = hbm_roofline("window_attn", window_bytes(w), t_win, peaks, workload=w.name)
    lin["ms_chained"] = round(t_lin_p, 5)
    win["ms_chained"] = round(t_win_p, 5)
    out = {"workload": prefill_config(w, world)["workload"],
           "tokens_per_s": round(world * w.B * w.L / (ms / 1e3), 1),
           "ms_per_step": round(ms, 5), "steps": n, "launches_per_step": launches,
           "kernels": {"linattn_prefill": lin, "window_attn": win}}
    if w.dtype == "f32":
        out["note"] = ("fp32 CUDA-core path; a few hundred tokens per head, so the launch "
                       "latency, not HBM, bounds it")
    return out


def run_e2e(args, w, lab, dev, world, warm):
    """Same step through the public API from pinned host buffers: every step
    copies its inputs host->device, runs both kernels (the linear attention
    with state export, as in the device-timed step), and copies both outputs
    and the exported states device->host.  Steps are pipelined the way a
    caller would run them: the inputs of step i+1 travel (copy stream) while
    step i computes (compute stream) and the outputs of step i-1 come back (a
    third stream), with two device buffer sets; PCIe carries both directions
    at once."""
    from linear_attention_lm_b200.inputs import prefill_inputs
    x = prefill_inputs(w, device=dev)
    n = max(2, min(args.steps, 30))
    host_in = {k: t.to("cpu").pin_memory() for k, t in x.items()}
    S_shape, z_shape = (w.B, w.H, 273, w.dv), (w.B, w.H, 273)

    def host_outs():
        return {"y": torch.empty(x["v"].shape, dtype=x["v"].dtype).pin_memory(),
                "yw": torch.empty(x["wq"].shape, dtype=x["wq"].dtype).pin_memory(),
                "S": torch.empty(S_shape, dtype=torch.float32).pin_memory(),
                "z": torch.empty(z_shape, dtype=torch.float32).pin_memory()}

    host_out = [host_outs() for _ in range(2)]
    dev_in = [{k: torch.empty_like(t, device=dev) for k, t in x.items()} for _ in range(2)]
    dev_out = [{"y": torch.empty_like(dev_in[0]["v"]), "yw": torch.empty_like(dev_in[0]["wq"]),
                "S": torch.empty(S_shape, dtype=torch.float32, device=dev),
                "z": torch.empty(z_shape, dtype=torch.float32, device=dev)} for _ in range(2)]
    del x
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
            o = dev_out[b]
            lab.based_linattn_fwd(dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["v"], o["y"], w.eps,
                                  o["S"], o["z"], stream=s_run)
            lab.based_window_attn_fwd(dev_in[b]["wq"], dev_in[b]["wk"], dev_in[b]["wv"], o["yw"],
                                      w.window, stream=s_run)
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            for k in host_out[b]:
                host_out[b][k].copy_(dev_out[b][k], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    warm(30.0)
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


def run_projections(args, lab, dev, world, peaks, warm):
    """The rows next to the hot path, each on layer_360m's shapes (synthetic):
    the six per-head input projections of one linear-attention and one window
    layer (x [8, 2048, 1024] bf16; q, k: 16 heads of 16; v and the window's q,
    k, v: 16 heads of 64), one BaseConv block (D = 1024, 3 taps), and the
    backward of both attention layers.  Four rotating x buffers (128 MB) keep
    L2 cold for the projections."""
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
        warm(30.0)
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

    w_cat = torch.cat(ws, 0).contiguous()

    def proj_step(i):
        # the six projections of a layer pair in one launch (x streamed once)
        lab.based_proj_heads_multi_fwd(xs[i % 4], w_cat, ys)

    def torch_proj_step(i):
        # the same product by torch's matmul (cuBLAS), row-major [B*L, 4608]
        # output, no split into heads: a lower bound on the library's time
        torch.matmul(xs[i % 4].view(B * L, dm), w_cat.t())

    def torch_conv_gemm(i):
        torch.matmul(xs[i % 4].view(B * L, dm), wb.t())

    def conv_step(i):
        lab.based_baseconv_fwd(xs[i % 4], wb, bias, taps, yb)

    # backward of both attention layers, layer_360m shape, CUDA cores (fp32 FMA)
    qb = (torch.randn(B, H, L, 16, device=dev, generator=g) * 0.25).to(torch.bfloat16)
    kb = (torch.randn(B, H, L, 16, device=dev, generator=g) * 0.25).to(torch.bfloat16)
    vb = torch.randn(B, H, L, 64, device=dev, generator=g).to(torch.bfloat16)
    dyb = torch.randn(B, H, L, 64, device=dev, generator=g).to(torch.bfloat16)
    gq, gk = torch.empty(B, H, L, 16, device=dev), torch.empty(B, H, L, 16, device=dev)
    gv = torch.empty(B, H, L, 64, device=dev)
    wsb = torch.empty(lab.based_linattn_bwd_workspace_bytes(B, H, L, 64), dtype=torch.uint8,
                      device=dev)
    wq_, wk_ = (torch.randn(B, H, L, 64, device=dev, generator=g) * 0.25).to(torch.bfloat16), \
        (torch.randn(B, H, L, 64, device=dev, generator=g) * 0.25).to(torch.bfloat16)
    gwq, gwk, gwv = (torch.empty(B, H, L, 64, device=dev) for _ in range(3))
    wsw = torch.empty(lab.based_window_attn_bwd_workspace_bytes(B, H, L), dtype=torch.uint8,
                      device=dev)

    def bwd_step(i):
        lab.based_linattn_bwd(qb, kb, vb, dyb, gq, gk, gv, 1e-6, workspace=wsb)

    def wbwd_step(i):
        lab.based_window_attn_bwd(wq_, wk_, vb, dyb, gwq, gwk, gwv, 64, workspace=wsw)

    out = {}
    peak = peaks["bf16_tflops"]
    # window backward: per (query, key) pair in the band, S, dP (2 x 2 dh), dq, dk, dv
    # (3 x 2 dh) -> 10 dh flop; W (W + 1) / 2 + W (L - W) pairs per head
    w_pairs = 64 * 65 / 2 + 64 * (L - 64)
    for name, fn, flops, launches, what in (
            ("proj", proj_step, 2.0 * B * L * dm * H * sum(heads), 1,
             "six per-head projections of x [8, 2048, 1024] in one launch: q, k 16x16; v 16x64; "
             "window q, k, v 16x64"),
            ("baseconv", conv_step, 2.0 * B * L * dm * dm, 1,
             "BaseConv block, x [8, 2048, 1024], dense 1024x1024 + bias, 3 causal taps"),
            ("linattn_bwd", bwd_step, 480.0 * B * H * L * (L + 1) / 2, 2,
             "gradient of the linear attention, bf16, B=8 H=16 L=2048 d=16 d_v=64 (quadratic "
             "form on the tensor cores; 480 flop per (t, s) pair counted)"),
            ("window_bwd", wbwd_step, 10.0 * 64 * B * H * w_pairs, 2,
             "gradient of the window attention, bf16, B=8 H=16 L=2048 d_h=64 W=64 on the "
             "tensor cores (q, k, v, dy read in bf16, dq, dk, dv written in fp32, 3 fp32 "
             "statistics per query written and read; 10 d_h flop per (query, key) pair in "
             "the band)")):
        ms = timed(fn, 10 if name == "linattn_bwd" else n)
        tf = flops / (ms / 1e3) / 1e12
        if name == "linattn_bwd":
            kern, bound, pk, src = "linattn_bwd_tc", "tensor", peak, peaks["source"]
        elif name == "window_bwd":
            kern, bound = "window_bwd_tc", "hbm"
        else:
            kern, bound, pk, src = "proj_tc", "tensor", peak, peaks["source"]
        out[name] = {"workload": what, "ms_per_step": round(ms, 5), "launches_per_step": launches,
                     "tokens_per_s": round(world * B * L / (ms / 1e3), 1)}
        if bound == "hbm":
            # bytes per token-head: 4 x 2 d_h (bf16 in) + 3 x 4 d_h (fp32 out) + 3 x 4 x 2
            nbytes = B * H * L * (4 * 2 * 64 + 3 * 4 * 64 + 24)
            out[name]["roofline"] = hbm_roofline(kern, nbytes, ms, peaks)
            out[name]["tflops"] = round(tf, 2)
        else:
            out[name]["roofline"] = {"kernel": kern, "bound": bound, "achieved": round(tf, 2),
                                     "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                                     "traffic": None, "peak_source": src}
        if name in ("proj", "baseconv"):
            # library context: torch.matmul of the same GEMM (no epilogue, no head split)
            tms = timed(torch_proj_step if name == "proj" else torch_conv_gemm, n)
            out[name]["torch_matmul"] = {"ms": round(tms, 5),
                                         "tflops": round(flops / (tms / 1e3) / 1e12, 2)}
    assert lab.based_get_device_error() == 0
    return out


def run_decode(args, lab, dev, world, peaks, warm):
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

    warm()
    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(n):
        one(i)
    e.record()
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    ms = s.elapsed_time(e) / n
    ms = max_over_ranks(ms, dev, world)
    b = decode_bytes(w)
    return {"workload": f"{w.name}: B={w.B} sequences, {w.H} linear heads (273x{w.dv} fp32 "
                        f"state) + {w.Hw} window heads ({w.window}-slot bf16 ring, d_h={w.dh}), "
                        f"after a {w.L}-token prefill",
            "value": round(world * w.B / (ms / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 5), "steps": n, "batch": w.B, "heads": w.H,
            "roofline": hbm_roofline("decode_step", b, ms, peaks, workload=w.name)}


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
    oracle.linattn_recurrent(ql, kl, vl, w.eps, threads=threads, return_state=True)
    oracle.window_attn(qw, kw, vw, w.window, threads=threads)
    return time.perf_counter() - t0


def cpu_baseline(w, threads=None):
    threads = threads or os.cpu_count() or 1
    n_seq = w.B * w.H  # one whole step of the workload
    sec = _oracle_step_sample(w, n_seq, w.B * w.Hw, w.L, threads)
    tok_per_s = w.B * w.L / sec  # tokens through all heads of both layers
    return {"value": round(tok_per_s, 1), "unit": UNIT, "cores": min(threads, n_seq),
            "kind": "oracle",
            "sample": f"one whole step of {w.name}: {n_seq} linear-attention sequences (fp64 "
                      f"recurrent form, with the final state) + {w.B * w.Hw} window sequences "
                      f"(direct window softmax) of L={w.L}"}


def cpu_baseline_decode(w, n_steps=4):
    """The oracle's decode steps (single-threaded C, as it stands) over all
    B x (H + H_w) sequences of the decode workload, for n_steps steps."""
    import oracle
    from linear_attention_lm_b200.inputs import decode_step_inputs, to_f64
    F = 273
    S = np.zeros((w.B, w.H, F, w.dv))
    z = np.zeros((w.B, w.H, F))
    kr = np.zeros((w.B, w.Hw, w.window, w.dh))
    vr = np.zeros_like(kr)
    ins = [{k: to_f64(t) for k, t in decode_step_inputs(w, s).items()} for s in range(n_steps)]
    oracle.build()
    t0 = time.perf_counter()
    for s, d in enumerate(ins):
        oracle.decode_linear(d["q"], d["k"], d["v"], S, z, w.eps)
        oracle.decode_window(d["wq"], d["wk"], d["wv"], kr, vr, w.L + s, w.window)
    sec = time.perf_counter() - t0
    return {"value": round(w.B * n_steps / sec, 1), "unit": "tokens/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{n_steps} decode steps of all {w.B} sequences x ({w.H} linear + {w.Hw} "
                      f"window heads) of {w.name}"}


def run_reference(args, rank, world):
    """The fp64 oracle on host cores as the reference arm, on the same
    workload, config, thread count and sample as the cpu_baseline leg: each
    step is one whole step of the layer_360m workload (all 128 linear-attention
    and 128 window sequences of L = 2048), run on all host cores."""
    from linear_attention_lm_b200.inputs import WORKLOADS
    w = WORKLOADS[PREFILL]
    threads = os.cpu_count() or 1
    n_seq = w.B * w.H
    for _ in range(args.warmup):
        _oracle_step_sample(w, n_seq, w.B * w.Hw, w.L, threads)
    t = 0.0
    for _ in range(args.steps):
        t += _oracle_step_sample(w, n_seq, w.B * w.Hw, w.L, threads)
    value = args.steps * w.B * w.L / t
    sample = (f"one whole step of {w.name}: {n_seq} linear-attention sequences (fp64 "
              f"recurrent form, with the final state) + {w.B * w.Hw} window sequences "
              f"(direct window softmax) of L={w.L}")
    return {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": prefill_config(w, world),
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT,
                             "cores": min(threads, n_seq), "kind": "oracle", "sample": sample},
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
