"""Benchmark: causal kernelized linear attention on B200.

One step = one pass of the hot path over one batch of synthetic input:
``la_prefill`` over the headline workload ``gdelta_bf16`` (the largest
single-GPU configuration: gated delta rule, B=1, H=32, N=65536,
d=dv=128, bf16 inputs, fp32 state).  The metric is prefill tokens/s
(tokens = B*N per step; each token carries H heads) and the roofline
fraction of the call's dominant kernel.

Timing: W untimed warm-up steps, then K timed steps.  Inputs stay resident in
HBM; L2 is flushed (a 256 MiB write, outside the timed events) before every
timed step.  Each step is timed with CUDA events on the stream the kernels
run on; for N GPUs every rank processes its own full batch (independent
problems: weak scaling, no data-path collective) and the time is the max
over ranks.  ``--gpus N`` starts the N ranks itself (one process per GPU)
unless it runs under torchrun, whose WORLD_SIZE must then equal N.

``other_workloads`` carries the other configurations, each with its own
roofline and end-to-end numbers: plain and decay kernelized prefill, the
fp32 prefill, the decode steps (kernelized and gated delta, 1000 chained
steps), GLA, the short causal convolution and a variable-length batch.

Printed: one JSON line (rank 0).  ``--impl reference`` times the float64 CPU
oracle (the only reference this method has) on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from causal_kernelized_linear_la_b200 import inputs  # noqa: E402

HEADLINE = "gdelta_bf16"
METRIC = "prefill tokens/s and decode state-updates/s on 1 B200; % of roofline"
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# work accounting (algorithmic bytes / flops per step: what the recurrence itself
# must read, write and compute, not the chunk form's extra work)

def prefill_units(p) -> dict:
    """Tokens, token-heads and the method's own bytes/flops for one prefill."""
    eb = 2 if p.dtype == "bf16" else 4
    th = p.B * p.H * p.N
    chains = p.B * p.H
    byts = th * (2 * p.d + 2 * p.dv) * eb + chains * p.d * p.dv * 4
    if p.mode == "gated_delta":
        byts += th * 8  # alpha, g fp32
        flops = th * 6 * p.d * p.dv
    elif p.mode == "gla":
        byts += th * p.d * 4  # the per-channel gate, fp32
        flops = th * 5 * p.d * p.dv
    else:
        byts += chains * p.d * 4
        flops = th * (4 * p.d * p.dv + 4 * p.d)
    return {"tokens": p.B * p.N, "token_heads": th, "bytes": byts, "flops": flops}


def decode_units(Bs, Hh, d, dv, eb=2, gated=False) -> dict:
    """Bytes one decode step must move: the fp32 state read and written, the
    token in and the output out (kernelized: z read and written too; gated
    delta: alpha and g in)."""
    states = Bs * Hh
    side = 8 if gated else 2 * d * 4
    byts = states * (2 * d * dv * 4 + side + (2 * d + 2 * dv) * eb)
    return {"state_updates": states, "tokens": Bs, "bytes": byts, "flops": states * 4 * d * dv}


def workload_desc(name: str) -> str:
    w = inputs.WORKLOADS[name]
    if w["kind"] == "decode":
        return f"{name}: decode step, {w['S']} sequences x {w['H']} heads, d=dv={w['d']}, fp32 state, bf16 tokens"
    if w["kind"] == "decode_gated_delta":
        return (f"{name}: gated delta decode step, {w['S']} sequences x {w['H']} heads, d=dv={w['d']}, "
                f"fp32 state, bf16 tokens, alpha and g per step")
    what = {"plain": "plain causal prefill with normaliser", "decay": "per-head decay prefill with decayed normaliser",
            "gated_delta": "gated delta rule prefill", "gla": "per-key-channel gated (GLA) prefill"}[
        w.get("mode", w["kind"])]
    return (f"{name}: B={w['B']} H={w['H']} N={w['N']} d=dv={w['d']} {w['dtype']} inputs, {what}")


# ----------------------------------------------------------------------------
# clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, path: str | None):
        self.idx = device_index
        self.path = path
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = open(self.path, "w") if self.path else subprocess.PIPE
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.text = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            if self.path:
                self.out.close()
                self.text = open(self.path).read()
            else:
                self.text = out or ""

    def summary(self) -> dict:
        rows = []
        for line in self.text.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append({"sm": float(f[1]), "max": float(f[2]), "util": float(f[4]),
                             "hw": f[6], "hwt": f[7], "swt": f[8], "pcap": f[9]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        busy = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(busy)}


# ----------------------------------------------------------------------------
# distributed plumbing (weak scaling: each rank owns an independent batch)

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Rank r processes an independent batch drawn with seed base + 1000 r."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------------------
# GPU arm

def _measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def _to_dev(x, torch):
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _prefill_device_args(p, torch):
    if p.dtype == "bf16":
        q, k, v = _to_dev(p.q_bits, torch), _to_dev(p.k_bits, torch), _to_dev(p.v_bits, torch)
    else:
        q, k, v = _to_dev(p.q, torch), _to_dev(p.k, torch), _to_dev(p.v, torch)
    kw = {}
    if p.mode == "decay":
        kw["gamma"] = _to_dev(p.gamma, torch)
    if p.mode == "gated_delta":
        kw["alpha"], kw["g"] = _to_dev(p.alpha, torch), _to_dev(p.g, torch)
    if p.mode == "gla":
        kw["alpha"] = _to_dev(p.alpha, torch)
    return q, k, v, kw


def time_prefill(p, steps, warmup, torch, la, flush):
    """Device time per step (ms) of la_prefill on resident inputs, L2 flushed
    before every timed step; returns (list of ms, launches per step, buffers)."""
    q, k, v, kw = _prefill_device_args(p, torch)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    out = torch.empty((B, H, N, dv), device="cuda", dtype=q.dtype)
    S_out = torch.empty((B, H, d, dv), device="cuda", dtype=torch.float32)
    z_out = None if p.mode in ("gated_delta", "gla") else torch.empty((B, H, d), device="cuda", dtype=torch.float32)
    ws_bytes = la.la_prefill_workspace_bytes(B, H, N, d, dv, p.dtype, p.mode)
    ws = torch.empty(max(ws_bytes, 16), device="cuda", dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step():
        la.la_prefill(q, k, v, mode=p.mode, eps=p.eps, out=out, S_out=S_out, z_out=z_out, workspace=ws, **kw)

    for _ in range(warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(1)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    la.la_prefill_check(ws)
    return [a.elapsed_time(b) for a, b in ev]


def _pinned(x, torch):
    """A pinned host tensor holding numpy array x (bf16 bit patterns as int16)."""
    if x is None:
        return None
    a = np.ascontiguousarray(x)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).pin_memory()


def time_e2e(host, call, steps, warmup, torch):
    """End to end through the public API with host buffers: every step copies
    the pinned host tensors ``host`` (name -> tensor) into device twins, runs
    ``call(device_tensors)`` (which returns the device results) and copies the
    results back into pinned host buffers, all inside the CUDA events.  Steps
    run as a serving loop would run them: the inputs of step i + 1 go in on one
    copy stream while step i computes and step i - 1's results come out on
    another (the two directions of the bus run at once); two sets of device
    input buffers alternate, and a step computes only after the previous
    step's results are out (so ``call`` may reuse its output buffers).
    Returns (ms per step, H2D bytes per step, D2H bytes per step)."""
    sets = [{n: torch.empty(t.shape, dtype=t.dtype, device="cuda") for n, t in host.items()} for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = torch.cuda.Event()
    outs_h = []
    state = {"i": 0}

    def step():
        i = state["i"]
        state["i"] += 1
        k = i % 2
        dev = sets[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[k])     # the set's previous step has computed
            for n, t in host.items():
                dev[n].copy_(t, non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[k])
            if i >= 1:
                s_comp.wait_event(out_done)       # the previous step's results are out
            outs = call(dev)
            comp_done[k].record(s_comp)
        if not outs_h:
            outs_h.extend(torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            for h, o in zip(outs_h, outs):
                h.copy_(o, non_blocking=True)
                o.record_stream(s_out)
            out_done.record(s_out)

    main = torch.cuda.current_stream()
    for st in (s_in, s_comp, s_out):
        st.wait_stream(main)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for st in (s_in, s_comp, s_out):
        st.wait_event(a)
    for _ in range(steps):
        step()
    for st in (s_in, s_comp, s_out):
        main.wait_stream(st)
    b.record(main)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    return a.elapsed_time(b) / steps, h2d, d2h


def time_prefill_e2e(p, steps, warmup, torch, la):
    """la_prefill end to end: q, k, v (and gamma / alpha / g) from pinned host
    memory, the output o copied back, every step inside the events."""
    host = {"q": _pinned(p.q_bits if p.dtype == "bf16" else p.q, torch),
            "k": _pinned(p.k_bits if p.dtype == "bf16" else p.k, torch),
            "v": _pinned(p.v_bits if p.dtype == "bf16" else p.v, torch)}
    if p.mode == "decay":
        host["gamma"] = _pinned(p.gamma, torch)
    if p.mode in ("gated_delta", "gla"):
        host["alpha"] = _pinned(p.alpha, torch)
    if p.mode == "gated_delta":
        host["g"] = _pinned(p.g, torch)
    tdt = torch.bfloat16 if p.dtype == "bf16" else torch.float32

    def call(d):
        kw = {n: d[n] for n in ("gamma", "alpha", "g") if n in d}
        o, _, _ = la.la_prefill(d["q"].view(tdt), d["k"].view(tdt), d["v"].view(tdt), mode=p.mode, eps=p.eps, **kw)
        return [o]

    return time_e2e(host, call, steps, warmup, torch)


def time_decode(steps, warmup, torch, la, seed, gated=False, Bs=256, Hh=32, d=128, dv=128, pool=8):
    """Device time per decode step (ms) over `steps` chained steps on the
    resident state; tokens come from a pool of `pool` pre-generated steps
    (identical cost per step).  Returns (ms per step, end-to-end record)."""
    st = inputs.make_decode_state(Bs, Hh, d, dv, seed=seed)
    S = torch.from_numpy(st.S).cuda()
    z = torch.from_numpy(st.z).cuda()
    toks = []
    for s in range(pool):
        if gated:
            t = inputs.make_gated_delta_decode_token(s, Bs, Hh, d, dv, seed=seed)
            arrs = (t.q_bits, t.k_bits, t.v_bits, t.alpha, t.g)
        else:
            t = inputs.make_decode_token(s, Bs, Hh, d, dv, seed=seed)
            arrs = (t.q_bits, t.k_bits, t.v_bits)
        toks.append(arrs)
    dtoks = [tuple(_to_dev(x, torch) for x in a) for a in toks]
    out = torch.empty((Bs, Hh, dv), device="cuda", dtype=torch.bfloat16)

    def run(tk, o):
        if gated:
            return la.la_gated_delta_decode_step(*tk, S, out=o)
        return la.la_decode_step(*tk, S, z, out=o)

    for i in range(warmup):
        run(dtoks[i % pool], out)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        run(dtoks[i % pool], out)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps

    # end to end: each step's token from pinned host memory, o back to the
    # host; the state stays resident on the device (the decode cache)
    names = ("q", "k", "v", "alpha", "g") if gated else ("q", "k", "v")
    hosts = [dict(zip(names, (_pinned(x, torch) for x in a))) for a in toks]
    cur = {"i": 0}
    host = dict(hosts[0])

    def call(dd):
        cur["i"] += 1
        for n in names:   # the next token's host buffers for the next step
            host[n] = hosts[cur["i"] % pool][n]
        tk = [dd["q"].view(torch.bfloat16), dd["k"].view(torch.bfloat16), dd["v"].view(torch.bfloat16)]
        if gated:
            tk += [dd["alpha"], dd["g"]]
        return [run(tk, None)]

    e_ms, h2d, d2h = time_e2e(host, call, 200, 5, torch)
    return ms, (e_ms, h2d, d2h)


def roofline_block(nbytes, kms, hbm_peak, peak_kind, workload, call_ms):
    """The roofline object of one call: algorithmic bytes over the dominant
    kernel's CUDA-event time, against the measured HBM copy bandwidth."""
    dom = max(kms, key=kms.get)
    achieved = nbytes / (kms[dom] / 1e3) / 1e9
    call_gbs = nbytes / (call_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
            "traffic": captured_traffic(workload, dom), "kernel": dom, "kernel_ms": kms[dom],
            "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": nbytes,
            "call_kernels_ms": kms, "whole_call": {"achieved": call_gbs, "frac": call_gbs / hbm_peak}}


def measure_prefill(name, p, steps, warmup, torch, la, flush, e2e_steps=10):
    """Device-timed throughput, per-kernel roofline and end-to-end numbers of
    one prefill workload.  Returns (record, list of per-step ms)."""
    hbm_peak, _, peak_kind = _measured_peaks()
    u = prefill_units(p)
    ms = time_prefill(p, steps, warmup, torch, la, flush)
    med = statistics.median(ms)
    kms = time_kernels(p, max(3, min(steps, 20)), torch, la, flush)
    e_ms, h2d, d2h = time_prefill_e2e(p, e2e_steps, 2, torch, la)
    rec = {"workload": workload_desc(name), "value": u["tokens"] / (med / 1e3), "unit": "tokens/s", "ms": med,
           "dtype": path_dtype(p), "roofline": roofline_block(u["bytes"], kms, hbm_peak, peak_kind, name, med),
           "e2e": {"value": u["tokens"] / (e_ms / 1e3), "unit": "tokens/s", "ms": e_ms,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
           "gpu_launches_per_call": la_launches_per_step(p)}
    return rec, ms


def measure_decode(name, torch, la, rank):
    hbm_peak, _, peak_kind = _measured_peaks()
    spec = inputs.WORKLOADS[name]
    gated = spec["kind"] == "decode_gated_delta"
    steps = spec["steps"]
    ms, (e_ms, h2d, d2h) = time_decode(steps, 20, torch, la, rank_seed(spec["seed"], rank), gated=gated,
                                       Bs=spec["S"], Hh=spec["H"], d=spec["d"], dv=spec["dv"])
    du = decode_units(spec["S"], spec["H"], spec["d"], spec["dv"], gated=gated)
    kernel = "decode_gated_delta" if gated else "decode_kernelized"
    gbs = du["bytes"] / (ms / 1e3) / 1e9
    return {"workload": workload_desc(name), "value": du["state_updates"] / (ms / 1e3), "unit": "state-updates/s",
            "tokens_per_s": du["tokens"] / (ms / 1e3), "ms_per_step": ms, "chained_steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": captured_traffic(name, kernel), "kernel": kernel, "kernel_ms": ms,
                         "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": du["bytes"]},
            "e2e": {"value": du["state_updates"] / (e_ms / 1e3), "unit": "state-updates/s", "ms": e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "note": "token in from pinned host memory and o out every step; the state stays resident"},
            "gpu_launches_per_call": 1}


def init_dist(world, local):
    """Process group of this rank (NCCL on GPUs, gloo where there are none)."""
    import datetime
    import torch
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return backend


def finish_line(line, world):
    """Close the rank's process group (after a last barrier) and print the
    line on rank 0."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if int(os.environ.get("RANK", "0")) == 0:
        print(json.dumps(line), flush=True)


def run_gpu(args, world, rank, local):
    import torch
    import causal_kernelized_linear_la_b200 as la

    torch.cuda.set_device(local)
    if world > 1:
        init_dist(world, local)
    hbm_peak, tc_peak, peak_kind = _measured_peaks()
    spec = inputs.WORKLOADS[args.workload]
    over = {"N": args.seq_len} if args.seq_len else {}
    p = inputs.make_workload(args.workload, seed=rank_seed(spec["seed"], rank), **over)
    u = prefill_units(p)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()

    # the SM clock record of the timed region: kept under --clocks-dir, else
    # in a temporary file that is removed once read
    if args.clocks_dir:
        clocks_path = os.path.join(args.clocks_dir, f"clocks_rank{rank}.csv")
    else:
        clocks_path = os.path.join(tempfile.gettempdir(), f"la_bench_clocks_{os.getpid()}_rank{rank}.csv")
    with ClockSampler(local, clocks_path) as clk:
        barrier()
        ms = time_prefill(p, args.steps, args.warmup, torch, la, flush)
        barrier()
        # the kernel split of the call, the other workloads: the device stays
        # busy, so the clock sampler sees the load
        kms = time_kernels(p, max(3, min(args.steps, 20)), torch, la, flush)
        extra = {}
        if not args.no_extra:
            extra = run_extra(args, torch, la, rank, flush)
    local_total_ms = sum(ms)
    total_ms = max_over_ranks(local_total_ms, world, device="cuda")
    ms_per_step = total_ms / args.steps
    value = aggregate_throughput(u["tokens"] * args.steps, world, total_ms / 1e3)
    e2e_ms, h2d, d2h = time_prefill_e2e(p, max(3, min(args.steps, 20)), 2, torch, la)
    e2e_ms = max_over_ranks(e2e_ms, world, device="cuda")
    e2e_value = aggregate_throughput(u["tokens"], world, e2e_ms / 1e3)
    clk_sum = clk.summary()
    if not args.clocks_dir:
        try:
            os.remove(clocks_path)
        except OSError:
            pass

    avg_launch_ms = local_total_ms / args.steps
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": path_dtype(p),
        "data": "synthetic (seeded numpy normal draws of the workload's shape and scale)",
        "config": {"workload": workload_desc(args.workload), "global_batch": p.B * world, "seq_len": p.N,
                   "heads": p.H, "d": p.d, "dv": p.dv, "parallelism": f"replicas x{world} (independent batches)",
                   "l2": "flushed before every timed step (256 MiB write outside the timed events); "
                         "the inputs also exceed L2"},
        "roofline": roofline_block(u["bytes"], kms, hbm_peak, peak_kind, args.workload, avg_launch_ms),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": la_launches_per_step(p) * args.steps,
        "clocks": clk_sum,
        "rank_seeds": [rank_seed(spec["seed"], r) for r in range(world)],
    }
    if args.seq_len:
        line["config"]["note"] = "seq_len overridden for profiling; not the benchmark configuration"
    if extra:
        line["other_workloads"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_seconds)
    finish_line(line, world)


def path_dtype(p) -> str:
    return "f32" if p.dtype == "f32" else "bf16"


def call_kernels(p) -> list:
    """The kernels one la_prefill call launches for this workload, in launch
    order (the dispatch documented with la_set_stage_events in include/la.h;
    the library reports how many)."""
    import causal_kernelized_linear_la_b200 as la
    n = la.la_prefill_kernel_count(p.B, p.H, p.N, p.d, p.dv, p.dtype, p.mode)
    if p.mode == "gla":
        names = ["gla_summary_kernel", "gla_scan_kernel", "gla_chunk_kernel"] if p.dtype == "bf16" else ["gla_token_simt"]
    elif p.dtype == "bf16" and p.mode in ("plain", "decay"):
        names = ["summary_kernel", "scan_kernel", "chunk_kernel"]
    elif p.dtype == "bf16":
        names = ["gd_prep_kernel", "gd_chain_kernel"] * (n // 2)   # one pair per part of the sequence
    elif p.mode == "gated_delta":
        names = ["gated_delta_token_simt"]
    else:   # fp32 kernelized: the parallel form for short sequences, else the chunk loop
        names = ["kernelized_parallel_simt", "kernelized_state_simt"] if n == 2 else ["kernelized_chunk_simt"]
    assert len(names) == n, (names, n)
    return names


def la_launches_per_step(p) -> int:
    """Kernels of ours one la_prefill call launches."""
    return len(call_kernels(p))


# DRAM traffic of one launch of a kernel, from a one-pass ncu capture of that
# kernel alone (--metrics dram__bytes_read.sum,dram__bytes_write.sum
# --clock-control none, one launch) in the workload's launch configuration.
# A capture holds only while the kernel's source is unchanged: the entry
# records the source file's sha256 at capture time, and the benchmark reports
# null when the file differs now.
TRAFFIC_CAPTURES = {
    # one call's eight chain launches (8 parts, 72 ... 204 chunks)
    ("gdelta_bf16", "gd_chain_kernel"): {
        "bytes": 2721121024 + 408967168, "source": "causal_kernelized_linear_la_b200/csrc/la_gdelta_tc.cu",
        "sha256": "16f1b3dfdea98f964829fc419b4ccc15394068910c17a373dc30ca1ff4b51191"},
    ("plain_bf16", "chunk_kernel"): {
        "bytes": 54631424 + 760064, "source": "causal_kernelized_linear_la_b200/csrc/la_prefill_tc.cu",
        "sha256": "2d1423379900cb8bcbda6d09bcd00835f6410ba5de2a92d2bc6ad2add4531edd"},
    ("decay_bf16", "chunk_kernel"): {
        "bytes": 824389888 + 209698560, "source": "causal_kernelized_linear_la_b200/csrc/la_prefill_tc.cu",
        "sha256": "2d1423379900cb8bcbda6d09bcd00835f6410ba5de2a92d2bc6ad2add4531edd"},
    ("gla_bf16", "gla_chunk_kernel"): {
        "bytes": 344009216 + 34973440, "source": "causal_kernelized_linear_la_b200/csrc/la_gla_tc.cu",
        "sha256": "635c8cade52f824b03c80c4f7dd276d836c8dc69d0eb41394c1641fffd759e46"},
}


def _file_sha256(rel):
    import hashlib
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def captured_traffic(workload, kernel):
    t = TRAFFIC_CAPTURES.get((workload, kernel))
    if not t or not t["sha256"]:
        return None
    try:
        return t["bytes"] if _file_sha256(t["source"]) == t["sha256"] else None
    except OSError:
        return None


def time_kernels(p, steps, torch, la, flush):
    """Average device time (ms) of each kernel of the call, from CUDA events the
    library records after each launch (la_set_stage_events) on the launching
    stream, L2 flushed before every step.  A separate pass from the headline
    timing, so the headline carries no extra event records."""
    q, k, v, kw = _prefill_device_args(p, torch)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    out = torch.empty((B, H, N, dv), device="cuda", dtype=q.dtype)
    S_out = torch.empty((B, H, d, dv), device="cuda", dtype=torch.float32)
    z_out = None if p.mode in ("gated_delta", "gla") else torch.empty((B, H, d), device="cuda", dtype=torch.float32)
    ws_bytes = la.la_prefill_workspace_bytes(B, H, N, d, dv, p.dtype, p.mode)
    ws = torch.empty(max(ws_bytes, 16), device="cuda", dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    names = call_kernels(p)
    start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    marks = [[torch.cuda.Event(enable_timing=True) for _ in names] for _ in range(steps)]
    for e in start + [m for row in marks for m in row]:
        e.record(stream)          # creates the underlying CUDA events
    torch.cuda.synchronize()
    per = [[] for _ in names]
    try:
        for i in range(steps):
            flush.fill_(1)
            la.la_set_stage_events(marks[i])
            start[i].record(stream)
            la.la_prefill(q, k, v, mode=p.mode, eps=p.eps, out=out, S_out=S_out, z_out=z_out, workspace=ws, **kw)
        torch.cuda.synchronize()
    finally:
        la.la_set_stage_events(None)
    for i in range(steps):
        prev = start[i]
        for j, m in enumerate(marks[i]):
            per[j].append(prev.elapsed_time(m))
            prev = m
    la.la_prefill_check(ws)
    # kernels launched more than once per call (one per part of the sequence)
    # are summed: the gaps between consecutive events are each kernel's share
    # of the call
    res = {}
    for n, t in zip(names, per):
        res[n] = res.get(n, 0.0) + sum(t) / len(t)
    return res


def _timed_calls(call, steps, flush, torch):
    """Median device time (ms) of `call`, L2 flushed before each, 3 warm-ups."""
    stream = torch.cuda.current_stream()
    for _ in range(3):
        flush.fill_(1)
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.fill_(1)
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def time_conv(torch, la, rank, flush, B=4, H=8, N=4096, d=64, w=4, steps=20):
    """The short causal convolution (with conv cache) over one q-shaped bf16
    stream of the plain workload's size, filter width 4: device time per
    call, L2 flushed before each, its bytes against HBM, and end to end."""
    hbm_peak, _, peak_kind = _measured_peaks()
    g = torch.Generator(device="cpu").manual_seed(rank_seed(77, rank))
    xh = (torch.randn((B, H, N, d), generator=g) / 8).to(torch.bfloat16)
    wt = (torch.randn((H, d, w), generator=g) / 2).cuda()
    c0h = torch.randn((B, H, w - 1, d), generator=g).to(torch.bfloat16)
    x, c0 = xh.cuda(), c0h.cuda()
    out = torch.empty_like(x)
    c1 = torch.empty_like(c0)
    ms = _timed_calls(lambda: la.la_causal_conv(x, wt, c0, out=out, cache_out=c1), steps, flush, torch)
    nbytes = 2 * x.numel() * 2 + wt.numel() * 4 + 2 * c0.numel() * 2
    host = {"x": xh.view(torch.int16).pin_memory(), "c": c0h.view(torch.int16).pin_memory()}

    def call(dd):
        o = torch.empty_like(x)
        c = torch.empty_like(c0)
        la.la_causal_conv(dd["x"].view(torch.bfloat16), wt, dd["c"].view(torch.bfloat16), out=o, cache_out=c)
        return [o, c]

    e_ms, h2d, d2h = time_e2e(host, call, 20, 3, torch)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": f"short causal conv, x [B={B},H={H},N={N},d={d}] bf16, w={w}, conv cache in and out",
            "value": B * N / (ms / 1e3), "unit": "tokens/s", "ms": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": None, "kernel": "causal_conv_kernel", "kernel_ms": ms,
                         "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": nbytes},
            "e2e": {"value": B * N / (e_ms / 1e3), "unit": "tokens/s", "ms": e_ms, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches_per_call": 1}


def time_varlen(torch, la, rank, flush, H=8, N=4096, d=64, steps=20):
    """A right-padded batch of eight plain bf16 sequences of mixed lengths
    (head size and padded length of the plain workload) through
    la_prefill_varlen, which runs it as one launch set: device time per call,
    L2 flushed before each."""
    hbm_peak, _, peak_kind = _measured_peaks()
    g = torch.Generator(device="cpu").manual_seed(rank_seed(91, rank))
    lens = [4096, 3000, 2048, 1500, 1000, 700, 300, 65]
    B = len(lens)
    q, k, v = ((torch.randn((B, H, N, d), generator=g) / 8).to(torch.bfloat16).cuda() for _ in range(3))
    out = torch.empty_like(v)
    S = torch.empty((B, H, d, d), device="cuda")
    z = torch.empty((B, H, d), device="cuda")
    ws = torch.empty(max(la.la_prefill_varlen_workspace_bytes(lens, H, d, d), 16), device="cuda",
                     dtype=torch.uint8)
    ms = _timed_calls(lambda: la.la_prefill_varlen(q, k, v, lens, out=out, S_out=S, z_out=z, workspace=ws),
                      steps, flush, torch)
    tokens = sum(lens)
    nbytes = tokens * H * 4 * d * 2 + B * H * (d * d + d) * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": f"variable-length batch: B={B} H={H} padded N={N} d=dv={d} bf16 plain, lengths {lens}",
            "value": tokens / (ms / 1e3), "unit": "tokens/s", "ms": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": None, "kernel": "whole call", "kernel_ms": ms,
                         "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": nbytes},
            "gpu_launches_per_call": 3}   # one launch set (summaries, scan, chunk loop) for the batch


def run_extra(args, torch, la, rank, flush):
    """The other workloads, each with its own roofline and end-to-end numbers."""
    res = {}
    names = [n for n in ("plain_bf16", "decay_bf16", "gdelta_bf16", "plain_f32", "gla_bf16") if n != args.workload]
    for name in names:
        spec = inputs.WORKLOADS[name]
        p = inputs.make_workload(name, seed=rank_seed(spec["seed"], rank))
        steps = {"plain_f32": 50, "gla_bf16": 3, "plain_bf16": 20}.get(name, 5)
        res[name], _ = measure_prefill(name, p, steps, 3, torch, la, flush, e2e_steps=3 if name == "gla_bf16" else 10)
        del p
    res["decode"] = measure_decode("decode", torch, la, rank)
    res["gdelta_decode"] = measure_decode("gdelta_decode", torch, la, rank)
    res["conv"] = time_conv(torch, la, rank, flush)
    res["varlen_bf16"] = time_varlen(torch, la, rank, flush)
    return res


# ----------------------------------------------------------------------------
# CPU arm: the float64 oracle

def cpu_baseline(workload: str, budget_s: float = 15.0, max_tokens: int | None = None) -> dict:
    """Time the oracle as it stands on a bounded sample of the workload: whole
    chains (or, with max_tokens, the first max_tokens tokens of each chain),
    as many as fit the budget; at least one call of as many chains as there
    are host threads (up to the workload's head count)."""
    import oracle
    spec = inputs.WORKLOADS[workload]
    threads = oracle.threads()
    H = max(1, min(spec["H"], threads))
    N = spec["N"] if max_tokens is None else min(spec["N"], max_tokens)
    p = inputs.make_workload(workload, B=1, H=H, N=N)
    chains = 0
    t0 = time.perf_counter()
    elapsed = 0.0
    while elapsed < budget_s or chains == 0:
        if p.mode == "gated_delta":
            oracle.gated_delta(p.q, p.k, p.v, p.alpha, p.g)
        elif p.mode == "gla":
            oracle.gla(p.q, p.k, p.v, p.alpha)
        else:
            oracle.kernelized(p.q, p.k, p.v, p.gamma, eps=p.eps)
        chains += H
        elapsed = time.perf_counter() - t0
    token_heads = chains * p.N
    value = token_heads / spec["H"] / elapsed  # tokens/s (a token carries H heads)
    what = "whole chains" if N == spec["N"] else f"chains cut to their first {N} tokens"
    return {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{chains} {what} of N={p.N} tokens ({token_heads} token-heads) of {workload}, "
                      f"{elapsed:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    spec = inputs.WORKLOADS[args.workload]
    # each step: one oracle call over as many chains as there are host
    # threads, cut to a prefix so the whole run stays within minutes
    prefix = 8192
    for _ in range(args.warmup):
        cpu_baseline(args.workload, budget_s=0.0, max_tokens=prefix)
    samples, per_step = [], []
    for _ in range(args.steps):
        cb = cpu_baseline(args.workload, budget_s=0.0, max_tokens=prefix)
        samples.append(cb)
        per_step.append(spec["B"] * spec["N"] / cb["value"] * 1e3)
    value = statistics.median(s["value"] for s in samples)
    cb = dict(samples[0])
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.median(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(args.workload)}, "impl": "reference",
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# entry point and rank launcher

def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_entry(rank, n, port, fn, fn_args):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    fn(*fn_args)


def spawn_ranks(n: int, fn, fn_args=()) -> None:
    """Run fn(*fn_args) in n fresh processes, one per GPU, with the torchrun
    environment (RANK = LOCAL_RANK = r, WORLD_SIZE = n, MASTER_ADDR =
    127.0.0.1 and a free MASTER_PORT); raises if any rank fails."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_entry, args=(n, _free_port(), fn, tuple(fn_args)), nprocs=n, join=True,
                       start_method="spawn")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=[k for k, v in inputs.WORKLOADS.items()
                                                              if not v["kind"].startswith("decode")])
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--clocks-dir", default=None,
                    help="keep the nvidia-smi clock samples of the timed region here (clocks_rank<r>.csv)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="profiling aid: the workload with this many tokens per chain instead of its own "
                         "(the line's config says so); not a benchmark configuration")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    args.steps = max(1, args.steps)
    args.gpus = max(1, args.gpus)
    return args


def run_rank(argv):
    """One rank of the benchmark (rank, world size from the environment)."""
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_gpu(args, world, rank, local)


def main(argv=None):
    args = parse_args(argv)
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        # no launcher: start one process per GPU here
        spawn_ranks(args.gpus, run_rank, (argv if argv is not None else sys.argv[1:],))
        return
    if env_world is not None and int(env_world) != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started WORLD_SIZE={env_world} ranks")
    run_rank(argv)


if __name__ == "__main__":
    main()
