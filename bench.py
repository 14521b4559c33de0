#!/usr/bin/env python
"""Store-h decode attention throughput on B200: cached positions per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one full decode step of the workload: for every loop iteration,
append the new token's h row (quantised) and run store-h attention with the
per-iteration safety check, for every lane.  Inputs are synthetic and seeded.
Timing: CUDA events on the launching stream, W untimed warm-up steps, K timed
steps bracketed by a barrier and a device synchronize, max over ranks.
Each rank (N > 1) runs its own independent batch (weak scaling, no collective
on the data path).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "store-h decode attention cached positions/s on 1 B200; % of roofline"
UNIT = "cached positions/s"
DEFAULT_WORKLOAD = "int4_2b"
DTYPE_OF_FMT = {0: "fp16", 1: "int8", 2: "int4"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-seconds", type=float, default=20.0, help="budget of the CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="decode: time the headline and per-step passes as eager calls instead of replays of "
                        "a CUDA graph of one step")
    p.add_argument("--path", default="decode", choices=["decode", "verify", "prefill", "delta", "rope"],
                   help="decode (the headline); verify / prefill: tree verification / chunked prefill over the "
                        "cache; delta: the iteration-axis delta cache; rope: the rotary-embedding variant")
    p.add_argument("--branches", type=int, default=4, help="verify: draft branches per lane")
    p.add_argument("--depth", type=int, default=4, help="verify: tokens per branch")
    p.add_argument("--tokens", type=int, default=16, help="prefill: tokens per lane per chunk")
    p.add_argument("--lanes", type=int, default=8, help="delta: lanes (the workload's shape otherwise)")
    p.add_argument("--split-rows", type=int, default=0,
                   help="context rows per split of every decode call (tl_decode_opts.split_rows; 0 = the default 1024)")
    return p.parse_args()


# ----------------------------------------------------------------------------- shared helpers
def workload_for_rank(name, rank):
    from synth.workloads import get_workload
    import dataclasses
    w = get_workload(name)
    if rank:
        w = dataclasses.replace(w, seed=w.seed + 1000 * rank)   # an independent batch per rank
    return w


def max_over_ranks(value, world, device):
    """The largest of every rank's `value` (each rank gets it); `value` itself on one rank."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, steps, ms_max, world):
    """Units all ranks processed per second, timed by the slowest rank (weak scaling: every rank
    has its own batch of the same shape)."""
    return world * steps * units_per_rank_step / (ms_max / 1000.0)


def row_bytes(w):
    return {0: 2 * w.d, 1: w.d + 4, 2: w.d // 2 + 2 * (w.d // 64)}[w.fmt]


def workload_config(w, n_gpus, extra=None):
    cfg = {"workload": w.name, "d_model": w.d, "n_heads": w.H, "head_dim": w.hd, "n_pre": w.n_pre,
           "L_max": w.L_max, "h_format": DTYPE_OF_FMT[w.fmt], "batch_per_gpu": w.B,
           "ctx_per_lane": (w.ctx[0] if len(set(w.ctx)) == 1 else "U[1024,8192] seeded"),
           "loops_per_lane": (w.loops[0] if len(set(w.loops)) == 1 else "16x4,16x16,16x32"),
           "global_batch": w.B * n_gpus, "parallelism": f"lanes x{n_gpus} (independent batches)",
           "cache_inputs_vs_l2": "cache read per step > 126 MB L2 (no flush needed)"}
    if extra:
        cfg.update(extra)
    return cfg


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class OracleSample:
    """A bounded sample of the workload for the plain C++ FP64 oracle: whole (lane, iteration)
    decodes -- append of the new row, exact dequantisation, explicit K/V rebuild, softmax,
    safety check -- each with its lane's cached rows quantised once beforehand (not timed)."""

    def __init__(self, w):
        self.w = w
        self.pairs = [(it, b) for it in range(w.L_max) for b in range(w.B) if it < w.loops[b]]
        self.prepared = {}
        self.W = [w.weight(k) for k in "qkv"]

    def _prepare(self, i):
        import oracle.cpp as ocpp
        if i not in self.prepared:
            w = self.w
            it, b = self.pairs[i % len(self.pairs)]
            codes, scales = ocpp.quantize_rows(w.h_rows(w.n_pre + it, b, 0, w.ctx[b]), w.fmt)
            self.prepared[i] = (it, b, codes, scales, w.h_new(it)[b], w.residual(it)[b])
        return self.prepared[i]

    def decode(self, i, threads):
        """Time the oracle as it stands on pair i with `threads` OpenMP threads (over heads)."""
        import oracle.cpp as ocpp
        it, b, codes, scales, hn, res = self._prepare(i)
        w = self.w
        t0 = time.perf_counter()
        ocpp.decode_lane(w.fmt, codes, scales, hn, *self.W, w.H, w.hd, residual=res, threshold=w.threshold, it=it,
                         loops=w.loops[b], form=0, threads=threads)
        return w.ctx[b], time.perf_counter() - t0

    def run(self, budget_s, threads, max_pairs=None, first=0):
        """Decode pairs first, first+1, ... until the budget is spent; returns (positions/s, s, n, positions)."""
        pos, spent, n = 0, 0.0, 0
        while n == 0 or (spent < budget_s and (max_pairs is None or n < max_pairs)):
            p, t = self.decode(first + n, threads)
            pos, spent, n = pos + p, spent + t, n + 1
        return pos / spent, spent, n, pos


def cpu_baseline(w, budget_s):
    """The C++ oracle on the host cores: single-threaded, and with OpenMP over the heads of a
    lane (the (lane, head) tasks of the sample), on a bounded sample of (lane, iteration) pairs
    of the workload, extrapolated linearly to the whole step (positions/s is per position)."""
    import oracle.cpp as ocpp
    sample = OracleSample(w)
    threads = min(ocpp.max_threads(), w.H)
    v1, s1, n1, p1 = sample.run(budget_s / 2, threads=1, max_pairs=1)
    vm, sm, nm, pm = sample.run(budget_s / 2, threads=threads, first=1)
    desc = (f"plain C++ FP64 oracle (append + exact dequant + explicit K/V rebuild + softmax + norm check) on "
            f"{nm} (lane, iteration) decodes of {w.name} ({pm} cached positions, {sm:.2f} s) with {threads} OpenMP "
            f"threads over the heads; single-threaded: {n1} decode ({p1} positions, {s1:.2f} s) = {v1:.4g} "
            f"positions/s; rates extrapolated linearly from the sample to the whole step "
            f"({w.cached_positions_per_step()} positions); host {os.cpu_count()} logical CPUs, {cpu_model()}")
    return {"value": vm, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
            "single_thread_value": v1, "nproc": os.cpu_count(), "cpu_model": cpu_model(), "extrapolated": True}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_sha():
    """Hash of the streaming kernel's translation unit: k_stream_tc.cu and every header it
    pulls in with #include "...", from the package sources or include/."""
    dirs = [os.path.join(ROOT, "store_kv_attention_b200", "csrc"), os.path.join(ROOT, "include")]
    seen, todo = {}, ["k_stream_tc.cu"]
    while todo:
        fn = todo.pop()
        if fn in seen:
            continue
        path = next(os.path.join(d, fn) for d in dirs if os.path.exists(os.path.join(d, fn)))
        with open(path, "rb") as f:
            seen[fn] = f.read()
        todo += re.findall(r'^\s*#\s*include\s+"([^"]+)"', seen[fn].decode(), flags=re.M)
    h = hashlib.sha256()
    for fn in sorted(seen):
        h.update(fn.encode() + seen[fn])
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch of the streaming kernel from a committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "stream_kernel_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(workload)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import torch
        ident = None
        try:
            ident = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        self.cmd = ["nvidia-smi", "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits", "-lms", "100"]
        if ident:
            self.cmd += ["-i", ident]
        self.proc = None

    def __enter__(self):
        import threading
        self.lines = []
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                if line.strip():
                    self.lines.append(line)
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        # the first sample comes after nvidia-smi has started: wait for it (bounded), so that the
        # timed region is covered
        t0 = time.time()
        while not self.lines and time.time() - t0 < 10.0 and self.proc.poll() is None:
            time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)  # one more sample period after the timed work
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle.cpp as ocpp
    w = workload_for_rank(args.workload, 0)
    sample = OracleSample(w)
    threads = min(ocpp.max_threads(), w.H)
    # a step = a bounded sample of the workload: one (lane, iteration) decode, OpenMP over its heads
    for k in range(args.warmup):
        sample.run(0.0, threads, max_pairs=1, first=k)
    t, pos = 0.0, 0
    for k in range(args.steps):
        _, s_, _, p_ = sample.run(0.0, threads, max_pairs=1, first=args.warmup + k)
        t += s_
        pos += p_
    value = pos / t
    desc = (f"per step: one (lane, iteration) decode of {w.name} by the plain C++ FP64 oracle (append + exact "
            f"dequant + explicit K/V rebuild + softmax + norm check), {threads} OpenMP threads over the heads; "
            f"{pos} cached positions in {t:.2f} s over {args.steps} steps, extrapolated linearly to the step's "
            f"{w.cached_positions_per_step()} positions; host {os.cpu_count()} logical CPUs, {cpu_model()}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * w.cached_positions_per_step() / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                             "nproc": os.cpu_count(), "cpu_model": cpu_model(), "extrapolated": True},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload

    torch.cuda.set_device(local_rank)
    w = workload_for_rank(args.workload, rank)
    dw = DeviceWorkload(w, device=f"cuda:{local_rank}", split_rows=args.split_rows)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        dw.step(fused_append=True)
    torch.cuda.synchronize()
    if tl.poll_status(dw.cache) != tl.TL_OK:
        raise RuntimeError("device status after warm-up: " + tl.lib.tl_last_error_message().decode())
    # One step (every loop iteration's tl_storeh_append_attn_decode call) captured as a CUDA graph:
    # the same launches with the same arguments, replayed without the host's per-call overhead.
    run_step = lambda: dw.step(fused_append=True)
    launch_mode = "eager calls"
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                dw.step(fused_append=True)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            with torch.cuda.graph(graph):
                dw.step(fused_append=True)
            for _ in range(max(3, args.warmup)):
                graph.replay()
            torch.cuda.synchronize()
            run_step = graph.replay
            launch_mode = ("replays of a CUDA graph of one step (the step's calls captured once); the kernel pass "
                           "and e2e run as eager calls")
        except RuntimeError as e:  # capture unsupported here: time eager calls and say so
            torch.cuda.synchronize()
            launch_mode = "eager calls (CUDA-graph capture failed: %s)" % str(e).splitlines()[0][:120]
        if tl.poll_status(dw.cache) != tl.TL_OK:
            raise RuntimeError("device status after graph warm-up: " + tl.lib.tl_last_error_message().decode())

    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.__enter__()  # samples through every timed pass below, the end-to-end one included
    # headline pass: the steps alone (an event between two kernels would stop the next one
    # from being scheduled during the previous one's tail, so none is recorded in here)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(K):
        run_step()
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    # per-step pass: the same K steps, each between its own pair of events (median reported)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b_ in step_ev:
        a.record(stream)
        run_step()
        b_.record(stream)
    torch.cuda.synchronize()
    step_ms_median = statistics.median(a.elapsed_time(b_) for a, b_ in step_ev)
    barrier()
    # kernel pass: the same K steps again, with events around every streaming-kernel launch
    with tl.ProfileHook(K * w.L_max) as prof:
        for _ in range(K):
            dw.step(fused_append=True)
        torch.cuda.synchronize()
    ms_max = max_over_ranks(start.elapsed_time(end), world, f"cuda:{local_rank}")
    step_ms_median = max_over_ranks(step_ms_median, world, f"cuda:{local_rank}")
    pos_step = w.cached_positions_per_step()
    value = whole_job_rate(pos_step, K, ms_max, world)

    # dominant kernel (context streaming): algorithmic bytes per launch / CUDA-event duration
    kms = prof.stream_kernel_ms()
    rb = row_bytes(w)
    bytes_per_launch = [sum((w.ctx[b] + 1) * rb for b in range(w.B) if it < w.loops[b]) for it in range(w.L_max)]
    total_bytes = sum(bytes_per_launch[i % w.L_max] for i in range(len(kms)))
    achieved_gbs = total_bytes / (sum(kms) / 1000.0) / 1e9
    peak, peak_kind = load_peaks()
    traffic = recorded_traffic(w.name)
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                "frac": achieved_gbs / peak, "traffic": traffic, "peak_source": peak_kind,
                "kernel": "stream (context streaming: dequant, scores, softmax, p.h)",
                "algorithmic_bytes_per_launch": statistics.mean(bytes_per_launch),
                "avg_launch_ms": statistics.mean(kms),
                "timed_in": "second pass of the same K steps, CUDA events around every streaming-kernel launch"}
    step_bytes = sum(bytes_per_launch) + 3 * 2 * w.d * w.d
    step_roofline_ms = step_bytes / (peak * 1e9) * 1e3

    # end to end through the public API: pinned host inputs in, results out, every step.  Inputs
    # and results are double-buffered on the device: step k+1's inputs are copied in (one copy
    # stream) while step k runs, and step k's results are read back (another copy stream) while
    # step k+1 runs; events order every reuse of a buffer.
    h_new_host = dw.h_new.cpu().pin_memory()
    res_host = dw.residual.cpu().pin_memory()
    out_host = torch.empty(dw.out.shape, dtype=torch.float32).pin_memory()
    flags_host = torch.empty(w.B, dtype=torch.uint8).pin_memory()
    first_host = torch.empty(w.B, dtype=torch.int32).pin_memory()
    h2d = h_new_host.numel() * 2 + res_host.numel() * 4
    d2h = out_host.numel() * 4 + w.B + w.B * 4
    names = ("h_new", "residual", "out", "flags", "first", "norms")
    sets = [{n: getattr(dw, n) for n in names}, {n: torch.empty_like(getattr(dw, n)) for n in names}]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    inputs_ready = [ev(), ev()]    # set i's inputs are on the device
    inputs_free = [ev(), ev()]     # the step that read set i's inputs is done
    results_read = [ev(), ev()]    # set i's results are on the host

    def upload(i):
        with torch.cuda.stream(up):
            up.wait_event(inputs_free[i])
            sets[i]["h_new"].copy_(h_new_host, non_blocking=True)
            sets[i]["residual"].copy_(res_host, non_blocking=True)
            inputs_ready[i].record(up)

    barrier()
    torch.cuda.synchronize()
    for i in range(2):
        inputs_free[i].record(stream)
        results_read[i].record(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    upload(0)
    for k in range(K):
        i = k & 1
        if k + 1 < K:
            upload(i ^ 1)
        stream.wait_event(inputs_ready[i])
        stream.wait_event(results_read[i])  # this set's results of two steps back are on the host
        for n in names:
            setattr(dw, n, sets[i][n])
        dw.reset_flags()
        dw.step(fused_append=True)
        inputs_free[i].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(inputs_free[i])
            out_host.copy_(dw.out, non_blocking=True)
            flags_host.copy_(dw.flags, non_blocking=True)
            first_host.copy_(dw.first, non_blocking=True)
            results_read[i].record(down)
    stream.wait_event(results_read[(K - 1) & 1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks.__exit__(None, None, None)
    for n in names:
        setattr(dw, n, sets[0][n])
    e2e_value = whole_job_rate(pos_step, K, max_over_ranks(e0.elapsed_time(e1), world, f"cuda:{local_rank}"), world)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": DTYPE_OF_FMT[w.fmt] + "-h codes, fp16 tensor operands, fp32 accumulate",
            "data": "synthetic (seeded generator: SplitMix64 + Box-Muller)",
            "config": workload_config(w, world, {"entry_point": ("tl_storeh_append_attn_decode per loop iteration" if not
                                                                 args.split_rows else
                                                                 "tl_storeh_decode_ex (append=1, split_rows=%d) per "
                                                                 "loop iteration" % args.split_rows),
                                                 "split_rows": args.split_rows or 1024,
                                                 "cached_positions_per_step_per_gpu": pos_step,
                                                 "step_roofline_ms_hbm": step_roofline_ms,
                                                 "ms_per_step_median_of_per_step_events": step_ms_median,
                                                 "timing": ("value and ms_per_step: K steps between one event "
                                                            "pair (no event between kernels); the median of K "
                                                            "per-step event pairs is reported beside it"),
                                                 "launch": launch_mode,
                                                 "step_frac_of_hbm_roofline": step_roofline_ms / (ms_max / K)}),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": prof.launches,
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- other paths
def load_tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s (the two have the same nominal rate on B200)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), "measured (bf16 burst; fp16 has the same nominal dense rate)"
    return 1590.0, "fallback"


def run_path(args, rank, world, local_rank):
    """One JSON line for a path other than the headline decode: its own units, the step time, and
    the roofline of its dominant kernel (events around every launch of it)."""
    import numpy as np
    import torch
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    w = workload_for_rank(args.workload, rank)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + w.seed)
    rb = row_bytes(w)
    extra = {}
    if args.path in ("verify", "prefill"):
        K, D = (args.branches, args.depth) if args.path == "verify" else (1, args.tokens)
        dw = DeviceWorkload(w, device=dev, max_ctx=max(w.ctx) + K * D + 1)
        # tree / chunk states: seeded normals on the device (timing inputs only)
        trees = [torch.randn((w.B, K, D, w.d), generator=gen, device=dev).half() for _ in range(w.L_max)]
        ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, K, D), dtype=torch.uint8, device=dev)
        out = torch.empty((w.B, K, D, w.H, w.hd), dtype=torch.float32, device=dev)

        def step():
            for it in range(w.L_max):
                tl.verify_attn(dw.cache, it, dw.loops, dw.ctx, trees[it], dw.W["q"], dw.W["k"], dw.W["v"], out, ws)

        act = [[b for b in range(w.B) if it < w.loops[b]] for it in range(w.L_max)]
        units = sum(w.ctx[b] * K * D + K * D * (D + 1) // 2 for it in range(w.L_max) for b in act[it])
        unit_name = "attended (query, row) pairs/s"
        launch_bytes = [sum((w.ctx[b] + K * D) * rb for b in act[it]) for it in range(w.L_max)]
        launches_per_it = -(-w.B * K * D // 64)
        extra = {"branches": K, "depth": D, "query_tokens_per_lane": K * D,
                 "roofline_note": "unique cache bytes (each row once from HBM) over the streaming launches of "
                                  "an iteration; every query token streams its rows as a lane of its own"}
        bound, peak, peak_kind, unit = "hbm", *load_peaks(), "GB/s"
    elif args.path == "delta":
        B = min(args.lanes, w.B)
        ctx = w.ctx[0]
        L = w.L_max
        desc = tl.DeltaDesc(w.d, w.H, w.hd, L, B, ctx + 1)
        cache = tl.DeltaCache(desc, device=dev, n_lanes=B)
        # trajectories on the device: h^0 ~ N(0,1), h^l = h^(l-1) + sigma_l z with the contraction
        # schedule of the synthetic generator (|dh|/|h| from 0.68 down to 0.04 over 32 iterations)
        traj = [torch.randn((B, ctx + 1, w.d), generator=gen, device=dev)]
        for l in range(1, L):
            rho = 0.68 * (0.04 / 0.68) ** ((l - 1) / 31)
            prev = traj[-1]
            sigma = rho * prev.norm(dim=2, keepdim=True) / math.sqrt(w.d * (1 - rho * rho))
            traj.append(prev + sigma * torch.randn(prev.shape, generator=gen, device=dev))
        traj = [t.half() for t in traj]
        zeros = torch.zeros(B, dtype=torch.int32, device=dev)
        for it in range(L):
            tl.delta_append(cache, it, traj[it][:, :ctx].contiguous(), zeros)
        loops = torch.full((B,), L, dtype=torch.int32, device=dev)
        ctx_d = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        h_new = [traj[it][:, ctx].contiguous() for it in range(L)]
        W = [torch.from_numpy(np.ascontiguousarray(w.weight(k)).view(np.int16)).view(torch.float16).to(dev)
             for k in "qkv"]
        out = torch.empty((B, w.d), dtype=torch.float32, device=dev)

        def step():
            for it in range(L):
                tl.delta_attn_decode(cache, it, loops, ctx_d, h_new[it], *W, out)

        units = B * ctx * L
        unit_name = UNIT
        launch_bytes = [B * (ctx + 1) * (2 * w.d + it * (w.d + 2 * w.H)) for it in range(L)]
        launches_per_it = 1
        extra = {"lanes": B, "delta_rows_per_position_at_iteration_l": "anchor (2d B) + l x (d + 2 H) B",
                 "inputs": "trajectories drawn on the device (seeded torch normals, the generator's schedule)"}
        bound, peak, peak_kind, unit = "hbm", *load_peaks(), "GB/s"
    else:  # rope
        dw = DeviceWorkload(w, device=dev)
        ws = torch.zeros(tl.rope_workspace_bytes(dw.desc, w.B), dtype=torch.uint8, device=dev)

        def step():
            for it in range(w.L_max):
                dw.append_new(it)
                tl.attn_decode_rope(dw.cache, it, dw.loops, dw.ctx, dw.h_new[it], dw.W["q"], dw.W["k"],
                                    dw.W["v"], dw.out[it], ws, residual=dw.residual[it], threshold=w.threshold,
                                    abort_flags=dw.flags, first_abort_iter=dw.first)

        units = w.cached_positions_per_step()
        unit_name = UNIT
        # the score kernel's contraction: K = h W_k^T for every attended row (2 d^2 FLOPs per row)
        launch_bytes = [sum(2.0 * (w.ctx[b] + 1) * w.d * w.d for b in range(w.B) if it < w.loops[b])
                        for it in range(w.L_max)]
        launches_per_it = 1
        extra = {"rope_base": 10000.0}
        bound, (peak, peak_kind), unit = "tensor", load_tensor_peak(), "TFLOP/s"

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K_ = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.__enter__()
    e0.record()
    for _ in range(K_):
        step()
    e1.record()
    torch.cuda.synchronize()
    with tl.ProfileHook(K_ * w.L_max * launches_per_it) as prof:
        for _ in range(K_):
            step()
        torch.cuda.synchronize()
    clocks.__exit__(None, None, None)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    kms = prof.stream_kernel_ms()
    per_it = [sum(kms[i * launches_per_it:(i + 1) * launches_per_it]) for i in range(len(kms) // launches_per_it)]
    total = sum(launch_bytes[i % w.L_max] for i in range(len(per_it)))
    achieved = total / (sum(per_it) / 1000.0) / (1e9 if unit == "GB/s" else 1e12)
    if rank != 0:
        return
    line = {"metric": f"{args.path} over the store-h cache: {unit_name} on 1 B200", "value":
            world * K_ * units / (ms / 1000.0), "unit": unit_name, "n_gpus": world, "steps": K_,
            "warmup": args.warmup, "ms_per_step": ms / K_, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "path": args.path,
            "config": workload_config(w, world, extra),
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                         "traffic": None, "peak_source": peak_kind,
                         "algorithmic_per_iteration": statistics.mean(launch_bytes),
                         "kernel_ms_per_iteration": statistics.mean(per_it)},
            "gpu_launches": prof.launches, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.path != "decode":
            run_path(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
