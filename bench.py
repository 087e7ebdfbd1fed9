"""Benchmark of the GQA attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one gqa_attention_fwd call (main kernel + LSE combine) over the
workload's inputs, already resident in HBM.  L2 is flushed (256 MB write)
between timed steps; each step is timed with CUDA events on the stream the
library launches on, and the reported time is the max over ranks.  The default
workload is the batched decode (B=16, Hq=32, Hkv=4, Tq=1, Tkv=16384, d=128,
ragged kv_len ~ U[1, 16384], NaN padding), measured in GB/s of algorithmic
bytes (K/V rows visible to some query row, plus Q, O and lse); prefill
workloads are measured in TFLOP/s (4*d flops per visible query/key pair).

By default the same run then times every other workload of the metric (tiny
prefill, short-q/long-kv prefill, full causal prefill, wide-head sink decode)
the same way, with fewer steps and a shorter oracle sample, and reports each in
a "workloads" block of the one JSON line (value, roofline, cpu_baseline, e2e,
clocks); --only keeps to --workload.  Step times are reported as mean (the
value) and median.

Multi-GPU: the path needs no exchange, so N GPUs run N independent replicas
(weak scaling); `value` sums the work of all ranks over the slowest rank's time.

--impl reference runs the fp64 oracle (the CPU reference of this build) on the
host cores, on bounded samples of the same workload, and prints the same line
with "impl": "reference".
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload, make_inputs, paginate  # noqa: E402

METRIC = "GQA fwd TFLOP/s (prefill) & KV HBM GB/s (decode), 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures (HGX HBM3e bandwidth, dense bf16 tensor rate), for context beside the measured peaks
SPEC_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
L2_FLUSH_BYTES = 256 << 20
PREFILL = {"full_causal_prefill"}


# ------------------------------------------------------------------ work counting

def visible_keys(w: Workload, n: int, i: int) -> int:
    last = (n - w.Tq + i) if w.causal else (n - 1)
    last = min(last, n - 1)
    return max(0, last + 1)


def unit_work(w: Workload, n: int):
    """Algorithmic bytes and flops of one (batch, KV head) unit with length n."""
    pairs_per_head = sum(visible_keys(w, n, i) for i in range(w.Tq))
    keys = max((visible_keys(w, n, i) for i in range(w.Tq)), default=0)
    kv_bytes = 2 * keys * w.d * (1 if w.kv_fp8 else 2)  # E4M3 caches: one byte per element
    q_o_bytes = 2 * w.G * w.Tq * w.d * 2 + w.G * w.Tq * 4
    flops = 4 * w.d * pairs_per_head * w.G
    return kv_bytes + q_o_bytes, flops


def workload_work(w: Workload, kv_lens):
    lens = [w.Tkv] * w.B if kv_lens is None else [int(x) for x in kv_lens]
    cache = {}
    tot_b = tot_f = 0
    for n in lens:
        if n not in cache:
            cache[n] = unit_work(w, n)
        b, f = cache[n]
        tot_b += b * w.Hkv
        tot_f += f * w.Hkv
    return tot_b, tot_f


def is_prefill(w: Workload) -> bool:
    return w.name in PREFILL


def metric_unit(w: Workload):
    return ("TFLOP/s", "tensor") if is_prefill(w) else ("GB/s", "hbm")


def throughput(w, nbytes, nflops, seconds):
    unit, _ = metric_unit(w)
    if unit == "TFLOP/s":
        return nflops / seconds / 1e12
    return nbytes / seconds / 1e9


# ------------------------------------------------------------------ environment

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(ws, x: float) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample(w: Workload, inp, target_seconds: float, seed: int = 0):
    """Time the oracle on whole (batch, KV head) units until about target_seconds.

    Returns (value in the metric's unit, description, cores)."""
    import oracle
    oracle.build()
    lens = [w.Tkv] * w.B if inp.kv_lens is None else [int(x) for x in inp.kv_lens]
    rng = np.random.default_rng(seed)
    units = rng.permutation(w.B * w.Hkv).tolist()

    def rows_of(u):
        b, g = divmod(u, w.Hkv)
        rows = []
        for h in range(g * w.G, (g + 1) * w.G):
            base = (b * w.Hq + h) * w.Tq
            rows.extend(range(base, base + w.Tq))
        return rows

    # rows of a unit are computed in full; for prefill units only a row subset
    max_rows_per_unit = w.G * w.Tq
    done_b = done_f = 0
    t_total = 0.0
    n_rows = 0
    n_units = 0
    # cycle over the units (repeating them if the workload is small) until the
    # time target is reached
    order = units * max(1, 64)
    for u in order:
        rows = rows_of(u)
        b = u // w.Hkv
        if len(rows) > 512:
            # a slice of the unit's rows: count exactly the work of those rows
            rows = sorted(rng.choice(rows, size=512, replace=False).tolist())
        t0 = time.perf_counter()
        if w.kv_fp8:
            oracle.attention_rows_fp8kv(inp.q, inp.k8, inp.v8, inp.k_scale, inp.v_scale, inp.kv_lens, inp.sink,
                                        inp.scale, inp.causal, np.array(rows, np.int64))
        else:
            oracle.attention_rows(inp.q, inp.k, inp.v, inp.kv_lens, inp.sink, inp.scale, inp.causal,
                                  np.array(rows, np.int64))
        t_total += time.perf_counter() - t0
        n = lens[b]
        if len(rows) == max_rows_per_unit:
            ub, uf = unit_work(w, n)
        else:
            pairs = sum(visible_keys(w, n, r % w.Tq) for r in rows)
            keys = max(visible_keys(w, n, r % w.Tq) for r in rows)
            ub = 2 * keys * w.d * (1 if w.kv_fp8 else 2) + len(rows) * (2 * w.d * 2 + 4)
            uf = 4 * w.d * pairs
        done_b += ub
        done_f += uf
        n_rows += len(rows)
        n_units += 1
        if t_total >= target_seconds:
            break
    val = throughput(w, done_b, done_f, t_total)
    desc = "%d query rows from %d (batch, kv-head) unit passes of %s, %.1f s" % (n_rows, n_units, w.name, t_total)
    return val, desc, oracle.num_threads(), t_total


# ------------------------------------------------------------------ arms

def run_reference(args, w, ws, rank):
    if rank != 0:
        return
    inp = make_inputs(w)
    unit, _ = metric_unit(w)
    # each step a bounded oracle sample; the whole run stays within about two minutes
    per_step = max(0.3, min(args.ref_step_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for s in range(args.warmup):
        oracle_sample(w, inp, per_step, seed=s)
    vals, times = [], []
    desc = ""
    cores = 0
    for s in range(args.steps):
        v, desc, cores, t = oracle_sample(w, inp, per_step, seed=1000 + s)
        vals.append(v)
        times.append(t)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.page_size),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w: Workload, page_size: int = 0):
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "G": w.G, "Tq": w.Tq, "Tkv": w.Tkv, "d": w.d,
         "kv_dtype": "e4m3 (per-tensor scales)" if w.kv_fp8 else "bf16",
         "causal": w.causal, "sink": w.sink, "seed": w.seed,
         "kv_len": "U[1,%d]" % w.Tkv if w.ragged else (w.kv_len or w.Tkv),
         "nan_padding": w.nan_pad, "sigma": w.sigma,
         "kv_layout": ("paged [num_pages, Hkv, %d, d], shuffled pages" % page_size) if page_size else "contiguous",
         "l2": "flushed between timed steps (256 MB write)"}
    return c


def paged_inputs(w: Workload, inp, page_size: int):
    """The workload's K/V as a paged cache (storage only; same logical keys)."""
    lens = inp.kv_lens if inp.kv_lens is not None else torch.full((w.B,), w.Tkv, dtype=torch.int32)
    kc, vc, table = paginate(inp.k, inp.v, lens, page_size, seed=w.seed)
    return kc, vc, table, lens


def measure(args, w, ws, rank, local, steps, cpu_seconds, with_e2e=True):
    """Time `steps` calls of the forward on workload w (inputs resident in HBM,
    L2 flushed before each call); returns the numbers of one JSON line."""
    from gqa_attention_forward_flash_b200 import binding
    binding.load()
    dev = torch.device("cuda", local if ws > 1 else 0)
    inp = make_inputs(w)
    if w.kv_fp8:
        q, k, v = inp.q.to(dev), inp.k8.to(dev), inp.v8.to(dev)
    else:
        q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    kv = None if inp.kv_lens is None else inp.kv_lens.to(dev)
    sink = None if inp.sink is None else inp.sink.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    nbytes, nflops = workload_work(w, inp.kv_lens)
    unit, bound = metric_unit(w)
    if args.page_size:
        kc, vc, table, lens = (t.to(dev) for t in paged_inputs(w, inp, args.page_size))
        del k, v

    def step(st=None):
        st = stream if st is None else st
        if args.page_size:
            binding.gqa_attention_fwd_paged(q, kc, vc, table, lens, sink, out, lse, scale=inp.scale,
                                            causal=inp.causal, stream=st)
        elif w.kv_fp8:
            binding.gqa_attention_fwd_fp8kv(q, k, v, inp.k_scale, inp.v_scale, kv, sink, out, lse, scale=inp.scale,
                                            causal=inp.causal, stream=st)
        else:
            binding.gqa_attention_fwd(q, k, v, kv, sink, out, lse, scale=inp.scale, causal=inp.causal,
                                      stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    err = binding.gqa_get_device_error(stream)
    if err != 0:
        raise RuntimeError("device error %d after warm-up" % err)

    # clocks: sample while this load runs (a burn of the same steps right before
    # the timed steps, and through them)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    t_end = time.time() + args.burn_seconds
    while time.time() < t_end:
        for _ in range(20):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    binding.gqa_profile_begin()
    barrier(ws)
    torch.cuda.synchronize(dev)
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(ws)
    clocks = sampler.stop()
    main_ms = binding.gqa_profile_take()
    err = binding.gqa_get_device_error(stream)
    if err != 0:
        raise RuntimeError("device error %d in the timed steps" % err)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = all_max(ws, sum(step_ms))
    ms_per_step = total_ms / steps
    value = throughput(w, nbytes * ws, nflops * ws, ms_per_step / 1e3)
    median_ms = all_max(ws, statistics.median(step_ms))

    peaks, peak_src = load_peaks()
    main_avg = all_max(ws, statistics.mean(main_ms)) if main_ms else float("nan")
    main_med = all_max(ws, statistics.median(main_ms)) if main_ms else float("nan")
    if bound == "hbm":
        achieved = nbytes / (main_avg / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
    else:
        achieved = nflops / (main_avg / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
    spec_peak = SPEC_PEAKS["hbm_gbs"] if bound == "hbm" else SPEC_PEAKS["bf16_tflops"]
    traffic = None if args.page_size else traffic_for(w)
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "peak_source": peak_src + (" (burst)" if bound == "tensor" else ""),
                "frac_of_spec": achieved / spec_peak, "spec_peak": spec_peak,
                "kernel": main_kernel_name(w), "kernel_ms": main_avg, "kernel_ms_median": main_med,
                "launches_per_step": launches_per_call(w),
                "algorithmic_bytes": nbytes, "algorithmic_flops": nflops}
    if w.name == "short_q_long_kv":
        # bandwidth-bound by its intensity (128 flop/B, below the ridge), but the
        # workload is a prefill: its tensor-core fraction too
        tf = nflops / (main_avg / 1e3) / 1e12
        roofline["tensor"] = {"achieved": tf, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                              "frac": tf / float(peaks["bf16_tflops"])}

    # back-to-back calls replayed from one CUDA graph (reported beside the timed steps)
    graph = graph_timing(args, w, step, dev, nbytes, nflops) if args.graph > 0 else None

    # end to end through the public API with host buffers
    e2e = None
    if with_e2e and not args.no_e2e:
        e2e = run_e2e(args, w, inp, dev, stream, nbytes, nflops, ws)

    cpu = None
    if ws == 1 and rank == 0 and not args.no_cpu_baseline and cpu_seconds > 0:
        val, desc, cores, _ = oracle_sample(w, inp, cpu_seconds)
        cpu = {"value": val, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc}
    del q, out, flush
    res = {"value": value, "unit": unit, "ms_per_step": ms_per_step, "ms_per_step_mean": ms_per_step,
           "ms_per_step_median": median_ms, "steps": steps, "roofline": roofline, "cpu_baseline": cpu,
           "e2e": e2e, "gpu_launches": len(main_ms) * launches_per_call(w), "clocks": clocks,
           "config": config_of(w, args.page_size)}
    if graph is not None:
        res["graph"] = graph
    return res


def run_ours(args, w, ws, rank, local):
    head = measure(args, w, ws, rank, local, args.steps, args.cpu_seconds)
    extra = {}
    if args.all_workloads:
        # the metric's other configurations, each timed the same way in this run
        # (fewer steps and a shorter CPU sample, so that the whole run stays short)
        for name in sorted(WORKLOADS):
            if name == w.name:
                continue
            r = measure(args, WORKLOADS[name], ws, rank, local, args.workload_steps, args.workload_cpu_seconds)
            torch.cuda.empty_cache()
            extra[name] = r
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "ms_per_step_median": head["ms_per_step_median"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": head["config"],
            "roofline": head["roofline"], "cpu_baseline": head["cpu_baseline"], "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        }
        if "graph" in head:
            line["graph"] = head["graph"]
        if extra:
            line["workloads"] = extra
        print(json.dumps(line), flush=True)


def graph_timing(args, w, step, dev, nbytes, nflops):
    """args.graph calls captured back to back in one CUDA graph and replayed: the
    time per call without host launch overhead, the way a layer loop replays a
    captured decode step.  No L2 flush between the calls (a small workload's
    inputs stay in L2), so this is a latency figure beside the timed steps, not
    the headline value."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(args.graph):
                step(s)
    torch.cuda.synchronize(dev)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(dev)
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / (reps * args.graph)
    return {"calls_per_graph": args.graph, "replays": reps, "us_per_call": us,
            "value": throughput(w, nbytes, nflops, us / 1e6), "l2": "not flushed between calls"}


def run_e2e(args, w, inp, dev, stream, nbytes, nflops, ws):
    from gqa_attention_forward_flash_b200 import binding
    paged = bool(getattr(args, "page_size", 0))
    if paged:
        kc, vc, table, lens = paged_inputs(w, inp, args.page_size)
        hq, hk, hv, hkv, htab = (t.pin_memory() for t in (inp.q, kc, vc, lens, table))
    else:
        kk, vv = (inp.k8, inp.v8) if w.kv_fp8 else (inp.k, inp.v)
        hq, hk, hv = inp.q.pin_memory(), kk.pin_memory(), vv.pin_memory()
        hkv = None if inp.kv_lens is None else inp.kv_lens.pin_memory()
        htab = None
    hs = None if inp.sink is None else inp.sink.pin_memory()
    dq, dk, dv = torch.empty_like(hq, device=dev), torch.empty_like(hk, device=dev), torch.empty_like(hv, device=dev)
    dkv = None if hkv is None else torch.empty_like(hkv, device=dev)
    dtab = None if htab is None else torch.empty_like(htab, device=dev)
    ds = None if hs is None else torch.empty_like(hs, device=dev)
    dout = torch.empty_like(dq)
    dlse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32, device=dev)
    hout = torch.empty_like(hq).pin_memory()
    hlse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hkv, hs, htab) if t is not None)
    d2h = hout.numel() * hout.element_size() + hlse.numel() * 4

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        if dkv is not None:
            dkv.copy_(hkv, non_blocking=True)
        if dtab is not None:
            dtab.copy_(htab, non_blocking=True)
        if ds is not None:
            ds.copy_(hs, non_blocking=True)
        if paged:
            binding.gqa_attention_fwd_paged(dq, dk, dv, dtab, dkv, ds, dout, dlse, scale=inp.scale,
                                            causal=inp.causal, stream=stream)
        elif w.kv_fp8:
            binding.gqa_attention_fwd_fp8kv(dq, dk, dv, inp.k_scale, inp.v_scale, dkv, ds, dout, dlse,
                                            scale=inp.scale, causal=inp.causal, stream=stream)
        else:
            binding.gqa_attention_fwd(dq, dk, dv, dkv, ds, dout, dlse, scale=inp.scale, causal=inp.causal,
                                      stream=stream)
        hout.copy_(dout, non_blocking=True)
        hlse.copy_(dlse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 20))
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = all_max(ws, e0.elapsed_time(e1)) / steps
    unit, _ = metric_unit(w)
    return {"value": throughput(w, nbytes * ws, nflops * ws, ms / 1e3), "unit": unit,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps}


def main_kernel_name(w: Workload) -> str:
    """The kernel gqa_attention_fwd launches for these sizes: the swap-AB decode
    kernel for head dim 128 with at most 16 packed rows per KV head, the two-lane
    kernel for the other head dims 64/128, the wide kernel for 256/512."""
    if w.d == 128 and w.G * w.Tq <= 16:
        return "gqa_dec_kernel"
    return "gqa_fwd2_kernel" if w.d <= 128 else "gqa_wide_kernel"


def launches_per_call(w: Workload) -> int:
    """Every kernel merges its split rows inside itself: one launch per call."""
    return 1


def kernel_source_digest() -> str:
    """sha256 over the library's CUDA sources (file name + contents, sorted)."""
    import hashlib
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "gqa_attention_forward_flash_b200", "csrc")
    for name in sorted(os.listdir(cs)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(cs, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def traffic_for(w: Workload):
    """DRAM bytes (read + write) per launch of the main kernel, from the ncu
    capture recorded in profiles/traffic.json, or None when there is none for
    this workload or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_sha256") != kernel_source_digest():
        return None
    e = d.get("workloads", {}).get(w.name)
    return None if e is None else e.get("bytes_per_launch")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="batched_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-step-seconds", type=float, default=3.0)
    ap.add_argument("--burn-seconds", type=float, default=1.5)
    ap.add_argument("--only", dest="all_workloads", action="store_false",
                    help="time only --workload (by default the other workloads follow in a 'workloads' block)")
    ap.add_argument("--workload-steps", type=int, default=40,
                    help="timed steps of each workload in the 'workloads' block")
    ap.add_argument("--workload-cpu-seconds", type=float, default=3.0,
                    help="oracle seconds of each workload in the 'workloads' block")
    ap.add_argument("--graph", type=int, default=0,
                    help="also time this many back-to-back calls captured in one CUDA graph")
    ap.add_argument("--page-size", type=int, default=0,
                    help="read K/V through gqa_attention_fwd_paged from a cache of pages of this many tokens "
                         "(0: contiguous K/V through gqa_attention_fwd)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, ws, rank)
        return
    ws, rank, local = dist_setup()
    try:
        run_ours(args, w, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
