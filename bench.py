"""Benchmark: prefill TFLOP/s and decode KV GB/s on B200, as a fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one launch sequence of the attention path over one batch of
synthetic, seeded bf16 inputs already resident in HBM.  The headline workload
is the GQA causal prefill (B1 Hq32 Hkv8 Sq=Skv=4096 D128).  All five base
workloads (tiny prefill, the headline, prefill at depth with D256, D512
split-KV decode with its LSE merge, 8-row speculative-verify decode) are timed
the same way and reported under "configs", the last key of the JSON line; the
widened workloads (logit terms, masks, windows, fp8, paged, fused, latent
cache, D512 prefill) come before it under "workloads".  Each carries the
roofline fraction of its whole step (a decode step is the split kernel plus
the merge, timed with no event between the two launches, as a caller runs
them) and, as kernel_frac, that of its first kernel alone (from a second
timed pass with an event after the split kernel).  L2 is
flushed between timed steps (a 256 MiB write, then a 256 MiB read so no dirty
lines are left behind); the flush is outside the timed events.

Under torchrun (N > 1) every rank runs the same problems independently (the
path does not shard: replicas only); times are the max over ranks and the
value is the work of all ranks divided by that time.

--impl reference times the float64 CPU oracle (the parity reference) on a
bounded row sample of the headline workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "gqa_causal_prefill_4k_d128"
# The five base workloads (tiny prefill, headline prefill, prefill at depth,
# D512 split-KV decode, 8-row verify decode): reported last in the JSON line,
# after the widened workloads, so that a reader of its tail sees all five.
BASE_CONFIGS = ["tiny_causal_gqa_prefill", "gqa_causal_prefill_4k_d128", "prefill_at_depth_d256",
                "split_kv_decode_d512", "spec_verify_decode_d128"]
METRIC = "prefill TFLOP/s and decode KV GB/s on 1 B200, as % of roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FLUSH_BYTES = 256 << 20


class L2Flush:
    """Leaves L2 holding none of the workload's data and no dirty lines: a
    write pass over one buffer larger than L2, then a read pass over another,
    so the next timed kernel neither hits in L2 nor pays for write-backs."""

    def __init__(self, device):
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def zero_(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="time only this workload (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle budget for cpu_baseline")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers --
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0.0)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "gqa_flash_attention_attn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "prefill": ["prefill_sm100.cu", "ptx.cuh"],
    # prefill that runs on the split-KV kernel in query-chunk mode
    "prefill_wide": ["decode_sm100.cu", "ptx.cuh"],
    "decode": ["decode_sm100.cu", "ptx.cuh"],
    "merge": ["merge.cu", "ptx.cuh"],
}


def prefill_sources(w):
    """Which kernel a prefill workload runs: the prefill kernel for D = Dv in
    {64, 128, 256} or (192, 128), else the split-KV kernel."""
    fast = (w.D == w.dv and w.D in (64, 128, 256)) or (w.D, w.dv) == (192, 128)
    return "prefill" if fast and w.kv_dtype == "bf16" and not w.page_size else "prefill_wide"


def profiled_traffic(kind, workload, sources=None):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    summary is missing or the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kind}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic-bytes-per-launch:\s*([0-9]+)", text)
    s = re.search(r"kernel-source-sha256:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != kernel_source_sha(KERNEL_SOURCES[sources or kind]):
        return None
    return int(m.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)  # let the first samples arrive before the timed work starts
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- the GPU arm --
def make_runner(ga, w, device):
    """Device-resident inputs/outputs and a closure that launches one step.
    Returns (step_fn, n_kernels_per_step, events_split) where the closure
    records optional inner events between the split and the merge."""
    from gqa_flash_attention_attn_b200.inputs import (make_fp8_kv, make_mask, make_paged, make_sinks,
                                                      make_workload_inputs)
    q, k, v = make_workload_inputs(w, seed=0, device=device)
    bt = None
    scales = {}
    if w.kv_dtype == "fp8":
        k, v, ks, vs = make_fp8_kv(k, v)
        scales = dict(k_scale=ks, v_scale=vs)
    if w.page_size:
        kc, vc, bt = make_paged(k.cpu(), v.cpu(), w.page_size, seed=0)
        k, v, bt = kc.to(device), vc.to(device), bt.to(device)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    out = torch.empty((w.B, w.Sq, w.Hq, w.dv), dtype=odt, device=device)
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=device)
    sinks = make_sinks(w.Hq, seed=0).to(device) if w.sinks else None
    mask = make_mask(w.mask_batch, w.Sq, w.Skv, seed=0).to(device) if w.mask_batch else None
    terms = dict(softcap=w.softcap, alibi_max_bias=w.alibi_max_bias, window=w.window, mask=mask)
    if w.kind == "prefill":
        def step(mid=None):
            if w.dv == w.D:
                ga.prefill(q, k, v, causal=w.causal, q_offset=w.q_offset, scale=w.scale, out=out, lse=lse,
                           sinks=sinks, **terms)
            else:
                ga.prefill_kv(q, k, v, causal=w.causal, q_offset=w.q_offset, scale=w.scale, out=out, lse=lse,
                              sinks=sinks, **terms)
        return step, 1, (q, k, v, out, lse)
    if w.fused:
        vv = k[..., :w.dv] if w.v_of_k else v

        def step(mid=None):
            ga.decode_fused(q, k, vv, w.num_splits, block_table=bt, causal=w.causal, q_offset=w.q_offset,
                            scale=w.scale, out=out, lse=lse, sinks=sinks, **scales, **terms)
        return step, 1, (q, k, v, out, lse)
    po = torch.empty((w.num_splits, w.B, w.Sq, w.Hq, w.dv), dtype=torch.float32, device=device)
    pl = torch.empty((w.num_splits, w.B, w.Hq, w.Sq), dtype=torch.float32, device=device)

    def step(mid=None):
        if bt is None and not scales and w.dv == w.D:
            ga.decode_split(q, k, v, w.num_splits, causal=w.causal, q_offset=w.q_offset, scale=w.scale,
                            partial_out=po, partial_lse=pl, **terms)
        else:
            ga.decode_split_kv(q, k, v, w.num_splits, block_table=bt, causal=w.causal, q_offset=w.q_offset,
                               scale=w.scale, partial_out=po, partial_lse=pl, **scales, **terms)
        if mid is not None:
            mid.record()
        ga.merge(po, pl, out=out, lse=lse, sinks=sinks)
    return step, 2, (q, k, v, out, lse)


def barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()


def max_over_ranks(x, dist_on, device):
    """The largest of every rank's x (a per-step time), same on all ranks."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(work_per_rank, ms_local, dist_on, device):
    """Whole-job rate for independent replicas: the work of all ranks divided
    by the slowest rank's time.  Returns (rate per second, max ms)."""
    world = torch.distributed.get_world_size() if dist_on else 1
    ms = max_over_ranks(ms_local, dist_on, device)
    return world * work_per_rank / (ms / 1e3), ms


def time_steps(step, steps, warmup, flush, dist_on, device, inner=False):
    for _ in range(warmup):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    barrier(dist_on)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, m, e in ev:
        s.record()
        step(m if inner else None)
        e.record()
        flush.zero_()
    torch.cuda.synchronize()
    barrier(dist_on)
    torch.cuda.synchronize()
    total = sum(s.elapsed_time(e) for s, _, e in ev)
    first = sum(s.elapsed_time(m) for s, m, _ in ev) if inner else total
    return total / steps, first / steps


def time_e2e(ga, w, steps, warmup, dist_on, device):
    """Same workload through the public call with pinned host buffers: every
    step copies its q, k, v host->device, runs the kernels and copies out and
    lse device->host; all of it is inside the timed region.  Steps are
    pipelined the way a streaming caller would run them: inputs double
    buffered on the device, uploads on one stream, kernels on another,
    downloads on a third, so step i's download overlaps step i+1's upload
    (PCIe is full duplex) and the kernels overlap both."""
    from gqa_flash_attention_attn_b200.inputs import make_workload_inputs
    q, k, v = make_workload_inputs(w, seed=0)
    # a V that is a view of K travels inside K
    host_in = [t.pin_memory() for t in ((q, k) if w.v_of_k else (q, k, v))]
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    ho = [torch.empty((w.B, w.Sq, w.Hq, w.dv), dtype=odt).pin_memory() for _ in range(2)]
    hl = [torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32).pin_memory() for _ in range(2)]
    dev_in = [[torch.empty_like(t, device=device) for t in host_in] for _ in range(2)]
    dev_out = [torch.empty((w.B, w.Sq, w.Hq, w.dv), dtype=odt, device=device) for _ in range(2)]
    dev_lse = [torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=device) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_comp = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event()
    state = {"in_free": [None, None], "out_free": [None, None]}

    def step(i):
        b = i & 1
        # upload into buffer b once the kernels of step i-2 stopped reading it
        with torch.cuda.stream(s_in):
            if state["in_free"][b] is not None:
                s_in.wait_event(state["in_free"][b])
            for dst, src in zip(dev_in[b], host_in):
                dst.copy_(src, non_blocking=True)
            uploaded = ev()
            uploaded.record(s_in)
        s_comp.wait_event(uploaded)
        if state["out_free"][b] is not None:
            s_comp.wait_event(state["out_free"][b])      # step i-2's download of out[b] is done
        dq, dk = dev_in[b][0], dev_in[b][1]
        dv = dk[..., :w.dv] if w.v_of_k else dev_in[b][2]
        kw = dict(causal=w.causal, q_offset=w.q_offset, scale=w.scale, out=dev_out[b], lse=dev_lse[b])
        if w.kind == "prefill":
            (ga.prefill if w.dv == w.D else ga.prefill_kv)(dq, dk, dv, **kw)
        else:
            if w.fused:
                ga.decode_fused(dq, dk, dv, w.num_splits, **kw)
            else:
                (ga.decode if w.dv == w.D else ga.decode_kv)(dq, dk, dv, w.num_splits, **kw)
        computed = ev()
        computed.record(s_comp)
        state["in_free"][b] = computed
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed)
            ho[b].copy_(dev_out[b], non_blocking=True)
            hl[b].copy_(dev_lse[b], non_blocking=True)
            downloaded = ev()
            downloaded.record(s_out)
        state["out_free"][b] = downloaded

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(dist_on)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    s_comp.wait_event(start)
    s_out.wait_event(start)
    for i in range(steps):
        step(warmup + i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_comp)
    end.record(s_in)
    torch.cuda.synchronize()
    barrier(dist_on)
    ms = max_over_ranks(start.elapsed_time(end) / steps, dist_on, device)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
    return ms, h2d, d2h


def workload_metric(w):
    """(unit, work per step) for a workload: TFLOP/s for prefill, KV GB/s for decode."""
    if w.kind == "prefill":
        return "TFLOP/s", w.flops() / 1e12
    return "GB/s", w.io_bytes() / 1e9


def cpu_baseline(w, seconds):
    """The float64 oracle, as it stands, on a bounded row sample of workload w."""
    import numpy as np
    import oracle
    from gqa_flash_attention_attn_b200.inputs import make_workload_inputs, sample_rows
    q, k, v = make_workload_inputs(w)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))

    def visible(s):
        return min(w.Skv, w.q_offset + s + 1) if w.causal else w.Skv

    def run(n, seed):
        rows = sample_rows(w, n, seed=seed, include_edges=False)
        t0 = time.perf_counter()
        oracle.attention_rows(qd, kd, vd, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
        dt = time.perf_counter() - t0
        flops = sum(2 * (w.D + w.dv) * visible(s) for _, _, s in rows)
        kv_bytes = sum(2 * (w.D + w.dv) * visible(s) for _, _, s in rows)  # K and V rows each row reads
        return dt, flops, kv_bytes, len(rows)

    dt, _, _, _ = run(256, 11)
    n2 = max(256, int(256 * seconds / max(dt, 1e-3)))
    dt, fl, kvb, n = run(n2, 12)
    unit, _ = workload_metric(w)
    value = fl / dt / 1e12 if unit == "TFLOP/s" else kvb / dt / 1e9
    return {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} random (b,h,s) rows of {w.name}, {fl / 1e9:.1f} GFLOP fp64 in {dt:.1f} s"}


def _sig(x, digits=4):
    return float(f"{x:.{digits}g}") if isinstance(x, float) else x


def compact(r):
    """One workload's figures for the JSON line: per step value and time,
    the roofline fraction of the step and of its first kernel, and the ncu
    DRAM bytes of that kernel (or null)."""
    roof = r["roofline"]
    return {"value": _sig(r["value"]), "unit": r["unit"], "ms_per_step": _sig(r["ms_per_step"]),
            "kernel_ms": _sig(r["kernel_ms"]), "roofline_frac": _sig(roof["frac"], 3),
            "kernel_frac": _sig(roof["kernel_frac"], 3), "bound": roof["bound"], "traffic": roof["traffic"]}


def workload_config(w, world):
    """The config object of the JSON line for workload w (same keys in both arms)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq, "Skv": w.Skv, "D": w.D,
            "q_offset": w.q_offset, "causal": w.causal, "out": w.out_dtype,
            "num_splits": w.num_splits if w.kind == "decode" else None,
            "l2": "flushed between timed steps (256 MiB write, then 256 MiB read)",
            "parallelism": f"replicas x{world}"}


def run_ours(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    import gqa_flash_attention_attn_b200 as ga
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS
    ga.library()  # fails loudly when the CUDA library is missing

    hbm, tf_burst, tf_sust, peak_src = peaks()
    flush = L2Flush(device)
    names = [args.workload] if args.workload else [HEADLINE] + [n for n in WORKLOADS if n != HEADLINE]
    sampler = ClockSampler(local)
    results = {}
    sampler.start()
    for name in names:
        w = WORKLOADS[name]
        step, nk, _ = make_runner(ga, w, device)
        ms, ms_first = time_steps(step, args.steps, args.warmup, flush, dist_on, device)
        if nk == 2:
            # The first kernel alone comes from a second timed pass with an
            # event between the two launches: in the step itself that event
            # would add its own time and keep the merge from being scheduled
            # while the split kernel drains.
            _, ms_first = time_steps(step, args.steps, args.warmup, flush, dist_on, device, inner=True)
        status = ga.last_status()
        if status != ga.ATTN_OK:
            raise RuntimeError(f"{name}: device status {ga.status_string(status)}")
        unit, work = workload_metric(w)
        value, ms = replica_throughput(work, ms, dist_on, device)
        ms_first = max_over_ranks(ms_first, dist_on, device)
        # The fraction is for the whole step (for a decode: the split kernel
        # and the merge); kernel_frac is the first kernel alone.
        if w.kind == "prefill":
            kind, achieved = "prefill", w.flops() / (ms / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                    "frac": achieved / tf_burst, "peak_source": f"{peak_src} bf16 burst"}
            kernel_frac = w.flops() / (ms_first / 1e3) / 1e12 / tf_burst
        else:
            kind, achieved = "decode", w.io_bytes() / (ms / 1e3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                    "peak_source": f"{peak_src} copy bandwidth"}
            kernel_frac = w.io_bytes() / (ms_first / 1e3) / 1e9 / hbm
        roof["kernel_frac"] = kernel_frac
        roof["kernel"] = kind
        roof["traffic"] = profiled_traffic(kind, name, prefill_sources(w) if kind == "prefill" else None)
        results[name] = {"value": value, "unit": unit, "ms_per_step": ms, "kernel_ms": ms_first,
                         "kernels_per_step": nk, "roofline": roof}
        del step
        torch.cuda.empty_cache()
    clocks = sampler.stop()

    head = results[names[0]]
    w = WORKLOADS[names[0]]
    e2e_ms, h2d, d2h = time_e2e(ga, w, max(3, args.steps // 5), max(1, args.warmup), dist_on, device)
    unit, work = workload_metric(w)
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1) cast to bf16)",
        "config": workload_config(w, world),
        "roofline": head["roofline"],
        "e2e": {"value": world * work / (e2e_ms / 1e3), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": head["kernels_per_step"] * args.steps,
        "clocks": clocks,
        "workloads": {n: compact(r) for n, r in results.items() if n not in BASE_CONFIGS},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    line["configs"] = {n: compact(results[n]) for n in BASE_CONFIGS if n in results}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_reference(args):
    """The float64 CPU oracle timed on a bounded sample per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_workload_inputs, sample_rows
    w = WORKLOADS[HEADLINE]
    q, k, v = make_workload_inputs(w)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))

    def one(n, seed):
        rows = sample_rows(w, n, seed=seed, include_edges=False)
        fl = sum(2 * (w.D + w.dv) * min(w.Skv, w.q_offset + s + 1) for _, _, s in rows)
        t0 = time.perf_counter()
        oracle.attention_rows(qd, kd, vd, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
        return time.perf_counter() - t0, fl

    dt, _ = one(128, 1)
    n = max(64, int(128 * 1.0 / max(dt, 1e-3)))   # about one second of oracle work per step
    for i in range(args.warmup):
        one(n, 100 + i)
    tot_t, tot_f = 0.0, 0
    for i in range(args.steps):
        dt, fl = one(n, 1000 + i)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded iid N(0,1) cast to bf16)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} random (b,h,s) rows of {w.name} per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
