#!/usr/bin/env python
"""Benchmark: one GQA decode step (one layer) per step, on N GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one gqa_decode call (one split-KV kernel, which also merges the
partials of the units it cut across CTAs) over one batch of the workload, with q, the KV cache and seq_lens resident in HBM.
The default workload is the Llama-2-70B-shaped ragged batch (B=32, 64 query /
8 KV heads, head_dim 128, lengths U[1, 32768]); its KV bytes per step
(~2.15 GB) exceed the 126 MB L2, so no flush is needed between steps.

Printed metric: achieved HBM GB/s of algorithmic traffic (K and V rows of
the live tokens, plus Q and the fp32 output) -- whole-job over N GPUs, each
GPU running its own independent batch (weak scaling, no collective on the
data path).  Timing: CUDA events on the launching stream, barrier and
synchronize around exactly K steps, max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the slow reference arm).
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gqa_mqa_kv_b200.workloads import (PREFILL_WORKLOADS, WORKLOADS, algorithmic_bytes,  # noqa: E402
                                       make_inputs, make_prefill_inputs, prefill_flops, prefill_lengths)

METRIC = "decode-attention achieved HBM GB/s (% of B200 peak) and µs per decode step"
PREFILL_METRIC = "prefill-attention achieved TFLOP/s (causal, algorithmic 4 d per visible query-head/key pair) and µs per step"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, DGX figure (7.7 TB/s on HGX)
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0  # the recipe's sustained figure under the power cap
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama2_70b_ragged", choices=sorted(WORKLOADS) + sorted(PREFILL_WORKLOADS),
                    help="a decode workload, or a multi-token (prefill) workload: prefill_*")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak-seconds", type=float, default=1.5,
                    help="untimed steps before the timed region so clocks settle and are sampled")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--kernel", default="auto", choices=["auto", "mma_sync", "tcgen05"],
                    help="split kernel (gqa_kernel); auto is the library's choice")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size B (reduced cases for profiler captures; the "
                         "JSON line's config then names the reduced workload and is not a bench line)")
    ap.add_argument("--path", default="decode", choices=["decode", "append_decode"],
                    help="decode: gqa_decode per step; append_decode: gqa_rope_append of the "
                         "newest token (re-appended at L_b - 1) followed by gqa_decode")
    return ap.parse_args(argv)


def decode_workload(args):
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        w = dataclasses.replace(w, name=f"{w.name}_B{args.batch}", B=args.batch)
    return w


def prefill_workload(args):
    w = PREFILL_WORKLOADS[args.workload]
    if args.batch is not None:
        w = dataclasses.replace(w, name=f"{w.name}_B{args.batch}", B=args.batch)
    return w


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist

    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- peaks, clocks, profiles

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: (burst, sustained, kind).  The burst figure is for a
    kernel timed alone; the sustained one (a seconds-long GEMM loop under the
    1 kW power cap) for a kernel that runs continuously, as the multi-token
    bench does (a soak, then back-to-back steps)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background (200 ms period)."""

    def __init__(self, device: torch.device):
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            sel = ["-i", self.uuid] if self.uuid else []
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, power, reasons = [], [], [], set()
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                power.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(REASON_NAMES, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "reasons": sorted(reasons), "samples": len(sm)}


# Sources each measured kernel is built from (the host file gqa_decode.cu and
# the shared headers count for both).
_PREFILL_ONLY = {"prefill_tc.cuh"}
_DECODE_ONLY = {"split_mma.cuh", "split_tc.cuh", "split_simt.cuh", "combine.cuh", "rope_append.cuh"}


def kernel_source_hash(kind: str = "decode") -> str:
    """sha256 (first 16 hex digits) over the csrc files of the decode or the
    prefill kernels."""
    skip = _PREFILL_ONLY if kind == "decode" else _DECODE_ONLY
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gqa_mqa_kv_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in skip:
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# The files each measured kernel is compiled from: its own header, the headers
# it includes and the host file that sets up its launch.
KERNEL_FILES = {
    "split_mma": ["gqa_decode.cu", "split_mma.cuh", "combine.cuh", "schedule.cuh", "ptx.cuh"],
    "split_tc": ["gqa_decode.cu", "split_tc.cuh", "tcgen05.cuh", "combine.cuh", "schedule.cuh", "ptx.cuh"],
    "prefill_tc": ["gqa_decode.cu", "prefill_tc.cuh", "tcgen05.cuh", "schedule.cuh", "ptx.cuh"],
}


def kernel_files_hash(kernel: str) -> str:
    """sha256 (first 16 hex digits) over the files one kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gqa_mqa_kv_b200", "csrc")
    for name in sorted(KERNEL_FILES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the workload's dominant kernel from the
    committed ncu summary, if it was taken on the current source of that
    kernel (the hash over the files that kernel is compiled from); else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec.get(workload)
        if ent and ent.get("kernel_files_hash") == kernel_files_hash(ent["kernel_family"]):
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- CPU oracle sample

def cpu_oracle_sample(w, inp, seconds: float):
    """Time the fp64 oracle on the first sequences of the batch (all query
    heads), sized to take about `seconds` of wall clock."""
    import oracle

    lens = inp["seq_lens"]
    H_Q = w.H_Q
    threads = oracle.hardware_threads()
    # calibrate on all heads of the first non-empty sequence
    b0 = int(torch.nonzero(lens > 0)[0])
    t0 = time.perf_counter()
    run = ((lambda pairs: oracle.gqa_decode_scaled(inp["q"], inp["k"], inp["v"], lens, w.softmax_scale,
                                                    inp["k_scale"], inp["v_scale"], pairs=pairs))
           if w.kv8 else
           (lambda pairs: oracle.gqa_decode(inp["q"], inp["k"], inp["v"], lens, w.softmax_scale, pairs=pairs,
                                            n_threads=0)))
    run([(b0, h) for h in range(H_Q)])
    per_token = max((time.perf_counter() - t0) / max(int(lens[b0]), 1), 1e-12)  # all heads, all threads
    est_full = per_token * int(lens.sum())
    if est_full <= seconds:
        nb, reps = w.B, max(1, min(3, int(seconds / max(est_full, 1e-3))))
    else:
        nb, acc = 0, 0.0
        while nb < w.B and (acc < seconds or nb == 0):
            acc += per_token * int(lens[nb])
            nb += 1
        reps = 1
    pairs = [(b, h) for b in range(nb) for h in range(H_Q)]
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        run(pairs)
        times.append(time.perf_counter() - t0)
    dt = statistics.median(times)
    e = 2 if w.dtype == "bf16" else 4
    e_kv = 1 if w.kv8 else e
    sample_bytes = (int(lens[:nb].to(torch.int64).sum()) * w.H_KV * w.D * e_kv * 2
                    + nb * H_Q * w.D * e + nb * H_Q * w.D * 4)
    what = "the whole step" if nb == w.B else f"sequences 0..{nb - 1} of {w.B}"
    return {
        "value": sample_bytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
        "sample": f"{what} (all {H_Q} query heads, {int(lens[:nb].sum())} cached tokens), fp64, "
                  f"median of {reps} run(s), {dt:.2f} s each",
        "seconds": dt, "us_per_full_step_equiv": dt * 1e6 * (algorithmic_bytes(w, lens) / sample_bytes),
    }


def run_reference(args):
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    w = decode_workload(args)
    inp = make_inputs(w)
    step_results = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm state; warm-up steps are no-ops by construction
    t_start = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_oracle_sample(w, inp, args.cpu_sample_seconds / max(args.steps, 1))
        step_results.append(last)
    total = time.perf_counter() - t_start
    value = statistics.median(r["value"] for r in step_results)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total * 1e3 / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w, args.gpus), split_kernel=args.kernel),
        "cpu_baseline": {k: last[k] for k in ("kind", "cores", "sample")} | {"value": value, "unit": "GB/s"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- L2 flush between timed steps

class L2Flush:
    """Writes a 256 MiB buffer (twice the 126 MB L2) and then reads another
    one, outside the timed events.  The write evicts the step's inputs from
    L2; the read then evicts the write's dirty lines, so their write-back to
    HBM happens here and not inside the next timed kernel (where it would add
    up to ~126 MB of DRAM writes to the kernel's own traffic)."""

    def __init__(self, dev):
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


L2_NOTE = "L2 flushed before every step (256 MiB written, then 256 MiB read so no dirty line is written back inside the timed kernel)"


# ---------------------------------------------------------------- end to end, copies overlapped

def overlapped_e2e(dev, stream, host_in, dev_in, call, dev_out, host_out, steps, warmup, dist):
    """Times `steps` end-to-end steps and returns ms per step (max over ranks).

    Every step copies its own inputs (host_in, pinned) into one of two device
    buffer sets, runs `call(slot)` on `stream` over that set, and copies its
    result (dev_out[slot]) back into pinned host memory.  The copies in run on
    one side stream and the copies out on another, ordered by events, so step
    i's copy in overlaps step i-1's kernels and its copy out overlaps step
    i+1's; a buffer set is refilled only after its previous step's kernels
    have read it and its result has been copied out."""
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    k_done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        s = i % 2
        if i >= 2:
            h2d_s.wait_event(k_done[s])
        with torch.cuda.stream(h2d_s):
            for h, d in zip(host_in, dev_in[s]):
                d.copy_(h, non_blocking=True)
        in_ready[s].record(h2d_s)
        stream.wait_event(in_ready[s])
        if i >= 2:
            stream.wait_event(out_read[s])
        call(s)
        k_done[s].record(stream)
        d2h_s.wait_event(k_done[s])
        with torch.cuda.stream(d2h_s):
            host_out[s].copy_(dev_out[s], non_blocking=True)
        out_read[s].record(d2h_s)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        one(i)
    for ev in out_read:  # the timed region ends when the last result is on the host
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return max_over_ranks(e0.elapsed_time(e1), dist, dev) / steps


# ---------------------------------------------------------------- GPU arm

def cache_capacity_bytes(w):
    """K plus V bytes at the workload's maximum length (the L2 comparison)."""
    e_kv = 1 if w.kv8 else (2 if w.dtype == "bf16" else 4)
    return w.seq_len * w.B * w.H_KV * w.D * e_kv * 2


def workload_config(w, n):
    return {"workload": w.name, "B": w.B, "H_Q": w.H_Q, "H_KV": w.H_KV, "head_dim": w.D,
            "seq_len": w.seq_len, "ragged": w.ragged, "page_size": w.page_size,
            "kv_dtype": "e4m3 (per-KV-head scales)" if w.kv8 else w.dtype, "global_batch": w.B * n,
            "l2": "inputs larger than L2 (no flush)" if cache_capacity_bytes(w) > 2 * 126e6
                  else L2_NOTE,
            "parallelism": f"dp{n} (independent batch per GPU, no collective)"}


def run_ours(args):
    import gqa_mqa_kv_b200 as gq

    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        print(f"WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    w = decode_workload(args)
    inp = make_inputs(w)
    lens_host = inp["seq_lens"]
    step_bytes = algorithmic_bytes(w, lens_host)
    paged = bool(w.page_size)
    kk = inp["k_paged"] if paged else inp["k"]
    vv = inp["v_paged"] if paged else inp["v"]
    q = inp["q"].to(dev)
    k = kk.to(dev)
    v = vv.to(dev)
    lens = lens_host.to(dev)
    table = inp["block_table"].to(dev) if paged else None
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    ks = inp["k_scale"].to(dev) if w.kv8 else None
    vs = inp["v_scale"].to(dev) if w.kv8 else None
    params = gq.make_params(q, k, lens, table)
    if w.kv8:
        params.qkv_dtype = gq.GQA_BF16
    ws = torch.zeros(gq.workspace_bytes(params), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    big = cache_capacity_bytes(w) > 2 * 126e6
    flush = None if big else L2Flush(dev)
    appending = args.path == "append_decode"
    if appending:
        # The newest token of every sequence is (re-)appended at position L_b - 1, so
        # each step rotates q and k and writes one cache row without growing the cache.
        gnew = torch.Generator().manual_seed(w.seed + 100)
        k_new = torch.randn(w.B, w.H_KV, w.D, generator=gnew).to(q.dtype).to(dev)
        v_new = torch.randn(w.B, w.H_KV, w.D, generator=gnew).to(q.dtype).to(dev)
        positions = (lens - 1).clamp(min=0)
        q_in = q.clone()
        step_bytes += w.B * w.D * q.element_size() * (2 * w.H_Q + 4 * w.H_KV)
    launches_per_step = 2 if appending else 1

    def append_call(events=None):
        if events is not None:
            events[0].record(stream)
        gq.gqa_rope_append(q_in, k_new, v_new, positions, k, v, table, q_out=q, workspace=ws,
                           stream=stream)
        if events is not None:
            events[1].record(stream)

    def decode_call(events=None, qq=None, ll=None, oo=None):
        qq = q if qq is None else qq
        ll = lens if ll is None else ll
        oo = out if oo is None else oo
        if w.kv8:  # 8-bit cache: events bracket the whole call (the split kernel)
            if events is not None:
                events[0].record(stream)
            gq.gqa_decode_fp8kv(qq, k, v, ks, vs, ll, table, scale=w.softmax_scale, out=oo,
                                workspace=ws, stream=stream, kernel=args.kernel)
            if events is not None:
                events[1].record(stream)
        elif events is not None:
            gq.gqa_decode_timed(events, qq, k, v, ll, table, scale=w.softmax_scale, out=oo,
                                workspace=ws, stream=stream, kernel=args.kernel)
        else:
            gq.gqa_decode(qq, k, v, ll, table, scale=w.softmax_scale, out=oo, workspace=ws,
                          stream=stream, kernel=args.kernel)

    def step():
        if flush is not None:
            flush()
        if appending:
            append_call()
        decode_call()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    with ClockSampler(dev) as clocks:
        t_soak = time.perf_counter()
        while time.perf_counter() - t_soak < args.soak_seconds:
            for _ in range(50):
                step()
            torch.cuda.synchronize(dev)
        # ------------------------------------------------ timed region: the headline
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev_begin = torch.cuda.Event(enable_timing=True)
        ev_end = torch.cuda.Event(enable_timing=True)
        step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)] if flush is not None else None
        ev_begin.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush()
                step_ev[i][0].record(stream)
            if appending:
                append_call()
            decode_call()
            if flush is not None:
                step_ev[i][1].record(stream)
        ev_end.record(stream)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        append_ev = split_ev = None
        if appending:
            # ------------------------------------------------ second pass: each kernel alone
            # Same K steps with events around the append and the decode kernel of
            # every step (the events break the launch chaining, so this pass is
            # not the headline).
            split_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                        for _ in range(args.steps)]
            append_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                         for _ in range(args.steps)]
            for i in range(args.steps):
                if flush is not None:
                    flush()
                append_call(append_ev[i])
                decode_call(split_ev[i])
            torch.cuda.synchronize(dev)
            if dist is not None:
                dist.barrier()
        # ------------------------------------------------ end of timed region
    # Whole region when nothing else runs in it; per-step sums when an L2 flush
    # sits between the steps.
    elapsed_ms = (ev_begin.elapsed_time(ev_end) if step_ev is None
                  else sum(a.elapsed_time(b) for a, b in step_ev))
    # The decode kernel's own duration per launch: a plain decode step is that
    # one kernel, so the timed region gives it directly; with the append the
    # second pass brackets the decode kernel alone.
    split_ms = (statistics.mean(a.elapsed_time(b) for a, b in split_ev) if appending
                else elapsed_ms / args.steps)
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    split_ms_max = max_over_ranks(split_ms, dist, dev)
    status = gq.read_status(ws)

    # ---------------------------------------------------- end to end through the public API
    q_host = inp["q"].pin_memory()
    lens_pin = lens_host.pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = q_host.numel() * q_host.element_size() + lens_pin.numel() * 4
    d2h = out_host[0].numel() * out_host[0].element_size()
    q_sets = [q, torch.empty_like(q)]
    lens_sets = [lens, torch.empty_like(lens)]
    out_sets = [out, torch.empty_like(out)]
    e2e_ms = overlapped_e2e(dev, stream, [q_host, lens_pin], list(zip(q_sets, lens_sets)),
                            lambda s: decode_call(qq=q_sets[s], ll=lens_sets[s], oo=out_sets[s]),
                            out_sets, out_host, args.e2e_steps, 3, dist)

    peak, peak_kind = hbm_peak()
    ms_per_step = elapsed_ms / args.steps
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9
    achieved = algorithmic_bytes(w, lens_host) / (split_ms_max * 1e-3) / 1e9
    traffic = recorded_traffic(w.name)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "pct_of_hbm_peak": 100.0 * (value / world) / peak, "peak_kind": peak_kind,
        "pct_of_nominal_hbm": 100.0 * (value / world) / NOMINAL_HBM_GBS,
        "hbm_target_note": ("the >=80% target is read against the measured copy rate "
                            f"({peak:.0f} GB/s, {peak_kind}); pct_of_nominal_hbm divides by the nominal "
                            f"{NOMINAL_HBM_GBS:.0f} GB/s"),
        "kernel_source_hash": kernel_source_hash("decode"),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 q, e4m3 KV" if w.kv8 else "bf16",
        "data": "synthetic", "config": dict(workload_config(w, world), split_kernel=args.kernel),
        "algorithmic_bytes_per_step_per_gpu": step_bytes,
        "clocks": clocks.summary(),
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "us_per_step": e2e_ms * 1e3, "h2d_bytes_per_step": world * h2d,
                "d2h_bytes_per_step": world * d2h,
                "path": "pinned q and seq_lens copied in, gqa_decode, out copied back, every step; copies "
                        "on two side streams overlap the neighbouring steps' kernels (two buffer sets); "
                        "KV cache resident in HBM"},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "split-KV decode kernel (partial merge included: the whole call)",
                     "kernel_us": split_ms_max * 1e3,
                     "kernel_timing": ("second pass, events around the decode kernel of every step" if appending
                                       else "the timed region: one decode kernel per step"),
                     "peak_note": f"{peak_kind} HBM copy bandwidth"},
        "device_status_flags": status,
    }
    if appending:
        append_us = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in append_ev), dist, dev) * 1e3
        line["config"]["path"] = "rope_append + decode"
        line["append_kernel_us"] = append_us
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w, inp, args.cpu_sample_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- multi-token (prefill) steps

def prefill_config(w, n):
    return {"workload": w.name, "B": w.B, "H_Q": w.H_Q, "H_KV": w.H_KV, "head_dim": w.D,
            "q_len": w.q_len, "prefix": w.prefix, "ragged": w.ragged, "page_size": w.page_size,
            "kv_dtype": "bf16", "out_dtype": "bf16", "global_batch": w.B * n,
            "l2": L2_NOTE,
            "parallelism": f"dp{n} (independent batch per GPU, no collective)"}


def cpu_oracle_prefill_sample(w, inp, seconds: float):
    """Time the fp64 oracle on the last query tokens of sequence 0 (all query
    heads; the tokens that see the most keys), sized to about `seconds`."""
    import numpy as np

    import oracle

    n, lens = prefill_lengths(w)
    cu = inp["cu_q"].numpy()
    threads = oracle.hardware_threads()

    def rows_for(count):
        lo = int(cu[1]) - count
        return [(i, h) for i in range(lo, int(cu[1])) for h in range(w.H_Q)]

    def run(count):
        t0 = time.perf_counter()
        oracle.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["seq_lens"], inp["cu_q"], w.softmax_scale,
                           rows=rows_for(count))
        return time.perf_counter() - t0

    per_tok = max(run(1), 1e-6)
    count = int(max(1, min(int(n[0]), seconds / per_tok)))
    dt = run(count)
    first = int(lens[0]) - count + 1  # keys seen by the first sampled token
    pairs = count * first + count * (count - 1) // 2
    flops = 4 * w.D * w.H_Q * pairs
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"last {count} query tokens of sequence 0 (all {w.H_Q} query heads, "
                      f"{first}..{int(lens[0])} visible keys each), fp64, {dt:.2f} s",
            "seconds": dt}


def run_reference_prefill(args):
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    w = prefill_workload(args)
    inp = make_prefill_inputs(w)
    t_start = time.perf_counter()
    results = [cpu_oracle_prefill_sample(w, inp, args.cpu_sample_seconds / max(args.steps, 1))
               for _ in range(args.steps)]
    total = time.perf_counter() - t_start
    value = statistics.median(r["value"] for r in results)
    last = results[-1]
    print(json.dumps({
        "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total * 1e3 / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": prefill_config(w, args.gpus),
        "cpu_baseline": {k: last[k] for k in ("kind", "cores", "sample")} | {"value": value, "unit": "TFLOP/s"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def run_ours_prefill(args):
    import gqa_mqa_kv_b200 as gq

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    w = prefill_workload(args)
    inp = make_prefill_inputs(w)
    n, lens_np = prefill_lengths(w)
    flops = prefill_flops(w, n, lens_np)
    paged = bool(w.page_size)
    q = inp["q"].to(dev)
    k = (inp["k_paged"] if paged else inp["k"]).to(dev)
    v = (inp["v_paged"] if paged else inp["v"]).to(dev)
    lens = inp["seq_lens"].to(dev)
    cu = inp["cu_q"].to(dev)
    table = inp["block_table"].to(dev) if paged else None
    max_q = inp["max_q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)

    def call(qq=None, oo=None):
        gq.gqa_prefill(q if qq is None else qq, k, v, lens, cu, max_q_len=max_q, block_table=table,
                       scale=w.softmax_scale, out=out if oo is None else oo, workspace=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush()
        call()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        t_soak = time.perf_counter()
        while time.perf_counter() - t_soak < args.soak_seconds:
            for _ in range(5):
                flush()
                call()
            torch.cuda.synchronize(dev)
        # ------------------------------------------------ timed region: K steps, L2 flushed between
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush()
            evs[i][0].record(stream)
            call()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    elapsed_ms = max_over_ranks(sum(step_ms), dist, dev)
    kernel_ms = max_over_ranks(statistics.mean(step_ms), dist, dev)
    status = gq.read_status(ws)

    # ---------------------------------------------------- end to end through the public API
    q_host = inp["q"].pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = q_host.numel() * q_host.element_size()
    d2h = out_host[0].numel() * out_host[0].element_size()
    q_sets = [q, torch.empty_like(q)]
    out_sets = [out, torch.empty_like(out)]
    e2e_ms = overlapped_e2e(dev, stream, [q_host], [[x] for x in q_sets],
                            lambda s: call(qq=q_sets[s], oo=out_sets[s]), out_sets, out_host,
                            max(1, min(args.e2e_steps, 20)), 2, dist)

    burst, sustained, peak_kind = tensor_peak()
    # The kernel runs back to back for seconds (soak, then the timed steps), so it
    # is in the sustained, power-capped regime; the clocks record shows it.
    peak = sustained
    ms_per_step = elapsed_ms / args.steps
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": world * flops / (ms_per_step * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "us_per_step": ms_per_step * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": prefill_config(w, world),
        "algorithmic_flops_per_step_per_gpu": flops, "kernel_source_hash": kernel_source_hash("prefill"),
        "clocks": clocks.summary(),
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "us_per_step": e2e_ms * 1e3,
                "h2d_bytes_per_step": world * h2d, "d2h_bytes_per_step": world * d2h,
                "path": "pinned q copied in, gqa_prefill, out copied back, every step; copies on two side "
                        "streams overlap the neighbouring steps' kernels (two buffer sets); KV cache resident in HBM"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(w.name),
                     "kernel": "prefill_tc_kernel (the whole call)", "kernel_us": kernel_ms * 1e3,
                     "peak_note": (f"{peak_kind} dense bf16 GEMM TFLOP/s, sustained (the kernel runs back to back "
                                   "for seconds under the power cap); frac_vs_burst divides by the burst figure"),
                     "peak_burst": burst, "frac_vs_burst": achieved / burst,
                     "tensor_work_note": "the value product runs twice (bf16 hi and lo parts of P): "
                                         "tensor-core work is 1.5x the algorithmic FLOPs"},
        "device_status_flags": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_prefill_sample(w, inp, args.cpu_sample_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    prefill = args.workload in PREFILL_WORKLOADS
    if args.impl == "reference":
        return run_reference_prefill(args) if prefill else run_reference(args)
    return run_ours_prefill(args) if prefill else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
