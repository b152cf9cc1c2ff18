#!/usr/bin/env python
"""Benchmark of the paged KV-cache segment attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--only decode]

Headline: multi-stream decode (16 one-row streams, 32/8 heads, head dim 128,
pages of 32 in a shuffled 8,192-page pool, 512-key partials + merge).  A step
is one decode pass over that batch: the split-KV partial kernel and the merge.
value = KV bytes a step reads (every visible key once per kv-head) / step time,
in GB/s, with inputs resident in HBM; three copies of the batch rotate between
steps (906 MB of KV, over seven times the L2), so no step finds its data in L2.
The timed steps replay CUDA graphs captured from the public calls, three
consecutive steps to a graph (one per input copy), so the Python binding's
host work never sits between two steps on the device and consecutive steps
meet at a kernel boundary inside a graph, as in a serving loop that captures
its steps; K steps are K // 3 graph replays plus the rest one step-graph
each.  The same step as one graph launch a step, and the calls issued
eagerly, are reported beside it.  A kernel's roofline divides its
algorithmic bytes (or FLOPs) by its average duration over launches issued
back to back, CUDA events at the two ends.  At N > 1 every rank runs its own replica of the batch
(independent streams, no collective on the data path) and value = all ranks'
bytes / the slowest rank's time ("weak" scaling).

Also reported (N = 1): the shared verify round (decode + merge + argmax), the
drafter ring, the 15,000-token prompt (TFLOP/s) and the 128,000-wide argmax
(rows/s), each with its own roofline; an end-to-end number through the public
API with host buffers; and the float64 oracle timed on the host cores.

--impl reference times the float64 oracle (the only reference there is) on
the same workload, metric and unit, a bounded sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "paged attn decode KV GB/s (% HBM peak); prompt attn TFLOP/s; argmax rows/s"
WORKLOAD = ("multi-stream decode: 16 streams x 1 row, 32 q / 8 kv heads, head dim 128, pages of 32 in a shuffled "
            "8,192-page pool, contexts U{1024..8192}, 512-key split-KV partials + merge, fp32 out")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


# ----------------------------------------------------------------------------- args / env

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--only", default="", help="comma list: decode,verify,ring,tree,prompt,argmax,block,append,e2e,cpu")
    ap.add_argument("--secondary-steps", type=int, default=24)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--secondary-cpu-seconds", type=float, default=3.0,
                    help="seconds of oracle time beside each secondary workload (0: one repetition)")
    return ap.parse_args()


def want(args, what):
    return not args.only or what in args.only.split(",")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {**FALLBACK_PEAKS, "source": "fallback"}


def load_traffic():
    """ncu DRAM bytes per launch recorded in profiles/ncu_traffic.json, valid
    only while the kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return {}
    out = {}
    for key, rec in d.items():
        src = os.path.join(ROOT, rec["source"])
        try:
            sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        except OSError:
            continue
        out[key] = rec["dram_bytes_per_launch"] if sha == rec["source_sha256"] else None
    return out


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while timing runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"tf_clocks_{os.getpid()}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, n = [], None, set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            n += 1
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        loaded = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": n}


def clocks_bad(c):
    if any(r in BAD_REASONS for r in c.get("reasons", [])):
        return True
    if c.get("sm_mhz") and c.get("sm_max_mhz") and c["sm_mhz"] < 0.5 * c["sm_max_mhz"] and not c.get("reasons"):
        return True
    return False


# ----------------------------------------------------------------------------- device helpers

def to_dev(a, dev):
    import torch

    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)


class DecodeRun:
    """Device buffers and the launches of one decode pass.  `copies` sets of
    the inputs live at different addresses; step k reads set k % copies, so
    with their total above the L2 size no step finds its data in L2."""

    def __init__(self, b, dev, logits=None, copies=3):
        import torch

        self.b = b
        rows, hq, d = b.q.shape
        self.sets = [dict(q=to_dev(b.q, dev), kp=to_dev(b.k_pool, dev), vp=to_dev(b.v_pool, dev),
                          pt=to_dev(b.page_table, dev), segs=to_dev(b.segs, dev),
                          logits=to_dev(logits, dev) if logits is not None else None)
                     for _ in range(copies)]
        c = b.n_splits_max
        self.po = torch.empty((rows, hq, c, d), device=dev)
        self.pm = torch.empty((rows, hq, c), device=dev)
        self.pl = torch.empty((rows, hq, c), device=dev)
        self.pf = torch.empty((rows, hq, c), dtype=torch.uint8, device=dev)
        self.out = torch.empty((rows, hq, d), device=dev)
        self.fl = torch.empty((rows, hq), dtype=torch.uint8, device=dev)
        self.st = torch.zeros(1, dtype=torch.int32, device=dev)
        if logits is not None:
            self.ids = torch.empty(logits.shape[0], dtype=torch.int32, device=dev)
            self.afl = torch.empty(logits.shape[0], dtype=torch.uint8, device=dev)

    def partial(self, k=0):
        import paged_kv_cache_segment_b200 as tf

        b, x = self.b, self.sets[k % len(self.sets)]
        tf.tf_paged_attn_decode(x["q"], x["kp"], x["vp"], x["pt"], x["segs"], scale=b.scale,
                                split_keys=b.split_keys, n_splits_max=b.n_splits_max, part_o=self.po,
                                part_m=self.pm, part_l=self.pl, part_flag=self.pf, status=self.st,
                                segs_host=b.segs)

    def merge(self, k=0):
        import paged_kv_cache_segment_b200 as tf

        tf.tf_attn_merge(self.po, self.pm, self.pl, self.pf, self.out, self.fl)

    def step(self, k=0):
        """One decode pass: partials, then the merge, back to back on the
        stream (the merge is a programmatic dependent of the partial kernel,
        so its launch overlaps the partial kernel's tail)."""
        self.partial(k)
        self.merge(k)

    def argmax(self, k=0):
        import paged_kv_cache_segment_b200 as tf

        tf.tf_argmax_rows(self.sets[k % len(self.sets)]["logits"], self.ids, self.afl)


def timed_steps(launches, steps):
    """Run `steps` steps, timing each launch of a step with CUDA events on the
    current stream.  Each launch gets the step index (it picks the input copy).
    Returns the per-launch total milliseconds and the step total."""
    import torch

    n = len(launches)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    for s in range(steps):
        evs[s][0].record()
        for k, fn in enumerate(launches):
            fn(s)
            evs[s][k + 1].record()
    torch.cuda.synchronize()
    per = [0.0] * n
    total = 0.0
    for s in range(steps):
        for k in range(n):
            per[k] += evs[s][k].elapsed_time(evs[s][k + 1])
        total += evs[s][0].elapsed_time(evs[s][n])
    return per, total


def graph_replayer(fn, copies):
    """Capture fn(k) for each input copy k in a CUDA graph (after one eager
    warm-up call each, which also loads the kernels) and return
    replay(k) -> replays copy k % copies.  The timed loop then launches a
    step's kernels without the Python binding's host work in between, so the
    device never waits for the host."""
    import torch

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for k in range(copies):
            fn(k)
    torch.cuda.current_stream().wait_stream(side)
    graphs = []
    for k in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn(k)
        graphs.append(g)

    def replay(k):
        graphs[k % copies].replay()

    replay.graphs = graphs
    return replay


def chain_replayer(fn, copies):
    """Capture fn(0), ..., fn(copies - 1) back to back in ONE CUDA graph
    (after an eager call of each, which also loads the kernels): consecutive
    steps then meet at a kernel boundary inside a graph, as in a serving loop
    that captures its decode steps, rather than at a graph launch, which costs
    the device a few microseconds of idle time per launch.  Returns
    run(steps) -> device milliseconds of exactly `steps` steps: steps // copies
    replays of the chain, then the remaining steps one graph each (step k
    always reads input copy k % copies), with CUDA events at the two ends."""
    import torch

    single = graph_replayer(fn, copies)
    chain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(chain, capture_error_mode="thread_local"):
        for k in range(copies):
            fn(k)

    def run(steps):
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps // copies):
            chain.replay()
        for k in range(steps - steps % copies, steps):
            single(k)
        z.record()
        torch.cuda.synchronize()
        return a.elapsed_time(z)

    run.single = single
    run.chain = chain
    return run


def time_cpu(fn, seconds, min_reps=1):
    """Repeat fn() until `seconds` have passed (at least min_reps times);
    returns (reps, elapsed seconds)."""
    t0 = time.perf_counter()
    reps = 0
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds and reps >= min_reps:
            return reps, el


def reduce_max(x: float, device, world: int) -> float:
    """The largest value of x over all ranks (every rank calls it, in the
    same order); the slowest rank's time is the job's time."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank's replica bytes over the slowest rank's time."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


def roofline(bound, achieved, peak, unit, traffic=None):
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4) if peak else None, "traffic": traffic}


# ----------------------------------------------------------------------------- the native arm

def bench_headline(args, wl, dev, world, peaks, traffic, barrier, max_over_ranks, local):
    """The headline: the multi-stream decode step (partials + merge) in KV GB/s."""
    b = wl.multi_stream_decode(2)
    kv_bytes = b.kv_bytes()
    run = DecodeRun(b, dev)
    # the step (partials + merge) captured three steps to a graph (one per
    # input copy) and replayed: the timed loop has no host work between steps,
    # and steps meet at kernel boundaries inside a graph; each kernel alone,
    # and the step as one graph launch each, for the record
    n_sets = len(run.sets)
    step_c = chain_replayer(run.step, n_sets)
    part_c = chain_replayer(run.partial, n_sets)
    step_g = step_c.single
    part_g = part_c.single
    merge_g = graph_replayer(run.merge, n_sets)
    for k in range(max(3, args.warmup)):
        step_g(k)
    step_c(n_sets)
    barrier()
    sampler = ClockSampler(local)
    result = None
    for attempt in range(2):
        sampler.start()
        barrier()
        # the timed region: exactly K steps, events at its two ends
        total = step_c(args.steps)
        barrier()
        # the partial kernel's launches back to back (chained the same way),
        # whose average duration is the roofline's denominator; then each
        # kernel with events around every launch, and the step as its own
        # graph launch
        part_b2b = part_c(args.steps) / args.steps
        per, _ = timed_steps([part_g, merge_g], args.steps)
        _, total_each = timed_steps([step_g], args.steps)
        barrier()
        clocks = sampler.stop()
        if not clocks_bad(clocks) or attempt == 1:
            break
    # the same step issued from Python through the binding every step, for
    # the record (host work per step then competes with the device's)
    n_eager = min(args.steps, 200)
    _, eager_total = timed_steps([run.step], n_eager)
    barrier()
    eager_ms = max_over_ranks(eager_total) / n_eager
    total_max = max_over_ranks(total)
    part_ms = part_b2b
    each_ms = max_over_ranks(total_each) / args.steps
    ms_step = total_max / args.steps
    assert int(run.st.item()) == 0, "device status set during the decode bench"
    value = whole_job_gbs(kv_bytes, world, ms_step)
    achieved = kv_bytes / (part_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded PCG64; bf16 ~N(0,1))",
        "config": {"workload": WORKLOAD, "streams": 16, "kv_bytes_per_step": kv_bytes,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: 3 rotating copies of the batch (906 MB of KV), step k reads copy k % 3"},
        "roofline": roofline("hbm", achieved, peaks["hbm_gbs"], "GB/s", traffic.get("decode_ws:multi_stream_decode")),
        "kernels": {"decode_partial_ms": round(part_ms, 5),
                    "decode_partial_ms_events_each": round(per[0] / args.steps, 5),
                    "merge_ms_alone": round(per[1] / args.steps, 5),
                    "merge_ms_in_step": round(ms_step - part_ms, 5),
                    "timing": "decode_partial_ms: the partial kernel's launches back to back (chained graphs), "
                              "events at the ends; *_events_each / merge_ms_alone: events around every launch"},
        "launch": "CUDA graphs of three consecutive steps (one per input copy, two kernels a step) replayed back "
                  "to back; K steps = K // 3 replays + the rest one step-graph each",
        "graph_each_step": {"ms_per_step": round(each_ms, 5), "value": round(whole_job_gbs(kv_bytes, world, each_ms), 2),
                            "path": "every step its own graph launch, an event between steps"},
        "eager": {"value": round(whole_job_gbs(kv_bytes, world, eager_ms), 2), "ms_per_step": round(eager_ms, 5),
                  "steps": n_eager, "path": "the same two calls issued through the Python binding every step"},
        "peaks_source": peaks["source"],
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    result["roofline"]["kernel"] = "decode_ws_kernel<128, paged>"
    result["roofline"]["frac_of"] = "measured" if peaks["source"] == "measured" else "fallback"
    result["roofline"]["frac_of_8tbs"] = round(achieved / 8000.0, 4)
    return result, b, run


def run_native(args):
    import torch
    import torch.distributed as dist

    from paged_kv_cache_segment_b200 import workloads as wl
    import paged_kv_cache_segment_b200 as tf

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    tf.load()
    peaks = load_peaks()
    traffic = load_traffic()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dev, world)

    # -------------------------------------------------------------- headline: decode
    b = run = None
    if want(args, "decode"):
        result, b, run = bench_headline(args, wl, dev, world, peaks, traffic, barrier, max_over_ranks, local)
    else:
        result = {"metric": METRIC, "only": args.only}

    # -------------------------------------------------------------- e2e through the public API, host buffers
    if want(args, "e2e") and run is not None:
        result["e2e"] = e2e_decode(b, run, min(args.steps, 500), barrier, max_over_ranks, world)

    # -------------------------------------------------------------- secondary workloads (N = 1 only)
    if world == 1:
        sec = {}
        ks = args.secondary_steps
        cs = args.secondary_cpu_seconds if want(args, "cpu") else 0.0
        if want(args, "verify") or want(args, "argmax"):
            sec.update(bench_verify(wl, dev, ks, peaks, traffic, cs))
        if want(args, "ring"):
            sec["ring"] = bench_ring(wl, tf, dev, ks, peaks, traffic, cs)
        if want(args, "tree"):
            sec["tree"] = bench_tree(wl, tf, dev, ks, peaks, traffic, cs)
        if want(args, "prompt"):
            sec["prompt"] = bench_prompt(wl, tf, dev, max(3, ks // 4), peaks, traffic, cs)
        if want(args, "block"):
            sec["block"] = bench_block(wl, tf, dev, ks, peaks, traffic, cs)
        if want(args, "append"):
            sec["append"] = bench_append(wl, tf, dev, ks, peaks, traffic, cs)
        result["secondary"] = sec
        result["gpu_launches_secondary"] = sum(v.get("launches", 0) for v in sec.values())
    if rank == 0 and world == 1 and want(args, "cpu") and b is not None:
        result["cpu_baseline"] = cpu_baseline(b, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def e2e_decode(b, run, steps, barrier, max_over_ranks, world):
    """The decode step through the public API with HOST inputs and outputs:
    pinned q / segment table / page table copied in, partials + merge, the
    output and flags copied back, every step inside the timed region.  The KV
    pool is the cache: it stays resident on the device (rotating copies).

    As a serving engine runs it, the copies overlap the compute: step k's
    inputs go in on a copy stream while step k-1 computes, and its results
    come back on another while step k+1 computes; events order each step's
    copy-in, compute and copy-out, and three staging buffers each way keep
    the steps in flight apart.  The timed region runs from before the first
    copy-in to after the last copy-out."""
    import torch

    import paged_kv_cache_segment_b200 as tf

    # one staging buffer each way a step, as a serving engine keeps them: the
    # step's inputs (q, segment table, page table) go in with one copy, its
    # results (output, flags) come back with one copy
    def align(n):
        return (n + 255) // 256 * 256

    qb, sb, pb = b.q.nbytes, b.segs.nbytes, b.page_table.nbytes
    o_in = [0, align(qb), align(qb) + align(sb)]
    n_in = o_in[2] + align(pb)
    stage_in = np.zeros(n_in, np.uint8)
    stage_in[0:qb] = np.frombuffer(np.ascontiguousarray(b.q).tobytes(), np.uint8)
    stage_in[o_in[1]:o_in[1] + sb] = np.frombuffer(np.ascontiguousarray(b.segs).tobytes(), np.uint8)
    stage_in[o_in[2]:o_in[2] + pb] = np.frombuffer(np.ascontiguousarray(b.page_table).tobytes(), np.uint8)
    in_h = torch.from_numpy(stage_in).pin_memory()
    ob, fb = run.out.numel() * 4, run.fl.numel()
    n_out = align(ob) + align(fb)
    dev = run.out.device
    nbuf = len(run.sets)
    out_h = [torch.empty(n_out, dtype=torch.uint8).pin_memory() for _ in range(nbuf)]
    staged = []
    for x in run.sets:
        buf = torch.empty(n_in, dtype=torch.uint8, device=dev)
        res = torch.empty(n_out, dtype=torch.uint8, device=dev)
        staged.append(dict(buf=buf, q=buf[0:qb].view(torch.int16).view(tuple(b.q.shape)),
                           segs=buf[o_in[1]:o_in[1] + sb].view(torch.int32).view(tuple(b.segs.shape)),
                           pt=buf[o_in[2]:o_in[2] + pb].view(torch.int32), kp=x["kp"], vp=x["vp"], res=res,
                           out=res[0:ob].view(torch.float32).view(tuple(run.out.shape)),
                           fl=res[align(ob):align(ob) + fb].view(tuple(run.fl.shape))))
    h2d = qb + sb + pb
    d2h = ob + fb
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = [dict(inp=torch.cuda.Event(), done=torch.cuda.Event(), out=torch.cuda.Event()) for _ in range(nbuf)]
    used = [False] * nbuf

    def step(k):
        i = k % nbuf
        x, e = staged[i], ev[i]
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(e["done"])  # the step before on this buffer has read its inputs
            x["buf"].copy_(in_h, non_blocking=True)
            e["inp"].record(s_in)
        comp.wait_event(e["inp"])
        if used[i]:
            comp.wait_event(e["out"])  # its results have been copied out
        tf.tf_paged_attn_decode(x["q"], x["kp"], x["vp"], x["pt"], x["segs"], scale=b.scale,
                                split_keys=b.split_keys, n_splits_max=b.n_splits_max, part_o=run.po, part_m=run.pm,
                                part_l=run.pl, part_flag=run.pf, status=run.st, segs_host=b.segs, stream=comp)
        tf.tf_attn_merge(run.po, run.pm, run.pl, run.pf, x["out"], x["fl"], stream=comp)
        e["done"].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e["done"])
            out_h[i].copy_(x["res"], non_blocking=True)
            e["out"].record(s_out)
        used[i] = True

    def run_steps(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(comp)
        s_in.wait_event(t0)
        for k in range(n):
            step(k)
        for e in ev:
            if used[ev.index(e)]:
                comp.wait_event(e["out"])
        t1.record(comp)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    run_steps(3)
    barrier()
    # the binding's host time a step (two calls, the copies and the events)
    t0 = time.perf_counter()
    for k in range(steps):
        step(k)
    host_us = (time.perf_counter() - t0) / steps * 1e6
    barrier()
    total = run_steps(steps)
    barrier()
    total = max_over_ranks(total)
    ms = total / steps
    return {"value": round(world * b.kv_bytes() / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "host_us_per_step": round(host_us, 1),
            "path": "binding tf_paged_attn_decode + tf_attn_merge issued every step; one pinned staging buffer in "
                    "(q, segment and page tables) and one out (output and flags) a step, copied on their own streams "
                    "so step k's copy-in and step k-1's copy-out overlap the compute"}


def oracle_cpu(fn, seconds, value_per_rep, unit, sample):
    """The float64 oracle as it stands, timed on this host's cores: fn() is
    one bounded unit of the workload, repeated for about `seconds`."""
    import oracle

    if seconds <= 0:
        return None
    reps, el = time_cpu(fn, seconds)
    return {"value": round(reps * value_per_rep / el, 6), "unit": unit, "cores": oracle.get().num_threads(),
            "kind": "oracle", "sample": f"{reps} x {sample} in {el:.1f} s"}


def bench_verify(wl, dev, steps, peaks, traffic, cpu_s):
    import oracle
    import paged_kv_cache_segment_b200 as tf

    # the split size the library chooses for this batch on this device
    b0 = wl.shared_verify(3)
    split, _ = tf.tf_choose_split_keys(b0.segs, n_q_heads=b0.n_q_heads, n_kv_heads=b0.n_kv_heads,
                                       head_dim=b0.head_dim)
    b = wl.shared_verify(3, split_keys=split)
    rows = b.n_rows_total
    logits = wl.verify_logits(3, rows)
    run = DecodeRun(b, dev, logits, copies=8)  # 8 x (151 MB of KV + 17 MB of logits)
    n = len(run.sets)
    part_c, arg_c = chain_replayer(run.partial, n), chain_replayer(run.argmax, n)
    pm_c = chain_replayer(lambda k: (run.partial(k), run.merge(k)), n)
    three_c = chain_replayer(lambda k: (run.partial(k), run.merge(k), run.argmax(k)), n)
    part_g, arg_g = part_c.single, arg_c.single
    merge_g = graph_replayer(run.merge, n)
    for k in range(3):
        part_g(k)
        merge_g(k)
        arg_g(k)
    per, _ = timed_steps([part_g, merge_g, arg_g], steps)
    pm_ms = pm_c(steps) / steps  # the verify step: partials + merge
    three_ms = three_c(steps) / steps  # the round as three calls

    # the same round as one call (tf_verify_round): merge and argmax launch as
    # programmatic dependents, timed at the round's ends
    def round_call(k):
        x = run.sets[k % len(run.sets)]
        tf.tf_verify_round(x["q"], x["kp"], x["vp"], x["pt"], x["segs"], scale=b.scale, split_keys=b.split_keys,
                           n_splits_max=b.n_splits_max, part_o=run.po, part_m=run.pm, part_l=run.pl,
                           part_flag=run.pf, out=run.out, flags=run.fl, status=run.st, logits=x["logits"],
                           ids=run.ids, id_flags=run.afl, segs_host=b.segs)

    round_c = chain_replayer(round_call, n)
    round_ms = round_c(steps) / steps
    # each kernel's launches back to back over the 8 copies (chained graphs),
    # events at the ends only: the average launch duration, the rooflines'
    # denominator
    part_b2b = part_c(steps) / steps
    arg_b2b = arg_c(steps) / steps
    kv = b.kv_bytes()
    pms, mms, ams = per[0] / steps, per[1] / steps, per[2] / steps
    flops = 4 * b.head_dim * sum(int(s[1]) * b.n_q_heads * (int(s[2]) - int(s[1]) + 1) + b.n_q_heads *
                                 int(s[1]) * (int(s[1]) - 1) // 2 for s in b.segs)
    arg_bytes = rows * 128000 * 2
    orc = oracle.get()
    cpu_verify = oracle_cpu(lambda: orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale),
                            cpu_s, kv / 1e9, "GB/s", "whole passes of the verify batch")
    cpu_arg = oracle_cpu(lambda: orc.argmax_rows(logits), cpu_s, rows, "rows/s",
                         f"whole passes of the {rows} x 128,000 logits")
    out = {
        "verify": {"workload": "shared verify: 8 streams x U{1..16} rows, 16/2 heads, D256, P32, contexts "
                               f"U{{2048..16384}}, {split}-key partials (tf_choose_split_keys) + merge", "rows": rows,
                   "split_keys": split,
                   "kv_gbs": round(kv / pm_ms / 1e6, 2), "ms_per_step": round(pm_ms, 5),
                   "ms_per_step_events_each": round(pms + mms, 5),
                   "tflops": round(flops / (part_b2b * 1e-3) / 1e12, 2),
                   "partial_ms": round(part_b2b, 5), "partial_ms_events_each": round(pms, 5),
                   "roofline": dict(roofline("hbm", kv / (part_b2b * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                                             traffic.get("prompt_tc:shared_verify")),
                                    kernel="prompt_tc_kernel<256, hilo, partial>"),
                   "cpu_baseline": cpu_verify,
                   "launches": 2 * steps, "l2": "8 rotating copies"},
        "round": {"workload": "the shared verify round in one call: partials, merge, argmax of its 62 rows",
                  "ms": round(round_ms, 5), "ms_three_calls": round(three_ms, 5),
                  "kv_plus_logit_gbs": round((kv + arg_bytes) / round_ms / 1e6, 2),
                  "launches": 3 * steps},
        "argmax": {"workload": f"{rows} rows x 128,000 bf16 ~N(0,3), ties in ~1/4 of rows",
                   "rows_per_s": round(rows / (arg_b2b * 1e-3), 1), "ms": round(arg_b2b, 5),
                   "ms_events_each": round(ams, 5),
                   "roofline": roofline("hbm", arg_bytes / (arg_b2b * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                                        traffic.get("argmax:verify_logits")),
                   "cpu_baseline": cpu_arg,
                   "launches": 2 * steps},
    }
    assert int(run.st.item()) == 0
    return out


def bench_ring(wl, tf, dev, steps, peaks, traffic, cpu_s):
    import torch

    import oracle
    from paged_kv_cache_segment_b200 import binding

    b = wl.drafter_ring(5)
    n = len(b.rsegs)
    hq, d = b.n_q_heads, b.head_dim
    sets = [dict(q=to_dev(b.q, dev), rk=to_dev(b.ring_k, dev), rv=to_dev(b.ring_v, dev),
                 rs=binding.rsegs_to_device(b.rsegs, dev)) for _ in range(3)]  # 3 x 146 MB of rings
    ws = torch.empty(tf.tf_ring_workspace_bytes(n, hq, d, b.n_splits_max), dtype=torch.uint8, device=dev)
    out = torch.empty((n, hq, d), device=dev)
    fl = torch.empty((n, hq), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(k):
        x = sets[k % 3]
        tf.tf_ring_attn(x["q"], x["rk"], x["rv"], x["rs"], scale=b.scale, split_slots=b.split_slots,
                        n_splits_max=b.n_splits_max, workspace=ws, out=out, flags=fl, status=st, rsegs_host=b.rsegs)

    c = chain_replayer(step, 3)
    c(3)
    ms = c(steps) / steps
    _, total_each = timed_steps([c.single], steps)
    kv = b.kv_bytes()
    assert int(st.item()) == 0
    orc = oracle.get()
    cpu = oracle_cpu(lambda: orc.ring_attn(b.q, b.ring_k, b.ring_v, b.rsegs, b.scale), cpu_s, kv / 1e9, "GB/s",
                     "whole passes of the 17 rings")
    return {"workload": "drafter ring: 17 rows, rings of 4,200 slots, random heads, U{1000..4200} valid, 16/2 heads, "
                        "D256, 320-slot partials + merge", "kv_gbs": round(kv / (ms * 1e-3) / 1e9, 2),
            "ms_per_step": round(ms, 5), "ms_per_step_graph_each": round(total_each / steps, 5),
            "pages_ms_reference": "0.24 ms a 4,200-slot draft step on GB10 (one stream)",
            "roofline": roofline("hbm", kv / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                                 traffic.get("decode_ws:drafter_ring")), "cpu_baseline": cpu,
            "launches": 2 * steps, "l2": "3 rotating copies"}


def bench_tree(wl, tf, dev, steps, peaks, traffic, cpu_s):
    """Draft trees over rings: 17 trees of 4-16 nodes (chain, star, binary,
    random) after windows of 1,000-4,184 slots of their own 4,200-slot rings,
    16/2 heads, D 256; 3 rotating copies of the rings."""
    import torch

    import oracle
    from paged_kv_cache_segment_b200 import binding

    b = wl.drafter_trees(6)
    rows, hq, d = b.q.shape
    sets = [dict(q=to_dev(b.q, dev), rk=to_dev(b.ring_k, dev), rv=to_dev(b.ring_v, dev),
                 ts=binding.tsegs_to_device(b.tsegs, dev), par=to_dev(b.parents, dev)) for _ in range(3)]
    ws = torch.empty(tf.tf_ring_tree_workspace_bytes(rows, hq, d, b.n_splits_max), dtype=torch.uint8, device=dev)
    out = torch.empty((rows, hq, d), device=dev)
    fl = torch.empty((rows, hq), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(k):
        x = sets[k % 3]
        tf.tf_ring_tree_attn(x["q"], x["rk"], x["rv"], x["ts"], x["par"], scale=b.scale, split_slots=b.split_slots,
                             n_splits_max=b.n_splits_max, workspace=ws, out=out, flags=fl, status=st,
                             tsegs_host=b.tsegs, parents_host=b.parents)

    c = chain_replayer(step, 3)
    c(3)
    ms = c(steps) / steps
    _, total_each = timed_steps([c.single], steps)
    kv = b.kv_bytes()
    assert int(st.item()) == 0
    orc = oracle.get()
    cpu = oracle_cpu(lambda: orc.ring_tree_attn(b.q, b.ring_k, b.ring_v, b.tsegs, b.parents, b.scale), cpu_s,
                     kv / 1e9, "GB/s", "whole passes of the 17 trees")
    return {"workload": "drafter trees: 17 trees of U{4..16} nodes (chain/star/binary/random) after windows of "
                        "U{1000..4184} slots of 4,200-slot rings, 16/2 heads, D256, "
                        f"{b.split_slots}-slot partials + merge", "nodes": rows,
            "kv_gbs": round(kv / (ms * 1e-3) / 1e9, 2), "ms_per_step": round(ms, 5),
            "ms_per_step_graph_each": round(total_each / steps, 5),
            "roofline": dict(roofline("hbm", kv / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                                      traffic.get("prompt_tc:drafter_trees")),
                             kernel="prompt_tc_kernel<256, hilo, partial, tree> + merge (the whole step)"),
            "cpu_baseline": cpu, "launches": 2 * steps, "l2": "3 rotating copies"}


def bench_prompt(wl, tf, dev, steps, peaks, traffic, cpu_s):
    import torch

    import oracle

    b, spans = wl.long_prompt(4)
    rows, hq, d = b.q.shape
    sets = [dict(q=to_dev(b.q, dev), kp=to_dev(b.k_pool, dev), vp=to_dev(b.v_pool, dev), pt=to_dev(b.page_table, dev))
            for _ in range(2)]  # 2 x 184 MB
    out = torch.empty((rows, hq, d), dtype=torch.bfloat16, device=dev)
    fl = torch.empty((rows, hq), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    segs = [wl.prompt_chunk_seg(b, r0, r1) for r0, r1 in spans]

    def step(k):
        x = sets[k % 2]
        for sg in segs:
            tf.tf_paged_attn_prompt(x["q"], x["kp"], x["vp"], x["pt"], sg, scale=b.scale, out=out, flags=fl,
                                    status=st)

    c = chain_replayer(step, 2)
    c(2)
    ms = c(steps) / steps
    _, total_each = timed_steps([c.single], steps)
    n = rows
    flops = 4 * d * hq * n * (n + 1) // 2
    assert int(st.item()) == 0
    tfl = flops / (ms * 1e-3) / 1e12
    # the oracle on a bounded sample: the prompt's last 32 rows, all heads
    orc = oracle.get()
    sel = np.zeros((rows, hq), np.uint8)
    sel[rows - 32:, :] = 1
    sample_flops = 4 * d * hq * sum(range(rows - 32 + 1, rows + 1))
    cpu = oracle_cpu(lambda: orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, sel=sel), cpu_s,
                     sample_flops / 1e12, "TFLOP/s", "the prompt's last 32 rows x 16 heads (14,969-15,000 keys each)")
    return {"workload": "long causal prompt: 15,000 tokens in 2,048-row chunks, 16/4 heads, D256, P32, 469 shuffled "
                        "pages, bf16 out", "tflops": round(tfl, 2), "ms_per_step": round(ms, 4),
            "ms_per_step_graph_each": round(total_each / steps, 4),
            "algorithmic_flops": flops,
            "roofline": dict(roofline("tensor", tfl, peaks["bf16_tflops"], "TFLOP/s",
                                      traffic.get("prompt_tc:long_prompt")), kernel="prompt_tc_kernel<256, bf16>",
                             traffic_is="DRAM bytes per chunk launch (mean of 8); the K/V of a chunk is re-read from L2"),
            "cpu_baseline": cpu,
            "launches": len(segs) * steps,
            "l2": "2 rotating copies"}


def bench_block(wl, tf, dev, steps, peaks, traffic, cpu_s):
    """A drafter-block round: 16 streams, each a block of 9 rows seeing all of
    its stream's keys (the FULL rule), contexts U{1,024..8,192}, 32/8 heads,
    D 128, pages of 32, 768-key partials (the fastest of 512-2,048 in a sweep
    on a B200) + merge; 3 rotating copies."""
    import oracle

    b0 = wl.multi_stream_decode(2)
    keys = [int(x) for x in b0.segs[:, 2]]
    b = wl.make_paged_batch(12, [9] * len(keys), keys, 32, 8, 128, 32, unused="nan", split_keys=768)
    run = DecodeRun(b, dev)

    def step(k):
        x = run.sets[k % len(run.sets)]
        tf.tf_paged_attn_block(x["q"], x["kp"], x["vp"], x["pt"], x["segs"], scale=b.scale,
                               split_keys=b.split_keys, n_splits_max=b.n_splits_max, part_o=run.po, part_m=run.pm,
                               part_l=run.pl, part_flag=run.pf, status=run.st, segs_host=b.segs)
        run.merge(k)

    c = chain_replayer(step, len(run.sets))
    c(len(run.sets))
    ms = c(steps) / steps
    _, total_each = timed_steps([c.single], steps)
    kv = b.kv_bytes()
    assert int(run.st.item()) == 0
    orc = oracle.get()
    sel = np.zeros((b.n_rows_total, b.n_q_heads), np.uint8)
    sel[:, :b.n_q_heads // b.n_kv_heads] = 1  # kv-head 0's q-heads: an eighth of the work
    cpu = oracle_cpu(lambda: orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, full=True,
                                            sel=sel), cpu_s, kv / b.n_kv_heads / 1e9, "GB/s",
                     "kv-head 0 of every block (all rows, its 4 q-heads)")
    return {"workload": "drafter blocks: 16 streams x 9 rows, every row over all its stream's keys, contexts "
                        "U{1024..8192}, 32/8 heads, D128, P32, 768-key partials + merge",
            "kv_gbs": round(kv / (ms * 1e-3) / 1e9, 2), "ms_per_step": round(ms, 5),
            "ms_per_step_graph_each": round(total_each / steps, 5),
            "roofline": dict(roofline("hbm", kv / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                                      traffic.get("prompt_tc:drafter_block")),
                             kernel="prompt_tc_kernel<128, hilo, partial> + merge (the whole step)"),
            "cpu_baseline": cpu,
            "launches": 2 * steps, "l2": "3 rotating copies"}


def bench_append(wl, tf, dev, steps, peaks, traffic, cpu_s):
    """The 15,000-token prompt's keys and values appended in one call (4
    kv-heads, D 256, pages of 32) into a shuffled pool; 3 rotating pool
    copies.  Bytes: every row read once from the row arrays and written once
    into the pools."""
    import torch

    import oracle

    b, _ = wl.long_prompt(4)
    n, hkv, d = b.n_rows_total, b.n_kv_heads, b.head_dim
    rng = np.random.default_rng(13)
    kr_h = wl.normal_bf16(rng, (n, hkv, d))
    vr_h = wl.normal_bf16(rng, (n, hkv, d))
    kr, vr = to_dev(kr_h, dev), to_dev(vr_h, dev)
    pools = [(to_dev(b.k_pool, dev), to_dev(b.v_pool, dev)) for _ in range(3)]
    pt = to_dev(b.page_table, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seg = b.segs[0]
    # one call over all rows: the kernel's own rate (chunk-sized calls of a
    # few microseconds each would time the host's launch path instead)
    sh = np.array([[0, n, n, seg[3], seg[4]]], np.int32)
    sd = to_dev(sh, dev)

    def step(k):
        kp, vp = pools[k % 3]
        tf.tf_kv_append(kr, vr, kp, vp, pt, sd, status=st, segs_host=sh)

    c = chain_replayer(step, 3)
    c(3)
    ms = c(steps) / steps
    _, total_each = timed_steps([c.single], steps)
    moved = 2 * 2 * n * hkv * d * 2  # K and V, read from the rows and written into the pages
    assert int(st.item()) == 0
    gbs = moved / (ms * 1e-3) / 1e9
    orc = oracle.get()
    cpu = oracle_cpu(lambda: orc.put_rows(kr_h, vr_h, b.k_pool, b.v_pool, b.page_table, sh), cpu_s, moved / 1e9,
                     "GB/s", "whole appends of the 15,000 rows (the oracle copies both pools first)")
    return {"workload": "append the 15,000-token prompt's K/V rows into 469 shuffled pages of 32 in one call "
                        "(4 kv-heads, D256)", "gbs": round(gbs, 2), "ms_per_step": round(ms, 5),
            "ms_per_step_graph_each": round(total_each / steps, 5),
            "bytes_per_step": moved, "roofline": dict(roofline("hbm", gbs, peaks["hbm_gbs"], "GB/s",
                                                               traffic.get("kv_append:long_prompt")),
                                                      kernel="kv_append_kernel<256>"),
            "cpu_baseline": cpu,
            "launches": steps, "l2": "3 rotating pool copies (rows arrays resident)"}


def cpu_baseline(b, seconds):
    """The float64 oracle, as it stands, on this host's cores: whole passes of
    the decode workload repeated for about `seconds`."""
    import oracle

    orc = oracle.get()
    t0 = time.perf_counter()
    reps = 0
    while True:
        orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(reps * b.kv_bytes() / el / 1e9, 4), "unit": "GB/s", "cores": orc.num_threads(),
            "kind": "oracle", "sample": f"{reps} whole passes of the 16-stream decode batch in {el:.1f} s"}


# ----------------------------------------------------------------------------- the reference arm (the oracle)

def run_reference(args):
    """The reference arm: the float64 oracle (there is no reference
    implementation to install: the pages hold no code) on the headline's own
    workload, a step being one whole pass over the 16-stream decode batch, as
    in the native arm; timed on the host cores.  Under torchrun only rank 0
    runs it."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from paged_kv_cache_segment_b200 import workloads as wl

    orc = oracle.get()
    b = wl.multi_stream_decode(2)

    def step():
        orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)

    for _ in range(args.warmup):
        step()
    budget = 150.0
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        step()
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    el = time.perf_counter() - t0
    v = done * b.kv_bytes() / el / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": done, "warmup": args.warmup, "ms_per_step": round(el / max(done, 1) * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": "whole passes of the 16-stream decode batch, one a step"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": orc.num_threads(), "kind": "oracle",
                         "sample": f"{done} whole passes of the 16-stream decode batch in {el:.1f} s"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
