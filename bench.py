#!/usr/bin/env python3
"""Benchmark of the any4 W4A16 matmul on B200: one JSON line.

Metric: any4 matmul HBM GB/s and us at M = 1, TFLOPS at M = 2048, % of roofline.

A step is one pass of the Llama3-8B-shaped decode layer at M = 1: the seven
any4_matmul calls of one transformer layer (q, k, v, o projections K = 4096;
gate and up K = 4096, N = 14336; down K = 14336, N = 4096), group size
G = 128, on seeded synthetic weights (no model weights exist here).  `value`
is the whole-job algorithmic HBM throughput (packed codes + scales/offsets +
tables + x + y per call, summed over the seven calls and over all ranks,
divided by the max-over-ranks device time).  Weights are rotated over enough
copies that the working set exceeds L2 (every step reads cold weights).

Also reported (same run, not part of the step): the prefill matmuls at
M = 2048 (TFLOPS), the roofline object of the decode kernel, the CPU oracle
as a baseline, the end-to-end number through the public API with host
buffers, the clocks seen during the timed region, the single-call latency of
each M = 1 shape, the time any4_quantize takes to learn the tables of the
Llama3-8B matrices (beside the oracle), and the any3 / any2 / any4 dequant rate.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 launch under torch.distributed.run; each rank runs an independent
replica on its own GPU (the path has no exchange step), `scaling` = "weak".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "any4 matmul HBM GB/s & µs (M=1), TFLOPS (M=2048), % of roofline"
L2_BYTES = 132644864
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except Exception:
        return dict(FALLBACK_PEAKS)


def kernel_source_hash() -> str:
    """Hash of the M = 1 weight-streaming decode kernel source (the only kernel of a step): a
    stored ncu traffic figure is only used while it was taken on this source."""
    h = hashlib.sha256()
    for fn in ("decode_tma.cu", "common.cuh"):
        with open(os.path.join(ROOT, "learned_bit_lut_any4_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic():
    """Per-launch DRAM bytes (read + write) of the decode kernel on this step,
    from the committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_tma_ffma_kernel_llama3_8b_layer_m1.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.]+)", text)
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_sum(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "clocks.mem")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"any4_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sms, maxs, mems, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
            if len(parts) > 9:
                try:
                    mems.append(float(parts[9]))
                except ValueError:
                    pass
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sms:
            return None
        return {"sm_mhz": float(np.median(sms)), "sm_max_mhz": float(max(maxs)),
                "reasons": sorted(reasons), "samples": len(sms),
                "mem_mhz": float(np.median(mems)) if mems else None}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _dev_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


_WS = {}


def ws_for(s):
    """One decode workspace shared by every call of this process (calls on one
    stream run in order, and the kernels touch it only after their
    predecessor has finished), grown to the largest size asked for."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    need = any4.any4_matmul_workspace_size(s.M, s.N, s.K, s.G)
    if s.M > 16:
        return None  # prefill: the binding allocates its workspace
    cur = _WS.get("decode")
    if cur is None or cur.numel() < need:
        cur = _WS["decode"] = torch.empty(max(need, 1 << 16), dtype=torch.uint8, device="cuda")
    return cur


def prepare_layer(shapes, copies):
    """Device copies of each shape's weights (packed on the device by
    any4_pack), plus x and y buffers."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    sets = []
    for s in shapes:
        p = workloads.make(s)
        packed = any4.any4_pack(torch.from_numpy(p.idx).cuda())
        lut, sc, of = _dev_bf16(p.lut), _dev_bf16(p.scale), _dev_bf16(p.offset)
        reps = [(packed, lut, sc, of)] + [(packed.clone(), lut.clone(), sc.clone(), of.clone())
                                          for _ in range(copies - 1)]
        x = _dev_bf16(p.x)
        y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device="cuda")
        sets.append((s, reps, x, y, p.x))
    torch.cuda.synchronize()
    return sets


def read_stream_rate(stream, nbytes=2 << 30, reps=10):
    """HBM read bandwidth (GB/s, median and best of `reps` launches) of
    any4_read_probe over a buffer of nbytes (16x the L2), CUDA events on
    `stream`: the read-only ceiling of the decode matmuls, which read about 250
    bytes for each byte they write."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(1, dtype=torch.int32, device="cuda")
    times = []
    with torch.cuda.stream(stream):
        for _ in range(3):
            any4.any4_read_probe(buf, out)
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            any4.any4_read_probe(buf, out)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b) * 1e-3)
    del buf
    rates = sorted(nbytes / t / 1e9 for t in times)
    return {"gbs_median": round(float(np.median(rates)), 1), "gbs_best": round(rates[-1], 1),
            "bytes": nbytes, "launches": reps, "kernel": "read_probe_kernel (any4_read_probe)"}


def _time_graph(stream, calls, n_rep):
    """µs per call of `calls` (a list of no-argument callables) captured once in
    a CUDA graph and replayed n_rep times on `stream` (events on that stream)."""
    import torch
    with torch.cuda.stream(stream):
        for f in calls:
            f()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for f in calls:
            f()
    with torch.cuda.stream(stream):
        g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_rep):
            g.replay()
        b.record(stream)
    b.synchronize()
    us = a.elapsed_time(b) * 1e3 / (n_rep * len(calls))
    del g
    return us


def fig3_square_sweep(stream, overlap):
    """The paper's speed study (Fig. 3): one row of x times square K x K weights,
    any4 (a table per row) against the one-table modes through the same kernels
    (nf4-style table from normal quantiles; int4 as the table {-8..7}) and
    against torch's dense bf16 matmul of the dequantised W (cuBLAS; context).
    Every variant cycles over weight copies larger than L2."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    from statistics import NormalDist
    nd = NormalDist()
    neg = [-nd.inv_cdf(0.5 + 0.5 * (1 - (i + 0.5) / 8)) for i in range(8)]
    pos = [nd.inv_cdf(0.5 + 0.5 * (i + 1) / 8.5) for i in range(7)]
    nf4 = np.array(sorted(neg + [0.0] + pos))
    nf4 = (nf4 / np.abs(nf4).max()).astype(np.float32)
    t_nf4 = torch.from_numpy(nf4).cuda().to(torch.bfloat16)
    t_int4 = torch.arange(-8, 8, dtype=torch.float32, device="cuda").to(torch.bfloat16)
    out = {}
    for K in (1024, 2048, 4096, 8192, 16384):
        s = workloads.Shape(f"fig3_{K}", 1, K, K, 128, 7000 + K, 7100 + K)
        wbytes = s.N * s.K // 2 + 4 * s.N * (s.K // s.G) + 32 * s.N
        copies = max(2, int(np.ceil(3 * L2_BYTES / wbytes)))
        (_, reps, x, y, _), = prepare_layer([s], copies)
        n_rep = max(3, 400 // copies)
        res = {}
        for name, table in (("any4", None), ("nf4_style", t_nf4), ("int4", t_int4)):
            calls = [(lambda w=w, t=table: any4.any4_matmul(
                x, w[0], w[1] if t is None else t, w[2], w[3], s.G, y=y, overlap_prior=overlap,
                workspace=ws_for(s)))
                for w in reps]
            res[name + "_us"] = round(_time_graph(stream, calls, n_rep), 3)
        W = any4.any4_dequant(reps[0][0], reps[0][1], reps[0][2], reps[0][3], s.G)
        dcopies = max(1, int(np.ceil(3 * L2_BYTES / (2 * s.N * s.K))))
        Ws = [W] + [W.clone() for _ in range(dcopies - 1)]
        xd = x.clone()
        calls = [(lambda Wc=Wc: torch.nn.functional.linear(xd, Wc)) for Wc in Ws]
        res["bf16_dense_us"] = round(_time_graph(stream, calls, max(3, 400 // dcopies)), 3)
        for name in ("any4", "nf4_style", "int4"):
            res[name + "_speedup_vs_bf16"] = round(res["bf16_dense_us"] / res[name + "_us"], 2)
        out[str(K)] = res
        del reps, x, y, W, Ws, xd
        torch.cuda.synchronize()
    return out


def time_weight_set(shapes, stream, overlap, peaks, decode_layout=False):
    """Time any4_matmul on one weight set (the shapes share a weight seed and
    differ in M and x) on rotating weight copies larger than L2, replayed in
    a CUDA graph; per shape µs per call, GB/s of its algorithmic bytes and the
    fraction of the HBM peak (+ TFLOPS for M > 16).  decode_layout: the codes
    repacked by any4_repack (set-up, untimed) and read with that flag."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    s0 = shapes[0]
    wbytes = s0.N * s0.K // 2 + 4 * s0.N * (s0.K // s0.G) + 32 * s0.N
    bc = max(2, int(np.ceil(3 * L2_BYTES / wbytes)))
    (_, reps, _, _, _), = prepare_layer([s0], bc)
    if decode_layout:
        reps = [(any4.any4_repack(w[0]), w[1], w[2], w[3]) for w in reps]
    out = {}
    for s in shapes:
        x = _dev_bf16(workloads.draw_x(s))
        y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device="cuda")
        ws = ws_for(s)
        calls = [(lambda w=w: any4.any4_matmul(x, w[0], w[1], w[2], w[3], s.G, y=y,
                                               overlap_prior=overlap, workspace=ws,
                                               decode_layout=decode_layout))
                 for w in reps]
        us = _time_graph(stream, calls, max(2, 200 // bc))
        gbs = s.alg_bytes() / (us * 1e-6) / 1e9
        r = {"M": s.M, "K": s.K, "N": s.N, "G": s.G, "us": round(us, 3), "GB/s": round(gbs, 1),
             "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        if s.M > 16:
            r["TFLOPS"] = round(s.flops() / (us * 1e-6) / 1e12, 2)
        out[s.name] = r
        del x, y
    del reps
    return out


# The layer's seven matmuls as the four calls a decoder makes: the projections
# that read the same activations run as one grouped call (q/k/v; gate/up).
LAYER_CALLS = (("8b_q", "8b_k", "8b_v"), ("8b_o",), ("8b_gate", "8b_up"), ("8b_down",))


def layer_plan(sets, grouped):
    """Index lists into `sets`: one list per call of a layer step."""
    names = [s.name for (s, *_r) in sets]
    if not grouped:
        return [[i] for i in range(len(sets))]
    return [[names.index(n) for n in call] for call in LAYER_CALLS]


def run_call(sets, idxs, c, copies, overlap, x=None, ys=None):
    """One call of a layer step on weight copy c: any4_matmul for one matrix,
    any4_matmul_grouped for matrices sharing x (the first matrix's x)."""
    import learned_bit_lut_any4_b200 as any4
    s0, reps0, x0, y0, _ = sets[idxs[0]]
    x = x0 if x is None else x
    if len(idxs) == 1:
        w = reps0[c % copies]
        any4.any4_matmul(x, w[0], w[1], w[2], w[3], s0.G, y=y0 if ys is None else ys[0],
                         overlap_prior=overlap, workspace=ws_for(s0))
    else:
        any4.any4_matmul_grouped(x, [sets[i][1][c % copies] for i in idxs], s0.G,
                                 ys=[sets[i][3] for i in idxs] if ys is None else ys,
                                 overlap_prior=overlap, workspace=ws_for(s0))


def gpu_arm(args, rank, world):
    import torch
    import learned_bit_lut_any4_b200 as any4

    peaks = load_peaks()
    shapes = workloads.LLAMA3_8B_DECODE
    layer_weight_bytes = sum(s.N * s.K // 2 + 4 * s.N * (s.K // s.G) + 32 * s.N for s in shapes)
    copies = max(2, int(np.ceil(3 * L2_BYTES / layer_weight_bytes)))
    sets = prepare_layer(shapes, copies)
    step_bytes = sum(s.alg_bytes() for s in shapes)
    overlap = not args.no_overlap
    stream = torch.cuda.Stream()

    plan = layer_plan(sets, grouped=not args.ungrouped)

    def step(c, plan=plan):
        for idxs in plan:
            run_call(sets, idxs, c, copies, overlap)

    # one graph = `copies` steps (each step on the next weight copy)
    with torch.cuda.stream(stream):
        for c in range(copies):
            step(c)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for c in range(copies):
            step(c)
    reps_needed = max(1, args.steps // copies)
    steps_timed = reps_needed * copies
    warm = max(1, int(np.ceil(args.warmup / copies)))
    with torch.cuda.stream(stream):
        for _ in range(warm):
            graph.replay()
    stream.synchronize()

    sampler = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first reading before the timed region
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps_needed):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms_local = e0.elapsed_time(e1)
    ms = allreduce_max(ms_local, world)
    ms_per_step = ms / steps_timed
    total_bytes = allreduce_sum(step_bytes * steps_timed, world)
    value_gbs = total_bytes / (ms * 1e-3) / 1e9

    # per-shape detail (each shape alone, same rotation, events on its stream)
    detail = {}
    for (s, reps, x, y, _) in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in range(copies):
                w = reps[c]
                any4.any4_matmul(x, w[0], w[1], w[2], w[3], s.G, y=y, overlap_prior=overlap,
                             workspace=ws_for(s))
        n_rep = max(1, 400 // copies)
        with torch.cuda.stream(stream):
            g.replay()
            stream.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n_rep):
                g.replay()
            b.record(stream)
        b.synchronize()
        us = a.elapsed_time(b) * 1e3 / (n_rep * copies)
        # 10 replays timed one by one: best and median µs per call
        per = []
        with torch.cuda.stream(stream):
            for _ in range(10):
                a.record(stream)
                g.replay()
                b.record(stream)
                b.synchronize()
                per.append(a.elapsed_time(b) * 1e3 / copies)
        gbs = s.alg_bytes() / (us * 1e-6) / 1e9
        detail[s.name] = {"us": round(us, 3), "GB/s": round(gbs, 1),
                          "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                          "us_best_of_10": round(min(per), 3),
                          "us_median_of_10": round(float(np.median(per)), 3)}
        del g

    # the layer both ways: the four calls of the step (q/k/v and gate/up
    # grouped) and seven separate calls, same rotation, one graph each
    layer_calls = {}
    for key, grouped in (("grouped_4_calls", True), ("separate_7_calls", False)):
        pl = layer_plan(sets, grouped)
        us = _time_graph(stream, [(lambda c=c, pl=pl: step(c, pl)) for c in range(copies)],
                         max(1, 200 // copies))
        gbs = step_bytes / (us * 1e-6) / 1e9
        layer_calls[key] = {"us_per_layer": round(us, 3), "GB/s": round(gbs, 1),
                            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                            "launches_per_layer": len(pl)}

    # single-call latency of each M = 1 shape: one launch between an event
    # pair, after a write of twice the L2 size (cold caches); 3 discarded, 20 kept
    single = {}
    try:  # a detail beside the step: its failure is reported, not fatal
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
        for (s, reps, x, y, _) in sets:
            w = reps[0]
            times = []
            with torch.cuda.stream(stream):
                for i in range(23):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    any4.any4_matmul(x, w[0], w[1], w[2], w[3], s.G, y=y, workspace=ws_for(s))
                    b.record(stream)
                    b.synchronize()
                    if i >= 3:
                        times.append(a.elapsed_time(b) * 1e3)
            single[s.name] = {"us_median": round(float(np.median(times)), 2),
                              "us_best": round(float(min(times)), 2)}
        del flush
        torch.cuda.synchronize()
    except Exception as e:  # pragma: no cover - only on a GPU machine
        single = {"error": f"{type(e).__name__}: {e}"}

    # prefill (M = 2048), TFLOPS against the bf16 peak
    prefill = {}
    if not args.skip_prefill:
        for s in workloads.PREFILL:
            p = workloads.make(s)
            packed = any4.any4_pack(torch.from_numpy(p.idx).cuda())
            lut, sc, of, x = (_dev_bf16(a) for a in (p.lut, p.scale, p.offset, p.x))
            y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device="cuda")
            flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
            with torch.cuda.stream(stream):
                for _ in range(3):
                    any4.any4_matmul(x, packed, lut, sc, of, s.G, y=y)
                times = []
                for _ in range(5):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    any4.any4_matmul(x, packed, lut, sc, of, s.G, y=y)
                    b.record(stream)
                    b.synchronize()
                    times.append(a.elapsed_time(b) * 1e3)
            us = float(np.median(times))
            tf = s.flops() / (us * 1e-6) / 1e12
            prefill[s.name] = {"us": round(us, 1), "TFLOPS": round(tf, 1),
                               "frac_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                               "frac_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4)}
            del packed, lut, sc, of, x, y, flush
        torch.cuda.synchronize()

    # the other M = 1 targets (tiny, the G = 64 variant, the 70B-shaped
    # matrices) and the batch sweep (M = 2 .. 32, 70B at M = 8): each weight set
    # once on rotating copies larger than L2, timed at every M it is used with
    more_m1, batch, decode_layout = {}, {}, {}
    if not args.skip_batch:
        groups = [workloads.TINY, [s for s in workloads.SKINNY_SWEEP if s.G == 64]]
        groups.append([s for s in workloads.SKINNY_SWEEP if s.G == 128])
        for nm in ("gate", "up", "down"):
            groups.append([s for s in workloads.LLAMA3_70B_DECODE if s.name.startswith(f"70b_{nm}_")])
        for grp in groups:
            res = time_weight_set(grp, stream, overlap, peaks)
            for s in grp:
                (more_m1 if s.M == 1 and s.name != "sweep_m1" else batch)[s.name] = res[s.name]
        torch.cuda.synchronize()
        # the same M = 1 shapes on codes in the decode layout (any4_repack)
        for s in ([s for s in workloads.LLAMA3_8B_DECODE if s.name in ("8b_gate", "8b_down")]
                  + [s for s in workloads.LLAMA3_70B_DECODE
                     if s.name in ("70b_gate_m1", "70b_down_m1")]):
            decode_layout[s.name] = time_weight_set([s], stream, overlap, peaks,
                                                    decode_layout=True)[s.name]
        torch.cuda.synchronize()

    fig3 = fig3_square_sweep(stream, overlap) if not args.skip_fig3 else {}

    # end to end through the public API with host buffers: every step copies
    # the step's inputs (every call's x) from pinned host memory in one
    # transfer and reads the step's results (every call's y) back in one
    lead = [idxs[0] for idxs in plan]  # the matrices whose x a call reads
    xs = [np.ascontiguousarray(sets[i][4]).view(np.int16).reshape(-1) for i in lead]
    x_off = np.cumsum([0] + [a.size for a in xs])
    host_x = torch.from_numpy(np.concatenate(xs)).pin_memory()
    dev_x = torch.empty(host_x.numel(), dtype=torch.int16, device="cuda")
    y_sizes = [s.M * s.N for (s, *_r) in sets]
    y_off = np.cumsum([0] + y_sizes)
    host_y = torch.empty(int(y_off[-1]), dtype=torch.int16).pin_memory()
    dev_y = torch.empty(int(y_off[-1]), dtype=torch.int16, device="cuda")
    x_views = [dev_x[x_off[j]:x_off[j + 1]].view(torch.bfloat16).view(sets[i][0].M, sets[i][0].K)
               for j, i in enumerate(lead)]
    y_views = [dev_y[y_off[i]:y_off[i + 1]].view(torch.bfloat16).view(s.M, s.N)
               for i, (s, *_r) in enumerate(sets)]
    h2d = host_x.numel() * 2
    d2h = host_y.numel() * 2
    e2e_steps = max(copies, min(steps_timed, 400))

    # the weights as a serving loop holds them: checked once (any4_prepare),
    # so that a call checks only its x and y
    prepared = [[any4.any4_prepare(*sets[i][1][c], sets[i][0].G) for i in range(len(sets))]
                for c in range(copies)]
    ys_of = [[y_views[i] for i in idxs] for idxs in plan]
    ws_of = [ws_for(sets[idxs[0]][0]) for idxs in plan]

    def e2e_step(c):
        dev_x.copy_(host_x, non_blocking=True)
        pc = prepared[c % copies]
        for j, idxs in enumerate(plan):
            any4.any4_matmul_grouped(x_views[j], [pc[i] for i in idxs], sets[idxs[0]][0].G,
                                     ys=ys_of[j], workspace=ws_of[j], overlap_prior=overlap)
        host_y.copy_(dev_y, non_blocking=True)

    with torch.cuda.stream(stream):
        for c in range(copies):
            e2e_step(c)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for c in range(e2e_steps):
            e2e_step(c)
        b.record(stream)
    b.synchronize()
    barrier(world)
    e2e_ms = allreduce_max(a.elapsed_time(b), world)
    e2e_gbs = allreduce_sum(step_bytes * e2e_steps, world) / (e2e_ms * 1e-3) / 1e9

    # the same step as a serving loop replays it: the host copies and the four
    # calls captured once (one step per weight copy) in a CUDA graph, so the
    # host issues one launch per `copies` steps instead of six operations a step
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        for c in range(copies):
            e2e_step(c)
    g_reps = max(1, e2e_steps // copies)
    with torch.cuda.stream(stream):
        e2e_graph.replay()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(g_reps):
            e2e_graph.replay()
        b.record(stream)
    b.synchronize()
    barrier(world)
    eg_ms = allreduce_max(a.elapsed_time(b), world)
    eg_gbs = allreduce_sum(step_bytes * g_reps * copies, world) / (eg_ms * 1e-3) / 1e9
    del e2e_graph
    read_stream = read_stream_rate(stream)

    return {
        "value": value_gbs, "ms_per_step": ms_per_step, "steps_timed": steps_timed,
        "clocks": clocks, "detail": detail, "layer_calls": layer_calls, "single": single,
        "prefill": prefill,
        "batch": batch, "more_m1": more_m1, "decode_layout": decode_layout, "fig3": fig3,
        "peaks": peaks,
        "copies": copies, "step_bytes": step_bytes,
        "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "read_stream": read_stream,
        "e2e_graph": {"value": round(eg_gbs, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h,
                      "us_per_step": round(eg_ms * 1e3 / (g_reps * copies), 2),
                      "how": "the e2e step (pinned H2D of x, four calls, D2H of y) "
                             "captured in a CUDA graph and replayed"},
        "launches": len(plan) * steps_timed,
    }


# ---------------------------------------------------------------------------
# CPU oracle (baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_layer_rate(max_seconds: float):
    """Time the oracle (dequant then fp64 matmul) over whole passes of the
    decode layer until about max_seconds of CPU work; GB/s on the same
    algorithmic bytes as the GPU arm."""
    import oracle
    shapes = workloads.LLAMA3_8B_DECODE
    probs = []
    for s in shapes:
        p = workloads.make(s)
        probs.append((s, oracle.pack(p.idx), p))
    step_bytes = sum(s.alg_bytes() for s in shapes)
    t0 = time.perf_counter()
    done_bytes = 0
    passes = 0
    while True:
        for (s, packed, p) in probs:
            oracle.any4_matmul(p.x, packed, p.lut, p.scale, p.offset, s.G)
        passes += 1
        done_bytes += step_bytes
        if time.perf_counter() - t0 >= max_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": round(done_bytes / dt / 1e9, 4), "unit": "GB/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{passes} full pass(es) of the 7-matmul Llama3-8B layer at M=1 "
                      f"(dequant + fp64 matmul), {dt:.1f} s"}


def oracle_single_thread():
    """The oracle on one host thread for the Tiny and 8B gate M = 1 configs:
    seconds of its dequant alone and of its whole matmul (dequant, then the
    fp64 product), one call each."""
    import oracle
    prev = oracle.num_threads()
    oracle.set_num_threads(1)
    out = {}
    try:
        for s in [workloads.TINY[0]] + [s for s in workloads.LLAMA3_8B_DECODE
                                        if s.name == "8b_gate"]:
            p = workloads.make(s)
            packed = oracle.pack(p.idx)
            t0 = time.perf_counter()
            oracle.dequant(packed, p.lut, p.scale, p.offset, s.G)
            t1 = time.perf_counter()
            oracle.any4_matmul(p.x, packed, p.lut, p.scale, p.offset, s.G)
            t2 = time.perf_counter()
            out[s.name] = {"dequant_s": round(t1 - t0, 4), "matmul_s": round(t2 - t1, 4),
                           "GB/s": round(s.alg_bytes() / (t2 - t1) / 1e9, 4)}
    finally:
        oracle.set_num_threads(prev)
    return {"cores": 1, "configs": out}


def reference_arm(args, rank, world):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    res = oracle_layer_rate(max_seconds=args.reference_seconds)
    line = {"metric": METRIC, "value": res["value"], "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generators, Llama3-8B shapes)",
            "config": {"workload": "llama3_8b_decode_layer_m1", "M": 1, "G": 128,
                       "shapes": [[s.name, s.K, s.N] for s in workloads.LLAMA3_8B_DECODE]},
            "impl": "reference", "cpu_baseline": res,
            "e2e": {"value": res["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def table_learning_detail(max_iter: int, cpu_seconds: float, reps: int = 3):
    """Time any4_quantize (learning the tables) on the Llama3-8B layer matrices
    with CUDA events on the launching stream, and the oracle beside it on a
    bounded sample of rows of each matrix (about cpu_seconds in all)."""
    import torch
    import oracle
    import learned_bit_lut_any4_b200 as any4
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    out = []
    for s in workloads.QUANTIZE_LLAMA3_8B:
        w_bits = workloads.draw_dense_weight(s)
        ex_np = workloads.draw_abs_act_mean(s)
        w = _dev_bf16(w_bits)
        ex = torch.from_numpy(ex_np).cuda()
        any4.any4_quantize(w, ex, s.G, max_iter)            # warm-up (module load, attributes)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            _, _, _, _, iters = any4.any4_quantize(w, ex, s.G, max_iter, return_iters=True)
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / reps
        it = iters.cpu().numpy().astype(np.int64)
        # algorithmic bytes: read w and E|x|, write codes, scale/offset and tables
        alg = 2 * s.N * s.K + 4 * s.K + s.N * s.K // 2 + 4 * s.N * (s.K // s.G) + 32 * s.N
        rows = 1
        t = time.perf_counter()
        while True:
            oracle.quantize(w_bits[:rows], ex_np, s.G, max_iter)
            dt = time.perf_counter() - t
            if dt >= cpu_seconds / len(workloads.QUANTIZE_LLAMA3_8B) or rows >= s.N:
                break
            rows = min(s.N, rows * 4)
            t = time.perf_counter()
        out.append({"shape": s.name, "N": s.N, "K": s.K, "G": s.G, "max_iter": max_iter,
                    "gpu_ms": round(ms, 3), "gpu_rows_per_s": round(s.N / ms * 1e3, 1),
                    "mean_m_steps": round(float(it.mean()), 2), "max_m_steps": int(it.max()),
                    "alg_bytes": alg, "gb_per_s": round(alg / ms / 1e6, 2),
                    "hbm_frac": round(alg / ms / 1e6 / peaks["hbm_gbs"], 5),
                    "mstep_columns_per_s": round(float(it.sum() * s.K) / ms * 1e3, 1),
                    "oracle_rows": rows, "oracle_rows_per_s": round(rows / dt, 2),
                    "oracle_cores": oracle.num_threads()})
    return out


def nbit_dequant_detail():
    """Time any4_dequant_bits for n = 2, 3, 4 on the Llama3-8B gate matrix
    (4096 -> 14336, G = 128) on rotating weight copies larger than L2, replayed
    in a CUDA graph (events on its stream): HBM GB/s of the algorithmic bytes
    (codes, scales, offsets and tables read, bf16 W written)."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    peaks = load_peaks()
    N, K, G = 14336, 4096, 128
    rng = np.random.default_rng(4600)
    stream = torch.cuda.Stream()
    out = {"N": N, "K": K, "G": G}
    for bits in (2, 3, 4):
        nq = 1 << bits
        alg = N * K * bits // 8 + 4 * N * (K // G) + 2 * nq * N + 2 * N * K
        copies = max(2, int(np.ceil(3 * L2_BYTES / alg)))
        packed = torch.from_numpy(rng.integers(0, 256, size=(N, bits * K // 8),
                                               dtype=np.uint8)).cuda()
        lut = _dev_bf16(workloads._to_bf16_bits(rng.normal(0, 0.5, (N, nq)).astype(np.float32)))
        scale = _dev_bf16(workloads._to_bf16_bits(
            (np.abs(rng.normal(0, 0.01, (N, K // G))) + 1e-3).astype(np.float32)))
        offset = _dev_bf16(workloads._to_bf16_bits(
            rng.normal(0, 0.002, (N, K // G)).astype(np.float32)))
        reps = [(packed, lut, scale, offset)] + [
            (packed.clone(), lut.clone(), scale.clone(), offset.clone()) for _ in range(copies - 1)]
        Ws = [torch.empty((N, K), dtype=torch.bfloat16, device="cuda") for _ in range(copies)]
        calls = [(lambda w=w, W=W: any4.any4_dequant_bits(w[0], w[1], w[2], w[3], G, bits, W=W))
                 for w, W in zip(reps, Ws)]
        us = _time_graph(stream, calls, max(2, 100 // copies))
        out[f"any{bits}"] = {"us": round(us, 2), "GB/s": round(alg / us / 1e3, 1),
                             "frac_hbm": round(alg / us / 1e3 / peaks["hbm_gbs"], 4)}
        del reps, Ws, packed, lut, scale, offset
        torch.cuda.synchronize()
    return out


def nbit_matmul_detail():
    """any4_matmul_bits at M = 1 (n = 2, 3, 4: the codes read directly by the
    weight-streaming kernel) on the Llama3-8B gate and Llama3-70B gate
    matrices, G = 128, on rotating weight copies larger than L2 replayed in a
    CUDA graph: us per call, GB/s of the algorithmic bytes (codes, scales,
    offsets, tables, x, y) and the fraction of the HBM peak."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    peaks = load_peaks()
    G = 128
    rng = np.random.default_rng(4700)
    stream = torch.cuda.Stream()
    out = {}
    for name, K, N in (("8b_gate", 4096, 14336), ("70b_gate", 8192, 28672)):
        res = {"K": K, "N": N, "G": G}
        for bits in (2, 3, 4):
            nq = 1 << bits
            wbytes = N * K * bits // 8 + 4 * N * (K // G) + 2 * nq * N
            copies = max(2, int(np.ceil(3 * L2_BYTES / wbytes)))
            packed = torch.from_numpy(rng.integers(0, 256, size=(N, bits * K // 8),
                                                   dtype=np.uint8)).cuda()
            lut = _dev_bf16(workloads._to_bf16_bits(
                np.sort(rng.normal(0, 0.5, (N, nq)), axis=1).astype(np.float32)))
            scale = _dev_bf16(workloads._to_bf16_bits(
                (np.abs(rng.normal(0, 0.01, (N, K // G))) + 1e-3).astype(np.float32)))
            offset = _dev_bf16(workloads._to_bf16_bits(
                rng.normal(0, 0.002, (N, K // G)).astype(np.float32)))
            reps = [(packed, lut, scale, offset)] + [
                (packed.clone(), lut.clone(), scale.clone(), offset.clone())
                for _ in range(copies - 1)]
            x = _dev_bf16(workloads._to_bf16_bits(rng.normal(0, 1, (1, K)).astype(np.float32)))
            y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
            calls = [(lambda w=w: any4.any4_matmul_bits(x, w[0], w[1], w[2], w[3], G, bits, y=y,
                                                        overlap_prior=True))
                     for w in reps]
            us = _time_graph(stream, calls, max(2, 200 // copies))
            alg = wbytes + 2 * K + 2 * N
            res[f"any{bits}"] = {"us": round(us, 3), "GB/s": round(alg / us / 1e3, 1),
                                 "frac_hbm": round(alg / us / 1e3 / peaks["hbm_gbs"], 4)}
            del reps, packed, lut, scale, offset, x, y
            torch.cuda.synchronize()
        out[name] = res
    return out


def profile_shape(name: str, calls: int, op: str = "matmul"):
    """Run a few calls of one operation (any4_matmul on the auto path,
    any4_dequant, or any4_quantize on the first 148 rows of a quantiser
    matrix, max_iter 20) on one workload shape: a small, fixed case for ncu."""
    import torch
    import learned_bit_lut_any4_b200 as any4
    if op == "quantize":
        qs = [q for q in workloads.QUANTIZE_LLAMA3_8B if q.name == name]
        if not qs:
            raise SystemExit(f"unknown quantiser matrix {name}")
        q = qs[0]
        w = _dev_bf16(workloads.draw_dense_weight(q)[:148])
        ex = torch.from_numpy(workloads.draw_abs_act_mean(q)).cuda()
        for _ in range(calls):
            any4.any4_quantize(w, ex, q.G, max_iter=20)
        torch.cuda.synchronize()
        print(f"profiled quantize {name}: 148 of {q.N} rows, K={q.K} G={q.G}, {calls} calls",
              flush=True)
        return
    shape = [s for s in workloads.all_shapes() if s.name == name]
    if not shape:
        raise SystemExit(f"unknown shape {name}; known: {[s.name for s in workloads.all_shapes()]}")
    s = shape[0]
    p = workloads.make(s)
    packed = any4.any4_pack(torch.from_numpy(p.idx).cuda())
    lut, sc, of, x = (_dev_bf16(a) for a in (p.lut, p.scale, p.offset, p.x))
    y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device="cuda")
    W = torch.empty((s.N, s.K), dtype=torch.bfloat16, device="cuda") if op == "dequant" else None
    for _ in range(calls):
        if op == "dequant":
            any4.any4_dequant(packed, lut, sc, of, s.G, W=W)
        else:
            any4.any4_matmul(x, packed, lut, sc, of, s.G, y=y)
    torch.cuda.synchronize()
    print(f"profiled {op} {name}: M={s.M} K={s.K} N={s.N} G={s.G}, {calls} calls", flush=True)


def target_summary(r, nbit, table, peaks):
    """The headline fractions in one small dict (fractions of the HBM peak
    for the memory-bound paths, of the bf16 burst peak for prefill)."""
    def get(d, *ks):
        for k in ks:
            if not isinstance(d, dict) or k not in d:
                return None
            d = d[k]
        return d
    t = {"peak_hbm_gbs": peaks["hbm_gbs"], "peak_bf16_tflops": peaks["bf16_tflops"],
         "m1_8b_layer_grouped": get(r, "layer_calls", "grouped_4_calls", "frac_hbm"),
         "m1_8b_layer_7_calls": get(r, "layer_calls", "separate_7_calls", "frac_hbm"),
         "m1_70b_gate": get(r, "more_m1", "70b_gate_m1", "frac_hbm"),
         "m1_70b_down": get(r, "more_m1", "70b_down_m1", "frac_hbm"),
         "m2": get(r, "batch", "sweep_m2", "frac_hbm"),
         "m4": get(r, "batch", "sweep_m4", "frac_hbm"),
         "m8": get(r, "batch", "sweep_m8", "frac_hbm"),
         "m16": get(r, "batch", "sweep_m16", "frac_hbm"),
         "m8_70b_gate": get(r, "batch", "70b_gate_m8", "frac_hbm"),
         "dequant_8b_gate": get(nbit, "any4", "frac_hbm"),
         "prefill_gate_burst": get(r, "prefill", "prefill_gate", "frac_bf16_burst"),
         "prefill_down_burst": get(r, "prefill", "prefill_down", "frac_bf16_burst")}
    if isinstance(table, dict) and isinstance(table.get("matrices"), list):
        for m in table["matrices"]:
            if m.get("shape") == "8b_down":
                t["quantize_8b_down_ms"] = m.get("gpu_ms")
    return t


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=40)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ungrouped", action="store_true",
                    help="run the layer step as seven separate any4_matmul calls instead of "
                         "four (q/k/v and gate/up as grouped calls)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the decode kernels without programmatic dependent launch")
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--skip-fig3", action="store_true",
                    help="skip the square K = N sweep at M = 1 (any4 / nf4-style / int4 / bf16)")
    ap.add_argument("--skip-batch", action="store_true",
                    help="skip the per-shape timing of the M = 2..16 and 70B M = 8 shapes")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=20.0)
    ap.add_argument("--profile-shape", default=None,
                    help="no timing: run --profile-calls any4_matmul calls on one named "
                         "workload shape (a small, fixed case for ncu captures)")
    ap.add_argument("--profile-calls", type=int, default=3)
    ap.add_argument("--profile-op", default="matmul", choices=["matmul", "dequant", "quantize"])
    ap.add_argument("--quantize-detail", action="store_true",
                    help="no step: time any4_quantize on the Llama3-8B matrices (and the "
                         "oracle on a sample of rows) and print one JSON line")
    ap.add_argument("--quantize-iters", type=int, default=100)
    ap.add_argument("--skip-table-learning", action="store_true",
                    help="leave the any4_quantize timing out of the JSON line")
    args = ap.parse_args()
    if args.profile_shape:
        profile_shape(args.profile_shape, args.profile_calls, args.profile_op)
        return
    if args.quantize_detail:
        print(json.dumps({"detail": "quantize",
                          "shapes": table_learning_detail(args.quantize_iters, args.cpu_seconds)}),
              flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3

    rank, world, _ = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            reference_arm(args, rank, world)
            return
        import torch
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        r = gpu_arm(args, rank, world)
        if rank != 0:
            return
        peaks = r["peaks"]
        cpu = oracle_layer_rate(max_seconds=args.cpu_seconds) if world == 1 else None
        if cpu is not None:
            cpu["single_thread"] = oracle_single_thread()
        table = None
        if world == 1 and not args.skip_table_learning:
            try:  # a detail beside the step: its failure is reported, not fatal
                table = {"max_iter": args.quantize_iters,
                         "matrices": table_learning_detail(args.quantize_iters, 4.0, reps=2)}
            except Exception as e:  # pragma: no cover - only on a GPU machine
                table = {"error": f"{type(e).__name__}: {e}"}
        nbit = nbit_mm = None
        if world == 1:
            try:  # a detail beside the step: its failure is reported, not fatal
                nbit = nbit_dequant_detail()
            except Exception as e:  # pragma: no cover - only on a GPU machine
                nbit = {"error": f"{type(e).__name__}: {e}"}
            try:
                nbit_mm = nbit_matmul_detail()
            except Exception as e:  # pragma: no cover - only on a GPU machine
                nbit_mm = {"error": f"{type(e).__name__}: {e}"}
        achieved = r["value"] / world  # per-GPU decode throughput over the whole step
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": stored_traffic(),
                    "kernel": "decode_tma_ffma_kernel (the only kernel of the step)",
                    "peak_source": peaks.get("source", "measured")}
        line = {
            "metric": METRIC, "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world,
            "steps": r["steps_timed"], "warmup": args.warmup,
            "ms_per_step": round(r["ms_per_step"], 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generators, Llama3-8B shapes, random any4 weights)",
            "config": {"workload": "llama3_8b_decode_layer_m1", "M": 1, "G": 128,
                       "shapes": [[s.name, s.K, s.N] for s in workloads.LLAMA3_8B_DECODE],
                       "parallelism": f"replicas{world}",
                       "l2": f"inputs larger than L2: {r['copies']} rotating weight copies",
                       "overlap_prior": not args.no_overlap,
                       "calls": ("q/k/v grouped, o, gate/up grouped, down (4 launches)"
                                 if not args.ungrouped else "7 separate calls")},
            "us_per_layer": round(r["ms_per_step"] * 1e3, 2),
            "roofline": roofline,
            "hbm_read_stream": dict(r["read_stream"], layer_frac=round(
                r["value"] / r["read_stream"]["gbs_median"], 4)),
            "cpu_baseline": cpu,
            "e2e": r["e2e"],
            "e2e_graph": r["e2e_graph"],
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
            # bulky details first; the target numbers (per-shape M = 1 and the
            # prefill fractions) close the line, where its tail is kept
            "fig3_square_m1": r["fig3"],
            "table_learning": table,
            "nbit_dequant": nbit,
            "nbit_matmul_m1": nbit_mm,
            "single_call_m1": r["single"],
            "detail_batch": r["batch"],
            "layer_m1_calls": r["layer_calls"],
            "detail_m1": r["detail"],
            "detail_m1_more": r["more_m1"],
            "m1_decode_layout": r["decode_layout"],
            "prefill_m2048": r["prefill"],
            # one compact summary of every target figure, last, where the
            # kept tail of the line always holds it
            "targets": target_summary(r, nbit, table, peaks),
        }
        print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
