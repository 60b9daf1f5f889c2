#!/usr/bin/env python
"""Decode-step throughput of shared-routing token-sparse attention on B200.

One step = one fused decode call over the whole batch: the routing score
scan over the K cache, the top-k select per (sequence, KV head), and the
gather attention of all L layers over that one set (CLSA article, sections
CLSAの仕組み and 計算コストの削減効果).  The default workload is the 128K-token
headline: B=1, N=131072, Hq=32, Hkv=8, d=128, k=2048, L=16, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Rank 0 prints one JSON line.  With N > 1 (torchrun, one process per GPU)
every rank runs its own replica on its own sequences: the path shards into
independent sequences with no exchange step, so the scaling is weak and the
only collectives are the barrier and the max-over-ranks of the timed region.

``--impl reference`` times the CPU oracle (the plain C reference under
oracle/) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from token_sparse_attention_sm_b200 import dist as sdist  # noqa: E402
from token_sparse_attention_sm_b200 import synth  # noqa: E402

METRIC = ("128K-context sparse decode steps/s (16 layers, k=2048); "
          "HBM GB/s vs roofline")
FALLBACK_HBM_GBS = 6650.0
QUERY_SETS = 8
TIMING = ("the K timed decode steps replayed back to back as one CUDA graph (query set "
          "i %% 8 at step i; %d kernels per step, programmatic dependent launch between "
          "them; for K > 256 a 64-step graph replayed plus a remainder graph), after the W "
          "warm-up steps; CUDA events on the launch stream; max over ranks")
TIMING_OTHER = ("the K timed steps replayed back to back as one CUDA graph (query set i %% 8 at "
                "step i; for K > 256 a 64-step graph replayed plus a remainder graph), after the "
                "W warm-up steps; CUDA events on the launch stream; max over ranks") % ()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s pool measurement)"


def algorithmic_bytes(w):
    """Bytes the method must move per step: the K cache once for routing plus
    the selected K and V rows once (the set and the cache are shared by all
    layers).  q, idx and out are < 0.3 MB and not counted."""
    scan = w.B * w.Hkv * w.N * w.d * w.esize
    gathered = 2 * w.B * w.Hkv * w.k * w.d * w.esize
    return scan, gathered


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
_SMI_FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw",
               "clocks_event_reasons.active",
               "clocks_event_reasons.hw_slowdown",
               "clocks_event_reasons.hw_thermal_slowdown",
               "clocks_event_reasons.sw_thermal_slowdown",
               "clocks_event_reasons.sw_power_cap"]


def _smi_id(local_rank: int) -> str:
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        return str(local_rank)


def _smi_time(s: str) -> float:
    from datetime import datetime
    return datetime.strptime(s.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()


class ClockSampler:
    """nvidia-smi sampling in the background; only samples taken between
    mark_start() and mark_stop() (the timed region) are summarised."""

    def __init__(self, local_rank: int, interval_ms: int = 50):
        self.dev = _smi_id(local_rank)
        self.interval = interval_ms
        self.proc = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}",
                 "--query-gpu=" + ",".join(_SMI_FIELDS),
                 "--format=csv,noheader,nounits", f"-lms", str(self.interval)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.15)

    def result(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        return summarize_clocks(out, self.t0, self.t1)


def summarize_clocks(out: str, t0=None, t1=None):
    """The clocks record of one timed region from nvidia-smi's CSV rows
    (_SMI_FIELDS, no header, no units): the median SM clock, the largest max
    clock and every throttle reason seen Active, over the rows stamped inside
    [t0, t1] (with 50 ms of slack); None when no row qualifies."""
    rows = [r for r in csv.reader(io.StringIO(out)) if len(r) == len(_SMI_FIELDS)]
    try:
        if t0 is not None and t1 is not None:
            rows = [r for r in rows if t0 - 0.05 <= _smi_time(r[0]) <= t1 + 0.05]
    except Exception:
        pass
    if not rows:
        return None
    sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
    mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4)
                      if r[5 + i].strip().lower() == "active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
            "samples": len(rows)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def time_graphs(graphs, steps: int, warmup: int, stream, sampler=None) -> float:
    """Replay graphs[i % len] for warmup + steps iterations; return the
    CUDA-event time (ms) of the last `steps` replays, bracketed by a barrier
    and device synchronisation."""
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    sdist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark_start()
    start.record(stream)
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_stop()
    sdist.barrier()
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def step_graphs(step_fns, count: int, stream, max_one: int = 256, chunk: int = 64):
    """CUDA graphs that together run `count` consecutive decode steps
    (step_fns[i % n] at step i): [(graph, replays)].  One graph of all the
    steps when count <= max_one, else a chunk-step graph replayed and one
    graph for the remainder (n must divide chunk so the cycle lines up)."""
    n = len(step_fns)
    if count <= max_one:
        return [(capture_loop([step_fns[i % n] for i in range(count)], stream), 1)]
    assert chunk % n == 0
    plan = [(capture_loop([step_fns[i % n] for i in range(chunk)], stream), count // chunk)]
    if count % chunk:
        plan.append((capture_loop([step_fns[i % n] for i in range(count % chunk)], stream), 1))
    return plan


def time_steps(step_fns, steps: int, warmup: int, stream, sampler=None) -> float:
    """Run warmup + steps decode steps, each phase as whole CUDA graph
    replays (step_graphs: the timed steps back to back in one graph when
    there are at most 256 of them); return the CUDA-event time (ms) of the
    `steps` timed steps, bracketed by a barrier and device synchronisation."""
    warm = step_graphs(step_fns, warmup, stream)
    timed = step_graphs(step_fns, steps, stream)
    # the timed graphs' work goes to the device now, not in their first
    # replay inside the timed region
    import token_sparse_attention_sm_b200 as sd
    for g, _ in timed:
        sd.graph_upload(g, stream)
    for g, reps in warm:
        for _ in range(reps):
            g.replay()
    torch.cuda.synchronize()
    sdist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark_start()
    start.record(stream)
    for g, reps in timed:
        for _ in range(reps):
            g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_stop()
    sdist.barrier()
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def step_distribution(g_loop, n_steps: int, stream, replays: int = 200) -> dict:
    """Median and p90 of the per-step time: `replays` replays of the
    n_steps-step graph, each bracketed by its own CUDA events (after the
    timed region; the per-step figure is a replay's time / n_steps)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(replays)]
    for a, b in evs:
        a.record(stream)
        g_loop.replay()
        b.record(stream)
    torch.cuda.synchronize()
    us = sorted(a.elapsed_time(b) * 1e3 / n_steps for a, b in evs)
    return {"median_us": round(statistics.median(us), 2),
            "p90_us": round(us[int(0.9 * (len(us) - 1))], 2), "replays": replays,
            "note": "per-step time of each %d-step graph replay" % n_steps}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def capture_loop(fn_list, stream):
    """One graph running every fn of fn_list in order."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fn_list:
            fn()
    return g


def kernels_per_step(w, reroute: int = 0) -> int:
    """Kernels one decode step launches: the routing scan, then -- where the
    library says the step runs fused (bf16, L*G <= 128 query vectors per
    head, N <= 131072, k or cap <= 32768) -- the one select + attention
    kernel, else the select (or threshold compaction) and the attention (one
    kernel for bf16, a partial and a merge kernel for fp32); once per group of
    `reroute` layers when routing is re-computed."""
    import token_sparse_attention_sm_b200 as sd
    lg = min(reroute, w.L) if reroute else w.L
    fused = sd.decode_step_fused(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, lg,
                                 k=w.k if w.mode == "topk" else None,
                                 cap=w.cap if w.mode != "topk" else None)
    per_group = 2 if fused else 2 + (1 if w.dtype == "bf16" else 2)
    groups = -(-w.L // reroute) if reroute else 1
    return per_group * groups


def capture(fn_list, stream):
    graphs = []
    for fn in fn_list:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs.append(g)
    return graphs


def kernel_source_sha(files) -> str:
    """sha256 over the concatenated source files of a kernel."""
    h = hashlib.sha256()
    for fn in files:
        with open(fn, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


SCORE_SOURCES = [os.path.join(ROOT, "token_sparse_attention_sm_b200", "csrc", n)
                 for n in ("score.cu", "scan.cuh")]


def traffic_record(files, workload: str = "decode_128k"):
    """ncu DRAM bytes per launch of the dominant kernel, valid only while the
    kernel source is unchanged since the capture and for the workload it was
    captured on."""
    path = os.path.join(ROOT, "profiles", "score_kernel_traffic.txt")
    try:
        with open(path) as f:
            rec = json.load(f)
        if (rec.get("source_sha256") == kernel_source_sha(files)
                and rec.get("workload", "").split(" ")[0] == workload):
            return rec
    except Exception:
        pass
    return None


def run_native(args, rank, world, local_rank):
    import token_sparse_attention_sm_b200 as sd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = synth.WORKLOADS[args.workload]
    # each rank decodes its own sequences (independent seeds)
    w = base.with_(seeds=tuple(s + 1000 * rank for s in base.seeds))
    x = synth.generate(w)
    variants = synth.query_variants(w, x, QUERY_SETS, seed=2000 + 1000 * rank)
    K = x["K"].to(dev)
    V = x["V"].to(dev)
    qs = [(qr.to(dev), ql.to(dev)) for qr, ql in variants]
    stream = torch.cuda.Stream(device=dev)
    ws = sd.Workspace(dev)
    # one workspace, sized up front for every op timed below, so that no
    # captured graph refers to a buffer that is later replaced
    ws.get(sd.workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, w.k, w.L))
    outs = [dict(out=torch.empty_like(ql), idx=torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev),
                 lse=torch.empty((w.L, w.B, w.Hq), dtype=torch.float32, device=dev)) for _, ql in qs]

    R = args.reroute
    if R:
        # routing re-computed every R layers: group g routes with the query
        # of its first layer (R = 1: every layer routes with its own query)
        ng = -(-w.L // R)
        qrs = [ql[::R].contiguous() for _, ql in qs]
        ws.get(sd.workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, w.k, min(R, w.L)))
        for o in outs:
            o["idx"] = torch.empty((ng, w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)

    def step_fn(i):
        qr, ql = qs[i]
        o = outs[i]
        if R:
            return lambda: sd.decode_step_grouped(qrs[i], ql, K, V, R, k=w.k, ws=ws, check=False,
                                                  out=o["out"], idx=o["idx"], lse=o["lse"])
        return lambda: sd.decode_step(qr, ql, K, V, k=w.k, ws=ws, check=False,
                                      out=o["out"], idx=o["idx"], lse=o["lse"])

    with torch.cuda.stream(stream):
        for i in range(len(qs)):          # warm the workspace and the library
            step_fn(i)()
        sd.read_device_status(ws)
        loop = capture_loop([step_fn(i) for i in range(len(qs))], stream)
        with ClockSampler(local_rank) as cs:
            ms = time_steps([step_fn(i) for i in range(len(qs))], args.steps, args.warmup,
                            stream, cs)
        clocks = cs.result()
        dist = step_distribution(loop, len(qs), stream)
        sd.read_device_status(ws)         # no device-side condition in the run

        # per-kernel durations, each kernel alone in a graph of back-to-back
        # launches over the rotating queries (CUDA events on this stream)
        S_buf = torch.empty((w.B, w.Hkv, w.N), dtype=torch.float32, device=dev)
        # one routing set per query set (computed here, outside any graph)
        sets = [torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev) for _ in qs]
        idx0 = sets[0]
        # size the workspace for every op before any capture
        sd.score(qs[0][0], K, ws=ws, check=False, out=S_buf)
        for qi in range(len(qs)):
            sd.route_topk(qs[qi][0], K, w.k, ws=ws, check=False, idx=sets[qi])
        sd.attn_gather(qs[0][1], K, V, idx0, ws=ws, check=False, out=outs[0]["out"],
                       lse=outs[0]["lse"])
        torch.cuda.synchronize()
        score_graphs = capture([lambda qr=qr: sd.score(qr, K, ws=ws, check=False, out=S_buf)
                                for qr, _ in qs], stream)
        n_k = max(args.steps // 4, 64)
        t_score = time_graphs(score_graphs, n_k, max(args.warmup, 3), stream) / n_k
        # the select kernel consumes the scan's histogram, so it is timed as
        # route (scan + select) minus the scan alone
        route_graphs = capture([lambda qr=qr: sd.route_topk(qr, K, w.k, ws=ws, check=False, idx=idx0)
                                for qr, _ in qs], stream)
        t_sel = time_graphs(route_graphs, n_k, max(args.warmup, 3), stream) / n_k - t_score
        attn_graphs = capture([lambda qi=qi: sd.attn_gather(qs[qi][1], K, V, sets[qi], ws=ws,
                                                            check=False, out=outs[qi]["out"],
                                                            lse=outs[qi]["lse"])
                               for qi in range(len(qs))], stream)
        t_attn = time_graphs(attn_graphs, n_k, max(args.warmup, 3), stream) / n_k
        sd.read_device_status(ws)
        dense = None
        if args.dense:
            # dense attention: every key selected (k = N), all L layers over one
            # read of K and V, and layer by layer (L reads)
            all_idx = torch.arange(w.N, dtype=torch.int32, device=dev).repeat(w.B, w.Hkv, 1)
            dense_out = torch.empty_like(qs[0][1])
            dense_lse = torch.empty((w.L, w.B, w.Hq), dtype=torch.float32, device=dev)
            ws.get(sd.workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, w.N, w.L))
            sd.attn_gather(qs[0][1], K, V, all_idx, ws=ws, check=True, out=dense_out,
                           lse=dense_lse)
            n_d = max(args.steps // 64, 16)
            g_all = capture([lambda qi=qi: sd.attn_gather(qs[qi][1], K, V, all_idx, ws=ws,
                                                          check=False, out=dense_out,
                                                          lse=dense_lse)
                             for qi in range(len(qs))], stream)
            t_dense_all = time_graphs(g_all, n_d, max(args.warmup, 3), stream) / n_d

            def per_layer(qi):
                def run():
                    for l in range(w.L):
                        sd.attn_gather(qs[qi][1][l:l + 1], K, V, all_idx, ws=ws, check=False,
                                       out=dense_out[l:l + 1], lse=dense_lse[l:l + 1])
                return run
            g_pl = capture([per_layer(qi) for qi in range(len(qs))], stream)
            t_dense_pl = time_graphs(g_pl, n_d, max(args.warmup, 3), stream) / n_d
            sd.read_device_status(ws)
            kv_b = 2 * w.B * w.Hkv * w.N * w.d * w.esize
            dense = {"all_layers_one_pass_us": round(t_dense_all * 1e3, 2),
                     "all_layers_one_pass_gbs": round(kv_b / (t_dense_all * 1e-3) / 1e9, 1),
                     "layer_by_layer_us": round(t_dense_pl * 1e3, 2),
                     "layer_by_layer_gbs": round(w.L * kv_b / (t_dense_pl * 1e-3) / 1e9, 1),
                     "note": "attn_gather with every key selected; the one-pass form reads K "
                             "and V once for all layers (the shared cache), the layer-by-layer "
                             "form L times"}

    ms_max = sdist.max_over_ranks(ms)
    t_score_max = sdist.max_over_ranks(t_score)
    ms_per_step = ms_max / args.steps
    value = world * args.steps / (ms_max / 1e3)

    # end to end through the public API: pinned host queries in, results out
    e2e = run_e2e(sd, w, variants, K, V, ws, stream, dev, args, world)

    peak, peak_src = load_peaks()
    scan_b, gath_b = algorithmic_bytes(w)
    achieved = scan_b / (t_score_max * 1e-3) / 1e9
    trec = traffic_record(SCORE_SOURCES, w.name)
    line = {
        "metric": METRIC if w.name == "decode_128k" else (
            "sparse decode steps/s on %s (B=%d, N=%d, %d layers, k=%d); HBM GB/s vs roofline"
            % (w.name, w.B, w.N, w.L, w.k)),
        "value": round(value, 2),
        "unit": "steps/s",
        # a step decodes one token of each of the B sequences
        **({"tokens_per_s": round(value * w.B, 2)} if w.B > 1 else {}),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded Gaussian K/V/q, planted heavy hitters, x8 outlier channel)",
        "config": {
            "workload": w.name, "B": w.B, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv,
            "d": w.d, "k": w.k, "L": w.L, "parallelism": f"replicas x{world}",
            "query_sets": QUERY_SETS,
            "l2": "inputs larger than L2 (K+V = %.0f MB per replica); the query "
                  "rotates over %d sets so the selected rows change every step"
                  % (2 * scan_b / 1e6, QUERY_SETS),
            "timing": TIMING % kernels_per_step(w, args.reroute),
            **({"reroute": args.reroute,
                "routing": "re-computed every %d layers (group g routes with its first "
                           "layer's query)" % args.reroute} if args.reroute else {}),
        },
        "roofline": {
            "bound": "hbm", "kernel": "score_kernel (routing scan)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": trec.get("traffic_bytes_per_launch") if trec else None,
            "algorithmic_bytes_per_launch": scan_b,
            "avg_launch_us": round(t_score_max * 1e3, 2),
            "peak_source": peak_src,
        },
        "step_roofline": {
            "unique_bytes_per_step": scan_b + gath_b,
            "achieved_gbs": round((scan_b + gath_b) / (ms_per_step * 1e-3) / 1e9, 1),
            "frac_of_measured_peak": round((scan_b + gath_b) / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        },
        "kernels_us": {"score": round(t_score * 1e3, 2),
                       "select_and_attention_in_step": round(ms_per_step * 1e3 - t_score * 1e3, 2),
                       "select_kernel": round(t_sel * 1e3, 2),
                       "attn_gather_all_layers": round(t_attn * 1e3, 2),
                       "note": "score (the routing scan) and attn_gather (attention over given "
                               "sets) timed alone in back-to-back graph launches (attention "
                               "alone may find its rows in L2); in the step the select runs "
                               "inside the attention kernel, whose share is the step time minus "
                               "the scan; select_kernel = route_topk (scan + the select as its "
                               "own kernel) minus the scan"},
        **({"dense_attention": dense} if dense else {}),
        "e2e": e2e,
        "gpu_launches": kernels_per_step(w, args.reroute) * args.steps,
        "clocks": clocks,
        "step_time": dist,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_full(w, x)
    return line


def run_e2e(sd, w, variants, K, V, ws, stream, dev, args, world):
    """Same metric through the public Python API with host buffers: every
    step copies its queries from pinned host memory to the device, runs the
    decode step, and brings the outputs and the index set back to pinned host
    memory (the outputs written there by the attention itself when the buffer
    is mapped), then waits for them -- all inside the timed region.  The step
    is the library's DecodeStepGraph (routing, attention and the transfers
    captured once as a CUDA graph, launched by one C call per step), one per
    query set, as a caller double-buffering its inputs keeps them; its pinned
    input views hold the set's queries."""
    graphs = []
    for qr, ql in variants:
        g = sd.DecodeStepGraph(K, V, w.L, w.Hq, k=w.k, ws=ws, stream=stream)
        g.q_route_host.copy_(qr)
        g.q_layers_host.copy_(ql)
        graphs.append(g)
    steps = min(args.steps, 2000)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            graphs[i % len(graphs)]()
        torch.cuda.synchronize()
        sdist.barrier()
        t0 = time.perf_counter()
        for i in range(steps):
            graphs[i % len(graphs)]()
        t1 = time.perf_counter()
        sdist.barrier()
        sd.read_device_status(ws)
    sec = sdist.max_over_ranks(t1 - t0)
    g0 = graphs[0]
    return {"value": round(world * steps / sec, 2), "unit": "steps/s",
            "h2d_bytes_per_step": g0.h2d_bytes, "d2h_bytes_per_step": g0.d2h_bytes,
            "steps": steps,
            "api": "token_sparse_attention_sm_b200.DecodeStepGraph (routing and the layers' "
                   "attention in one CUDA graph with the host transfers: the routing query "
                   "crosses PCIe first, the layers' queries on a second stream while the "
                   "routing scan runs; fused=%s: the select + attention kernel writes the "
                   "outputs and the index set into mapped pinned host memory "
                   "(results_direct=%s); synchronised every step)" % (g0.fused,
                                                                      g0.results_direct)}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def cpu_baseline_full(w, x, budget_s: float = 10.0):
    """The C oracle, as it stands, on full decode steps of the same workload,
    repeated until about `budget_s` seconds of CPU work."""
    import oracle
    qr, ql = synth.f32(x["q_route"]), synth.f32(x["q_layers"])
    Kf, Vf = synth.f32(x["K"]), synth.f32(x["V"])
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_step(qr, ql, Kf, Vf, k=w.k)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    sec = time.perf_counter() - t0
    return {"value": round(n / sec, 4), "unit": "steps/s", "cores": oracle.num_threads(),
            "kind": "oracle", "cpu": cpu_model(),
            "sample": f"{n} full decode steps of {w.name} (all {w.B * w.Hkv} KV heads, "
                      f"{w.L} layers) by the plain C oracle with OpenMP, {sec:.1f} s"}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle timed on bounded samples of the workload.
    A sample is the whole step (every sequence and KV head, so the oracle's
    parallel loops see the same work split as on a full step) over the first
    n keys of the cache with k (or cap) scaled in proportion, sized so the
    whole run takes about a minute; steps/s is scaled to full steps by the
    fraction n / N of the keys the sample covers."""
    import oracle
    w = synth.WORKLOADS[args.workload]
    x = synth.generate(w)
    G = w.G
    qr = synth.f32(x["q_route"])
    ql = synth.f32(x["q_layers"])
    K_all = synth.f32(x["K"])
    V_all = synth.f32(x["V"])

    threshold = w.mode == "threshold"

    def prepare(n):
        """Contiguous inputs of the n-key sample and its k or tau (untimed)."""
        Kn = np.ascontiguousarray(K_all[:, :, :n])
        Vn = np.ascontiguousarray(V_all[:, :, :n])
        if threshold:  # tau of the sample's own scores
            tau = oracle.percentile_tau(oracle.scores(qr, Kn), *w.tau_pct)
            return Kn, Vn, dict(tau=tau, cap=max(1, round(w.cap * n / w.N)))
        return Kn, Vn, dict(k=max(1, round(w.k * n / w.N)))

    def sample(inputs):
        Kn, Vn, sel = inputs
        t0 = time.perf_counter()
        oracle.decode_step(qr, ql, Kn, Vn, **sel)
        return time.perf_counter() - t0

    t_full = sample(prepare(w.N))                   # calibration, untimed
    budget = 60.0 / max(1, args.steps + args.warmup)
    n = int(min(w.N, max(1024, w.N * budget / max(t_full, 1e-6))))
    inputs = prepare(n)
    for _ in range(args.warmup):
        sample(inputs)
    sec = 0.0
    for _ in range(args.steps):
        sec += sample(inputs)
    frac = n / w.N                                  # share of one full step
    value = args.steps * frac / sec
    sel = (f"tau = {w.tau_pct[0]}th-percentile score, cap {max(1, round(w.cap * n / w.N))}"
           if threshold else f"k={max(1, round(w.k * n / w.N))}")
    desc = (f"{args.steps} samples, each the oracle decode step of all {w.B * w.Hkv} KV "
            f"heads (G={G}, L={w.L}) over the first {n} of {w.N} keys with "
            f"{sel}; value scaled by {frac:.3g} step per sample")
    return {
        "metric": (LOUVER_METRIC if args.louver else
                   THRESHOLD_METRIC if threshold else METRIC), "value": round(value, 5),
        "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 / value, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 attention / f32 scores (CPU oracle)", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv,
                   "d": w.d, "k": w.k, "L": w.L, "parallelism": "host cores"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 5), "unit": "steps/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "cpu": cpu_model(), "sample": desc},
        "e2e": {"value": round(value, 5), "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# Louver-index threshold step
# ---------------------------------------------------------------------------

LOUVER_METRIC = ("128K-context threshold sparse decode steps/s through the Louver index "
                 "(16 layers, tau = 97th-percentile score per head)")


def percentile_tau_device(sd, q_route, K, ws, num=97, den=100):
    """tau per (sequence, KV head): the nearest-rank num/den percentile of the
    head's routing scores (the library's scores; workload set-up, untimed)."""
    S = sd.score(q_route, K, ws=ws)
    N = S.shape[-1]
    rank = -(-num * N // den)
    return torch.kthvalue(S, rank, dim=-1).values.contiguous()


def run_native_louver(args, rank, world, local_rank):
    """One step = one sparse_louver_decode_step: threshold routing through the
    Louver index (ball tests, exact checks of the surviving clusters, the
    ordered set) and the attention of all L layers over that set.  The
    full-scan threshold step (score scan, threshold select, attention) is
    timed beside it."""
    import token_sparse_attention_sm_b200 as sd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = synth.WORKLOADS[args.workload]
    w = base.with_(seeds=tuple(s + 1000 * rank for s in base.seeds))
    r = args.louver
    x = synth.generate(w)
    variants = synth.query_variants(w, x, QUERY_SETS, seed=2000 + 1000 * rank)
    K = x["K"].to(dev)
    V = x["V"].to(dev)
    qs = [(qr.to(dev), ql.to(dev)) for qr, ql in variants]
    stream = torch.cuda.Stream(device=dev)
    ws = sd.Workspace(dev)
    ws.get(sd.workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, w.cap, w.L))
    cap = w.cap
    with torch.cuda.stream(stream):
        taus = [percentile_tau_device(sd, qr, K, ws, *w.tau_pct) for qr, _ in qs]
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        ix = sd.louver_build(K, r)
        ev1.record(stream)
        torch.cuda.synchronize()
        build_ms = ev0.elapsed_time(ev1)
        outs = [dict(out=torch.empty_like(ql),
                     idx=torch.empty((w.B, w.Hkv, cap), dtype=torch.int32, device=dev),
                     count=torch.empty((w.B, w.Hkv), dtype=torch.int32, device=dev),
                     surv=torch.empty((w.B, w.Hkv, 2), dtype=torch.int32, device=dev),
                     lse=torch.empty((w.L, w.B, w.Hq), dtype=torch.float32, device=dev))
                for _, ql in qs]

        def route_fn(i):
            o = outs[i]
            return lambda: sd.louver_route_threshold(qs[i][0], K, ix, taus[i], cap, check=False,
                                                     idx=o["idx"], count=o["count"])

        def attn_fn(i):
            o = outs[i]
            return lambda: sd.attn_gather(qs[i][1], K, V, o["idx"], count=o["count"], ws=ws,
                                          check=False, out=o["out"], lse=o["lse"])

        def step_fn(i):
            o = outs[i]
            return lambda: sd.louver_decode_step(qs[i][0], qs[i][1], K, V, ix, taus[i], cap,
                                                 ws=ws, check=False, out=o["out"],
                                                 idx=o["idx"], count=o["count"], lse=o["lse"])

        def full_fn(i):
            o = outs[i]
            return lambda: sd.decode_step(qs[i][0], qs[i][1], K, V, tau=taus[i], cap=cap, ws=ws,
                                          check=False, out=o["out"], idx=o["idx"],
                                          count=o["count"], lse=o["lse"])

        # survivors and set sizes per query set (untimed); equality with the
        # full-scan set is the tests' business, the sizes are reported here
        surv, counts = [], []
        for i in range(len(qs)):
            sd.louver_route_threshold(qs[i][0], K, ix, taus[i], cap, check=True,
                                      return_survivors=True, idx=outs[i]["idx"],
                                      count=outs[i]["count"], survivors=outs[i]["surv"])
            surv.append(outs[i]["surv"].cpu())
            counts.append(outs[i]["count"].cpu())
            step_fn(i)()
            full_fn(i)()
        sd.read_device_status(ws)
        sd.read_device_status(ix.ws)
        loop = capture_loop([step_fn(i) for i in range(len(qs))], stream)
        with ClockSampler(local_rank) as cs:
            ms = time_steps([step_fn(i) for i in range(len(qs))], args.steps, args.warmup,
                            stream, cs)
        clocks = cs.result()
        dist = step_distribution(loop, len(qs), stream)
        sd.read_device_status(ws)
        sd.read_device_status(ix.ws)
        n_k = max(args.steps // 4, 64)
        wk = max(args.warmup, 3)
        t_route = time_graphs(capture([route_fn(i) for i in range(len(qs))], stream), n_k, wk,
                              stream) / n_k
        t_attn = time_graphs(capture([attn_fn(i) for i in range(len(qs))], stream), n_k, wk,
                             stream) / n_k
        ms_full = time_steps([full_fn(i) for i in range(len(qs))], n_k, wk, stream) / n_k
        full_route = capture([lambda i=i: sd.route_threshold(qs[i][0], K, taus[i], cap, ws=ws,
                                                             check=False)
                              for i in range(len(qs))], stream)
        t_full_route = time_graphs(full_route, n_k, wk, stream) / n_k
        sd.read_device_status(ws)
        sd.read_device_status(ix.ws)

    ms_max = sdist.max_over_ranks(ms)
    t_route_max = sdist.max_over_ranks(t_route)
    ms_per_step = ms_max / args.steps
    value = world * args.steps / (ms_max / 1e3)
    e2e = run_e2e_louver(sd, w, variants, K, V, ix, taus, ws, stream, dev, args, world)

    peak, peak_src = load_peaks()
    nc = w.N // r
    BH = w.B * w.Hkv
    mean_surv = float(np.mean([s[..., 0].sum().item() for s in surv]))
    mean_leaves = float(np.mean([s[..., 1].sum().item() for s in surv]))
    mean_count = float(np.mean([np.minimum(c.numpy(), cap).sum() for c in counts]))
    # cluster balls, the leaf balls of the surviving clusters, the surviving
    # leaves' keys and key ids, the set written
    route_b = (BH * nc * (w.d + 1) * 4 + mean_surv * (r // 32) * (w.d + 1) * 4
               + mean_leaves * 32 * (w.d * w.esize + 4) + mean_count * 4)
    attn_b = 2 * mean_count * w.d * w.esize
    achieved = route_b / (t_route_max * 1e-3) / 1e9
    line = {
        "metric": LOUVER_METRIC,
        "value": round(value, 2),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded clustered keys: 64 centres per head plus noise; Gaussian q, V)",
        "config": {
            "workload": w.name, "B": w.B, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "L": w.L, "cap": cap, "tau": "nearest-rank 97th percentile score per head",
            "louver_r": r, "parallelism": f"replicas x{world}", "query_sets": QUERY_SETS,
            "l2": "inputs larger than L2 (K+V = %.0f MB, index keys %.0f MB per replica); the "
                  "query rotates over %d sets" % (2 * BH * w.N * w.d * w.esize / 1e6,
                                                    BH * w.N * w.d * w.esize / 1e6, QUERY_SETS),
            "timing": TIMING_OTHER,
            "index_build_ms": round(build_ms, 3),
            "surviving_clusters_per_query": round(mean_surv, 1),
            "surviving_leaves_per_query": round(mean_leaves, 1),
            "clusters_per_query": BH * nc,
            "mean_set_size_per_query": round(mean_count, 1),
        },
        "roofline": {
            "bound": "hbm", "kernel": "louver_query_kernel (routing: ball tests, exact checks, ordered set)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": None,
            "algorithmic_bytes_per_launch": int(route_b),
            "avg_launch_us": round(t_route_max * 1e3, 2),
            "peak_source": peak_src,
        },
        "step_roofline": {
            "unique_bytes_per_step": int(route_b + attn_b),
            "achieved_gbs": round((route_b + attn_b) / (ms_per_step * 1e-3) / 1e9, 1),
            "frac_of_measured_peak": round((route_b + attn_b) / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        },
        "kernels_us": {"louver_route": round(t_route * 1e3, 2),
                       "attn_gather_all_layers": round(t_attn * 1e3, 2),
                       "full_scan_route_threshold": round(t_full_route * 1e3, 2),
                       "full_scan_threshold_step": round(ms_full * 1e3, 2)},
        "e2e": e2e,
        "gpu_launches": (1 + (1 if w.dtype == "bf16" else 2)) * args.steps,
        "clocks": clocks,
        "step_time": dist,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_threshold(w, x)
    return line


THRESHOLD_METRIC = ("128K-context threshold sparse decode steps/s (16 layers, tau = "
                    "97th-percentile score per head, full scan)")


def run_native_threshold(args, rank, world, local_rank):
    """One step = one sparse_decode_step in threshold mode: the marking scan
    over the whole K cache (bits 'score >= tau' per key), the ordered sets
    written from the bitmaps, and the attention of all L layers over them."""
    import token_sparse_attention_sm_b200 as sd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = synth.WORKLOADS[args.workload]
    w = base.with_(seeds=tuple(s + 1000 * rank for s in base.seeds))
    x = synth.generate(w)
    variants = synth.query_variants(w, x, QUERY_SETS, seed=2000 + 1000 * rank)
    K = x["K"].to(dev)
    V = x["V"].to(dev)
    qs = [(qr.to(dev), ql.to(dev)) for qr, ql in variants]
    stream = torch.cuda.Stream(device=dev)
    ws = sd.Workspace(dev)
    ws.get(sd.workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.d, w.torch_dtype, w.cap, w.L))
    cap = w.cap
    with torch.cuda.stream(stream):
        taus = [percentile_tau_device(sd, qr, K, ws, *w.tau_pct) for qr, _ in qs]
        outs = [dict(out=torch.empty_like(ql),
                     idx=torch.empty((w.B, w.Hkv, cap), dtype=torch.int32, device=dev),
                     count=torch.empty((w.B, w.Hkv), dtype=torch.int32, device=dev),
                     lse=torch.empty((w.L, w.B, w.Hq), dtype=torch.float32, device=dev))
                for _, ql in qs]

        def step_fn(i):
            o = outs[i]
            return lambda: sd.decode_step(qs[i][0], qs[i][1], K, V, tau=taus[i], cap=cap, ws=ws,
                                          check=False, out=o["out"], idx=o["idx"],
                                          count=o["count"], lse=o["lse"])

        def route_fn(i):
            o = outs[i]
            return lambda: sd.route_threshold(qs[i][0], K, taus[i], cap, ws=ws, check=False,
                                              idx=o["idx"], count=o["count"])

        def attn_fn(i):
            o = outs[i]
            return lambda: sd.attn_gather(qs[i][1], K, V, o["idx"], count=o["count"], ws=ws,
                                          check=False, out=o["out"], lse=o["lse"])

        counts = []
        for i in range(len(qs)):
            step_fn(i)()
            counts.append(outs[i]["count"].cpu())
        sd.read_device_status(ws)
        loop = capture_loop([step_fn(i) for i in range(len(qs))], stream)
        with ClockSampler(local_rank) as cs:
            ms = time_steps([step_fn(i) for i in range(len(qs))], args.steps, args.warmup,
                            stream, cs)
        clocks = cs.result()
        dist = step_distribution(loop, len(qs), stream)
        sd.read_device_status(ws)
        n_k = max(args.steps // 4, 64)
        wk = max(args.warmup, 3)
        t_route = time_graphs(capture([route_fn(i) for i in range(len(qs))], stream), n_k, wk,
                              stream) / n_k
        t_attn = time_graphs(capture([attn_fn(i) for i in range(len(qs))], stream), n_k, wk,
                             stream) / n_k
        sd.read_device_status(ws)

    ms_max = sdist.max_over_ranks(ms)
    t_route_max = sdist.max_over_ranks(t_route)
    ms_per_step = ms_max / args.steps
    value = world * args.steps / (ms_max / 1e3)
    e2e = run_e2e_threshold(sd, w, variants, K, V, taus, ws, stream, dev, args, world)
    peak, peak_src = load_peaks()
    scan_b = w.B * w.Hkv * w.N * w.d * w.esize
    mean_count = float(np.mean([np.minimum(c.numpy(), cap).sum() for c in counts]))
    gath_b = 2 * mean_count * w.d * w.esize
    achieved = scan_b / (t_route_max * 1e-3) / 1e9
    line = {
        "metric": THRESHOLD_METRIC,
        "value": round(value, 2),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded Gaussian K/V/q, planted heavy hitters)",
        "config": {
            "workload": w.name, "B": w.B, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "L": w.L, "cap": cap, "tau": "nearest-rank 97th percentile score per head",
            "parallelism": f"replicas x{world}", "query_sets": QUERY_SETS,
            "l2": "inputs larger than L2 (K+V = %.0f MB per replica); the query rotates over "
                  "%d sets" % (2 * scan_b / 1e6, QUERY_SETS),
            "timing": TIMING_OTHER,
            "mean_set_size_per_query": round(mean_count, 1),
        },
        "roofline": {
            "bound": "hbm", "kernel": "threshold_mark_kernel + bitmap_compact_kernel (routing)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": None,
            "algorithmic_bytes_per_launch": scan_b,
            "avg_launch_us": round(t_route_max * 1e3, 2),
            "peak_source": peak_src,
        },
        "step_roofline": {
            "unique_bytes_per_step": int(scan_b + gath_b),
            "achieved_gbs": round((scan_b + gath_b) / (ms_per_step * 1e-3) / 1e9, 1),
            "frac_of_measured_peak": round((scan_b + gath_b) / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        },
        "kernels_us": {"route_threshold": round(t_route * 1e3, 2),
                       "attn_gather_all_layers": round(t_attn * 1e3, 2)},
        "e2e": e2e,
        "gpu_launches": (2 + (1 if w.dtype == "bf16" else 2)) * args.steps,
        "clocks": clocks,
        "step_time": dist,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_threshold(w, x)
    return line


def run_e2e_threshold(sd, w, variants, K, V, taus, ws, stream, dev, args, world):
    """The threshold step through the public API with host buffers (queries in
    from pinned memory, outputs, set and counts back, per-step sync):
    DecodeStepGraph, one per query set."""
    return _e2e_graphs(sd, w, variants, K, V, taus, ws, stream, args, world, None,
                       "route_threshold (full scan)")


def run_e2e_louver(sd, w, variants, K, V, ix, taus, ws, stream, dev, args, world):
    """The Louver step through the public API with host buffers:
    DecodeStepGraph over the index, one per query set."""
    return _e2e_graphs(sd, w, variants, K, V, taus, ws, stream, args, world, ix,
                       "louver_route_threshold (through the index)")


def _e2e_graphs(sd, w, variants, K, V, taus, ws, stream, args, world, index, what):
    graphs = []
    for (qr, ql), tau in zip(variants, taus):
        g = sd.DecodeStepGraph(K, V, w.L, w.Hq, tau=tau, cap=w.cap, ws=ws, stream=stream,
                               index=index)
        g.q_route_host.copy_(qr)
        g.q_layers_host.copy_(ql)
        graphs.append(g)
    steps = min(args.steps, 2000)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            graphs[i % len(graphs)]()
        torch.cuda.synchronize()
        sdist.barrier()
        t0 = time.perf_counter()
        for i in range(steps):
            graphs[i % len(graphs)]()
        t1 = time.perf_counter()
        sdist.barrier()
        sd.read_device_status(ws)
    sec = sdist.max_over_ranks(t1 - t0)
    g0 = graphs[0]
    return {"value": round(world * steps / sec, 2), "unit": "steps/s",
            "h2d_bytes_per_step": g0.h2d_bytes, "d2h_bytes_per_step": g0.d2h_bytes,
            "steps": steps,
            "api": "token_sparse_attention_sm_b200.DecodeStepGraph (%s and the layers' "
                   "attention in one CUDA graph with the host transfers: the layers' queries "
                   "and the index set cross PCIe on a second stream while routing and "
                   "attention run, the attention writes its outputs into mapped pinned host "
                   "memory (mapped_out=%s); synchronised every step)" % (what, g0.mapped_out)}


def cpu_baseline_threshold(w, x, budget_s: float = 10.0):
    """The C oracle, as it stands, on full threshold decode steps of the same
    workload (its set is the one the Louver index returns), repeated for
    about `budget_s` seconds."""
    import oracle
    qr, ql = synth.f32(x["q_route"]), synth.f32(x["q_layers"])
    Kf, Vf = synth.f32(x["K"]), synth.f32(x["V"])
    tau = oracle.percentile_tau(oracle.scores(qr, Kf), *w.tau_pct)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_step(qr, ql, Kf, Vf, tau=tau, cap=w.cap)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    sec = time.perf_counter() - t0
    return {"value": round(n / sec, 4), "unit": "steps/s", "cores": oracle.num_threads(),
            "kind": "oracle", "cpu": cpu_model(),
            "sample": f"{n} full threshold decode steps of {w.name} (all {w.B * w.Hkv} KV "
                      f"heads, {w.L} layers, full scan) by the plain C oracle, {sec:.1f} s"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="decode_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reroute", type=int, default=0,
                    help="re-route every R layers (1: per-layer routing); default: route "
                         "once per step, the method's shared routing")
    ap.add_argument("--dense", action="store_true",
                    help="also time dense attention over all N keys (k = N), all layers in "
                         "one pass and layer by layer, as the comparison for per-layer routing")
    ap.add_argument("--louver", type=int, default=0, metavar="R",
                    help="threshold steps routed through the Louver index with clusters of "
                         "R keys (workload louver_128k unless --workload names another "
                         "threshold workload)")
    args = ap.parse_args()
    if args.louver and synth.WORKLOADS[args.workload].mode != "threshold":
        args.workload = "louver_128k"
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = sdist.env_rank_world()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    sdist.init("nccl")
    try:
        if args.louver:
            line = run_native_louver(args, rank, world, local_rank)
        elif synth.WORKLOADS[args.workload].mode == "threshold":
            line = run_native_threshold(args, rank, world, local_rank)
        else:
            line = run_native(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        sdist.finalize()


if __name__ == "__main__":
    main()
