#!/usr/bin/env python3
"""Benchmark of the attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on stdout (rank 0).  Two timed phases, each of exactly K steps
after W warm-up steps, bracketed by a barrier and a device synchronisation on
both sides, timed with CUDA events on the launching stream, max over ranks:

Timed steps are CUDA-graph replays of one step's launches (captured through the
public API; ``--no-graph`` launches them directly); the roofline figures come
from a second pass with CUDA events around each library call.

* prefill (headline ``value``): the 70B-shaped causal GQA workload
  (b1 S8192 H64 Hkv8 D128, RoPE theta 1e4 with linear factor 2.0, bf16).  One
  step = RoPE table from position ids + llama_attn_prefill (K rotation pass +
  tcgen05 attention kernel).  Throughput counts only unmasked FLOPs:
  4 * D * (S(S+1)/2) * b * H per step.
* decode: the GQA decode workload (b32 H64 Hkv8 D128, cache lengths uniform
  in [512, 4096], max 4096).  One step = RoPE row for the query positions +
  llama_attn_decode (split-KV kernel + combine).  Bytes = K and V rows read,
  2 * sum(len_b) * Hkv * D * 2.

``e2e``: the same metrics through the public API with the inputs in pinned
host memory.  Prefill copies each step's q, k, v and positions in and the
output out, pipelined over three streams; decode keeps the caches resident
(model state) and copies each step's q, lengths and positions in and the
output out, steps in sequence on one stream.

``--phase configs`` instead times every named workload (the five shapes the
parity tests cover) through the public API, one JSON line per workload, with
CUDA events around each call (direct launches); it is a report, not the
benchmark line.

Inputs are larger than L2 (126 MB) in both phases (prefill: q 134 MB, out
134 MB; decode: two alternating 537 MB caches, ~302 MB read per step), so no
L2 flush is needed between steps.  Multi-GPU runs are independent replicas
(the path has no cross-GPU exchange): ``value`` is the sum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from llama_gqa_causal_b200 import replicas, workloads as W  # noqa: E402

PREFILL = W.LLAMA70B
DECODE = W.DECODE70B
METRIC = "causal GQA prefill TFLOP/s and KV-decode HBM GB/s, % of B200 roofline"


def _traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu record, or None
    when the CUDA sources changed since that capture."""
    import glob
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    except Exception:
        return None
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "llama_gqa_causal_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        h.update(open(f, "rb").read())
    if h.hexdigest()[:16] != rec.get("csrc_sha256_16") or kernel not in rec:
        return None
    return rec[kernel]["dram_read_bytes"] + rec[kernel]["dram_write_bytes"]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# ----------------------------------------------------------------------------- distributed plumbing

def _barrier(ws):
    replicas.barrier(ws)


def _max_over_ranks(x: float, ws: int) -> float:
    return replicas.max_over_ranks(x, ws, device="cuda")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling (every 10 ms) of SM clock, power and throttle
    reasons; `summary()` keeps only the samples taken inside the windows marked
    with `mark()` (wall-clock spans in which the GPU runs the timed work), so
    idle moments between phases do not dilute the figure."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.windows = []

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def mark(self, t0: float, t1: float):
        self.windows.append((t0, t1))

    def summary(self):
        import datetime
        out = {"sm_mhz": None, "sm_max_mhz": None, "power_w": None, "reasons": [], "samples": 0,
               "window_s": round(sum(b - a for a, b in self.windows), 4)}
        if not self.path or not os.path.exists(self.path):
            return out
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), float(f[4]), f[6], f[7], f[8], f[9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if self.windows:
            inside = [r for r in rows if any(a <= r[0] <= b for a, b in self.windows)]
            rows = inside if inside else rows
        if not rows:
            return out
        out["samples"] = len(rows)
        out["sm_mhz"] = statistics.median(r[1] for r in rows)
        out["sm_max_mhz"] = max(r[2] for r in rows)
        out["power_w"] = round(statistics.median(r[3] for r in rows), 1)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[4:]):
                if v.lower() == "active":
                    reasons.add(n)
        out["reasons"] = sorted(reasons)
        return out


def _capture(step_fn):
    """Capture one step (its kernel launches, through the public API) into a CUDA
    graph; None if capture is not possible here (the steps then launch directly)."""
    try:
        return _capture_or_raise(step_fn)
    except Exception as e:  # noqa: BLE001
        print(f"bench: CUDA graph capture failed ({e}); launching directly", file=sys.stderr)
        torch.cuda.synchronize()
        return None


def _capture_or_raise(step_fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step_fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step_fn()
    torch.cuda.synchronize()
    return graph


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, ws, local):
    from llama_gqa_causal_b200 import api
    api.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peak_burst, peak_sus, hbm, peak_src = _peaks()

    line = {
        "metric": METRIC,
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v, cast to bf16)",
    }
    launches = 0
    if args.phase in ("all", "prefill"):
        launches += _prefill_phase(args, ws, local, dev, stream, line)
    if args.phase in ("all", "decode"):
        launches += _decode_phase(args, ws, local, dev, stream, line)
    line["gpu_launches"] = launches
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    return line


def _prefill_phase(args, ws, local, dev, stream, line):
    from llama_gqa_causal_b200 import api
    peak_burst, peak_sus, hbm, peak_src = _peaks()
    cfg = PREFILL
    x = W.prefill_inputs(cfg)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    pos = x["pos"].to(dev)
    out = torch.empty(cfg.bsz, cfg.seq, cfg.n_heads * cfg.head_dim, device=dev, dtype=cfg.dtype)
    wsp = torch.empty(api.prefill_workspace_bytes(cfg.bsz, cfg.n_heads, cfg.n_kv_heads, cfg.seq,
                                                  cfg.head_dim, cfg.dtype, True),
                      device=dev, dtype=torch.uint8)

    def prefill_step(ev=None):
        cos, sin = api.rope_table(pos, cfg.head_dim, cfg.theta, cfg.factor)
        if ev is not None:
            ev[0].record(stream)
        api.prefill(q, k, v, cos, sin, causal=True, scale=cfg.scale, out=out, workspace=wsp)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        prefill_step()
    torch.cuda.synchronize()
    graph = None if args.no_graph else _capture(prefill_step)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        # whole steps (CUDA-graph replays of rope_table + llama_attn_prefill)
        for _ in range(args.warmup):
            graph.replay() if graph is not None else prefill_step()
        _barrier(ws)
        torch.cuda.synchronize()
        w0 = time.time()
        t0.record(stream)
        for i in range(args.steps):
            graph.replay() if graph is not None else prefill_step()
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark(w0, time.time())
        _barrier(ws)
        # the prefill call alone, events around each call (roofline figure)
        w0 = time.time()
        for i in range(args.steps):
            prefill_step(evs[i])
        torch.cuda.synchronize()
        clk.mark(w0, time.time())
    clocks = clk.summary()
    ms_total = _max_over_ranks(t0.elapsed_time(t1), ws)
    ms_call = _max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), ws)
    flops = cfg.flops()
    value = replicas.job_throughput(flops, args.steps, ms_total, ws) / 1e12
    achieved = flops / (ms_call * 1e-3) / 1e12
    assert api.device_status() == api.LLAMA_OK

    # e2e: pinned host inputs -> device, compute, result -> pinned host, every
    # step, pipelined the way a serving loop runs it: step i+1's inputs are
    # copied in on one stream while step i computes on another and step i-1's
    # output is copied out on a third (two device buffer sets; events order
    # each buffer's reuse).  The timed region spans the first copy-in to the
    # last copy-out.
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    hpos = x["pos"].pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = 0 if args.no_e2e else max(args.steps, 10)
    if e2e_steps:
        sets = [dict(q=q, k=k, v=v, pos=pos, out=out)]
        sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_done = [ev(), ev()]
        comp_done = [ev(), ev()]
        out_done = [ev(), ev()]

        def e2e_pipeline(n_steps):
            for i in range(n_steps):
                j = i % 2
                d = sets[j]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(comp_done[j])  # step i-2 has read these inputs
                    d["q"].copy_(hq, non_blocking=True)
                    d["k"].copy_(hk, non_blocking=True)
                    d["v"].copy_(hv, non_blocking=True)
                    d["pos"].copy_(hpos, non_blocking=True)
                    in_done[j].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(in_done[j])
                    if i >= 2:
                        s_comp.wait_event(out_done[j])  # step i-2's output has been copied out
                    cos, sin = api.rope_table(d["pos"], cfg.head_dim, cfg.theta, cfg.factor)
                    api.prefill(d["q"], d["k"], d["v"], cos, sin, causal=True, scale=cfg.scale,
                                out=d["out"], workspace=wsp)
                    comp_done[j].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[j])
                    hout.copy_(d["out"], non_blocking=True)
                    out_done[j].record(s_out)
            cur = torch.cuda.current_stream()
            for st_ in (s_in, s_comp, s_out):
                cur.wait_stream(st_)

        e2e_pipeline(2)  # warm-up (allocations, first copies)
        torch.cuda.synchronize()
        _barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_stream(stream)
        e2e_pipeline(e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize()
        _barrier(ws)
        ms_e2e = _max_over_ranks(e0.elapsed_time(e1), ws)
        assert api.device_status() == api.LLAMA_OK
        e2e_value = replicas.job_throughput(flops, e2e_steps, ms_e2e, ws) / 1e12
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hpos))
        d2h = hout.numel() * hout.element_size()
        del sets
    else:
        e2e_value, h2d, d2h = None, 0, 0
    del hq, hk, hv, hout, q, k, v, out, wsp, x
    torch.cuda.empty_cache()
    line.update({
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "ms_per_step": round(ms_total / args.steps, 4),
        "config": {
            "workload": "llama70b causal GQA prefill b1 S8192 H64 Hkv8 D128, RoPE theta 1e4 "
                        "linear x2 (value); decode70b GQA decode b32 H64 Hkv8 D128 lens U[512,4096] "
                        "(decode)",
            "global_batch": cfg.bsz * ws,
            "seq_len": cfg.seq,
            "parallelism": f"replicas x{ws}",
            "l2": "inputs larger than L2 (no flush)",
            "launch": "cuda-graph replay" if graph is not None else "direct",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": "llama_attn_prefill (K rotation pass + prefill_sm100_kernel)",
            "achieved": round(achieved, 2),
            "peak": peak_burst,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak_burst, 4),
            "peak_source": f"{peak_src} bf16 burst",
            "traffic": _traffic("prefill_sm100_kernel<128>"),
            "traffic_unit": "bytes per launch (ncu dram read+write)",
        },
        "e2e": {
            "value": None if e2e_value is None else round(e2e_value, 3),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "steps": e2e_steps,
            "launch": "3-stream pipeline (copy-in, compute, copy-out), direct launches",
        },
        "clocks": clocks,
    })
    # rope_table + K rotation + attention kernel per timed step
    return args.steps * 3


def _pack_step_inputs(tensors, dev):
    """One device byte buffer holding `tensors` back to back (each at a 16-byte
    aligned offset) and typed views of it, shaped like the inputs."""
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 15) // 16 * 16
    stage = torch.empty(total, dtype=torch.uint8, device=dev)
    views = []
    for t, o in zip(tensors, offs):
        n = t.numel() * t.element_size()
        v = stage[o:o + n].view(t.dtype).view(t.shape)
        v.copy_(t.to(dev))
        views.append(v)
    return stage, views


def _decode_phase(args, ws, local, dev, stream, line):
    from llama_gqa_causal_b200 import api
    peak_burst, peak_sus, hbm, peak_src = _peaks()
    dcfg = DECODE
    insts = []
    for rep in range(2):  # two caches, alternated, so no step reads L2-resident data
        y = W.decode_inputs(dcfg)
        d = {n: y[n].to(dev) for n in ("k_cache", "v_cache")}
        # a step's own inputs (q, lengths, positions) sit in one staging buffer,
        # so the end-to-end run copies them in with a single transfer
        d["stage"], views = _pack_step_inputs([y["q"], y["lens"], y["qpos"]], dev)
        d["q"], d["lens"], d["qpos"] = views
        insts.append(d)
    lens_cpu = y["lens"].to(torch.int64)
    dbytes = int(2 * lens_cpu.sum().item() * dcfg.n_kv_heads * dcfg.head_dim * 2)
    dout = torch.empty(dcfg.bsz, dcfg.n_heads * dcfg.head_dim, device=dev, dtype=dcfg.dtype)
    dws = torch.empty(api.decode_workspace_bytes(dcfg.bsz, dcfg.n_heads, dcfg.max_cache_len,
                                                 dcfg.head_dim), device=dev, dtype=torch.uint8)

    def decode_step(i, ev=None):
        d = insts[i % 2]
        cos, sin = api.rope_table(d["qpos"].view(-1, 1), dcfg.head_dim, dcfg.theta, dcfg.factor)
        if ev is not None:
            ev[0].record(stream)
        api.decode(d["q"], d["k_cache"], d["v_cache"], d["lens"], cos.view(dcfg.bsz, -1),
                   sin.view(dcfg.bsz, -1), scale=dcfg.scale, out=dout, workspace=dws)
        if ev is not None:
            ev[1].record(stream)

    dsteps = max(args.steps, 20)
    for i in range(max(args.warmup, 3)):
        decode_step(i)
    torch.cuda.synchronize()
    graphs = None if args.no_graph else [_capture(lambda i=i: decode_step(i)) for i in range(2)]
    if graphs is not None and any(g_ is None for g_ in graphs):
        graphs = None
    devs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(dsteps)]
    for i in range(max(args.warmup, 3)):
        graphs[i % 2].replay() if graphs is not None else decode_step(i)
    _barrier(ws)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for i in range(dsteps):
        graphs[i % 2].replay() if graphs is not None else decode_step(i)
    d1.record(stream)
    torch.cuda.synchronize()
    _barrier(ws)
    # the decode call alone (roofline figure).  Events between direct launches
    # would also time the split kernel's launch, which the call otherwise
    # overlaps with the previous grid, so with graphs the call (split +
    # combine, tables formed beforehand) is replayed as a graph of its own and
    # the train's mean is taken; without graphs, events go around each call.
    tabs = [api.rope_table(d["qpos"].view(-1, 1), dcfg.head_dim, dcfg.theta, dcfg.factor)
            for d in insts]

    def decode_call(i):
        d = insts[i % 2]
        cos, sin = tabs[i % 2]
        api.decode(d["q"], d["k_cache"], d["v_cache"], d["lens"], cos.view(dcfg.bsz, -1),
                   sin.view(dcfg.bsz, -1), scale=dcfg.scale, out=dout, workspace=dws)

    call_graphs = None if graphs is None else [_capture(lambda i=i: decode_call(i)) for i in range(2)]
    if call_graphs is not None and all(g_ is not None for g_ in call_graphs):
        for i in range(max(args.warmup, 3)):
            call_graphs[i % 2].replay()
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for i in range(dsteps):
            call_graphs[i % 2].replay()
        c1.record(stream)
        torch.cuda.synchronize()
        ms_dec_call = _max_over_ranks(c0.elapsed_time(c1) / dsteps, ws)
        call_timing = "graph replays of the call alone (train mean)"
    else:
        for i in range(dsteps):
            decode_step(i, devs[i])
        torch.cuda.synchronize()
        ms_dec_call = _max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in devs), ws)
        call_timing = "events around each direct call"
    del call_graphs
    ms_dec_total = _max_over_ranks(d0.elapsed_time(d1), ws)
    dec_value = replicas.job_throughput(dbytes, dsteps, ms_dec_total, ws) / 1e9
    dec_achieved = dbytes / (ms_dec_call * 1e-3) / 1e9
    assert api.device_status() == api.LLAMA_OK

    # e2e: the KV caches are model state resident in HBM; every step copies its
    # own inputs (the new token's q, the cache lengths, the query positions)
    # from pinned host memory, runs the public API, and reads the output back.
    # A decode step needs the previous step's output, so the steps run one
    # after another on one stream.
    dec_e2e = None
    if not args.no_e2e:
        hosts = [insts[r]["stage"].cpu().pin_memory() for r in range(2)]
        hout = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()

        def e2e_step(i):
            insts[i % 2]["stage"].copy_(hosts[i % 2], non_blocking=True)
            decode_step(i)
            hout.copy_(dout, non_blocking=True)

        for i in range(max(args.warmup, 3)):
            e2e_step(i)
        torch.cuda.synchronize()
        _barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(dsteps):
            e2e_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        _barrier(ws)
        ms_e2e = _max_over_ranks(e0.elapsed_time(e1), ws)
        assert api.device_status() == api.LLAMA_OK
        dec_e2e = {
            "value": round(replicas.job_throughput(dbytes, dsteps, ms_e2e, ws) / 1e9, 1),
            "unit": "GB/s",
            "ms_per_step": round(ms_e2e / dsteps, 4),
            "h2d_bytes_per_step": hosts[0].numel() * hosts[0].element_size(),
            "d2h_bytes_per_step": hout.numel() * hout.element_size(),
            "steps": dsteps,
            "launch": "one stream, steps in sequence, direct launches; caches resident; the step's "
                      "q, lengths and positions copied in as one pinned buffer",
        }
        del hosts, hout

    line["decode"] = {
        "launch": "cuda-graph replay" if graphs is not None else "direct",
        "value": round(dec_value, 1),
        "unit": "GB/s",
        "ms_per_step": round(ms_dec_total / dsteps, 4),
        "steps": dsteps,
        "bytes_per_step": dbytes,
        "roofline": {
            "bound": "hbm",
            "kernel": "llama_attn_decode (decode_bf16_kernel + decode_combine_kernel)",
            "timing": call_timing,
            "achieved": round(dec_achieved, 1),
            "peak": hbm,
            "unit": "GB/s",
            "frac": round(dec_achieved / hbm, 4),
            "peak_source": f"{peak_src} copy bandwidth",
            "traffic": _traffic("decode_bf16_kernel<128>"),
            "traffic_unit": "bytes per launch of the split kernel (ncu dram read+write)",
        },
        "e2e": dec_e2e,
    }
    if "value" not in line:  # decode-only run: the decode numbers are the line's
        line.update({"value": line["decode"]["value"], "unit": "GB/s",
                     "ms_per_step": line["decode"]["ms_per_step"],
                     "config": {"workload": "decode70b GQA decode b32 H64 Hkv8 D128 lens U[512,4096]",
                                "global_batch": dcfg.bsz * ws, "seq_len": dcfg.max_cache_len,
                                "parallelism": f"replicas x{ws}",
                                "l2": "two alternating caches larger than L2"}})
    # rope_table + split kernel + combine kernel per timed step
    return dsteps * 3


# ----------------------------------------------------------------------------- oracle arms

def _oracle_sample_prefill(cfg, rows):
    """Run the fp64 oracle on all heads of `rows` (lo, hi) of the workload; returns (seconds, flops)."""
    import oracle
    x = W.prefill_inputs(cfg)
    lo, hi = rows
    t = time.perf_counter()
    oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                   scale=cfg.scale, causal=cfg.causal, rows=rows)
    dt = time.perf_counter() - t
    keys = sum(min(cfg.seq, i + 1) if cfg.causal else cfg.seq for i in range(lo, hi))
    flops = 4 * cfg.head_dim * keys * cfg.bsz * cfg.n_heads
    return dt, flops


def _config_cpu_baseline(cfg, x):
    """The fp64 oracle timed on a bounded sample of one named workload, on all
    host cores and on one core; the value in the workload's own unit."""
    import oracle
    out = {"kind": "oracle"}
    for key, nthreads in (("value", 0), ("one_core", 1)):
        if isinstance(cfg, W.DecodeConfig):
            # the whole step: every cached row attended once
            t = time.perf_counter()
            oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"], theta=cfg.theta,
                          factor=cfg.factor, scale=cfg.scale, nthreads=nthreads)
            dt = time.perf_counter() - t
            nbytes = 2 * int(x["lens"].to(torch.int64).sum()) * cfg.n_kv_heads * cfg.head_dim * 2
            out[key] = round(nbytes / dt / 1e9, 4)
            out.update(unit="GB/s", sample="the whole step (all batch entries and heads)")
            continue
        # prefill: all heads of the last rows (every row for the small workloads)
        lo = 0 if cfg.seq <= 256 else cfg.seq - 64
        reps = 20 if cfg.seq <= 64 else 1
        t = time.perf_counter()
        for _ in range(reps):
            oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                           scale=cfg.scale, causal=cfg.causal, rows=(lo, cfg.seq), nthreads=nthreads)
        dt = (time.perf_counter() - t) / reps
        keys = sum(min(cfg.seq, i + 1) if cfg.causal else cfg.seq for i in range(lo, cfg.seq))
        flops = 4 * cfg.head_dim * keys * cfg.bsz * cfg.n_heads
        out[key] = round(flops / dt / 1e12, 6)
        out.update(unit="TFLOP/s",
                   sample=("every row" if lo == 0 else f"query rows [{lo}, {cfg.seq})")
                   + f" of all {cfg.n_heads} heads and {cfg.bsz} batch "
                   + ("entry" if cfg.bsz == 1 else "entries") + f" ({flops / 1e9:.3g} GFLOP)")
    out["cores"] = oracle.max_threads()
    return out


def cpu_baseline(rows=None):
    import oracle
    cfg = PREFILL
    rows = rows or (cfg.seq - 1024, cfg.seq)
    dt, flops = _oracle_sample_prefill(cfg, rows)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"llama70b prefill, all 64 heads, query rows [{rows[0]}, {rows[1]}) "
                      f"({flops / 1e9:.1f} GFLOP fp64, {dt:.1f} s, includes rotating all K)"}


def run_reference(args, rank, ws):
    if rank != 0:
        return None
    import oracle
    cfg = PREFILL
    rows = (cfg.seq - 4, cfg.seq)
    times, flops = [], 0
    for i in range(args.warmup + args.steps):
        dt, fl = _oracle_sample_prefill(cfg, rows)
        if i >= args.warmup:
            times.append(dt)
            flops = fl
    total = sum(times)
    value = flops * len(times) / total / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total / len(times) * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/k/v, cast to bf16)",
        "config": {"workload": "llama70b causal GQA prefill b1 S8192 H64 Hkv8 D128, RoPE theta 1e4 "
                               "linear x2 (bounded sample per step)",
                   "global_batch": 1, "seq_len": cfg.seq, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"all 64 heads, query rows [{rows[0]}, {rows[1]}) per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_configs(args):
    """One JSON line per named workload: mean device time of the library call
    (a train of CUDA-graph replays of the call; events around each direct call
    with --no-graph)."""
    from llama_gqa_causal_b200 import api
    api.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peak_burst, _, hbm, peak_src = _peaks()
    steps = max(args.steps, 1)

    def timed(call):
        """Mean device time of one call: the call captured as a CUDA graph and
        replayed `steps` times between two events (so that the binding's host
        work, which exceeds the small workloads' kernel time, is not what is
        timed); events around each direct call where capture is not possible."""
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        graph = None if args.no_graph else _capture(call)
        if graph is not None:
            for _ in range(args.warmup):
                graph.replay()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                graph.replay()
            b.record(stream)
            torch.cuda.synchronize()
            assert api.device_status() == api.LLAMA_OK
            del graph
            return a.elapsed_time(b) / steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        assert api.device_status() == api.LLAMA_OK
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    def wanted(cfg):
        return args.workload in (None, cfg.name)

    for cfg in W.PREFILL_CONFIGS.values():
        if not wanted(cfg):
            continue
        x = W.prefill_inputs(cfg)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        cos = sin = None
        x_pos = None
        if x["pos"] is not None:
            x_pos = x["pos"].to(dev)
            cos, sin = api.rope_table(x_pos, cfg.head_dim, cfg.theta, cfg.factor)
        out = torch.empty(cfg.bsz, cfg.seq, cfg.n_heads * cfg.head_dim, device=dev, dtype=cfg.dtype)
        wsp = torch.empty(max(1, api.prefill_workspace_bytes(cfg.bsz, cfg.n_heads, cfg.n_kv_heads,
                                                             cfg.seq, cfg.head_dim, cfg.dtype,
                                                             cos is not None)),
                          device=dev, dtype=torch.uint8)
        ms = timed(lambda: api.prefill(q, k, v, cos, sin, causal=cfg.causal, scale=cfg.scale,
                                       out=out, workspace=wsp))
        tflops = cfg.flops() / (ms * 1e-3) / 1e12
        cline = {"phase": "configs", "workload": cfg.name, "dtype": str(cfg.dtype).split(".")[-1],
                 "ms_per_call": round(ms, 5), "value": round(tflops, 2), "unit": "TFLOP/s",
                 "frac": round(tflops / peak_burst, 4),
                 "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}
        if not args.no_cpu_baseline:
            cline["cpu_baseline"] = _config_cpu_baseline(cfg, x)
        print(json.dumps(cline), flush=True)
        if cfg.name == "llama7b":
            # the same batch right-padded: the second entry holds about half its rows
            lens = [cfg.seq] + [cfg.seq // 2 + 37] * (cfg.bsz - 1)
            sl = torch.tensor(lens, dtype=torch.int32, device=dev)
            vflops = sum(4 * cfg.head_dim * n * (n + 1) // 2 * cfg.n_heads for n in lens)
            ms = timed(lambda: api.prefill_varlen(q, k, v, sl, cos, sin, causal=True,
                                                  scale=cfg.scale, out=out, workspace=wsp))
            tflops = vflops / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+varlen{lens}",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5),
                              "value": round(tflops, 2), "unit": "TFLOP/s",
                              "frac": round(tflops / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
        if cfg.name == "llama7b":
            # the same heads with four sequences packed back to back
            plens = [cfg.seq, cfg.seq // 2 + 37, 700, 300]
            T = sum(plens)
            g = torch.Generator().manual_seed(cfg.seed + 3)
            pq = W.normal((T, cfg.n_heads, cfg.head_dim), cfg.dtype, g).to(dev)
            pk = W.normal((T, cfg.n_kv_heads, cfg.head_dim), cfg.dtype, g).to(dev)
            pv = W.normal((T, cfg.n_kv_heads, cfg.head_dim), cfg.dtype, g).to(dev)
            ppos = torch.cat([torch.arange(n) for n in plens]).to(dev)
            pc, ps = api.rope_table(ppos.view(1, -1), cfg.head_dim, cfg.theta, cfg.factor)
            pc, ps = pc.view(T, -1), ps.view(T, -1)
            cu = torch.tensor([0] + list(np.cumsum(plens)), dtype=torch.int32, device=dev)
            pout = torch.empty(T, cfg.n_heads * cfg.head_dim, device=dev, dtype=cfg.dtype)
            pws = torch.empty(api.prefill_workspace_bytes(1, cfg.n_heads, cfg.n_kv_heads, T,
                                                          cfg.head_dim, cfg.dtype, True),
                              device=dev, dtype=torch.uint8)
            pflops = sum(4 * cfg.head_dim * n * (n + 1) // 2 * cfg.n_heads for n in plens)
            ms = timed(lambda: api.prefill_packed(pq, pk, pv, cu, max(plens), pc, ps, causal=True,
                                                  scale=cfg.scale, out=pout, workspace=pws))
            tflops = pflops / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+packed{plens}",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5),
                              "value": round(tflops, 2), "unit": "TFLOP/s",
                              "frac": round(tflops / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
            del pq, pk, pv, pout, pws
        if cfg.causal and cfg.dtype == torch.bfloat16 and cfg.seq > 4096:
            # the same workload with a 4096-key sliding window (visible pairs only)
            window = 4096
            pairs = sum(min(i + 1, window) for i in range(cfg.seq))
            wflops = 4 * cfg.head_dim * pairs * cfg.n_heads * cfg.bsz
            ms = timed(lambda: api.prefill_window(q, k, v, cos, sin, window=window, scale=cfg.scale,
                                                  out=out, workspace=wsp))
            tflops = wflops / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+window{window}",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5),
                              "value": round(tflops, 2), "unit": "TFLOP/s",
                              "frac": round(tflops / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
        if cfg.name == "llama70b":
            # the NTK-aware scaled RoPE table for the workload's positions (alpha 4)
            # a small kernel: replay the captured call, so that the binding's
            # host work (more than the kernel's time) is not what is timed
            for _ in range(args.warmup):
                api.rope_table_ntk(x_pos, cfg.head_dim, cfg.theta, 4.0)
            torch.cuda.synchronize()
            tgraph = _capture(lambda: api.rope_table_ntk(x_pos, cfg.head_dim, cfg.theta, 4.0))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(50):
                tgraph.replay() if tgraph is not None else api.rope_table_ntk(
                    x_pos, cfg.head_dim, cfg.theta, 4.0)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / 50
            del tgraph
            nbytes = 2 * x_pos.numel() * cfg.head_dim * 4
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+rope_table_ntk",
                              "dtype": "float32", "ms_per_call": round(ms, 5),
                              "value": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                              "frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4),
                              "peak": f"{hbm} GB/s ({peak_src} copy)"}), flush=True)
        if cfg.name == "llama70b":
            # the projections around the attention of this shape (hidden 8192):
            # q/k/v with RoPE in the GEMM epilogue, then the output projection
            hidden = cfg.n_heads * cfg.head_dim
            n_qkv = (cfg.n_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
            T = cfg.bsz * cfg.seq
            g = torch.Generator().manual_seed(cfg.seed + 4)
            px = W.normal((T, hidden), cfg.dtype, g).to(dev)
            pw = (torch.randn(n_qkv, hidden, generator=g) / hidden ** 0.5).to(cfg.dtype).to(dev)
            pwo = (torch.randn(hidden, hidden, generator=g) / hidden ** 0.5).to(cfg.dtype).to(dev)
            bufs = (torch.empty(T, cfg.n_heads, cfg.head_dim, device=dev, dtype=cfg.dtype),
                    torch.empty(T, cfg.n_kv_heads, cfg.head_dim, device=dev, dtype=cfg.dtype),
                    torch.empty(T, cfg.n_kv_heads, cfg.head_dim, device=dev, dtype=cfg.dtype))
            ct, st_ = cos.view(T, -1), sin.view(T, -1)
            # (the attention lines run before the GEMM timings: sustained GEMMs
            # raise the power draw and can lower the clock of what follows)
            api.qkv_rope(px, pw, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, ct, st_, out=bufs)
            torch.cuda.synchronize()
            # the attention of the same shape on the q/k the projection has
            # already rotated (no cos/sin: no K rotation pass, no Q rotation)
            ms = timed(lambda: api.prefill(bufs[0].view(cfg.bsz, cfg.seq, cfg.n_heads, -1),
                                           bufs[1].view(cfg.bsz, cfg.seq, cfg.n_kv_heads, -1),
                                           bufs[2].view(cfg.bsz, cfg.seq, cfg.n_kv_heads, -1),
                                           causal=True, scale=cfg.scale, out=out))
            tf = cfg.flops() / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+prerotated_qk",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5), "value": round(tf, 2),
                              "unit": "TFLOP/s", "frac": round(tf / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
            ms = timed(lambda: api.qkv_rope(px, pw, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, ct,
                                            st_, out=bufs))
            tf = 2.0 * T * hidden * n_qkv / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+qkv_rope_proj",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5), "value": round(tf, 2),
                              "unit": "TFLOP/s", "frac": round(tf / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
            py = torch.empty(T, hidden, device=dev, dtype=cfg.dtype)
            ms = timed(lambda: api.out_proj(bufs[0].view(T, hidden), pwo, out=py))
            tf = 2.0 * T * hidden * hidden / (ms * 1e-3) / 1e12
            print(json.dumps({"phase": "configs", "workload": f"{cfg.name}+out_proj",
                              "dtype": "bfloat16", "ms_per_call": round(ms, 5), "value": round(tf, 2),
                              "unit": "TFLOP/s", "frac": round(tf / peak_burst, 4),
                              "peak": f"{peak_burst} TFLOP/s ({peak_src} bf16 burst)"}), flush=True)
            del px, pw, pwo, bufs, py
        del q, k, v, out, wsp, x

    for cfg in W.DECODE_CONFIGS.values():
        if not wanted(cfg):
            continue
        x = W.decode_inputs(cfg)
        d = {n: x[n].to(dev) for n in ("q", "k_cache", "v_cache", "lens", "qpos")}
        cos, sin = api.rope_table(d["qpos"].view(-1, 1), cfg.head_dim, cfg.theta, cfg.factor)
        cos, sin = cos.view(cfg.bsz, -1), sin.view(cfg.bsz, -1)
        out = torch.empty(cfg.bsz, cfg.n_heads * cfg.head_dim, device=dev, dtype=cfg.dtype)
        wsp = torch.empty(api.decode_workspace_bytes(cfg.bsz, cfg.n_heads, cfg.max_cache_len,
                                                     cfg.head_dim), device=dev, dtype=torch.uint8)
        ms = timed(lambda: api.decode(d["q"], d["k_cache"], d["v_cache"], d["lens"], cos, sin,
                                      scale=cfg.scale, out=out, workspace=wsp))
        nbytes = int(2 * x["lens"].to(torch.int64).sum().item() * cfg.n_kv_heads * cfg.head_dim * 2)
        gbs = nbytes / (ms * 1e-3) / 1e9
        cline = {"phase": "configs", "workload": cfg.name, "dtype": str(cfg.dtype).split(".")[-1],
                 "ms_per_call": round(ms, 5), "value": round(gbs, 1), "unit": "GB/s",
                 "frac": round(gbs / hbm, 4), "peak": f"{hbm} GB/s ({peak_src} copy)"}
        if not args.no_cpu_baseline:
            cline["cpu_baseline"] = _config_cpu_baseline(cfg, x)
        print(json.dumps(cline), flush=True)
        # the same step with the new token's own key/value appended at row
        # p = min(len, L - 1) and attended (rows 0..p); every call rewrites the
        # same rows with the same values
        g = torch.Generator().manual_seed(cfg.seed + 2)
        k_new = W.normal((cfg.bsz, cfg.n_kv_heads, cfg.head_dim), cfg.dtype, g).to(dev)
        v_new = W.normal((cfg.bsz, cfg.n_kv_heads, cfg.head_dim), cfg.dtype, g).to(dev)
        ms = timed(lambda: api.decode_append(d["q"], k_new, v_new, d["k_cache"], d["v_cache"],
                                             d["lens"], cos, sin, scale=cfg.scale, out=out,
                                             workspace=wsp))
        rows = x["lens"].to(torch.int64).clamp(0, cfg.max_cache_len - 1) + 1
        nbytes = int(2 * rows.sum().item() * cfg.n_kv_heads * cfg.head_dim * 2)
        gbs = nbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"phase": "configs", "workload": cfg.name + "+append",
                          "dtype": str(cfg.dtype).split(".")[-1], "ms_per_call": round(ms, 5),
                          "value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / hbm, 4),
                          "peak": f"{hbm} GB/s ({peak_src} copy)"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer e2e measurement")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step directly instead of replaying a captured CUDA graph")
    ap.add_argument("--phase", choices=["all", "prefill", "decode", "configs"], default="all",
                    help="run only one timed phase (for profiling one kernel; the JSON line "
                         "then carries only that phase), or 'configs': one line per named "
                         "workload, single GPU")
    ap.add_argument("--workload", default=None,
                    choices=sorted(list(W.PREFILL_CONFIGS) + list(W.DECODE_CONFIGS)),
                    help="with --phase configs: time only this named workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.phase == "configs":
        if int(os.environ.get("RANK", "0")) == 0:
            run_configs(args)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, ws, local = replicas.init("nccl")
    try:
        line = run_ours(args, rank, ws, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        replicas.shutdown(ws)


if __name__ == "__main__":
    main()
