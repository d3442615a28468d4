#!/usr/bin/env python
"""Benchmark of the Gated MLA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole decode path over the batch-32 decode workload
(d_model 2048, 16 heads, d_h 128, d_c 512, NoPE, per-channel gate, cache
lengths uniform in [1024, 8192], seed 0): gmla_latent_project (writes each
sequence's new latent row) -> gmla_decode (absorbed split-K attention, W_v
and gate) -> gmla_gate_out (W_o). The metric is latent-cache bytes read per
step over the step time (GB/s). Inputs are synthetic, drawn by ``synth``.

Timing: W untimed warm-up steps; then K steps, each replayed from a CUDA
graph between CUDA events on the launching stream, with a 256 MiB memset
flushing L2 before every step (outside the events); barrier + synchronize on
both sides; the max over ranks of the summed step times. Under torchrun every
rank runs its own replica of the workload (weak scaling; no data-path
collective). Rank 0 prints one JSON line.

``--impl reference`` times the fp64 oracle (the CPU restatement of the method
that the tests check the library against) on this machine's host cores, each
step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Gated-MLA decode latent-cache GB/s (latent_project + decode + gate_out step)"
UNIT = "GB/s"
WORKLOAD = "decode_b32"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def src_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


DECODE_SRC = ["gated_mla_b200/csrc/decode_tc.cu", "gated_mla_b200/csrc/ptx.cuh", "gated_mla_b200/csrc/common.cuh"]


def ncu_traffic():
    """DRAM bytes per decode_attn launch from the committed ncu summary, if it
    was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "decode_attn_decode_b32.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("src_sha") != src_hash(DECODE_SRC):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"gmla_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                                 "active": parts[4], "hw": parts[5], "hwt": parts[6], "swt": parts[7],
                                 "pcap": parts[8]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                            ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(inp, seconds: float, start: int = 0):
    """Run the fp64 oracle's decode over whole sequences from `start` until the
    time budget is spent. Returns (latent bytes processed, seconds, sequences)."""
    import oracle
    w = inp["workload"]
    p = oracle.params(inp)
    row_bytes = w.row * 2
    done, nbytes = [], 0
    t0 = time.perf_counter()
    b = start
    while True:
        oracle.decode(p, inp["x"], inp["past"], seqs=[b % w.batch])
        nbytes += int(inp["lengths"][b % w.batch]) * row_bytes
        done.append(b % w.batch)
        b += 1
        if time.perf_counter() - t0 >= seconds or len(done) >= w.batch:
            break
    return nbytes, time.perf_counter() - t0, done


def run_reference(args):
    import synth
    if int(os.environ.get("RANK", "0")) != 0:
        return
    w = synth.workload(WORKLOAD)
    inp = synth.generate(w, seed=0)
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(inp, per_step, start=i)
    tot_b, tot_s, seqs = 0, 0.0, []
    for i in range(args.steps):
        nb, s, d = oracle_sample(inp, per_step, start=args.warmup + i)
        tot_b += nb
        tot_s += s
        seqs += d
    value = tot_b / tot_s / 1e9
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, inp),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(seqs)} whole sequences over {args.steps} steps, fp64 explicit form "
                                   f"(per-head K/V rebuilt from latents), numpy/BLAS"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, inp):
    lens = inp["lengths"]
    return {"workload": f"{WORKLOAD}: batch {w.batch} decode, d_model {w.d_model}, H {w.n_heads}, d_h {w.d_h}, "
                        f"d_c {w.d_c}, NoPE, per-channel gate, lengths uniform[{w.len_lo},{w.len_hi}] seed 0",
            "batch": w.batch, "d_model": w.d_model, "n_heads": w.n_heads, "d_h": w.d_h, "d_c": w.d_c,
            "d_rope": w.d_rope, "sum_len": int(lens.sum()),
            "latent_bytes_per_step": int(lens.sum()) * w.row * 2,
            "l2": "flushed before every timed step (256 MiB memset, outside the events)",
            "parallelism": "replica per GPU"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    from gated_mla_b200 import _lib
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from gpu_pipeline import make_decode_cache, make_model

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    w = synth.workload(WORKLOAD)
    inp = synth.generate(w, seed=0)
    lens_np = inp["lengths"]
    latent_bytes = int(lens_np.sum()) * w.row * 2
    model = make_model(inp, device=dev)
    cache = make_decode_cache(inp, device=dev, paged=False, fill=0.0)
    B = w.batch
    x = torch.from_numpy(inp["x"]).to(dev, torch.bfloat16)
    seq_lens = torch.tensor(lens_np, dtype=torch.int32, device=dev)
    positions = (seq_lens - 1).contiguous()
    seq_ids = torch.arange(B, dtype=torch.int32, device=dev)
    q = torch.empty(B, w.n_heads, w.d_h + w.d_rope, dtype=torch.bfloat16, device=dev)
    g = torch.empty(B, w.gate_width, dtype=torch.float32, device=dev)
    o = torch.empty(B, w.n_heads * w.d_h, dtype=torch.bfloat16, device=dev)
    y = torch.empty(B, w.d_model, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def step():
        model.latent_project(x, positions, seq_ids, cache, q_out=q, gate_logits=g)
        model.decode(q, g, cache, seq_lens, o_out=o)
        model.gate_out(o, y_out=y)

    # eager warm-up (also sizes the workspaces) and launches per step
    step()
    torch.cuda.synchronize()
    model.sync_status()
    n0 = _lib.gmla_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = _lib.gmla_launch_count() - n0

    # capture one step in a CUDA graph
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    model.sync_status()

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        for i in range(K):
            flush.zero_()
            ev0[i].record(stream)
            graph.replay()
            ev1[i].record(stream)
        torch.cuda.synchronize()
        # keep the GPU busy long enough for the clock sampler to see it
        extra = 0
        while time.perf_counter() - t_wall < 1.0 and extra < 20000:
            flush.zero_()
            graph.replay()
            extra += 1
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    times = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    total_ms = sum(times)
    tt = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    max_total_ms = float(tt.item())
    value = world * latent_bytes * K / (max_total_ms / 1e3) / 1e9
    model.sync_status()

    # dominant kernel: per-launch CUDA events on the launching stream. The step is
    # captured with the library's event records inside the graph, so the records
    # bracket the kernel nodes with no host time in between; each replay
    # overwrites them and they are read after it.
    _lib.gmla_profile_enable(1)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        step()
    torch.cuda.synchronize()
    n_rec = _lib.gmla_profile_count()
    by = {}
    for _ in range(K):
        flush.zero_()
        pgraph.replay()
        torch.cuda.synchronize()
        for i in range(n_rec):
            name, ms = _lib.gmla_profile_get(i)
            by.setdefault(name, []).append(ms)
    _lib.gmla_profile_enable(0)
    del pgraph
    attn_ms = statistics.mean(by["decode_attn"])
    achieved = latent_bytes / (attn_ms / 1e3) / 1e9
    pk = peaks()
    kernel_ms = {k: statistics.mean(v) * (len(v) // K) for k, v in by.items()}   # per step

    # end to end through the public API, host buffers (pinned), copies inside the events
    x_h = torch.from_numpy(inp["x"]).to(torch.bfloat16).pin_memory()
    lens_h = torch.tensor(lens_np, dtype=torch.int32).pin_memory()
    pos_h = (lens_h - 1).pin_memory()
    ids_h = torch.arange(B, dtype=torch.int32).pin_memory()
    y_h = torch.empty(B, w.d_model, dtype=torch.bfloat16).pin_memory()
    x_d, lens_d, pos_d, ids_d = (torch.empty_like(t, device=dev) for t in (x_h, lens_h, pos_h, ids_h))
    h2d = sum(t.numel() * t.element_size() for t in (x_h, lens_h, pos_h, ids_h))
    d2h = y_h.numel() * y_h.element_size()

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        lens_d.copy_(lens_h, non_blocking=True)
        pos_d.copy_(pos_h, non_blocking=True)
        ids_d.copy_(ids_h, non_blocking=True)
        yy = model.decode_step(x_d, cache, lens_d, pos_d, ids_d)
        y_h.copy_(yy, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        e0[i].record(stream)
        e2e_step()
        e1[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(e0, e1))
    et = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(et, op=dist.ReduceOp.MAX)
    e2e_value = world * latent_bytes * K / (float(et.item()) / 1e3) / 1e9
    model.sync_status()

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        nb, sec, seqs = oracle_sample(inp, args.cpu_seconds)
        cpu = {"value": nb / sec / 1e9, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(seqs)} of {B} sequences ({nb / 1e6:.1f} MB of latent rows) of the same workload, "
                         f"fp64 explicit form, numpy/BLAS, {sec:.1f} s"}
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": max_total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": dict(config_dict(w, inp), cuda_graph=True),
            "roofline": {"bound": "hbm", "kernel": "decode_attn", "achieved": achieved, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "peak_source": pk["source"],
                         "traffic": ncu_traffic(), "launch_ms": attn_ms,
                         "algorithmic_bytes_per_launch": latent_bytes},
            "kernel_ms": kernel_ms,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches_per_step * K),
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        del graph
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
