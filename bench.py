#!/usr/bin/env python
"""Benchmark of the Gated MLA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--prefill-workload NAME|none]

One run measures two workloads on the same GPU, one after the other:

* the JSON line itself: the long-context decode (batch 8 x 131072 cached rows,
  d_model 7168, 128 heads, d_h 128, d_c 512 + decoupled RoPE 64, per-channel
  gate, seed 0), the largest decode workload. A decode step is
  gmla_latent_project (writes each sequence's new latent row) -> gmla_decode
  (absorbed split-K attention, W_v and gate) -> gmla_gate_out (W_o); its metric
  is latent-cache bytes read per step over the step time (GB/s);
* its ``prefill`` object: the batch-4 x 4096 causal prefill (d_model 7168,
  64 heads), a step being gmla_latent_project -> gmla_prefill -> gmla_gate_out
  over whole prompts, with explicit-form algorithmic FLOPs per second (TFLOP/s).

``--workload`` picks another decode (or prefill) workload for the line;
``--prefill-workload none`` leaves the prefill object out. Inputs are
synthetic, drawn by ``synth``.

Timing: W untimed warm-up steps; then K steps, each replayed from a CUDA
graph between CUDA events on the launching stream, with L2 flushed before
every step by a 256 MiB memset and a read of it (outside the events); barrier
+ synchronize on both sides; the max over ranks of the summed step times.
Under torchrun every rank runs its own replica of the workload (weak scaling;
no data-path collective). Rank 0 prints one JSON line.

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

DECODE_METRIC = "Gated-MLA decode latent-cache GB/s (latent_project + decode + gate_out step)"
PREFILL_METRIC = "Gated-MLA prefill TFLOP/s (latent_project + prefill + gate_out step, explicit-form FLOPs)"
DEFAULT_WORKLOAD = "decode_long_rope"
DEFAULT_PREFILL = "prefill_b4_s4096"
WORKLOAD_NAMES = ["decode_b32", "decode_long_rope", "decode_paged_head", "prefill_b4_s4096",
                  "prefill_b1_s4096_h16", "tiny_prefill_f32", "decode_long_rope_qc", "prefill_b4_s4096_qc",
                  "decode_paged_head_top8", "decode_long_rope_top32", "decode_long_rope_b2", "decode_b32_fp8",
                  "decode_paged_head_fp8"]
# Denominators used when no measured peaks file is present: a B200's HBM copy
# bandwidth (GB/s), its dense bf16 GEMM throughput as a short burst, and the
# same GEMM held for seconds under the 1 kW power cap (TFLOP/s).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}



def flush_l2(buf):
    """Evicts L2 between timed steps: a write of a buffer twice the size of L2,
    then a read of it, so the next step finds none of its inputs cached and no
    dirty line left to write back on its time."""
    buf.zero_()
    buf.sum()

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_NAMES)
    ap.add_argument("--prefill-workload", default=DEFAULT_PREFILL, choices=WORKLOAD_NAMES + ["none"],
                    help="prefill workload measured in the same run (its own object in the line)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cp-shares", type=int, default=1,
                    help="decode only: run the step as a context-parallel decode of this many position "
                         "ranges, all on this GPU (gmla_decode_partial per range, then gmla_decode_merge)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def src_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


DECODE_SRC = ["gated_mla_b200/csrc/decode_tc.cu", "gated_mla_b200/csrc/ptx.cuh", "gated_mla_b200/csrc/common.cuh"]
KERNEL_SRC = {
    "decode_attn": DECODE_SRC,
    "prefill_attn": ["gated_mla_b200/csrc/prefill_tc.cu", "gated_mla_b200/csrc/ptx.cuh",
                     "gated_mla_b200/csrc/common.cuh"],
    "gemm_project": ["gated_mla_b200/csrc/gemm_tc.cu", "gated_mla_b200/csrc/ptx.cuh",
                     "gated_mla_b200/csrc/common.cuh"],
}


def ncu_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu summary profiles/<kernel>_<workload>.json, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    if not os.path.exists(p) or kernel not in KERNEL_SRC:
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("src_sha") != src_hash(KERNEL_SRC[kernel]):
        return None
    return d.get("dram_bytes_per_launch")


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


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
# workload accounting
# ---------------------------------------------------------------------------

def cache_elem_bytes(w):
    """Bytes per cached element: 1 for an FP8 latent cache, else the dtype's."""
    return 1 if w.cache_fp8 else (2 if w.dtype == "bf16" else 4)


def prefill_flops(w, lengths):
    """Explicit-form algorithmic FLOPs of one prefill step, per kernel."""
    T = int(sum(lengths))
    H, dh, dc, dr, dm = w.n_heads, w.d_h, w.d_c, w.d_rope, w.d_model
    pairs = sum(int(L) * (int(L) + 1) // 2 for L in lengths)
    out = {}
    if w.d_cq:   # low-rank query: x -> [c | k^R | c^Q | g], then c^Q -> [q | q^R]
        out["gemm_project"] = 2.0 * T * dm * (dc + dr + w.d_cq + w.gate_width)
        out["gemm_query_up"] = 2.0 * T * w.d_cq * (H * dh + H * dr)
    else:
        out["gemm_project"] = 2.0 * T * dm * (dc + dr + H * dh + H * dr + w.gate_width)
    out.update({"gemm_kv": 2.0 * T * dc * 2 * H * dh,
                "prefill_attn": 4.0 * (dh + dr) * H * pairs,
                "gemm_out": 2.0 * T * H * dh * dm})
    return out


def config_dict(w, inp):
    lens = inp["lengths"]
    if w.mode == "decode":
        desc = (f"{w.name}: batch {w.batch} decode, d_model {w.d_model}, H {w.n_heads}, d_h {w.d_h}, d_c {w.d_c}"
                + (f" + RoPE {w.d_rope}" if w.d_rope else ", NoPE")
                + (", paged (page 64)" if w.paged else "")
                + f", {w.gate_mode} gate, lengths {w.len_law}[{w.len_lo},{w.len_hi}]"
                + (f", low-rank query d_cq {w.d_cq}" if w.d_cq else "")
                + (f", top-{w.gate_topk} of {w.n_heads} heads" if w.gate_mode == "head_topk" else "")
                + (f", FP8 E4M3 cache (scale {w.cache_scale})" if w.cache_fp8 else "") + ", seed 0")
        extra = {"sum_len": int(lens.sum()), "latent_bytes_per_step": int(lens.sum()) * w.row * cache_elem_bytes(w)}
    else:
        desc = (f"{w.name}: batch {w.batch} x {w.seq_len} causal prefill, d_model {w.d_model}, H {w.n_heads}, "
                f"d_h {w.d_h}, d_c {w.d_c}, " + (f"RoPE {w.d_rope}" if w.d_rope else "NoPE")
                + f", {w.gate_mode} gate" + (f", low-rank query d_cq {w.d_cq}" if w.d_cq else "")
                + f", {w.dtype}, seed 0")
        extra = {"flops_per_step": sum(prefill_flops(w, lens).values())}
    return dict({"workload": desc, "batch": w.batch, "d_model": w.d_model, "n_heads": w.n_heads, "d_h": w.d_h,
                 "d_c": w.d_c, "d_rope": w.d_rope, "d_cq": w.d_cq,
                 "l2": "flushed before every timed step (256 MiB memset then a read of it, outside the events)",
                 "parallelism": "replica per GPU"}, **extra)


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
    """Run the fp64 oracle on a bounded sample of the workload. Decode: whole
    sequences from `start` until the time budget is spent (work = latent bytes
    read). Prefill: a prefix of sequence 0 (same dimensions, shorter prompt;
    work = its algorithmic FLOPs). Returns (work, seconds, description)."""
    import oracle
    w = inp["workload"]
    p = oracle.params(inp)
    t0 = time.perf_counter()
    if w.mode == "decode":
        # units of (sequence, 8 heads), sequences in turn (wrapping around the
        # batch) until the time budget is spent; work = that share of the
        # sequence's latent bytes
        units, nbytes, b = 0, 0.0, start
        hc = min(8, w.n_heads)
        while time.perf_counter() - t0 < seconds:
            seq = b % w.batch
            for h0 in range(0, w.n_heads, hc):
                heads = list(range(h0, min(w.n_heads, h0 + hc)))
                oracle.decode(p, inp["x"], inp["past"], seqs=[seq], heads=heads)
                nbytes += int(inp["lengths"][seq]) * w.row * cache_elem_bytes(w) * len(heads) / w.n_heads
                units += 1
                if time.perf_counter() - t0 >= seconds:
                    break
            b += 1
        return nbytes, time.perf_counter() - t0, f"{units} (sequence, {hc}-head) units from {b - start} sequences"
    # prefill: prompts of the first min(L, 512) tokens of successive sequences
    # until the time budget is spent
    flops, n, b = 0.0, 0, start
    while time.perf_counter() - t0 < seconds:
        seq = b % w.batch
        off = int(sum(int(L) for L in inp["lengths"][:seq]))
        S = min(int(inp["lengths"][seq]), 512)
        oracle.prefill(p, inp["x"][off:off + S], [S])
        flops += sum(prefill_flops(w, [S]).values())
        n += 1
        b += 1
    return flops, time.perf_counter() - t0, f"{n} prefills of the first min(L, 512) tokens of successive sequences"


def work_unit(w):
    return (1e9, "GB/s") if w.mode == "decode" else (1e12, "TFLOP/s")


def job_throughput(local_ms, world, units_per_step, steps, scale, dist=None, device="cpu"):
    """Whole-job throughput of `world` replicas: every rank processed `units_per_step`
    units per step for `steps` steps; the job time is the slowest rank's (an
    all-reduce MAX of the ranks' own device times when world > 1). Returns
    (value in units/s / scale, max_ms)."""
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    return world * units_per_step * steps / (max_ms / 1e3) / scale, max_ms


def reference_fields(name, args, per_step):
    """The oracle timed on a bounded sample of workload `name` per step."""
    import synth
    w = synth.workload(name)
    inp = synth.generate(w, seed=0)
    scale, unit = work_unit(w)
    for i in range(args.warmup):
        oracle_sample(inp, per_step, start=i)
    tot_w, tot_s, desc = 0.0, 0.0, ""
    for i in range(args.steps):
        wk, sec, desc = oracle_sample(inp, per_step, start=args.warmup + i)
        tot_w += wk
        tot_s += sec
    value = tot_w / tot_s / scale
    return {
        "metric": DECODE_METRIC if w.mode == "decode" else PREFILL_METRIC,
        "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_dict(w, inp),
        "cpu_baseline": {"value": value, "unit": unit, "cores": blas_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": f"per step: {desc}; fp64 explicit form (per-head K/V rebuilt from "
                                   f"latents), numpy/BLAS"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args):
    import synth
    if int(os.environ.get("RANK", "0")) != 0:
        return
    with_prefill = synth.workload(args.workload).mode == "decode" and args.prefill_workload != "none"
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    if with_prefill:
        per_step /= 2
    line = dict(impl="reference", **reference_fields(args.workload, args, per_step))
    if with_prefill:
        line["prefill"] = reference_fields(args.prefill_workload, args, per_step)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class DecodeRunner:
    def __init__(self, inp, dev, cp_shares=1):
        import torch
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from gpu_pipeline import make_decode_cache, make_model
        w = self.w = inp["workload"]
        self.dev = dev
        self.model = make_model(inp, device=dev)
        self.cache = make_decode_cache(inp, device=dev, fill=0.0)
        B = w.batch
        self.x = torch.from_numpy(inp["x"]).to(dev, torch.bfloat16)
        self.seq_lens = torch.tensor(inp["lengths"], dtype=torch.int32, device=dev)
        self.positions = (self.seq_lens - 1).contiguous()
        self.seq_ids = torch.arange(B, dtype=torch.int32, device=dev)
        self.q = torch.empty(B, w.n_heads, w.d_h + w.d_rope, dtype=torch.bfloat16, device=dev)
        self.g = torch.empty(B, w.gate_width, dtype=torch.float32, device=dev)
        self.o = torch.empty(B, w.n_heads * w.d_h, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(B, w.d_model, dtype=torch.bfloat16, device=dev)
        self.work = float(inp["lengths"].sum()) * w.row * cache_elem_bytes(w)   # latent bytes per step
        self.dominant = "decode_attn"
        self.kernel_work = {"decode_attn": self.work}
        # host copies for the end-to-end leg
        self.host_in = [t.cpu().pin_memory() for t in (self.x, self.seq_lens, self.positions, self.seq_ids)]
        self.dev_in = [torch.empty_like(t) for t in (self.x, self.seq_lens, self.positions, self.seq_ids)]
        self.y_host = torch.empty(B, w.d_model, dtype=torch.bfloat16).pin_memory()
        # context-parallel emulation: the ranges of every share, run one after another here
        self.cp = cp_shares
        if cp_shares > 1:
            from gated_mla_b200 import context_parallel as cpm
            self.cpm = cpm
            lens = [int(n) for n in inp["lengths"]]
            self.shares = [tuple(t.to(dev) for t in cpm.shard_table(lens, cp_shares, r)) for r in range(cp_shares)]
            self.parts = torch.empty(cp_shares, B, w.n_heads, w.d_c + cpm.PARTIAL_PAD, dtype=torch.float32,
                                     device=dev)

    def step(self):
        m = self.model
        m.latent_project(self.x, self.positions, self.seq_ids, self.cache, q_out=self.q, gate_logits=self.g)
        if self.cp > 1:
            for r, (starts, ends) in enumerate(self.shares):
                self.cpm.decode_partial(m, self.q, self.g, self.cache, starts, ends, out=self.parts[r])
            self.cpm.decode_merge(m, self.parts, self.g, out=self.o)
        else:
            m.decode(self.q, self.g, self.cache, self.seq_lens, o_out=self.o)
        m.gate_out(self.o, y_out=self.y)

    def e2e_step(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)
        x, lens, pos, ids = self.dev_in
        yy = self.model.decode_step(x, self.cache, lens, pos, ids)
        self.y_host.copy_(yy, non_blocking=True)


class PrefillRunner:
    def __init__(self, inp, dev):
        import numpy as np
        import torch
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from gpu_pipeline import make_model
        from gated_mla_b200 import LatentCache
        w = self.w = inp["workload"]
        self.dev = dev
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.model = make_model(inp, device=dev)
        lens = [int(L) for L in inp["lengths"]]
        self.max_len = max(lens)
        self.cache = LatentCache(data=torch.zeros(len(lens), self.max_len, w.row, dtype=dt, device=dev))
        self.x = torch.from_numpy(inp["x"]).to(dev, dt)
        self.cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
        self.positions = torch.from_numpy(np.concatenate([np.arange(L) for L in lens]).astype(np.int32)).to(dev)
        self.seq_ids = torch.from_numpy(
            np.concatenate([np.full(L, b) for b, L in enumerate(lens)]).astype(np.int32)).to(dev)
        T = self.x.shape[0]
        self.q = torch.empty(T, w.n_heads, w.d_h + w.d_rope, dtype=dt, device=dev)
        self.g = torch.empty(T, w.gate_width, dtype=torch.float32, device=dev)
        self.o = torch.empty(T, w.n_heads * w.d_h, dtype=dt, device=dev)
        self.y = torch.empty(T, w.d_model, dtype=dt, device=dev)
        self.kernel_work = prefill_flops(w, lens)
        self.work = sum(self.kernel_work.values())
        self.dominant = None   # picked from the measured kernel times
        self.host_in = [t.cpu().pin_memory() for t in (self.x, self.positions, self.seq_ids, self.cu)]
        self.dev_in = [torch.empty_like(t) for t in (self.x, self.positions, self.seq_ids, self.cu)]
        self.y_host = torch.empty(T, w.d_model, dtype=dt).pin_memory()

    def step(self):
        m = self.model
        m.latent_project(self.x, self.positions, self.seq_ids, self.cache, q_out=self.q, gate_logits=self.g)
        m.prefill(self.q, self.g, self.cache, self.cu, self.max_len, o_out=self.o)
        m.gate_out(self.o, y_out=self.y)

    def e2e_step(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)
        x, pos, ids, cu = self.dev_in
        yy = self.model.prefill_step(x, self.cache, cu, self.max_len, pos, ids)
        self.y_host.copy_(yy, non_blocking=True)


def measure(name, args, world, rank, dev, dist, cpu_leg):
    """Time one workload as described in the module docstring; returns the
    fields of its JSON line (or object)."""
    import torch

    import synth
    from gated_mla_b200 import _lib

    w = synth.workload(name)
    inp = synth.generate(w, seed=0)
    run = DecodeRunner(inp, dev, args.cp_shares) if w.mode == "decode" else PrefillRunner(inp, dev)
    scale, unit = work_unit(w)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    # eager warm-up (also sizes the workspaces) and launches per step
    run.step()
    torch.cuda.synchronize()
    run.model.sync_status()
    n0 = _lib.gmla_launch_count()
    run.step()
    torch.cuda.synchronize()
    launches_per_step = _lib.gmla_launch_count() - n0

    # capture one step in a CUDA graph
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run.step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run.step()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        flush_l2(flush)
        graph.replay()
    torch.cuda.synchronize()
    run.model.sync_status()

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_wall = time.perf_counter()
        for i in range(K):
            flush_l2(flush)
            ev0[i].record(stream)
            graph.replay()
            ev1[i].record(stream)
        torch.cuda.synchronize()
        # keep the GPU busy long enough for the clock sampler to see it
        extra = 0
        while time.perf_counter() - t_wall < 1.0 and extra < 20000:
            flush_l2(flush)
            graph.replay()
            extra += 1
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))
    value, max_total_ms = job_throughput(total_ms, world, run.work, K, scale, dist, dev)
    run.model.sync_status()

    # per-kernel times: the step captured with the library's event records inside
    # the graph (no host time between a record and its kernel); each replay
    # overwrites the records and they are read after it
    _lib.gmla_profile_enable(1)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        run.step()
    torch.cuda.synchronize()
    n_rec = _lib.gmla_profile_count()
    by = {}
    for _ in range(K):
        flush_l2(flush)
        pgraph.replay()
        torch.cuda.synchronize()
        for i in range(n_rec):
            kname, ms = _lib.gmla_profile_get(i)
            by.setdefault(kname, []).append(ms)
    _lib.gmla_profile_enable(0)
    del pgraph
    kernel_ms = {k: statistics.mean(v) * (len(v) // K) for k, v in by.items()}   # per step
    pk = peaks()
    if w.mode == "decode":
        dom = "decode_attn"
        achieved = run.kernel_work[dom] / (kernel_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "peak_source": pk["source"],
                "traffic": ncu_traffic(dom, name),
                "launch_ms": kernel_ms[dom], "algorithmic_bytes_per_launch": run.kernel_work[dom]}
    else:
        per = {k: v for k, v in run.kernel_work.items() if k in kernel_ms}
        if not per:   # fp32 path: its kernels are not split the same way; use the whole step
            per = {"step": run.work}
            kernel_ms["step"] = max_total_ms / K
        dom = max(per, key=lambda k: kernel_ms[k])
        achieved = per[dom] / (kernel_ms[dom] / 1e3) / 1e12
        # the prefill step runs for seconds back to back under the power cap:
        # the sustained bf16 figure is the denominator (the burst one is kept beside it)
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops_sustained"],
                "peak_source": pk["source"] + " sustained", "peak_burst": pk["bf16_tflops"],
                "frac_of_burst": achieved / pk["bf16_tflops"],
                "traffic": ncu_traffic(dom, name), "launch_ms": kernel_ms[dom],
                "algorithmic_flops_per_launch": per[dom],
                "per_kernel_tflops": {k: per[k] / (kernel_ms[k] / 1e3) / 1e12 for k in per},
                "step_frac_of_sustained": value / pk["bf16_tflops_sustained"]}

    # end to end through the public API, host buffers (pinned), copies inside the events
    h2d = sum(t.numel() * t.element_size() for t in run.host_in)
    d2h = run.y_host.numel() * run.y_host.element_size()
    for _ in range(3):
        run.e2e_step()
    torch.cuda.synchronize()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for i in range(K):
        flush_l2(flush)
        e0[i].record(stream)
        run.e2e_step()
        e1[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(e0, e1))
    e2e_value, _ = job_throughput(e2e_ms, world, run.work, K, scale, dist, dev)
    run.model.sync_status()

    cpu = None
    if cpu_leg:
        wk, sec, desc = oracle_sample(inp, args.cpu_seconds)
        cpu = {"value": wk / sec / scale, "unit": unit, "cores": blas_threads(), "cpu_model": cpu_model(),
               "kind": "oracle",
               "sample": f"{desc} of the same workload, fp64 explicit form, numpy/BLAS, {sec:.1f} s"}
    out = {
        "metric": DECODE_METRIC if w.mode == "decode" else PREFILL_METRIC, "value": value, "unit": unit,
        "ms_per_step": max_total_ms / K,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "config": dict(config_dict(w, inp), cuda_graph=True,
                       **({"context_parallel_shares_on_one_gpu": args.cp_shares}
                          if w.mode == "decode" and args.cp_shares > 1 else {})),
        "roofline": roof, "kernel_ms": kernel_ms, "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches_per_step * K),
        "clocks": clk.summary(),
    }
    del graph
    del run
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    cpu_leg = rank == 0 and not args.no_cpu_baseline
    main_fields = measure(args.workload, args, world, rank, dev, dist, cpu_leg)
    pre = None
    import synth
    if synth.workload(args.workload).mode == "decode" and args.prefill_workload != "none":
        pre = measure(args.prefill_workload, args, world, rank, dev, dist, cpu_leg)
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {"metric": main_fields.pop("metric"), "value": main_fields.pop("value"),
                "unit": main_fields.pop("unit"), "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": main_fields.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "data": "synthetic"}
        line.update(main_fields)
        if pre is not None:
            line["prefill"] = dict(pre, n_gpus=world, steps=args.steps, warmup=args.warmup,
                                   higher_is_better=True, scaling="weak", vs_baseline=None, data="synthetic")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
