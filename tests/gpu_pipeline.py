"""Run the CUDA library on seeded synthetic inputs (test helper).

Builds device weights, the latent cache (contiguous or paged, with every row
that no sequence owns filled with NaN so masking bugs surface), runs the C-ABI
calls through ``gated_mla_b200`` and returns host copies of every output.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import synth


def metrics(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    return {"max_abs": float(np.max(np.abs(d))) if d.size else 0.0,
            "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)) if d.size else 0.0}


BF16_TOL = {"max_abs": 2e-2, "rel_l2": 1e-2}
F32_TOL = {"max_abs": 1e-4, "rel_l2": 1e-4}


def assert_close(got, ref, tol, what=""):
    m = metrics(got, ref)
    assert m["max_abs"] <= tol["max_abs"] and m["rel_l2"] <= tol["rel_l2"], f"{what}: {m} vs {tol}"
    return m


def _dt(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def make_model(inp, device="cuda"):
    from gated_mla_b200 import GatedMLA
    w = inp["workload"]
    dt = _dt(w)
    dev = lambda a, t=dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device, t)
    weights = {k: dev(inp.get(k)) for k in ("W_c", "W_kr", "W_q", "W_qr", "W_k", "W_v", "W_g", "W_o",
                                            "W_dq", "W_uq")}
    weights["b_g"] = dev(inp["b_g"], torch.float32)
    return GatedMLA(d_model=w.d_model, n_heads=w.n_heads, d_h=w.d_h, d_c=w.d_c, d_rope=w.d_rope,
                    gate_mode=w.gate_mode, softmax_scale=w.softmax_scale, rope_base=w.rope_base,
                    dtype=dt, weights=weights, d_cq=w.d_cq, gate_topk=w.gate_topk, cache_fp8=w.cache_fp8,
                    cache_scale=w.cache_scale)


def _filled(shape, fill, dt, device):
    if dt == torch.float8_e4m3fn:   # NaN is the code 0x7f, zero the code 0x00
        code = 0x7F if fill != fill else 0x00
        return torch.full(shape, code, dtype=torch.uint8, device=device).view(torch.float8_e4m3fn)
    return torch.full(shape, fill, dtype=dt, device=device)


def make_decode_cache(inp, device="cuda", paged=None, capacity=None, fill=float("nan")):
    """Latent cache holding each sequence's past rows (positions < L-1)."""
    from gated_mla_b200 import LatentCache
    w = inp["workload"]
    dt = _dt(w)
    lens = [int(L) for L in inp["lengths"]]
    B = w.batch
    paged = w.paged if paged is None else paged
    if w.cache_fp8:   # E4M3 codes of the stored values / cache_scale (exact: the values are on the grid)
        dt = torch.float8_e4m3fn
        scale = np.float32(w.cache_scale)
        inp = dict(inp, past=[r / scale for r in inp["past"]])
    if not paged:
        cap = capacity or max(1, max(lens))
        data = _filled((B, cap, w.row), fill, dt, device)
        for b, rows in enumerate(inp["past"]):
            if len(rows):
                data[b, :len(rows)] = torch.from_numpy(rows).to(device, dt)
        return LatentCache(data=data)
    ps = w.page_size
    npg = [max(1, math.ceil(L / ps)) for L in lens]
    total = sum(npg)
    perm = inp.get("page_perm")
    if perm is None or len(perm) != total:
        perm = np.random.default_rng(7).permutation(total)
    mpps = max(npg)
    bt = np.full((B, mpps), -1, dtype=np.int32)
    data = _filled((total, ps, w.row), fill, dt, device)
    k = 0
    for b in range(B):
        for p in range(npg[b]):
            bt[b, p] = perm[k]
            k += 1
        rows = inp["past"][b]
        for p in range(npg[b]):
            seg = rows[p * ps:(p + 1) * ps]
            if len(seg):
                data[bt[b, p], :len(seg)] = torch.from_numpy(seg).to(device, dt)
    return LatentCache(data=data, block_table=torch.from_numpy(bt).to(device))


def run_decode(inp, paged=None, device="cuda"):
    w = inp["workload"]
    model = make_model(inp, device)
    cache = make_decode_cache(inp, device, paged=paged)
    dt = _dt(w)
    B = w.batch
    lens = torch.tensor(inp["lengths"], dtype=torch.int32, device=device)
    x = torch.from_numpy(inp["x"]).to(device, dt)
    positions = (lens - 1).to(torch.int32)
    seq_ids = torch.arange(B, dtype=torch.int32, device=device)
    q, g = model.latent_project(x, positions, seq_ids, cache)
    o = model.decode(q, g, cache, lens)
    y = model.gate_out(o)
    model.sync_status()
    torch.cuda.synchronize()
    f = lambda t: t.float().cpu().numpy()
    return {"q": f(q), "glogit": f(g), "o": f(o), "y": f(y), "cache": cache, "model": model}


def run_prefill(inp, device="cuda"):
    from gated_mla_b200 import LatentCache
    w = inp["workload"]
    model = make_model(inp, device)
    dt = _dt(w)
    lens = [int(L) for L in inp["lengths"]]
    B = len(lens)
    cap = max(lens)
    data = torch.full((B, cap, w.row), float("nan"), dtype=dt, device=device)
    cache = LatentCache(data=data)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=device)
    positions = torch.from_numpy(np.concatenate([np.arange(L) for L in lens]).astype(np.int32)).to(device)
    seq_ids = torch.from_numpy(np.concatenate([np.full(L, b) for b, L in enumerate(lens)]).astype(np.int32)).to(device)
    x = torch.from_numpy(inp["x"]).to(device, dt)
    q, g = model.latent_project(x, positions, seq_ids, cache)
    o = model.prefill(q, g, cache, cu, cap)
    y = model.gate_out(o)
    model.sync_status()
    torch.cuda.synchronize()
    f = lambda t: t.float().cpu().numpy()
    return {"q": f(q), "glogit": f(g), "o": f(o), "y": f(y), "cache": cache, "model": model}


def small_decode(name, batch, lens, **kw):
    w = synth.workload(name, batch=batch, **kw)
    return synth.generate(w, seed=0, lengths=np.array(lens))
