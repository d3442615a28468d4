"""Seeded synthetic inputs for the Gated MLA hot path.

This module is shared by the GPU path's tests/benchmark and by the oracle's
tests. It holds no arithmetic of the method itself: it only draws random
numbers, rounds them to bfloat16 when the workload is bf16, and lays out
lengths and page tables. Every stored cache row (latent ``c_s`` and, where the
workload has one, the decoupled RoPE key ``k^R_s``) is a plain Gaussian draw:
a rotated Gaussian vector has the same law as an unrotated one, so no rotation
is applied here.

Workloads (sizes as named in the problem statement of Gated MLA):

* ``tiny_prefill_f32``   batch 1, seq 64, d_model 256, H 4, d_h 64, d_c 64, NoPE, fp32.
* ``decode_b32``         batch 32 decode, d_model 2048, H 16, d_h 128, d_c 512,
                         lengths uniform in [1024, 8192], bf16.
* ``prefill_b4_s4096``   batch 4, seq 4096, d_model 7168, H 64, d_h 128, d_c 512,
                         gate bias N(0, 2), bf16.
* ``prefill_b1_s4096_h16`` batch 1, seq 4096, d_model 2048, H 16 (else as prefill_b4_s4096):
  a reduced prefill for full ncu captures.
* ``decode_long_rope``   batch 8, length 131072, d_model 7168, H 128, d_h 128,
                         d_c 512, decoupled RoPE d_R 64 (base 10000), bf16.
* ``decode_paged_head``  batch 64 paged (page 64), lengths log-uniform in
                         [256, 32768], d_model 4096, H 32, d_h 128, d_c 512,
                         per-head gate with bias, bf16.
* ``decode_long_rope_qc``, ``prefill_b4_s4096_qc``: the long-context decode
                         and the batch-4 prefill with a low-rank query,
                         d_cq 1536.
* ``decode_b32_fp8``, ``decode_paged_head_fp8``: the batch-32 and the paged decode
                         over an FP8 E4M3 latent cache (one scale, 1/64).
* ``decode_paged_head_top8``, ``decode_long_rope_top32``: the paged decode and
                         the long-context decode with hard top-k per-head
                         gates (8 of 32, 32 of 128 heads).

Drawing order is fixed: x, W_c, W_kr, W_q (or W_dq, W_uq with a compressed
query), W_qr, W_k, W_v, W_g, b_g, W_o, lengths, page permutation, cache rows.
Weights are N(0, 1/fan_in).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "generate", "bf16_round", "e4m3_round",
           "bf16_bits", "bits_to_f32"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str               # "prefill" or "decode"
    dtype: str              # "f32" or "bf16"
    batch: int
    d_model: int
    n_heads: int
    d_h: int
    d_c: int
    d_rope: int = 0         # 0 = NoPE
    rope_base: float = 10000.0
    gate_mode: str = "channel"   # "channel", or per head: "head", "head_topk", "head_binary", "head_ternary"
    gate_topk: int = 0           # k of "head_topk"
    gate_bias: bool = False
    gate_bias_var: float = 2.0
    seq_len: int = 0        # prefill: tokens per sequence
    len_law: str = "fixed"  # decode: "fixed", "uniform", "loguniform"
    len_lo: int = 1
    len_hi: int = 1
    paged: bool = False
    page_size: int = 64
    d_cq: int = 0           # query low-rank compression width; 0 = full-rank query
    cache_fp8: bool = False  # FP8 E4M3 latent cache with one fp32 scale
    cache_scale: float = 1.0 / 64.0

    @property
    def softmax_scale(self) -> float:
        # 1/sqrt(d_h) over the content key; with a decoupled RoPE key the
        # score is over the concatenated key [k; k^R] of d_h + d_R dims.
        return 1.0 / math.sqrt(self.d_h + self.d_rope)

    @property
    def gate_width(self) -> int:
        return self.n_heads * self.d_h if self.gate_mode == "channel" else self.n_heads

    @property
    def row(self) -> int:
        """Cached elements per token: d_c + d_R."""
        return self.d_c + self.d_rope

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_prefill_f32": Workload(
        name="tiny_prefill_f32", mode="prefill", dtype="f32", batch=1, seq_len=64,
        d_model=256, n_heads=4, d_h=64, d_c=64),
    "decode_b32": Workload(
        name="decode_b32", mode="decode", dtype="bf16", batch=32, d_model=2048,
        n_heads=16, d_h=128, d_c=512, len_law="uniform", len_lo=1024, len_hi=8192),
    "prefill_b4_s4096": Workload(
        name="prefill_b4_s4096", mode="prefill", dtype="bf16", batch=4, seq_len=4096,
        d_model=7168, n_heads=64, d_h=128, d_c=512, gate_bias=True),
    # a reduced prefill (one sequence, 16 heads) that a full ncu capture can replay quickly
    "prefill_b1_s4096_h16": Workload(
        name="prefill_b1_s4096_h16", mode="prefill", dtype="bf16", batch=1, seq_len=4096,
        d_model=2048, n_heads=16, d_h=128, d_c=512, gate_bias=True),
    "decode_long_rope": Workload(
        name="decode_long_rope", mode="decode", dtype="bf16", batch=8, d_model=7168,
        n_heads=128, d_h=128, d_c=512, d_rope=64, rope_base=10000.0,
        len_law="fixed", len_lo=131072, len_hi=131072),
    # the long-context decode with 2 sequences instead of 8 (0.3 GB of cache), for ncu captures
    "decode_long_rope_b2": Workload(
        name="decode_long_rope_b2", mode="decode", dtype="bf16", batch=2, d_model=7168,
        n_heads=128, d_h=128, d_c=512, d_rope=64, rope_base=10000.0,
        len_law="fixed", len_lo=131072, len_hi=131072),
    "decode_paged_head": Workload(
        name="decode_paged_head", mode="decode", dtype="bf16", batch=64, d_model=4096,
        n_heads=32, d_h=128, d_c=512, gate_mode="head", gate_bias=True,
        len_law="loguniform", len_lo=256, len_hi=32768, paged=True, page_size=64),
    # the long-context decode and the batch-4 prefill with a low-rank query of
    # 1536 dims (the pages give the form, not a width)
    "decode_long_rope_qc": Workload(
        name="decode_long_rope_qc", mode="decode", dtype="bf16", batch=8, d_model=7168,
        n_heads=128, d_h=128, d_c=512, d_rope=64, rope_base=10000.0,
        len_law="fixed", len_lo=131072, len_hi=131072, d_cq=1536),
    # hard top-k per-head gates (heads outside the top k are skipped in decode):
    # the paged per-head-gate decode keeping 8 of 32 heads, and the long-context
    # decode with per-head gates keeping 32 of 128 heads
    "decode_paged_head_top8": Workload(
        name="decode_paged_head_top8", mode="decode", dtype="bf16", batch=64, d_model=4096,
        n_heads=32, d_h=128, d_c=512, gate_mode="head_topk", gate_topk=8, gate_bias=True,
        len_law="loguniform", len_lo=256, len_hi=32768, paged=True, page_size=64),
    "decode_long_rope_top32": Workload(
        name="decode_long_rope_top32", mode="decode", dtype="bf16", batch=8, d_model=7168,
        n_heads=128, d_h=128, d_c=512, d_rope=64, rope_base=10000.0, gate_mode="head_topk", gate_topk=32,
        gate_bias=True, len_law="fixed", len_lo=131072, len_hi=131072),
    # the batch-32 and the paged decode over an FP8 (E4M3) latent cache, scale 1/64
    "decode_b32_fp8": Workload(
        name="decode_b32_fp8", mode="decode", dtype="bf16", batch=32, d_model=2048,
        n_heads=16, d_h=128, d_c=512, len_law="uniform", len_lo=1024, len_hi=8192, cache_fp8=True),
    "decode_paged_head_fp8": Workload(
        name="decode_paged_head_fp8", mode="decode", dtype="bf16", batch=64, d_model=4096,
        n_heads=32, d_h=128, d_c=512, gate_mode="head", gate_bias=True,
        len_law="loguniform", len_lo=256, len_hi=32768, paged=True, page_size=64, cache_fp8=True),
    "prefill_b4_s4096_qc": Workload(
        name="prefill_b4_s4096_qc", mode="prefill", dtype="bf16", batch=4, seq_len=4096,
        d_model=7168, n_heads=64, d_h=128, d_c=512, gate_bias=True, d_cq=1536),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


# ---------------------------------------------------------------------------
# bfloat16 helpers (data formatting only)
# ---------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs only: the largest finite pattern plus the rounding
    # increment stays below 2**32
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def e4m3_round(a: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest FP8 E4M3 value (ties to even,
    saturating at +-448), kept as float32: torch's float8 conversion."""
    import torch
    t = torch.from_numpy(np.clip(np.ascontiguousarray(a, dtype=np.float32), -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).to(torch.float32).numpy()


def bf16_round(a: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bfloat16 value, kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32)


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------

def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.mode == "prefill":
        return np.full(w.batch, w.seq_len, dtype=np.int64)
    if w.len_law == "fixed":
        return np.full(w.batch, w.len_hi, dtype=np.int64)
    if w.len_law == "uniform":   # integers, inclusive on both ends
        return rng.integers(w.len_lo, w.len_hi + 1, size=w.batch).astype(np.int64)
    if w.len_law == "loguniform":
        u = rng.uniform(math.log(w.len_lo), math.log(w.len_hi), size=w.batch)
        return np.clip(np.floor(np.exp(u)), w.len_lo, w.len_hi).astype(np.int64)
    raise ValueError(w.len_law)


def generate(w: Workload, seed: int = 0, lengths: Optional[np.ndarray] = None) -> dict:
    """Draw every input of workload ``w``.

    Returns a dict of float32 arrays whose values are exactly representable in
    the workload's dtype (bf16-rounded for bf16 workloads):

    ``x``      [T, d_model]  hidden states of the tokens of this call
               (prefill: all prompt tokens, packed by sequence; decode: the one
               new token per sequence)
    ``W_c``    [d_c, d_model]        ``W_kr`` [d_R, d_model] or None
    ``W_q``    [H*d_h, d_model] (None with a compressed query)
    ``W_dq``   [d_cq, d_model], ``W_uq`` [H*d_h, d_cq] (compressed query only, else None)
    ``W_qr``   [H*d_R, d_model] or [H*d_R, d_cq] with a compressed query, or None
    ``W_k``    [H, d_h, d_c]         ``W_v``  [H, d_h, d_c]
    ``W_g``    [G, d_model]          ``b_g``  [G] or None   (G = H*d_h or H)
    ``W_o``    [d_model, H*d_h]
    ``lengths`` int64 [B]: prefill tokens per sequence, or decode cache length
               including the new token
    ``past``   decode only: list of [L_b - 1, d_c + d_R] cached rows per sequence
    ``page_perm`` paged decode only: permutation of the page pool
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    H, dh, dc, dr, dm = w.n_heads, w.d_h, w.d_c, w.d_rope, w.d_model
    G = w.gate_width
    rnd = bf16_round if w.dtype == "bf16" else (lambda a: a)

    if w.mode == "prefill":
        pre_lens = (np.asarray(lengths, dtype=np.int64) if lengths is not None
                    else np.full(w.batch, w.seq_len, dtype=np.int64))
        n_tok = int(pre_lens.sum())
    else:
        n_tok = w.batch
    out: dict = {"workload": w}
    out["x"] = rnd(_normal(rng, (n_tok, dm), 1.0))
    out["W_c"] = rnd(_normal(rng, (dc, dm), 1.0 / math.sqrt(dm)))
    out["W_kr"] = rnd(_normal(rng, (dr, dm), 1.0 / math.sqrt(dm))) if dr else None
    dcq = w.d_cq
    if dcq:
        # compressed query: c^Q = W_dq x, q = W_uq c^Q, q^R from c^Q (fan-in d_cq)
        out["W_q"] = None
        out["W_dq"] = rnd(_normal(rng, (dcq, dm), 1.0 / math.sqrt(dm)))
        out["W_uq"] = rnd(_normal(rng, (H * dh, dcq), 1.0 / math.sqrt(dcq)))
    else:
        out["W_q"] = rnd(_normal(rng, (H * dh, dm), 1.0 / math.sqrt(dm)))
        out["W_dq"] = out["W_uq"] = None
    q_in = dcq or dm
    out["W_qr"] = rnd(_normal(rng, (H * dr, q_in), 1.0 / math.sqrt(q_in))) if dr else None
    out["W_k"] = rnd(_normal(rng, (H, dh, dc), 1.0 / math.sqrt(dc)))
    out["W_v"] = rnd(_normal(rng, (H, dh, dc), 1.0 / math.sqrt(dc)))
    out["W_g"] = rnd(_normal(rng, (G, dm), 1.0 / math.sqrt(dm)))
    out["b_g"] = rnd(_normal(rng, (G,), math.sqrt(w.gate_bias_var))) if w.gate_bias else None
    out["W_o"] = rnd(_normal(rng, (dm, H * dh), 1.0 / math.sqrt(H * dh)))
    lens = _lengths(w, rng) if w.mode == "decode" else pre_lens
    if lengths is not None:
        lens = np.asarray(lengths, dtype=np.int64)
        assert lens.shape == (w.batch,)
    out["lengths"] = lens
    if w.mode == "decode":
        if w.paged:
            n_pages = int(sum((int(L) + w.page_size - 1) // w.page_size for L in lens))
            out["page_perm"] = rng.permutation(n_pages).astype(np.int64)
        if w.cache_fp8:   # stored values: scale * an E4M3 code
            sc = np.float32(w.cache_scale)
            cache_rnd = lambda a: e4m3_round(a / sc) * sc
        else:
            cache_rnd = rnd
        out["past"] = [cache_rnd(_normal(rng, (int(L) - 1, w.row), 1.0)) if L > 1
                       else np.zeros((0, w.row), np.float32) for L in lens]
    return out
