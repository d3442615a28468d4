"""Inputs whose softmax must be rescaled inside the attention kernels, and the
CPU checks that prove it (test helper).

Both tensor-core attention kernels raise a row's running max only when a later
tile's max exceeds it by more than 8 (in log2 units), and only then rescale
the accumulated output in tensor memory. With plain N(0, 1) inputs the scores
never jump that far after the first tile, so those branches would stay cold.

Here a few keys are planted: a cached latent row (decode) or a prompt token's
hidden state (prefill) is replaced by one whose latent points along a chosen
head's absorbed query W_k^T q, with a length that gives that one score a set
value (e.g. 16 log2 units, against about 4 for the other keys). Every other
score stays as drawn, so magnitudes of o and y stay ordinary and the bf16
tolerances keep their meaning. The planted values are computed from the
oracle's fp64 projections and rounded to bf16 like every other input.

The functions below recompute the log2-domain scores in fp64 from the actual
inputs and count, for the kernels' tiling, how many raises must happen, so a
test can assert on the CPU that its input really reaches those branches.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
import synth

LOG2E = 1.0 / math.log(2.0)
TILE = 128
RAISE = 8.0          # the kernels' threshold (log2 units)


def _rnd(inp):
    return synth.bf16_round if inp["workload"].dtype == "bf16" else (lambda a: np.asarray(a, np.float32))


def plant_decode(inp, plan):
    """plan: (sequence b, cached position, head h, score in log2 units). The
    row's latent part becomes alpha * q_lat / |q_lat| with q_lat = W_k^(h)T q of
    sequence b's query; its RoPE part is kept."""
    p = oracle.params(inp)
    x = np.asarray(inp["x"], np.float64)
    lens = np.array([len(r) + 1 for r in inp["past"]])
    pr = oracle.project(p, x, lens - 1)
    dc = p["d_c"]
    out = dict(inp)
    out["past"] = [r.copy() for r in inp["past"]]
    for b, pos, h, score in plan:
        ql = pr["q"][b, h] @ p["W_k"][h]
        alpha = score / (p["scale"] * LOG2E * np.linalg.norm(ql))
        out["past"][b][pos, :dc] = _rnd(inp)((alpha * ql / np.linalg.norm(ql)).astype(np.float32))
    return out


def plant_prefill(inp, plan):
    """plan: (sequence b, key position s, query position t > s, head h, score in
    log2 units). Token s's hidden state becomes the least-norm x with
    W_c x = alpha * q_lat / |q_lat|, q_lat the absorbed query of (t, h)."""
    p = oracle.params(inp)
    lengths = [int(L) for L in inp["lengths"]]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    positions = np.concatenate([np.arange(L) for L in lengths])
    x = np.asarray(inp["x"], np.float64).copy()
    pr = oracle.project(p, x, positions)
    Wc = p["W_c"]
    pinv = Wc.T @ np.linalg.inv(Wc @ Wc.T)
    for b, s, t, h, score in plan:
        assert s < t < lengths[b]
        ql = pr["q"][starts[b] + t, h] @ p["W_k"][h]
        alpha = score / (p["scale"] * LOG2E * np.linalg.norm(ql))
        x[starts[b] + s] = pinv @ (alpha * ql / np.linalg.norm(ql))
    out = dict(inp)
    out["x"] = _rnd(inp)(x.astype(np.float32))
    return out


def decode_head_group(H):
    """Heads per attention CTA and the number of head groups (as the decode kernel picks them)."""
    HG = 16 if H <= 16 else (64 if H % 64 == 0 else (32 if H % 32 == 0 else 16))
    return HG, (H + HG - 1) // HG


def decode_segments(lengths, G):
    """The decode split plan: 128-token tiles of all sequences, concatenated and cut
    into G equal ranges; returns (sequence, first tile, end tile) per segment."""
    tiles = [(int(L) + TILE - 1) // TILE for L in lengths]
    total = sum(tiles)
    tpc = (total + G - 1) // G if total else 1
    segs, P = [], 0
    for b, t in enumerate(tiles):
        if t:
            for g in range(P // tpc, (P + t - 1) // tpc + 1):
                lo, hi = max(P, g * tpc), min(P + t, (g + 1) * tpc)
                segs.append((b, lo - P, hi - P))
        P += t
    return segs


def decode_scores_log2(inp, b):
    """[H, L_b] log2-domain scores of sequence b's query over its L_b cached rows (fp64)."""
    p = oracle.params(inp)
    x = np.asarray(inp["x"], np.float64)
    lens = np.array([len(r) + 1 for r in inp["past"]])
    pr = oracle.project(p, x, lens - 1)
    dc = p["d_c"]
    rows = np.asarray(inp["past"][b], np.float64)
    C = np.concatenate([rows[:, :dc], pr["c"][b:b + 1]])
    KR = np.concatenate([rows[:, dc:], pr["kR"][b:b + 1]])
    z = np.stack([(pr["q"][b, h] @ p["W_k"][h]) @ C.T + (pr["qR"][b, h] @ KR.T if KR.shape[1] else 0.0)
                  for h in range(p["H"])])
    return p["scale"] * z * LOG2E


def count_raises(z_row, lo, hi):
    """Raises of the running max over tiles lo..hi-1 of one score row (the kernels' rule)."""
    n = 0
    m = z_row[lo * TILE:(lo + 1) * TILE].max()
    for t in range(lo + 1, hi):
        seg = z_row[t * TILE:(t + 1) * TILE]
        if seg.size and seg.max() > m + RAISE:
            m = seg.max()
            n += 1
    return n


def decode_raises(inp, num_sms):
    """Total in-kernel raises over every (segment, head) of a decode input, and the
    largest gap between the maxima of two segments of one sequence."""
    w = inp["workload"]
    HG, n_hg = decode_head_group(w.n_heads)
    segs = decode_segments(inp["lengths"], max(1, num_sms // n_hg))
    raises, gap = 0, 0.0
    by_seq = {}
    for b, lo, hi in segs:
        by_seq.setdefault(b, []).append((lo, hi))
    for b, ranges in by_seq.items():
        z = decode_scores_log2(inp, b)
        for h in range(z.shape[0]):
            maxima = []
            for lo, hi in ranges:
                raises += count_raises(z[h], lo, hi)
                maxima.append(z[h, lo * TILE:hi * TILE].max())
            gap = max(gap, max(maxima) - min(maxima))
    return raises, gap


def prefill_raises(inp):
    """In-kernel raises over every (query row, head) of a prefill input: row t of a
    sequence sees key tiles 0..t // 128, the first always setting the max."""
    p = oracle.params(inp)
    x = np.asarray(inp["x"], np.float64)
    lengths = [int(L) for L in inp["lengths"]]
    positions = np.concatenate([np.arange(L) for L in lengths])
    pr = oracle.project(p, x, positions)
    n, start = 0, 0
    for L in lengths:
        sl = slice(start, start + L)
        start += L
        for h in range(p["H"]):
            K, _ = oracle.head_kv(p, h, pr["c"][sl])
            z = p["scale"] * (pr["q"][sl, h] @ K.T) * LOG2E
            for t in range(TILE, L):
                n += count_raises(z[t, :t + 1], 0, t // TILE + 1)
    return n
