"""fp64 CPU oracle of Gated Multi-head Latent Attention (test infrastructure).

This module is the reference the CUDA path is checked against. It is slow and
plain on purpose: every quantity is built from its definition, in float64,
with numpy matmuls as the only library primitive. It shares no code with the
CUDA library, and only tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import it. The product path never calls it.

Sources (cited by page title and section):

* [MLA-gate] "Gated MLA 计算公式：输出门与 FFN 的区别" (hackcha.cn):
  §一 latent and per-head up-projections; §二 causal softmax attention,
  head concatenation and the boxed per-channel output gate; §四 NoPE;
  §五 the gate depends only on the current token.
* [MLA-notes] "LLM 注意力与计算内核精读笔记 · 03 注意力头变体：MQA / GQA / MLA"
  (zzszmyf.github.io): §5.1 low-rank joint KV compression and weight
  absorption; §5.2 decoupled RoPE and the cached row ``d_c + d_h^R``;
  §5.3 table of KV elements per token; §7 worked cache ledgers; 题4 the
  absorption identity; 题6 ``kv_bytes_per_token``.
* [Gated-MLA concept] "Gated Multi-head Latent Attention (Gated MLA)"
  (codewithdark-git.github.io): "Gating Mechanism" and "Mathematical
  Formulation", the per-head gate ``g_h = sigmoid(W_g x + b_g)``.

Readings where the pages leave a step open (each is a convention shared with
the CUDA path through its configuration):

* the query of head h is ``q^(h) = W_q^(h) x_t`` (full rank, no bias);
* the softmax scale is ``1/sqrt(d_h)``; with a decoupled RoPE key the key is
  the concatenation ``[k; k^R]`` so the scale is ``1/sqrt(d_h + d_R)``;
* RoPE rotates the pairs (2i, 2i+1) by ``pos * base**(-2i/d_R)``; ``k^R`` is
  stored already rotated, shared by all heads; ``q^R`` has ``d_R`` dims per
  head and is rotated at the query position;
* a decode query sits at position ``L - 1`` of its sequence and attends to
  all ``L`` cached rows, the last of which it writes itself.

Parity status: the formulas of [MLA-gate] §一/§二 and the absorbed form of
[MLA-notes] §5.1/题4 are pinned by closed forms, invariants and a brute-force
restatement. The four readings above are conventions, not facts the pages
fix: parity unpinned against the pages for those readings (they are pinned
only as self-consistent rotations and scalings).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "params", "sigmoid", "rope", "round_e4m3", "cache_store", "latent", "project", "project_latent", "project_query", "head_kv",
    "attention_explicit", "attention_absorbed", "head_gate_values", "gate", "output",
    "prefill", "decode", "kv_elements_per_token", "kv_bytes_per_token",
]


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------

def params(inputs: dict) -> dict:
    """fp64 copy of a workload's weights plus the configuration values.

    ``inputs`` is the dict drawn by the seeded generator (or any dict with the
    same keys). Weight layouts are [out, in]: W_c [d_c, d_model],
    W_kr [d_R, d_model], W_q [H*d_h, d_model], W_qr [H*d_R, d_model]
    (with a compressed query: W_dq [d_cq, d_model], W_uq [H*d_h, d_cq],
    W_qr [H*d_R, d_cq] and no W_q),
    W_k / W_v [H, d_h, d_c], W_g [G, d_model], b_g [G], W_o [d_model, H*d_h].
    """
    w = inputs["workload"]
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    return {
        "H": w.n_heads, "d_h": w.d_h, "d_c": w.d_c, "d_R": w.d_rope,
        "d_model": w.d_model, "gate_mode": w.gate_mode, "gate_topk": w.gate_topk,
        "cache_fp8": w.cache_fp8, "cache_scale": w.cache_scale,
        "scale": w.softmax_scale, "rope_base": w.rope_base,
        "W_c": f(inputs["W_c"]), "W_kr": f(inputs.get("W_kr")),
        "W_q": f(inputs.get("W_q")), "W_qr": f(inputs.get("W_qr")),
        "W_dq": f(inputs.get("W_dq")), "W_uq": f(inputs.get("W_uq")),
        "W_k": f(inputs["W_k"]), "W_v": f(inputs["W_v"]),
        "W_g": f(inputs["W_g"]), "b_g": f(inputs.get("b_g")),
        "W_o": f(inputs["W_o"]),
    }


# ---------------------------------------------------------------------------
# elementary steps
# ---------------------------------------------------------------------------

def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + e^-z), written to avoid overflow for large |z|."""
    z = np.asarray(z, dtype=np.float64)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def rope(v: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotary position rotation of the last axis ([MLA-notes] §5.2: a
    position-dependent rotation applied to q and k).

    Reading: pair (2i, 2i+1) of a d_R-vector at position p is rotated by the
    angle p * base**(-2i/d_R). ``pos`` broadcasts against v's leading axes.
    """
    v = np.asarray(v, dtype=np.float64)
    d = v.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)                             # [d/2]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta  # [..., d/2]
    cos, sin = np.cos(ang), np.sin(ang)
    x0, x1 = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


E4M3_MAX = 448.0


def round_e4m3(v: np.ndarray) -> np.ndarray:
    """Nearest FP8 E4M3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; subnormals below 2^-6 in steps of 2^-9; largest finite 448), ties to
    the even code, saturating to +-448. Values are returned as float64."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)                        # a = f * 2^e, f in [0.5, 1)
    ulp = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)   # 3 mantissa bits; subnormal step 2^-9
    q = np.round(a / ulp) * ulp               # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, v)


def cache_store(p: dict, row: np.ndarray) -> np.ndarray:
    """The value a cached element holds: itself in a bf16/fp32 cache; with an
    FP8 latent cache, cache_scale * e4m3(row / cache_scale) (reading: one fp32
    scale for the whole cache, codes rounded to nearest even and saturated;
    the [K3 blog] §7 warns that such quantisation errors compound, so the
    oracle models the stored value exactly)."""
    if not p.get("cache_fp8"):
        return row
    s = p["cache_scale"]
    return s * round_e4m3(np.asarray(row, np.float64) / s)


def latent(W_c: np.ndarray, x: np.ndarray) -> np.ndarray:
    """c_s = W_c x_s ([MLA-gate] §一; [MLA-notes] §5.1 c^KV = W^DKV h). x [T, d_model]."""
    return x @ W_c.T


def project_latent(p: dict, x: np.ndarray, positions: np.ndarray) -> dict:
    """What a token writes into the cache ([MLA-gate] §一; [MLA-notes] §5.2):

    * c  [T, d_c]   latent c = W_c x
    * kR [T, d_R]   RoPE(W_kr x) at the token's position (shared by all heads)

    Both are returned as the cache stores them (cache_store: rounded to FP8
    E4M3 times the cache scale for an FP8 latent cache).
    """
    x = np.asarray(x, dtype=np.float64)
    out = {"c": cache_store(p, latent(p["W_c"], x))}
    if p["d_R"]:
        out["kR"] = cache_store(p, rope(x @ p["W_kr"].T, positions, p["rope_base"]))
    else:
        out["kR"] = np.zeros((x.shape[0], 0))
    return out


def project_query(p: dict, x: np.ndarray, positions: np.ndarray) -> dict:
    """What a token needs as a query:

    * q  [T, H, d_h]     q^(h) = W_q^(h) x (reading: full-rank query), or with
                         the low-rank query of [MLA-notes] §5.1
                         c^Q = W_dq x (d_cq dims, returned as ``cq``), q = W_uq c^Q
    * qR [T, H, d_R]     RoPE(W_qr^(h) x) at the token's position ([MLA-notes]
                         §5.2); with the low-rank query RoPE(W_qr^(h) c^Q), as
                         §5.2 writes q^R = RoPE(W^QR c^Q)
    * glogit [T, G]      W_g x (+ b_g): gate logits ([MLA-gate] §二 boxed
                         equation, per channel; [Gated-MLA concept] "Gating
                         Mechanism", per head with bias)
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    H, dh, dR = p["H"], p["d_h"], p["d_R"]
    if p.get("W_dq") is not None:
        q_in = x @ p["W_dq"].T                                     # c^Q [T, d_cq]
        out = {"cq": q_in, "q": (q_in @ p["W_uq"].T).reshape(T, H, dh)}
    else:
        q_in = x
        out = {"q": (x @ p["W_q"].T).reshape(T, H, dh)}
    if dR:
        qr = (q_in @ p["W_qr"].T).reshape(T, H, dR)
        out["qR"] = rope(qr, np.asarray(positions)[:, None], p["rope_base"])
    else:
        out["qR"] = np.zeros((T, H, 0))
    g = x @ p["W_g"].T
    if p["b_g"] is not None:
        g = g + p["b_g"]
    out["glogit"] = g
    return out


def project(p: dict, x: np.ndarray, positions: np.ndarray) -> dict:
    """Everything computed from the tokens' own hidden states x [T, d_model]:
    the cached row (project_latent) and the query side (project_query)."""
    out = project_latent(p, x, positions)
    out.update(project_query(p, x, positions))
    return out


def head_kv(p: dict, h: int, C: np.ndarray):
    """Explicit per-head key and value from cached latents ([MLA-gate] §一):
    k_s^(h) = W_k^(h) c_s, v_s^(h) = W_v^(h) c_s. C [L, d_c] -> K, V [L, d_h]."""
    return C @ p["W_k"][h].T, C @ p["W_v"][h].T


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    """Softmax over the last axis; -inf entries get weight exactly 0."""
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_explicit(p: dict, h: int, q: np.ndarray, qR: np.ndarray,
                       C: np.ndarray, KR: np.ndarray, q_pos: np.ndarray,
                       return_weights: bool = False):
    """Causal softmax attention of head h in the explicit (non-absorbed) form.

    [MLA-gate] §二: a_{t,s} = Softmax_{s<=t}(q_t . k_s / sqrt(d_h)),
    o_t = sum_{s<=t} a_{t,s} v_s, with k, v rebuilt from the cached latents
    (§一). With a decoupled RoPE key the score adds q^R_t . k^R_s before
    scaling ([MLA-notes] §5.2, reading: concatenated key).

    q [n, d_h], qR [n, d_R] are the queries at positions ``q_pos`` [n];
    C [L, d_c], KR [L, d_R] are the cached rows of positions 0..L-1.
    Returns o [n, d_h] (and the weights a [n, L] when asked).
    """
    K, V = head_kv(p, h, C)
    z = q @ K.T
    if KR.shape[1]:
        z = z + qR @ KR.T
    z = p["scale"] * z
    s = np.arange(C.shape[0])
    mask = s[None, :] > np.asarray(q_pos)[:, None]            # future keys
    z = np.where(mask, -np.inf, z)
    a = _softmax_rows(z)
    o = a @ V
    return (o, a) if return_weights else o


def attention_absorbed(p: dict, h: int, q: np.ndarray, qR: np.ndarray,
                       C: np.ndarray, KR: np.ndarray, q_pos: np.ndarray,
                       return_weights: bool = False):
    """The same attention with W_k folded into the query and W_v applied after
    the weighted sum ([MLA-notes] §5.1 and 题4: q^T W^UK c = ((W^UK)^T q)^T c).

    q_lat = W_k^(h)T q; z_s = scale (q_lat . c_s + q^R . k^R_s);
    O_lat = sum_s a_s c_s; o = W_v^(h) O_lat.
    """
    q_lat = q @ p["W_k"][h]                                    # [n, d_c]
    z = q_lat @ C.T
    if KR.shape[1]:
        z = z + qR @ KR.T
    z = p["scale"] * z
    s = np.arange(C.shape[0])
    z = np.where(s[None, :] > np.asarray(q_pos)[:, None], -np.inf, z)
    a = _softmax_rows(z)
    o_lat = a @ C                                              # [n, d_c]
    o = o_lat @ p["W_v"][h].T
    return (o, a) if return_weights else o


HEAD_GATE_MODES = ("head", "head_topk", "head_binary", "head_ternary")


def head_gate_values(p: dict, glogit: np.ndarray) -> np.ndarray:
    """Per-head gate values [T, H] from the gate logits [T, H].

    * "head": sigmoid(z) ([Gated-MLA concept] "Mathematical Formulation").
    * "head_topk" ([Gated-MLA concept] "Variants / Extensions", Hard Gating:
      top-k heads per token): 1 for the k = p["gate_topk"] heads with the
      largest logits of the token, 0 for the others. Reading: the discrete
      forward values (the straight-through estimator the page names concerns
      training only); equal logits go to the lower head index.
    * "head_binary" (same list, Quantized Gates): 1 where sigmoid(z) >= 1/2,
      i.e. z >= 0, else 0.
    * "head_ternary" (same list): sigmoid(z) rounded to the nearest of
      {0, 1/2, 1} (reading: the three levels of a [0, 1] gate), halfway
      values rounded up; the cuts are sigmoid(z) = 1/4 and 3/4, z = -+ln 3.
    """
    z = np.asarray(glogit, dtype=np.float64)
    mode = p["gate_mode"]
    if mode == "head":
        return sigmoid(z)
    if mode == "head_topk":
        k = int(p["gate_topk"])
        order = np.argsort(-z, axis=1, kind="stable")          # ties: lower index first
        g = np.zeros_like(z)
        np.put_along_axis(g, order[:, :k], 1.0, axis=1)
        return g
    if mode == "head_binary":
        return (z >= 0.0).astype(np.float64)
    if mode == "head_ternary":
        return np.floor(2.0 * sigmoid(z) + 0.5) / 2.0
    raise ValueError(mode)


def gate(p: dict, glogit: np.ndarray, o_tilde: np.ndarray) -> np.ndarray:
    """Output gate applied to the concatenated heads.

    Per channel ([MLA-gate] §二 boxed equation): Sigmoid(W_g x_t) ⊙ õ_t with
    G = H*d_h. Per head ([Gated-MLA concept] "Mathematical Formulation" and
    "Variants / Extensions"): gate values [.., H] (head_gate_values) broadcast
    over each head's d_h channels.
    """
    if p["gate_mode"] == "channel":
        return sigmoid(glogit) * o_tilde
    g = head_gate_values(p, glogit)
    T = o_tilde.shape[0]
    return (g[:, :, None] * o_tilde.reshape(T, p["H"], p["d_h"])).reshape(T, -1)


def output(p: dict, gated: np.ndarray) -> np.ndarray:
    """y_t = W_o [gated õ_t] ([MLA-gate] §二 boxed equation)."""
    return gated @ p["W_o"].T


# ---------------------------------------------------------------------------
# whole calls
# ---------------------------------------------------------------------------

def prefill(p: dict, x: np.ndarray, lengths: Sequence[int],
            rows: Optional[dict] = None, absorbed: bool = False) -> dict:
    """Causal prefill of a packed batch starting from an empty cache.

    x [T, d_model] holds the sequences back to back; ``lengths`` their token
    counts. ``rows`` optionally maps a sequence index to the list of query
    positions to evaluate (default: all; sequences not in ``rows`` are
    evaluated in full). Returns c, kR for all tokens and, for the evaluated
    rows, ``index`` (packed row ids), q, qR, glogit, o [n, H, d_h], o_tilde,
    gated and y.
    """
    x = np.asarray(x, dtype=np.float64)
    lengths = [int(L) for L in lengths]
    starts = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    positions = np.concatenate([np.arange(L) for L in lengths]) if lengths else np.zeros(0, np.int64)
    lat = project_latent(p, x, positions)
    attn = attention_absorbed if absorbed else attention_explicit
    H = p["H"]
    sel = []
    for b, L in enumerate(lengths):
        t_sel = np.arange(L) if rows is None or b not in rows else np.asarray(sorted(rows[b]), dtype=np.int64)
        sel.append(t_sel)
    index = np.concatenate([starts[b] + t for b, t in enumerate(sel)]) if sel else np.zeros(0, np.int64)
    qs = project_query(p, x[index], positions[index])
    o_rows, k = [], 0
    for b, L in enumerate(lengths):
        t_sel = sel[b]
        n = len(t_sel)
        if n == 0:
            continue
        sl = slice(starts[b], starts[b] + L)
        C, KR = lat["c"][sl], lat["kR"][sl]
        o = np.stack([attn(p, h, qs["q"][k:k + n, h], qs["qR"][k:k + n, h], C, KR, t_sel)
                      for h in range(H)], axis=1)              # [n, H, d_h]
        o_rows.append(o)
        k += n
    out = dict(lat)
    out.update(qs)
    out["index"] = index
    o = np.concatenate(o_rows) if o_rows else np.zeros((0, H, p["d_h"]))
    out["o"] = o
    out["o_tilde"] = o.reshape(o.shape[0], -1)                 # Concat_h ([MLA-gate] §二)
    out["gated"] = gate(p, qs["glogit"], out["o_tilde"])
    out["y"] = output(p, out["gated"])
    return out


def decode(p: dict, x: np.ndarray, past: Sequence[np.ndarray],
           heads: Optional[Sequence[int]] = None,
           seqs: Optional[Sequence[int]] = None, absorbed: bool = False) -> dict:
    """One decode step per sequence over a latent cache.

    x [B, d_model] is the new token of each sequence; ``past[b]`` holds the
    L_b - 1 cached rows [c | k^R] of its earlier positions. The new token sits
    at position L_b - 1: its own latent row is appended (as the library
    writes it into the cache) and it attends to all L_b rows.

    ``heads``/``seqs`` restrict the attention to a subset (for large cases);
    y is produced only when every head of a sequence was evaluated.
    Returns c, kR, q, qR, glogit [B, ...], o [nb, nh, d_h] and, with all
    heads, o_tilde, gated, y [nb, ...].
    """
    x = np.asarray(x, dtype=np.float64)
    B = x.shape[0]
    dc = p["d_c"]
    lens = np.array([len(r) + 1 for r in past], dtype=np.int64)
    pr = project(p, x, lens - 1)
    heads = list(range(p["H"])) if heads is None else list(heads)
    seqs = list(range(B)) if seqs is None else list(seqs)
    attn = attention_absorbed if absorbed else attention_explicit
    o = np.zeros((len(seqs), len(heads), p["d_h"]))
    for i, b in enumerate(seqs):
        rows = np.asarray(past[b], dtype=np.float64)
        C = np.concatenate([rows[:, :dc], pr["c"][b:b + 1]])
        KR = np.concatenate([rows[:, dc:], pr["kR"][b:b + 1]])
        t = np.array([lens[b] - 1])
        for j, h in enumerate(heads):
            o[i, j] = attn(p, h, pr["q"][b:b + 1, h], pr["qR"][b:b + 1, h], C, KR, t)[0]
    out = dict(pr)
    out["lengths"] = lens
    out["o"] = o
    if len(heads) == p["H"]:
        out["o_tilde"] = o.reshape(len(seqs), -1)
        out["gated"] = gate(p, pr["glogit"][seqs], out["o_tilde"])
        out["y"] = output(p, out["gated"])
    return out


# ---------------------------------------------------------------------------
# cache accounting ([MLA-notes] §5.3 table, §7 ledgers, 题1 and 题6)
# ---------------------------------------------------------------------------

def kv_elements_per_token(mechanism: str, h: int = 0, g: int = 0, d_h: int = 0,
                          d_c: int = 0, d_r: int = 0) -> int:
    """Cached KV elements per token per layer: MHA 2 h d_h, GQA-g 2 g d_h,
    MQA 2 d_h, MLA d_c + d_R (independent of the head count)."""
    m = mechanism.upper()
    if m == "MHA":
        return 2 * h * d_h
    if m == "GQA":
        return 2 * g * d_h
    if m == "MQA":
        return 2 * d_h
    if m == "MLA":
        return d_c + d_r
    raise ValueError(mechanism)


def kv_bytes_per_token(mechanism: str, h: int = 0, g: int = 0, d_h: int = 0,
                       d_c: int = 0, d_r: int = 0, layers: int = 1,
                       bytes: int = 2) -> int:
    """Cache bytes per token over all layers ([MLA-notes] 题6)."""
    return kv_elements_per_token(mechanism, h, g, d_h, d_c, d_r) * layers * bytes
