"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test ties the oracle to something other than itself: a closed form, an
invariant of the definitions, a brute-force restatement written with plain
Python loops, or a number printed on the pages (tests/golden/). The last group
plants plausible mistakes in the oracle (on the CPU) and checks that some pin
fails for each one.
"""
import math
import os

import numpy as np
import pytest

import synth
import oracle
from oracle import core

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(d_rope=0, gate_mode="channel", gate_bias=True, lengths=(3, 5), **kw):
    w = synth.Workload(name="tiny", mode="prefill", dtype="f32", batch=len(lengths),
                       d_model=6, n_heads=2, d_h=3, d_c=4, d_rope=d_rope,
                       rope_base=10000.0, gate_mode=gate_mode, gate_bias=gate_bias, **kw)
    return synth.generate(w, seed=1, lengths=np.array(lengths))


def tiny_decode(d_rope=0, lens=(1, 4, 7), gate_mode="channel"):
    w = synth.Workload(name="tinyd", mode="decode", dtype="f32", batch=len(lens),
                       d_model=6, n_heads=2, d_h=3, d_c=4, d_rope=d_rope,
                       gate_mode=gate_mode, gate_bias=True)
    return synth.generate(w, seed=2, lengths=np.array(lens))


# ---------------------------------------------------------------------------
# brute force: the page formulas as plain loops (no numpy linear algebra)
# ---------------------------------------------------------------------------

def _mv(W, v):
    return [sum(W[i][j] * v[j] for j in range(len(v))) for i in range(len(W))]


def _rot(v, pos, base):
    d = len(v)
    out = list(v)
    for i in range(d // 2):
        ang = pos * base ** (-2.0 * i / d)
        c, s = math.cos(ang), math.sin(ang)
        out[2 * i] = v[2 * i] * c - v[2 * i + 1] * s
        out[2 * i + 1] = v[2 * i] * s + v[2 * i + 1] * c
    return out


def brute_prefill(inp):
    """y_t = W_o[Sigmoid(W_g x_t + b_g) ⊙ Concat_h sum_{s<=t} a_ts v_s] with
    k = W_k c, v = W_v c, c = W_c x, written out loop by loop."""
    w = inp["workload"]
    H, dh, dR = w.n_heads, w.d_h, w.d_rope
    X = inp["x"].astype(float).tolist()
    Wc, Wk, Wv, Wg, Wo = (np.asarray(inp[k], float).tolist() for k in ("W_c", "W_k", "W_v", "W_g", "W_o"))
    compressed = inp.get("W_dq") is not None
    if compressed:   # [MLA-notes] §5.1 c^Q = W^DQ h, q = W^UQ c^Q; §5.2 q^R = RoPE(W^QR c^Q)
        Wdq, Wuq = np.asarray(inp["W_dq"], float).tolist(), np.asarray(inp["W_uq"], float).tolist()
    else:
        Wq = np.asarray(inp["W_q"], float).tolist()
    bg = np.asarray(inp["b_g"], float).tolist() if inp["b_g"] is not None else None
    Wkr = np.asarray(inp["W_kr"], float).tolist() if dR else None
    Wqr = np.asarray(inp["W_qr"], float).tolist() if dR else None
    scale = 1.0 / math.sqrt(dh + dR)
    ys = []
    start = 0
    for L in inp["lengths"]:
        L = int(L)
        xs = X[start:start + L]
        start += L
        c = [_mv(Wc, x) for x in xs]
        kr = [_rot(_mv(Wkr, x), s, w.rope_base) for s, x in enumerate(xs)] if dR else None
        for t in range(L):
            x = xs[t]
            q_in = _mv(Wdq, x) if compressed else x
            qfull = _mv(Wuq, q_in) if compressed else _mv(Wq, x)
            qrfull = _mv(Wqr, q_in) if dR else None
            o_cat = []
            for h in range(H):
                q = qfull[h * dh:(h + 1) * dh]
                qr = _rot(qrfull[h * dR:(h + 1) * dR], t, w.rope_base) if dR else []
                z = []
                for s in range(t + 1):
                    k = _mv(Wk[h], c[s])
                    dot = sum(q[i] * k[i] for i in range(dh))
                    if dR:
                        dot += sum(qr[i] * kr[s][i] for i in range(dR))
                    z.append(scale * dot)
                m = max(z)
                e = [math.exp(zz - m) for zz in z]
                den = sum(e)
                o = [0.0] * dh
                for s in range(t + 1):
                    v = _mv(Wv[h], c[s])
                    for i in range(dh):
                        o[i] += e[s] / den * v[i]
                o_cat += o
            logit = _mv(Wg, x)
            if bg is not None:
                logit = [logit[i] + bg[i] for i in range(len(logit))]
            gsig = [1.0 / (1.0 + math.exp(-l)) for l in logit]
            if w.gate_mode == "head_topk":       # the k largest logits, ties to the lower head
                ranked = sorted(range(H), key=lambda hh: (-logit[hh], hh))
                gsig = [1.0 if hh in ranked[:w.gate_topk] else 0.0 for hh in range(H)]
            elif w.gate_mode == "head_binary":
                gsig = [1.0 if l >= 0.0 else 0.0 for l in logit]
            elif w.gate_mode == "head_ternary":  # nearest of 0, 1/2, 1
                gsig = [min((0.0, 0.5, 1.0), key=lambda v: (abs(v - g_), -v)) for g_ in gsig]
            if w.gate_mode == "channel":
                gated = [gsig[i] * o_cat[i] for i in range(H * dh)]
            else:
                gated = [gsig[i // dh] * o_cat[i] for i in range(H * dh)]
            ys.append(_mv(Wo, gated))
    return np.array(ys)


@pytest.mark.parametrize("d_rope", [0, 2])
@pytest.mark.parametrize("gate_mode", ["channel", "head"])
def test_bruteforce_prefill(d_rope, gate_mode):
    inp = tiny(d_rope=d_rope, gate_mode=gate_mode)
    p = oracle.params(inp)
    got = oracle.prefill(p, inp["x"], inp["lengths"])["y"]
    ref = brute_prefill(inp)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("d_rope", [0, 2])
def test_bruteforce_prefill_compressed_query(d_rope):
    inp = tiny(d_rope=d_rope, d_cq=3)
    assert inp["W_q"] is None and inp["W_dq"].shape == (3, 6) and inp["W_uq"].shape == (6, 3)
    if d_rope:
        assert inp["W_qr"].shape == (2 * 2, 3)     # q^R is read from c^Q
    p = oracle.params(inp)
    got = oracle.prefill(p, inp["x"], inp["lengths"])["y"]
    np.testing.assert_allclose(got, brute_prefill(inp), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("d_rope", [0, 2])
def test_compressed_query_equals_full_rank_with_the_product_weight(d_rope):
    """q = W_uq (W_dq x) is the full-rank query of W_q = W_uq W_dq, and
    q^R = RoPE(W_qr (W_dq x)) the one of W_qr W_dq: the two oracle paths agree."""
    inp = tiny(d_rope=d_rope, d_cq=4)
    p = oracle.params(inp)
    full = dict(p, W_q=p["W_uq"] @ p["W_dq"], W_dq=None, W_uq=None)
    if d_rope:
        full["W_qr"] = p["W_qr"] @ p["W_dq"]
    a = oracle.prefill(p, inp["x"], inp["lengths"])
    b = oracle.prefill(full, inp["x"], inp["lengths"])
    for k in ("q", "qR", "o", "y"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-13, err_msg=k)
    np.testing.assert_allclose(a["cq"], np.asarray(inp["x"], float) @ p["W_dq"].T, rtol=1e-15)


@pytest.mark.parametrize("gate_mode,k", [("head_topk", 1), ("head_topk", 2), ("head_binary", 0),
                                         ("head_ternary", 0)])
def test_bruteforce_prefill_hard_and_quantized_head_gates(gate_mode, k):
    inp = tiny(d_rope=2, gate_mode=gate_mode, gate_topk=k, lengths=(4, 6))
    p = oracle.params(inp)
    got = oracle.prefill(p, inp["x"], inp["lengths"])["y"]
    np.testing.assert_allclose(got, brute_prefill(inp), rtol=1e-12, atol=1e-12)


def _hard(gate_mode, k=0, H=6, seed=3, T=40):
    w = synth.Workload(name="hard", mode="prefill", dtype="f32", batch=1, d_model=8, n_heads=H, d_h=3, d_c=4,
                       gate_mode=gate_mode, gate_topk=k, gate_bias=True)
    inp = synth.generate(w, seed=seed, lengths=np.array([T]))
    p = oracle.params(inp)
    return inp, p, oracle.project(p, inp["x"], np.arange(T))["glogit"]


def test_topk_gates_select_the_k_largest_logits():
    for k in range(1, 7):
        inp, p, z = _hard("head_topk", k)
        g = oracle.head_gate_values(p, z)
        assert np.all(g.sum(axis=1) == k)
        for t in range(z.shape[0]):
            chosen = set(np.flatnonzero(g[t]))
            assert z[t, list(chosen)].min() >= np.max(np.delete(z[t], list(chosen)), initial=-np.inf)
    # equal logits: the lower head index wins
    p = {"gate_mode": "head_topk", "gate_topk": 2}
    assert np.array_equal(oracle.head_gate_values(p, np.array([[1.0, 3.0, 3.0, 3.0]])), [[0, 1, 1, 0]])


def test_topk_with_every_head_is_ungated_mla():
    inp, p, _ = _hard("head_topk", 6)
    y = oracle.prefill(p, inp["x"], inp["lengths"])
    np.testing.assert_allclose(y["y"], oracle.output(p, y["o_tilde"]), rtol=1e-13, atol=1e-15)


def test_binary_gate_is_the_saturated_sigmoid():
    inp, p, z = _hard("head_binary")
    g = oracle.head_gate_values(p, z)
    far = np.abs(z) > 1e-2
    np.testing.assert_array_equal(g[far], oracle.sigmoid(1e5 * z[far]))
    assert set(np.unique(g)) <= {0.0, 1.0}


def test_ternary_gate_is_the_nearest_of_three_levels():
    inp, p, z = _hard("head_ternary", T=200)
    g = oracle.head_gate_values(p, z)
    s = oracle.sigmoid(z)
    assert set(np.unique(g)) <= {0.0, 0.5, 1.0}
    assert np.all(np.abs(g - s) <= 0.25 + 1e-15)
    order = np.argsort(z.ravel())
    assert np.all(np.diff(g.ravel()[order]) >= 0)               # monotone in the logit
    cut = math.log(3.0)                                            # sigmoid(+-ln 3) = 3/4, 1/4
    np.testing.assert_array_equal(oracle.head_gate_values(p, np.array([[-cut - 1e-9, -cut + 1e-9, 0.0,
                                                                        cut - 1e-9, cut + 1e-9]])),
                                  [[0.0, 0.5, 0.5, 0.5, 1.0]])


@pytest.mark.parametrize("gate_mode,k", [("head_topk", 2), ("head_binary", 0), ("head_ternary", 0)])
def test_zero_gated_heads_do_not_reach_y(gate_mode, k):
    """Head skipping is exact: a head whose gate is 0 for a token contributes
    nothing to that token's y, whatever its attention computes."""
    inp, p, z = _hard(gate_mode, k)
    g = oracle.head_gate_values(p, z)
    y = oracle.prefill(p, inp["x"], inp["lengths"])["y"]
    for h in range(p["H"]):
        p2 = dict(p, W_v=p["W_v"].copy(), W_k=p["W_k"].copy())
        p2["W_v"][h] *= 1e3
        p2["W_k"][h] *= -7.0
        y2 = oracle.prefill(p2, inp["x"], inp["lengths"])["y"]
        off = g[:, h] == 0.0
        np.testing.assert_allclose(y2[off], y[off], rtol=1e-12, atol=1e-14)
        if (~off).any():
            assert np.abs(y2[~off] - y[~off]).max() > 1e-3


def test_two_token_closed_form():
    """H=1, d_h=d_c=1: o_1 = v_0 sigmoid(z_0 - z_1) + v_1 sigmoid(z_1 - z_0)."""
    w = synth.Workload(name="t2", mode="prefill", dtype="f32", batch=1, d_model=1,
                       n_heads=1, d_h=1, d_c=1, gate_bias=True)
    inp = synth.generate(w, seed=0, lengths=np.array([2]))
    inp.update(x=np.array([[0.7], [-1.3]]), W_c=np.array([[1.5]]), W_q=np.array([[2.0]]),
               W_k=np.array([[[0.8]]]), W_v=np.array([[[-0.6]]]), W_g=np.array([[0.0]]),
               b_g=np.array([50.0]), W_o=np.array([[1.0]]))
    p = oracle.params(inp)
    y = oracle.prefill(p, inp["x"], [2])["y"][:, 0]
    c0, c1 = 1.5 * 0.7, 1.5 * -1.3
    q1 = 2.0 * -1.3
    z0, z1 = q1 * 0.8 * c0, q1 * 0.8 * c1          # scale 1/sqrt(1) = 1
    v0, v1 = -0.6 * c0, -0.6 * c1
    sig = lambda u: 1.0 / (1.0 + math.exp(-u))
    o1 = v0 * sig(z0 - z1) + v1 * sig(z1 - z0)
    g = sig(50.0)
    np.testing.assert_allclose(y, [g * v0, g * o1], rtol=1e-13)


def test_scale_is_inverse_sqrt_dh():
    """d_h = 4, d_c = 9: two keys whose scaled scores differ by exactly 1 get
    weights e/(1+e) and 1/(1+e) (pins the 1/sqrt(d_h) factor of [MLA-gate] §二)."""
    w = synth.Workload(name="s", mode="decode", dtype="f32", batch=1, d_model=4,
                       n_heads=1, d_h=4, d_c=9)
    inp = synth.generate(w, seed=0, lengths=np.array([2]))
    W_c = np.zeros((9, 4)); W_c[0, 0] = 1.0                  # c = (x_0, 0, ..., 0)
    W_k = np.zeros((1, 4, 9)); W_k[0, 0, 0] = 1.0             # k = (c_0, 0, 0, 0)
    W_v = np.zeros((1, 4, 9)); W_v[0, 0, 0] = 1.0             # v = (c_0, 0, 0, 0)
    W_q = np.zeros((4, 4)); W_q[0, 0] = 2.0                   # q = (2 x_0, 0, 0, 0)
    inp.update(x=np.array([[1.0, 0.0, 0.0, 0.0]]), W_c=W_c, W_k=W_k, W_v=W_v, W_q=W_q,
               W_g=np.zeros((4, 4)), W_o=np.eye(4))
    past = [np.zeros((1, 9))]
    past[0][0, 0] = 2.0                                       # c_0 = 2 e_0, c_1 = e_0
    p = oracle.params(inp)
    out = oracle.decode(p, inp["x"], past)
    # z_0 = (2*2)/sqrt(4) = 2, z_1 = (2*1)/sqrt(4) = 1
    a0 = math.e / (1.0 + math.e)
    np.testing.assert_allclose(out["o"][0, 0, 0], a0 * 2.0 + (1 - a0) * 1.0, rtol=1e-14)


# ---------------------------------------------------------------------------
# invariants of the definitions
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d_rope", [0, 2])
def test_softmax_rows_sum_to_one_and_causal(d_rope):
    inp = tiny(d_rope=d_rope, lengths=(7,))
    p = oracle.params(inp)
    pr = oracle.project(p, inp["x"], np.arange(7))
    for h in range(2):
        _, a = oracle.attention_explicit(p, h, pr["q"][:, h], pr["qR"][:, h], pr["c"],
                                         pr["kR"], np.arange(7), return_weights=True)
        assert np.max(np.abs(a.sum(1) - 1.0)) < 1e-12
        assert np.all(a[np.triu_indices(7, 1)] == 0.0)
        assert np.all(a[np.tril_indices(7)] > 0.0)


def test_single_token_gives_v0():
    """L = 1 (prefill row t=0 and decode with a one-row cache): o^(h) = W_v^(h) c_0."""
    inp = tiny(lengths=(1, 4))
    p = oracle.params(inp)
    out = oracle.prefill(p, inp["x"], [1, 4])
    for row in (0, 1):                          # t=0 of both sequences
        c0 = np.asarray(inp["W_c"], float) @ np.asarray(inp["x"][row], float)
        for h in range(2):
            np.testing.assert_allclose(out["o"][row, h], np.asarray(inp["W_v"][h], float) @ c0,
                                       rtol=1e-13, atol=1e-15)
    d = tiny_decode(lens=(1, 3))
    p = oracle.params(d)
    out = oracle.decode(p, d["x"], d["past"])
    c0 = np.asarray(d["W_c"], float) @ np.asarray(d["x"][0], float)
    for h in range(2):
        np.testing.assert_allclose(out["o"][0, h], np.asarray(d["W_v"][h], float) @ c0,
                                   rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("gate_mode", ["channel", "head"])
def test_gate_saturation(gate_mode):
    """Logits +30 give ungated MLA (y = W_o õ); -30 give y ~ 0."""
    inp = tiny(gate_mode=gate_mode)
    inp["W_g"] = np.zeros_like(inp["W_g"])
    p = oracle.params(inp)
    for b, check in ((30.0, "open"), (-30.0, "closed")):
        p["b_g"] = np.full_like(p["b_g"], b)
        out = oracle.prefill(p, inp["x"], inp["lengths"])
        ungated = out["o_tilde"] @ p["W_o"].T
        if check == "open":
            assert np.linalg.norm(out["y"] - ungated) <= 1e-12 * np.linalg.norm(ungated)
        else:
            assert np.linalg.norm(out["y"]) <= 1e-12 * np.linalg.norm(ungated)


def test_per_head_gate_zero_weights_scales_heads_by_sigmoid_bias():
    inp = tiny(gate_mode="head")
    inp["W_g"] = np.zeros_like(inp["W_g"])
    inp["b_g"] = np.array([-1.0, 2.0])
    p = oracle.params(inp)
    out = oracle.prefill(p, inp["x"], inp["lengths"])
    o = out["o"]
    s = 1.0 / (1.0 + np.exp(-np.array([-1.0, 2.0])))
    np.testing.assert_allclose(out["gated"].reshape(o.shape), o * s[None, :, None], rtol=1e-14)


@pytest.mark.parametrize("d_rope", [0, 2])
def test_absorbed_equals_explicit(d_rope):
    inp = tiny(d_rope=d_rope, lengths=(5, 2))
    p = oracle.params(inp)
    a = oracle.prefill(p, inp["x"], inp["lengths"])
    b = oracle.prefill(p, inp["x"], inp["lengths"], absorbed=True)
    np.testing.assert_allclose(a["y"], b["y"], rtol=1e-12, atol=1e-14)
    d = tiny_decode(d_rope=d_rope)
    p = oracle.params(d)
    a = oracle.decode(p, d["x"], d["past"])
    b = oracle.decode(p, d["x"], d["past"], absorbed=True)
    np.testing.assert_allclose(a["y"], b["y"], rtol=1e-12, atol=1e-14)


def test_decode_equals_last_prefill_row():
    """A decode step over the cache a prefill would have written equals the
    prefill's last row (same definitions, two entry points)."""
    inp = tiny(d_rope=2, lengths=(6,))
    p = oracle.params(inp)
    full = oracle.prefill(p, inp["x"], [6])
    past = np.concatenate([full["c"][:5], full["kR"][:5]], axis=1)
    dec = oracle.decode(p, inp["x"][5:6], [past])
    np.testing.assert_allclose(dec["y"][0], full["y"][5], rtol=1e-12, atol=1e-14)


def test_uniform_attention_when_query_is_zero():
    inp = tiny(lengths=(6,))
    inp["W_q"] = np.zeros_like(inp["W_q"])
    p = oracle.params(inp)
    out = oracle.prefill(p, inp["x"], [6])
    c = out["c"]
    for h in range(2):
        v = c @ p["W_v"][h].T
        mean = np.cumsum(v, 0) / np.arange(1, 7)[:, None]
        np.testing.assert_allclose(out["o"][:, h], mean, rtol=1e-13, atol=1e-15)


def test_constant_cache_gives_wv_c():
    d = tiny_decode(lens=(5,))
    p = oracle.params(d)
    x = np.asarray(d["x"], float)
    c_new = p["W_c"] @ x[0]
    past = [np.tile(c_new, (4, 1))]
    out = oracle.decode(p, x, past)
    for h in range(2):
        np.testing.assert_allclose(out["o"][0, h], p["W_v"][h] @ c_new, rtol=1e-13)


def test_causality_future_tokens_do_not_change_past_rows():
    inp = tiny(lengths=(6,))
    p = oracle.params(inp)
    y0 = oracle.prefill(p, inp["x"], [6])["y"]
    x2 = np.array(inp["x"], float)
    x2[4:] += 3.0
    y1 = oracle.prefill(p, x2, [6])["y"]
    assert np.array_equal(y0[:4], y1[:4])
    assert not np.allclose(y0[4:], y1[4:])


def test_rope_closed_forms():
    base = 10000.0
    v = np.array([1.0, 0.0])
    for pos in (0, 1, 5, 1000):                       # d_R = 2: angle = pos radians
        np.testing.assert_allclose(oracle.rope(v, np.array(pos), base),
                                   [math.cos(pos), math.sin(pos)], rtol=1e-14, atol=1e-15)
    v4 = np.array([0.0, 0.0, 1.0, 0.0])               # d_R = 4: pair 1 angle = pos * 0.01
    np.testing.assert_allclose(oracle.rope(v4, np.array(7), base),
                               [0, 0, math.cos(0.07), math.sin(0.07)], atol=1e-15)
    rng = np.random.default_rng(0)
    u = rng.standard_normal((3, 64))
    np.testing.assert_array_equal(oracle.rope(u, np.zeros(3), base), u)
    r = oracle.rope(u, np.array([3, 17, 131071]), base)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(u, axis=1), rtol=1e-13)


def test_rope_scores_depend_on_offset_only():
    """q^R(t) . k^R(s) is unchanged when both positions shift by the same amount."""
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for t, s, d in ((10, 3, 100), (0, 0, 131000), (5000, 17, 7)):
        a = oracle.rope(q, np.array(t), 1e4) @ oracle.rope(k, np.array(s), 1e4)
        b = oracle.rope(q, np.array(t + d), 1e4) @ oracle.rope(k, np.array(s + d), 1e4)
        assert abs(a - b) < 1e-11 * max(1.0, abs(a))


def test_rope_branch_closed_form_in_attention():
    """NoPE branch switched off (W_q = 0): the scores come from the decoupled
    RoPE key alone. With unit vectors of d_R = 2 at angle 0 the score of key s
    for the query at t is scale * cos(t - s)."""
    d = tiny_decode(d_rope=2, lens=(5,))
    p = oracle.params(d)
    p["W_q"] = np.zeros_like(p["W_q"])
    x = np.zeros((1, 6)); x[0, 0] = 1.0
    p["W_qr"] = np.zeros_like(p["W_qr"]); p["W_qr"][0, 0] = 1.0; p["W_qr"][2, 0] = 1.0
    p["W_kr"] = np.zeros_like(p["W_kr"]); p["W_kr"][0, 0] = 1.0
    past = np.zeros((4, 6))
    past[:, :4] = np.random.default_rng(3).standard_normal((4, 4))
    for s in range(4):                              # cached k^R_s = RoPE((1,0), s)
        past[s, 4:] = [math.cos(s), math.sin(s)]
    out = oracle.decode(p, x, [past])
    t = 4
    C = np.concatenate([past[:, :4], (p["W_c"] @ x[0])[None]])
    z = p["scale"] * np.cos(t - np.arange(5))
    a = np.exp(z - z.max()); a /= a.sum()
    for h in range(2):
        np.testing.assert_allclose(out["o"][0, h], p["W_v"][h] @ (a @ C), rtol=1e-13)


def test_nope_decode_invariant_to_cache_row_order():
    d = tiny_decode(lens=(6,))
    p = oracle.params(d)
    y0 = oracle.decode(p, d["x"], d["past"])["y"]
    perm = np.random.default_rng(0).permutation(5)
    y1 = oracle.decode(p, d["x"], [d["past"][0][perm]])["y"]
    np.testing.assert_allclose(y0, y1, rtol=1e-13)


def test_linearity_in_wo_and_wv():
    inp = tiny()
    p = oracle.params(inp)
    y = oracle.prefill(p, inp["x"], inp["lengths"])["y"]
    p2 = dict(p, W_o=2.5 * p["W_o"])
    np.testing.assert_allclose(oracle.prefill(p2, inp["x"], inp["lengths"])["y"], 2.5 * y, rtol=1e-13)
    p3 = dict(p, W_v=-0.5 * p["W_v"])
    np.testing.assert_allclose(oracle.prefill(p3, inp["x"], inp["lengths"])["y"], -0.5 * y, rtol=1e-13)


def test_gate_never_changes_attention_weights():
    inp = tiny(lengths=(6,))
    p = oracle.params(inp)
    pr = oracle.project(p, inp["x"], np.arange(6))
    _, a = oracle.attention_explicit(p, 1, pr["q"][:, 1], pr["qR"][:, 1], pr["c"], pr["kR"],
                                     np.arange(6), return_weights=True)
    p2 = dict(p, W_g=np.random.default_rng(9).standard_normal(p["W_g"].shape))
    pr2 = oracle.project(p2, inp["x"], np.arange(6))
    _, a2 = oracle.attention_explicit(p2, 1, pr2["q"][:, 1], pr2["qR"][:, 1], pr2["c"],
                                      pr2["kR"], np.arange(6), return_weights=True)
    assert np.array_equal(a, a2)


# ---------------------------------------------------------------------------
# subset evaluation: the large-case parity tests ask the oracle for a few rows,
# sequences or heads; each answer must equal the matching slice of the full one
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d_rope", [0, 2])
def test_prefill_row_subset_equals_full_rows(d_rope):
    inp = tiny(d_rope=d_rope, lengths=(5, 7, 4))
    p = oracle.params(inp)
    full = oracle.prefill(p, inp["x"], inp["lengths"])
    rows = {0: [4, 0, 2], 1: [6], 2: []}
    sub = oracle.prefill(p, inp["x"], inp["lengths"], rows=rows)
    want = np.array([0, 2, 4, 5 + 6])
    assert np.array_equal(sub["index"], want)
    # equal up to the summation order BLAS picks for a different number of rows
    for k in ("q", "qR", "glogit", "o", "o_tilde", "gated", "y"):
        np.testing.assert_allclose(sub[k], full[k][want], rtol=1e-13, atol=1e-15, err_msg=k)
    # the whole cache side is always evaluated in full
    np.testing.assert_array_equal(sub["c"], full["c"])


@pytest.mark.parametrize("absorbed", [False, True])
def test_decode_sequence_and_head_subsets_equal_full(absorbed):
    d = tiny_decode(d_rope=2, lens=(1, 4, 7, 3))
    p = oracle.params(d)
    full = oracle.decode(p, d["x"], d["past"], absorbed=absorbed)
    seqs, heads = [3, 1], [1]
    sub = oracle.decode(p, d["x"], d["past"], seqs=seqs, heads=heads, absorbed=absorbed)
    np.testing.assert_allclose(sub["o"], full["o"][np.ix_(seqs, heads)], rtol=1e-13, atol=1e-15)
    assert "y" not in sub   # y needs every head
    sub = oracle.decode(p, d["x"], d["past"], seqs=seqs, absorbed=absorbed)
    for k in ("o", "o_tilde", "gated", "y"):
        np.testing.assert_allclose(sub[k], full[k][seqs], rtol=1e-13, atol=1e-15, err_msg=k)


# ---------------------------------------------------------------------------
# printed numbers ([MLA-notes] §5.3, §7, 题1, 题5)
# ---------------------------------------------------------------------------

def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            fields, cite = line.split("|", 1)
            yield fields.split(), cite.strip()


def test_kv_accounting_matches_printed_values():
    n = 0
    for f, cite in _golden("kv_accounting.txt"):
        mech, h, g, dh, dc, dr, layers, nb, want = f[0], *map(int, f[1:])
        got = oracle.kv_bytes_per_token(mech, h, g, dh, dc, dr, layers, nb)
        assert got == want, cite
        n += 1
    assert n == 6


def test_kv_context_totals_match_printed_values():
    for f, cite in _golden("kv_context_totals.txt"):
        mech, h, g, dh, dc, dr, layers, nb, ctx = f[0], *map(int, f[1:9])
        printed = f[9]
        gib = oracle.kv_bytes_per_token(mech, h, g, dh, dc, dr, layers, nb) * ctx / 2 ** 30
        decimals = len(printed.split(".")[1]) if "." in printed else 0
        assert round(gib, decimals) == float(printed), cite


def test_mla_cache_is_independent_of_heads_and_about_57x_smaller():
    mla = oracle.kv_bytes_per_token("MLA", d_c=512, d_r=64, layers=60, bytes=2)
    for h in (1, 16, 128):
        assert oracle.kv_bytes_per_token("MLA", h=h, d_c=512, d_r=64, layers=60, bytes=2) == mla
    mha = oracle.kv_bytes_per_token("MHA", h=128, d_h=128, layers=60, bytes=2)
    assert round(mha / mla) == 57
    assert oracle.kv_elements_per_token("MLA", d_c=512, d_r=64) == 4.5 * 128   # ≈ 9/2 d_h


def test_workload_cache_rows():
    assert synth.workload("decode_long_rope").row == 576
    assert synth.workload("decode_b32").row == 512


# ---------------------------------------------------------------------------
# planted mistakes: every one must break at least one pin above
# ---------------------------------------------------------------------------

def _pins_fail(fns):
    failed = 0
    for fn in fns:
        try:
            fn()
        except Exception:       # a failed assertion or a crash both expose the mistake
            failed += 1
    return failed


def _run_all_pins():
    return _pins_fail([
        lambda: test_bruteforce_prefill(0, "channel"),
        lambda: test_bruteforce_prefill(2, "head"),
        test_two_token_closed_form,
        test_scale_is_inverse_sqrt_dh,
        test_single_token_gives_v0,
        lambda: test_gate_saturation("channel"),
        lambda: test_gate_saturation("head"),
        test_per_head_gate_zero_weights_scales_heads_by_sigmoid_bias,
        test_causality_future_tokens_do_not_change_past_rows,
        test_rope_closed_forms,
        test_rope_branch_closed_form_in_attention,
        lambda: test_softmax_rows_sum_to_one_and_causal(2),
    ])


MUTANTS = {
    "sigmoid_sign": ("sigmoid", lambda orig: (lambda z: orig(-np.asarray(z)))),
    "no_causal_mask": ("attention_explicit", None),
    "scale_sqrt_dc": ("params", lambda orig: (lambda inp: dict(orig(inp), scale=1.0 / math.sqrt(inp["workload"].d_c + inp["workload"].d_rope)))),
    "rope_negative_angle": ("rope", lambda orig: (lambda v, pos, base: orig(v, -np.asarray(pos), base))),
    "rope_dropped": ("rope", lambda orig: (lambda v, pos, base: np.asarray(v, float))),
    "gate_head_tiled": ("gate", None),
    "value_from_key_weights": ("head_kv", lambda orig: (lambda p, h, C: (C @ p["W_k"][h].T, C @ p["W_k"][h].T))),
}


def _mutant_attention_no_mask(p, h, q, qR, C, KR, q_pos, return_weights=False):
    K, V = core.head_kv(p, h, C)
    z = p["scale"] * (q @ K.T + (qR @ KR.T if KR.shape[1] else 0.0))
    a = core._softmax_rows(z)
    return (a @ V, a) if return_weights else a @ V


def _mutant_gate_tiled(p, glogit, o_tilde):
    g = core.sigmoid(glogit)
    if p["gate_mode"] == "channel":
        return g * o_tilde
    return np.tile(g, (1, p["d_h"])) * o_tilde      # wrong broadcast order


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, make = MUTANTS[name]
    if name == "no_causal_mask":
        new = _mutant_attention_no_mask
    elif name == "gate_head_tiled":
        new = _mutant_gate_tiled
    else:
        new = make(getattr(core, attr))
    monkeypatch.setattr(core, attr, new)
    monkeypatch.setattr(oracle, attr, new, raising=False)
    assert _run_all_pins() >= 1, f"planted mistake {name} passed every pin"


# ---------------------------------------------------------------------------
# the rescale-path GPU inputs have teeth: simulated on the CPU with the
# kernels' tiling and raise rule, dropping the rescale of the partial output
# moves the result far outside the bf16 tolerance
# ---------------------------------------------------------------------------

def _online_latent(z2, C, tile=128, raise_by=8.0, rescale=True):
    """sum_s 2^(z2_s - m) c_s / sum_s 2^(z2_s - m) by tiles, raising the running
    max m only by more than raise_by; with rescale=False the accumulated sum is
    not multiplied by 2^(m_old - m_new) when m rises (the mistake to expose)."""
    m, l, O = -np.inf, 0.0, np.zeros(C.shape[1])
    for t0 in range(0, len(z2), tile):
        zt, Ct = z2[t0:t0 + tile], C[t0:t0 + tile]
        if t0 == 0 or zt.max() > m + raise_by:
            mn = max(m, zt.max())
            alpha = 0.0 if m == -np.inf else 2.0 ** (m - mn)
            l *= alpha
            if rescale:
                O *= alpha
            m = mn
        p = 2.0 ** (zt - m)
        l += p.sum()
        O += p @ Ct
    return O / l


def test_peaked_decode_input_needs_the_rescale():
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from gpu_pipeline import small_decode
    from rescale_inputs import decode_scores_log2, plant_decode
    inp = small_decode("decode_b32", 2, [2000, 1500])
    inp = plant_decode(inp, [(b, 300 + 61 * h, h, 16.0) for b in range(2) for h in range(16)])
    dc = inp["workload"].d_c
    worst = 0.0
    for b in range(2):
        z = decode_scores_log2(inp, b)
        p = oracle.params(inp)
        c_new = oracle.project_latent(p, np.asarray(inp["x"], float)[b:b + 1], np.array([len(inp["past"][b])]))["c"]
        C = np.concatenate([np.asarray(inp["past"][b], float)[:, :dc], c_new])
        for h in range(z.shape[0]):
            exact = oracle.core._softmax_rows((z[h] * math.log(2.0))[None])[0] @ C
            good = _online_latent(z[h], C)
            np.testing.assert_allclose(good, exact, rtol=1e-9, atol=1e-12)
            bad = _online_latent(z[h], C, rescale=False)
            worst = max(worst, np.linalg.norm(bad - exact) / np.linalg.norm(exact))
    assert worst > 1.0, worst


# ---------------------------------------------------------------------------
# FP8 latent cache: the stored value is cache_scale * e4m3(c / cache_scale)
# ---------------------------------------------------------------------------

def _e4m3_table():
    """Every finite E4M3 value, decoded from its bits by the format's
    definition: sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals at
    exponent 0, and the all-ones code (S.1111.111) left out as NaN."""
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(-mag if s else mag)
    return np.array(sorted(set(vals)))


def test_e4m3_rounding_matches_the_format_definition():
    table = _e4m3_table()
    assert table.max() == 448.0 and np.min(np.abs(table[table != 0])) == 2.0 ** -9
    np.testing.assert_array_equal(oracle.round_e4m3(table), table)      # representable values are fixed
    # midpoints between neighbours go to the even code; positive magnitudes in
    # increasing order are the codes 0x00, 0x01, ... so a code's parity is its index's
    pos = table[table >= 0]
    mids = (pos[1:] + pos[:-1]) / 2
    got = oracle.round_e4m3(mids)
    want = np.where(np.arange(len(mids)) % 2 == 0, pos[:-1], pos[1:])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(oracle.round_e4m3(-mids), -want)
    assert oracle.round_e4m3(np.array([500.0, -1e9]))[0] == 448.0 and oracle.round_e4m3(np.array([-1e9]))[0] == -448.0
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000) * 50
    q = oracle.round_e4m3(x)
    # the nearest representable value: no table entry is closer
    idx = np.searchsorted(table, x)
    lo = table[np.clip(idx - 1, 0, len(table) - 1)]
    hi = table[np.clip(idx, 0, len(table) - 1)]
    assert np.all(np.abs(q - x) <= np.minimum(np.abs(lo - x), np.abs(hi - x)) + 1e-12)


def test_e4m3_rounding_agrees_with_torch_float8():
    import torch
    x = np.random.default_rng(1).standard_normal(200000).astype(np.float32) * 40
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_e4m3(x), ref)


def test_fp8_cache_rows_and_their_error_bound():
    w = synth.Workload(name="f8", mode="decode", dtype="bf16", batch=2, d_model=16, n_heads=2, d_h=4, d_c=8,
                       cache_fp8=True, cache_scale=1 / 32)
    inp = synth.generate(w, seed=0, lengths=np.array([5, 9]))
    p = oracle.params(inp)
    for rows in inp["past"]:                                             # past rows are already stored values
        np.testing.assert_array_equal(oracle.cache_store(p, rows.astype(np.float64)), rows)
    c = oracle.latent(p["W_c"], np.asarray(inp["x"], float))
    stored = oracle.project_latent(p, inp["x"], np.array([4, 8]))["c"]
    s = p["cache_scale"]
    assert np.all(np.abs(stored - c) <= 2.0 ** -4 * np.abs(c) + 2.0 ** -10 * s)
    codes = stored / s
    np.testing.assert_array_equal(oracle.round_e4m3(codes), codes)
    # a bf16 cache stores values as they are
    assert oracle.cache_store(dict(p, cache_fp8=False), c) is c
