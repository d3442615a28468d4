"""Prefill parity: latent_project -> prefill (explicit K/V rebuild + causal
flash attention with the gate fused) -> gate_out, against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from gpu_pipeline import BF16_TOL, F32_TOL, assert_close, run_prefill

pytestmark = pytest.mark.gpu


def _check(inp, gpu, tol, rows=None):
    w = inp["workload"]
    p = oracle.params(inp)
    ref = oracle.prefill(p, inp["x"], inp["lengths"], rows=rows)
    idx = ref["index"]
    dh = w.d_h
    assert_close(gpu["q"][idx][:, :, :dh], ref["q"], tol, "q")
    assert_close(gpu["glogit"][idx], ref["glogit"], tol, "gate logits")
    assert_close(gpu["o"][idx], ref["gated"], tol, "gated o")
    assert_close(gpu["y"][idx], ref["y"], tol, "y")
    # cached latents written by latent_project
    cache = gpu["cache"].data.float().cpu().numpy()
    starts = np.concatenate([[0], np.cumsum(inp["lengths"])])
    for b, L in enumerate(inp["lengths"]):
        assert_close(cache[b, :L, :w.d_c], ref["c"][starts[b]:starts[b] + L], tol, f"cached latents seq {b}")
        if w.d_rope:
            assert_close(cache[b, :L, w.d_c:], ref["kR"][starts[b]:starts[b] + L], tol, f"cached k^R seq {b}")
    if w.d_rope:
        assert_close(gpu["q"][idx][:, :, dh:], ref["qR"], tol, "q^R (rotated)")


def test_prefill_tiny_fp32_full_config():
    """The tiny fp32 workload (batch 1, seq 64, d_model 256, H 4, d_h 64, d_c 64) at 1e-4."""
    inp = synth.generate(synth.workload("tiny_prefill_f32"), seed=0)
    _check(inp, run_prefill(inp), F32_TOL)


def test_prefill_fp32_ragged_batch():
    inp = synth.generate(synth.workload("tiny_prefill_f32", batch=3), seed=1, lengths=np.array([1, 17, 64]))
    _check(inp, run_prefill(inp), F32_TOL)


def test_prefill_bf16_ragged_tiles():
    """Lengths 1, 127, 128, 129, 300: tile edges and ragged tails, 4 heads."""
    inp = synth.generate(synth.workload("prefill_b4_s4096", batch=5, d_model=512, n_heads=4), seed=0,
                         lengths=np.array([1, 127, 128, 129, 300]))
    _check(inp, run_prefill(inp), BF16_TOL)


def test_prefill_bf16_long_sequence_many_heads():
    inp = synth.generate(synth.workload("prefill_b4_s4096", batch=2, d_model=1024, n_heads=16), seed=2,
                         lengths=np.array([1000, 700]))
    _check(inp, run_prefill(inp), BF16_TOL)


def test_prefill_bf16_decoupled_rope_ragged():
    """Decoupled RoPE ("精读笔记 03" §5.2): scores add q^R . k^R with k^R read from
    the cache rows; lengths 1, 127, 128, 129, 300."""
    inp = synth.generate(synth.workload("prefill_b4_s4096", batch=5, d_model=512, n_heads=4, d_rope=64), seed=3,
                         lengths=np.array([1, 127, 128, 129, 300]))
    _check(inp, run_prefill(inp), BF16_TOL)


def test_prefill_bf16_decoupled_rope_long_positions():
    """A 1500-token prompt of the long-context shape (d_c 512 + RoPE 64, base
    10000) with 16 heads: angles of positions up to 1499."""
    inp = synth.generate(synth.workload("prefill_b4_s4096", batch=2, d_model=1024, n_heads=16, d_rope=64,
                                        gate_bias=False), seed=4, lengths=np.array([1500, 260]))
    _check(inp, run_prefill(inp), BF16_TOL)


def test_prefill_first_row_is_gated_v0():
    """Row t = 0 of every sequence attends only to itself: o = sigmoid(g) W_v c_0."""
    inp = synth.generate(synth.workload("prefill_b4_s4096", batch=3, d_model=512, n_heads=4), seed=3,
                         lengths=np.array([5, 1, 9]))
    gpu = run_prefill(inp)
    p = oracle.params(inp)
    starts = np.concatenate([[0], np.cumsum(inp["lengths"])])[:-1]
    x0 = np.asarray(inp["x"][starts], float)
    c0 = x0 @ p["W_c"].T
    v0 = np.einsum("hid,nd->nhi", p["W_v"], c0).reshape(len(starts), -1)
    g = oracle.sigmoid(x0 @ p["W_g"].T + p["b_g"])
    assert_close(gpu["o"][starts], g * v0, BF16_TOL, "row 0 = gated v_0")


@pytest.mark.slow
def test_prefill_full_config_sampled_rows():
    """The full bf16 prefill workload (batch 4 x 4096, d_model 7168, H 64);
    the oracle evaluates 12 seeded rows per sequence, always t = 0 and t = S-1."""
    w = synth.workload("prefill_b4_s4096")
    inp = synth.generate(w, seed=0)
    gpu = run_prefill(inp)
    rng = np.random.default_rng(0)
    rows = {b: sorted({0, w.seq_len - 1, *rng.choice(w.seq_len, 10, replace=False).tolist()})
            for b in range(w.batch)}
    _check(inp, gpu, BF16_TOL, rows=rows)
