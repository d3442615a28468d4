"""Hard top-k, binary and ternary per-head gates ("Gated Multi-head Latent
Attention", "Variants / Extensions": Hard Gating, Quantized Gates). Decode
skips every head whose gate is 0; prefill and the fp32 path multiply by the
gate value. Each case first checks on the CPU that no token's gate decision
lies within 1e-3 of its cut (the k-th / (k+1)-th largest logits, z = 0,
z = -+ln 3), so the fp32 logits of the GPU and the fp64 ones of the oracle
decide alike; then the CUDA path is compared with the fp64 oracle."""
import math

import numpy as np
import pytest

import oracle
import synth
from gpu_pipeline import BF16_TOL, F32_TOL, assert_close, run_decode, run_prefill, small_decode

pytestmark = pytest.mark.gpu
MARGIN = 1e-3


def decision_margin(inp):
    """Smallest distance of a gate logit to its decision cut, over all tokens."""
    w = inp["workload"]
    p = oracle.params(inp)
    x = np.asarray(inp["x"], np.float64)
    z = x @ p["W_g"].T + (p["b_g"] if p["b_g"] is not None else 0.0)
    if w.gate_mode == "head_topk":
        s = -np.sort(-z, axis=1)
        return float(np.min(s[:, w.gate_topk - 1] - s[:, w.gate_topk])) if w.gate_topk < w.n_heads else np.inf
    if w.gate_mode == "head_binary":
        return float(np.min(np.abs(z)))
    if w.gate_mode == "head_ternary":
        c = math.log(3.0)
        return float(min(np.min(np.abs(z - c)), np.min(np.abs(z + c))))
    raise ValueError(w.gate_mode)


def first_clear_seed(make):
    for seed in range(50):
        inp = make(seed)
        if decision_margin(inp) > MARGIN:
            return inp
    raise AssertionError("no seed gives clear gate decisions")


def _check_decode(inp):
    gpu = run_decode(inp)
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    g = oracle.head_gate_values(oracle.params(inp), ref["glogit"])
    assert (g == 0).any() and (g != 0).any()          # some heads skipped, some kept
    assert_close(gpu["o"], ref["gated"], BF16_TOL, "gated o")
    assert_close(gpu["y"], ref["y"], BF16_TOL, "y")
    # skipped heads give exactly 0
    H, dh = inp["workload"].n_heads, inp["workload"].d_h
    o = gpu["o"].reshape(len(g), H, dh)
    assert np.all(o[g == 0] == 0.0)


@pytest.mark.parametrize("mode,k", [("head_topk", 8), ("head_binary", 0), ("head_ternary", 0)])
def test_decode_paged_32_heads_hard_gates(mode, k):
    lens = [1, 63, 64, 65, 300, 1000, 2500, 129]
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("decode_paged_head", batch=8, gate_mode=mode, gate_topk=k), seed=s, lengths=np.array(lens)))
    _check_decode(inp)


def test_decode_topk_16_of_16_heads_is_the_ungated_path():
    inp = small_decode("decode_b32", 3, [10, 200, 129], gate_mode="head_topk", gate_topk=16)
    gpu = run_decode(inp)
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    assert_close(gpu["o"], ref["o_tilde"], BF16_TOL, "o (all gates 1)")


def test_decode_rope_128_heads_top_32():
    """Top-32 of 128 heads: the attention runs one 32-head group instead of two
    64-head groups, so every cached row is read once."""
    lens = [1, 129, 1500, 700]
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("decode_long_rope", batch=4, d_model=512, gate_mode="head_topk", gate_topk=32,
                       gate_bias=True), seed=s, lengths=np.array(lens)))
    _check_decode(inp)


def test_decode_split_k_with_skipped_heads():
    """A long sequence over many CTAs (split-K merge) with binary gates."""
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("decode_b32", batch=2, gate_mode="head_binary", gate_bias=True), seed=s,
        lengths=np.array([30000, 40])))
    _check_decode(inp)


@pytest.mark.parametrize("mode,k", [("head_topk", 2), ("head_binary", 0), ("head_ternary", 0)])
def test_prefill_bf16_hard_gates(mode, k):
    lens = [300, 129, 1]
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("prefill_b4_s4096", batch=3, d_model=512, n_heads=4, gate_mode=mode, gate_topk=k),
        seed=s, lengths=np.array(lens)))
    gpu = run_prefill(inp)
    ref = oracle.prefill(oracle.params(inp), inp["x"], inp["lengths"])
    assert_close(gpu["o"], ref["gated"], BF16_TOL, "gated o")
    assert_close(gpu["y"], ref["y"], BF16_TOL, "y")


def test_prefill_fp32_ternary_gates():
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("tiny_prefill_f32", batch=2, gate_mode="head_ternary", gate_bias=True), seed=s,
        lengths=np.array([64, 17])))
    gpu = run_prefill(inp)
    ref = oracle.prefill(oracle.params(inp), inp["x"], inp["lengths"])
    assert_close(gpu["y"], ref["y"], F32_TOL, "y")


def test_gate_out_applies_hard_gates_to_ungated_o():
    """gmla_gate_out given ungated o and the logits applies the same gate values."""
    import torch
    inp = first_clear_seed(lambda s: synth.generate(
        synth.workload("decode_paged_head", batch=5, gate_mode="head_topk", gate_topk=4), seed=s,
        lengths=np.array([5, 70, 300, 1, 900])))
    gpu = run_decode(inp)
    model = gpu["model"]
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    o_un = torch.from_numpy(ref["o_tilde"].astype(np.float32)).to("cuda", torch.bfloat16)
    g = torch.from_numpy(gpu["glogit"]).to("cuda")
    y = model.gate_out(o_un, g).float().cpu().numpy()
    model.sync_status()
    assert_close(y, ref["y"], BF16_TOL, "y from ungated o")
