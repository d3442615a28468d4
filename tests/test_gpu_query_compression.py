"""Low-rank query ("精读笔记 03" §5.1: c^Q = W^DQ h, q = W^UQ c^Q; §5.2:
q^R = RoPE(W^QR c^Q)): gmla_latent_project runs a second GEMM over c^Q. The
whole path is compared with the fp64 oracle, whose compressed query is pinned
to its full-rank form by the CPU tests."""
import numpy as np
import pytest

import oracle
import synth
from gpu_pipeline import BF16_TOL, F32_TOL, assert_close, run_decode, run_prefill, small_decode
from test_gpu_decode import _check as check_decode
from test_gpu_prefill import _check as check_prefill

pytestmark = pytest.mark.gpu


def test_decode_compressed_query_16_heads():
    inp = small_decode("decode_b32", 5, [1, 127, 300, 1000, 2500], d_cq=384)
    assert inp["W_q"] is None
    check_decode(inp, run_decode(inp))


def test_decode_compressed_query_rope_128_heads():
    inp = small_decode("decode_long_rope", 3, [1, 129, 1500], d_model=512, d_cq=256)
    check_decode(inp, run_decode(inp))


def test_decode_compressed_query_batch_beyond_one_token_tile():
    """40 tokens: the few-token GEMMs use a wider token tile and K splits."""
    lens = np.random.default_rng(2).integers(1, 900, 40).tolist()
    inp = small_decode("decode_paged_head", 40, lens, d_cq=512)
    check_decode(inp, run_decode(inp))


def test_prefill_compressed_query_bf16():
    """556 tokens: the many-token orientation for both GEMMs."""
    w = synth.workload("prefill_b4_s4096", batch=3, d_model=512, n_heads=4, d_cq=256)
    inp = synth.generate(w, seed=4, lengths=np.array([300, 129, 127]))
    check_prefill(inp, run_prefill(inp), BF16_TOL)


def test_prefill_compressed_query_fp32():
    w = synth.workload("tiny_prefill_f32", batch=2, d_cq=96)
    inp = synth.generate(w, seed=5, lengths=np.array([64, 33]))
    check_prefill(inp, run_prefill(inp), F32_TOL)
