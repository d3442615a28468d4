"""Parity on inputs that force the online-softmax rescale branches.

The decode and prefill attention kernels keep a running max per (row, head)
and raise it, rescaling the partial output held in tensor memory, only when a
later tile beats it by more than 8 in log2 units; the split-K merge rescales
partials whose maxima differ. The softmax these must reproduce is the causal
softmax over s <= t of "Gated MLA 计算公式：输出门与 FFN 的区别" §二. Each case
plants keys aligned with chosen heads' absorbed queries (see rescale_inputs),
asserts first, on the CPU, that its input makes the branch run (the counts come
from fp64 scores and the kernels' tiling), then compares the CUDA path with
the fp64 oracle at the bf16 tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_pipeline import BF16_TOL, assert_close, run_decode, run_prefill, small_decode
from rescale_inputs import decode_raises, plant_decode, plant_prefill, prefill_raises

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _check_decode(inp, seqs=None):
    gpu = run_decode(inp)
    p = oracle.params(inp)
    seqs = list(range(inp["workload"].batch)) if seqs is None else seqs
    ref = oracle.decode(p, inp["x"], inp["past"], seqs=seqs)
    assert_close(gpu["o"][seqs], ref["gated"], BF16_TOL, "gated o")
    assert_close(gpu["y"][seqs], ref["y"], BF16_TOL, "y")


def decode_plan(lens, H, seed, per_seq=4, score=16.0):
    """Per sequence, `per_seq` heads each get one planted row in a tile after the
    first (positions spread over the cache)."""
    rng = np.random.default_rng(seed)
    plan = []
    for b, L in enumerate(lens):
        for h in rng.choice(H, per_seq, replace=False):
            plan.append((b, int(rng.integers(256, L - 1)), int(h), score))
    return plan


def test_decode_rescale_contiguous_16_heads():
    lens = np.random.default_rng(3).integers(900, 3000, 32).tolist()
    inp = small_decode("decode_b32", 32, lens)
    inp = plant_decode(inp, decode_plan(lens, 16, 0))
    raises, _ = decode_raises(inp, _sms())
    assert raises >= 40, raises
    _check_decode(inp)


def test_decode_rescale_paged_32_heads_per_head_gate():
    lens = np.random.default_rng(4).integers(700, 2500, 24).tolist()
    inp = small_decode("decode_paged_head", 24, lens)
    inp = plant_decode(inp, decode_plan(lens, 32, 1))
    raises, _ = decode_raises(inp, _sms())
    assert raises >= 30, raises
    _check_decode(inp)


def test_decode_rescale_rope_128_heads():
    lens = np.random.default_rng(5).integers(1500, 4000, 6).tolist()
    inp = small_decode("decode_long_rope", 6, lens, d_model=512)
    inp = plant_decode(inp, decode_plan(lens, 128, 2, per_seq=16))
    raises, _ = decode_raises(inp, _sms())
    assert raises >= 30, raises
    _check_decode(inp)


def test_decode_merge_of_far_apart_segment_maxima():
    """One 40000-token sequence spread over every CTA; every head has a planted
    row in one segment that beats every other segment's max by far, so the
    merge weights partials by 2^0 and by 2^-(large)."""
    inp = small_decode("decode_b32", 2, [40000, 300])
    plan = [(0, 23456 + 97 * h, h, 20.0) for h in range(16)]
    inp = plant_decode(inp, plan)
    _, gap = decode_raises(inp, _sms())
    assert gap >= 12, gap
    _check_decode(inp)


def test_prefill_rescale_planted_keys():
    w = synth.workload("prefill_b4_s4096", batch=3, d_model=1024, n_heads=4)
    lens = [700, 300, 129]
    inp = synth.generate(w, seed=8, lengths=np.array(lens))
    rng = np.random.default_rng(9)
    plan = []
    for b, L in enumerate(lens):
        for _ in range(12 if L > 256 else 2):
            t = int(rng.integers(128, L))
            s = int(rng.integers(max(1, (t // 128) * 128 - 60), t))    # often in t's own or a late tile
            if s >= 128 or t >= 256:
                plan.append((b, s, t, int(rng.integers(0, 4)), 16.0))
    inp = plant_prefill(inp, plan)
    raises = prefill_raises(inp)
    assert raises >= 10, raises
    gpu = run_prefill(inp)
    ref = oracle.prefill(oracle.params(inp), inp["x"], inp["lengths"])
    assert_close(gpu["o"], ref["gated"], BF16_TOL, "gated o")
    assert_close(gpu["y"], ref["y"], BF16_TOL, "y")
