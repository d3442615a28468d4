"""FP8 (E4M3) latent cache: one byte per cached element, a code of value /
cache_scale (one fp32 scale for the cache). gmla_latent_project writes the
new token's codes; gmla_decode reads the codes directly in kind::f8f6f4
tensor-core products, with the absorbed query and the softmax weights carried
as hi + lo e4m3 pairs. The oracle's quantised-cache mode stores the same codes
(its E4M3 rounding is pinned to the format's definition and to torch's float8
conversion on the CPU) and then computes in fp64; the GPU must match it at the
bf16 tolerances."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_pipeline import BF16_TOL, assert_close, run_decode

pytestmark = pytest.mark.gpu


def _fp8(name, B, lens, seed=0, **kw):
    w = synth.workload(name, batch=B, cache_fp8=True, cache_scale=1 / 64, **kw)
    return synth.generate(w, seed=seed, lengths=np.array(lens))


def _check(inp, seqs=None):
    w = inp["workload"]
    gpu = run_decode(inp)
    p = oracle.params(inp)
    seqs = list(range(w.batch)) if seqs is None else seqs
    ref = oracle.decode(p, inp["x"], inp["past"], seqs=seqs)
    assert_close(gpu["o"][seqs], ref["gated"], BF16_TOL, "gated o")
    assert_close(gpu["y"][seqs], ref["y"], BF16_TOL, "y")
    # the new token's stored codes: equal, except where c / scale lies within a
    # hair of a rounding boundary (the GPU rounds its fp32 c, the oracle its fp64 c)
    cache = gpu["cache"]
    for b in seqs[:4]:
        L = int(inp["lengths"][b])
        if cache.paged:
            ps = cache.data.shape[1]
            got = cache.data[int(cache.block_table[b, (L - 1) // ps]), (L - 1) % ps]
        else:
            got = cache.data[b, L - 1]
        got = got.float().cpu().numpy().astype(np.float64) * w.cache_scale
        want = ref["c"][b]
        diff = got != want
        assert diff.mean() < 0.01, diff.mean()
        assert np.all(np.abs(got - want)[diff] <= 2.0 ** -3 * np.abs(want[diff]) + 1e-12)
    return gpu


def test_fp8_cache_decode_tile_edges_16_heads():
    _check(_fp8("decode_b32", 5, [1, 127, 128, 129, 3000]))


def test_fp8_cache_decode_paged_32_heads_per_head_gate():
    _check(_fp8("decode_paged_head", 6, [1, 63, 64, 65, 700, 2500]))


def test_fp8_cache_decode_many_segments():
    _check(_fp8("decode_b32", 2, [40000, 3]))


def test_fp8_cache_decode_64_heads_in_groups_of_32():
    _check(_fp8("decode_b32", 3, [300, 1500, 70], n_heads=64, d_model=1024))


def test_fp8_cache_decode_hard_top_k():
    _check(_fp8("decode_paged_head", 4, [900, 2000, 130, 5], gate_mode="head_topk", gate_topk=8))


def test_fp8_cache_full_batch32_shape():
    """The batch-32 decode's lengths and shapes over an FP8 cache."""
    w = synth.workload("decode_b32", cache_fp8=True, cache_scale=1 / 64)
    inp = synth.generate(w, seed=0)
    seqs = sorted(np.random.default_rng(1).choice(32, 6, replace=False).tolist())
    _check(inp, seqs=seqs)
