"""Decode parity: the CUDA path (latent_project -> decode -> gate_out through the
C ABI) against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_pipeline import BF16_TOL, assert_close, metrics, run_decode, small_decode

pytestmark = pytest.mark.gpu


def _check(inp, gpu, seqs=None, absorbed=False, tol=BF16_TOL, check_cache=True):
    w = inp["workload"]
    p = oracle.params(inp)
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    ref = oracle.decode(p, inp["x"], inp["past"], seqs=seqs, absorbed=absorbed)
    H, dh = w.n_heads, w.d_h
    out = {}
    out["q"] = assert_close(gpu["q"][:, :, :dh], ref["q"], tol, "q")
    if w.d_rope:
        out["qR"] = assert_close(gpu["q"][:, :, dh:], ref["qR"], tol, "qR (rotated)")
    out["glogit"] = assert_close(gpu["glogit"], ref["glogit"], tol, "gate logits")
    out["o_gated"] = assert_close(gpu["o"][seqs], ref["gated"], tol, "gated o")
    out["y"] = assert_close(gpu["y"][seqs], ref["y"], tol, "y")
    if check_cache:
        cache = gpu["cache"]
        for b in seqs[:4]:
            L = int(inp["lengths"][b])
            if cache.paged:
                ps = cache.data.shape[1]
                page = int(cache.block_table[b, (L - 1) // ps])
                row = cache.data[page, (L - 1) % ps].float().cpu().numpy()
            else:
                row = cache.data[b, L - 1].float().cpu().numpy()
            assert_close(row[:w.d_c], ref["c"][b], tol, "cached latent of the new token")
            if w.d_rope:
                assert_close(row[w.d_c:], ref["kR"][b], tol, "cached rotated k^R")
    return out


def test_decode_contiguous_tile_edges():
    """Lengths 1, 127, 128, 129, 300: single token, tile boundary +-1, ragged tail."""
    inp = small_decode("decode_b32", 5, [1, 127, 128, 129, 300])
    _check(inp, run_decode(inp))


def test_decode_single_token_gives_gated_wv_c():
    """L = 1 everywhere: o^(h) = W_v^(h) c_0 exactly in the method; checks the
    whole chain with no softmax freedom."""
    inp = small_decode("decode_b32", 3, [1, 1, 1])
    _check(inp, run_decode(inp))


def test_decode_paged_per_head_gate():
    inp = small_decode("decode_paged_head", 6, [1, 63, 64, 65, 200, 1000])
    _check(inp, run_decode(inp))


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
def test_decode_paged_equals_contiguous(page_size):
    """Pages smaller than a 128-token tile are copied one per lane; pages of 128 or
    more hold whole tiles, copied as one box at the tile's offset in the page."""
    inp = small_decode("decode_b32", 4, [65, 300, 1, 1000])
    a = run_decode(inp, paged=False)
    w = inp["workload"].replace(paged=True, page_size=page_size)
    inp2 = dict(inp, workload=w)
    b = run_decode(inp2, paged=True)
    m = metrics(b["o"], a["o"])
    assert m["rel_l2"] < 1e-5, m


def test_decode_rope_128_heads():
    """128 heads (two 64-head groups), d_c 512 + decoupled RoPE d_R 64."""
    inp = small_decode("decode_long_rope", 3, [1, 129, 1500], d_model=512)
    _check(inp, run_decode(inp))


def test_decode_heads_not_multiple_of_16():
    inp = small_decode("decode_b32", 3, [5, 130, 260], n_heads=4, d_model=256)
    _check(inp, run_decode(inp))


def test_decode_head_dim_256():
    """d_h = 256: the query absorption takes W_k^(h) in boxes of 256 rows and K = 256
    (16 MMAs), and the W_v product spans two 128-row tiles per head."""
    inp = small_decode("decode_b32", 3, [5, 130, 700], n_heads=4, d_h=256, d_model=512)
    _check(inp, run_decode(inp))


def test_decode_more_than_128_sequences():
    """136 sequences: the query absorption takes its sequences in chunks of 128
    (the second chunk ragged), each chunk one column block of its MMA."""
    lens = [1 + (37 * b) % 300 for b in range(136)]
    inp = small_decode("decode_b32", 136, lens, n_heads=4, d_model=256)
    _check(inp, run_decode(inp), check_cache=False)


def test_decode_many_segments_per_sequence():
    """One long sequence spread over every CTA (split-K merge across ~148 partials)."""
    inp = small_decode("decode_b32", 2, [40000, 3])
    _check(inp, run_decode(inp))


def test_decode_zero_length_sequence_gives_zero():
    inp = small_decode("decode_b32", 3, [10, 20, 30])
    gpu = run_decode(inp)
    model, cache = gpu["model"], gpu["cache"]
    q = torch.from_numpy(gpu["q"]).to("cuda", torch.bfloat16)
    g = torch.from_numpy(gpu["glogit"]).to("cuda")
    lens = torch.tensor([10, 0, 30], dtype=torch.int32, device="cuda")
    o = model.decode(q, g, cache, lens)
    model.sync_status()
    o = o.float().cpu().numpy()
    assert np.all(o[1] == 0.0)
    np.testing.assert_allclose(o[[0, 2]], gpu["o"][[0, 2]], rtol=1e-2, atol=1e-3)


def test_decode_length_beyond_cache_reports_range():
    from gated_mla_b200 import _lib
    inp = small_decode("decode_b32", 2, [10, 20])
    gpu = run_decode(inp)
    model, cache = gpu["model"], gpu["cache"]
    q = torch.from_numpy(gpu["q"]).to("cuda", torch.bfloat16)
    lens = torch.tensor([10, cache.data.shape[1] + 5], dtype=torch.int32, device="cuda")
    model.decode(q, None, cache, lens)
    with pytest.raises(_lib.GmlaError) as e:
        model.sync_status()
    assert e.value.status == _lib.GMLA_ERR_DEVICE_RANGE
    # the workspace status is sticky until cleared
    ws = model._ws["decode"]
    _lib.check(_lib.gmla_clear_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream), "clear")
    model.sync_status()


@pytest.mark.slow
def test_decode_full_batch32_config():
    """The full decode workload (batch 32, lengths U[1024, 8192], H 16, d_c 512)."""
    inp = synth.generate(synth.workload("decode_b32"), seed=0)
    _check(inp, run_decode(inp))


@pytest.mark.slow
def test_decode_full_paged_config_sampled():
    """The full paged per-head-gate workload; oracle on 8 seeded sequences."""
    inp = synth.generate(synth.workload("decode_paged_head"), seed=0)
    gpu = run_decode(inp)
    seqs = sorted(np.random.default_rng(0).choice(64, 8, replace=False).tolist())
    _check(inp, gpu, seqs=seqs)


@pytest.mark.slow
def test_decode_full_long_context_rope_sampled():
    """The long-context workload (batch 8 x 131072 cached rows, H 128, d_c 512 +
    decoupled RoPE 64). The oracle evaluates y of one sequence in the absorbed
    form (pinned equal to the explicit form by the oracle's own tests) and the
    explicit per-head output o of two (sequence, head) pairs."""
    inp = synth.generate(synth.workload("decode_long_rope"), seed=0)
    gpu = run_decode(inp)
    w = inp["workload"]
    p = oracle.params(inp)
    # y of sequence 3, all heads (absorbed form)
    ref = oracle.decode(p, inp["x"], inp["past"], seqs=[3], absorbed=True)
    assert_close(gpu["q"][:, :, :w.d_h], ref["q"], BF16_TOL, "q")
    assert_close(gpu["q"][:, :, w.d_h:], ref["qR"], BF16_TOL, "qR (rotated at position 131071)")
    assert_close(gpu["o"][[3]], ref["gated"], BF16_TOL, "gated o, sequence 3")
    assert_close(gpu["y"][[3]], ref["y"], BF16_TOL, "y, sequence 3")
    # explicit form for two single heads
    for b, h in ((0, 5), (7, 127)):
        ex = oracle.decode(p, inp["x"], inp["past"], seqs=[b], heads=[h])
        g = oracle.sigmoid(ex["glogit"][b, h * w.d_h:(h + 1) * w.d_h])
        assert_close(gpu["o"][b, h * w.d_h:(h + 1) * w.d_h], g * ex["o"][0, 0], BF16_TOL, f"o[{b}, head {h}]")
