"""Context-parallel decode on one GPU, its ranks emulated one after another:
every rank's gmla_decode_partial runs on a copy of the cache whose rows
outside the rank's positions are NaN (so a row read from the wrong range would
poison the result), the partials are stacked in rank order as the all-gather
would, and gmla_decode_merge gives o_gated. It must match gmla_decode on the
whole cache and the fp64 oracle. (The kernels of different ranks never wait on
one another, so running them one after another on one GPU is the same
computation.)"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gated_mla_b200 import context_parallel as cp
from gpu_pipeline import BF16_TOL, assert_close, metrics, run_decode, small_decode

pytestmark = pytest.mark.gpu


def _emulate(inp, world):
    gpu = run_decode(inp)                      # the whole-cache decode (and the projected q, gates)
    model, cache = gpu["model"], gpu["cache"]
    q = torch.from_numpy(gpu["q"]).to("cuda", torch.bfloat16)
    g = torch.from_numpy(gpu["glogit"]).to("cuda")
    lens = [int(n) for n in inp["lengths"]]
    parts = []
    for r in range(world):
        starts, ends = cp.shard_table(lens, world, r)
        local = cache.data.clone()
        for b, (s, e) in enumerate(zip(starts.tolist(), ends.tolist())):
            local[b, :s] = float("nan")
            local[b, e:] = float("nan")
        rank_cache = type(cache)(data=local)
        parts.append(cp.decode_partial(model, q, g, rank_cache, starts.cuda(), ends.cuda()))
    o = cp.decode_merge(model, torch.stack(parts), g)
    model.sync_status()
    return o.float().cpu().numpy(), gpu


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_matches_whole_cache_decode(world):
    inp = small_decode("decode_b32", 4, [3000, 129, 1000, 5000])
    o, gpu = _emulate(inp, world)
    assert np.all(np.isfinite(o))
    m = metrics(o, gpu["o"])
    assert m["rel_l2"] < 3e-3, m
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    assert_close(o, ref["gated"], BF16_TOL, "gated o")


def test_context_parallel_rope_128_heads_with_an_empty_range():
    """Sequence 1 is shorter than one tile, so ranks 0 and 1 hold nothing of it."""
    inp = small_decode("decode_long_rope", 3, [2000, 100, 700], d_model=512)
    o, gpu = _emulate(inp, 3)
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    assert_close(o, ref["gated"], BF16_TOL, "gated o")


def test_context_parallel_with_hard_top_k_gates():
    inp = synth.generate(synth.workload("decode_paged_head", batch=3, gate_mode="head_topk", gate_topk=8,
                                        paged=False), seed=1, lengths=np.array([900, 2600, 300]))
    o, gpu = _emulate(inp, 2)
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    assert_close(o, ref["gated"], BF16_TOL, "gated o")


def test_context_parallel_long_shares():
    """Two sequences of 76,800 rows: the whole cache and each rank's share hold
    enough 128-token tiles (600 per share) that the split plan charges each
    sequence start its virtual tiles, in the partial decode as in the whole one.
    The oracle checks sequence 0 in the absorbed form (pinned equal to the
    explicit form by the oracle's tests)."""
    inp = small_decode("decode_b32", 2, [76800, 76800])
    o, gpu = _emulate(inp, 2)
    assert np.all(np.isfinite(o))
    m = metrics(o, gpu["o"])
    assert m["rel_l2"] < 3e-3, m
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"], seqs=[0], absorbed=True)
    assert_close(o[[0]], ref["gated"], BF16_TOL, "gated o, sequence 0")
