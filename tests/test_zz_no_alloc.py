"""gmla_decode_noalloc: the decode call for callers that cannot allocate device
memory (engines with their own memory pools, loops that cannot afford
cudaMalloc's synchronisation). It keeps its scratch in a static device
array inside the library; here it must reproduce gmla_decode, which uses a
caller-provided workspace, on two calls in a row through the C ABI.

This file is collected last on purpose (its name sorts last), so a run that
stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from gpu_pipeline import BF16_TOL, assert_close, make_decode_cache, make_model, small_decode

pytestmark = pytest.mark.gpu


def _decode_both(inp):
    from gated_mla_b200 import _lib
    w = inp["workload"]
    model = make_model(inp)
    cache = make_decode_cache(inp)
    B = w.batch
    lens = torch.tensor(inp["lengths"], dtype=torch.int32, device="cuda")
    x = torch.from_numpy(inp["x"]).to("cuda", torch.bfloat16)
    q, g = model.latent_project(x, (lens - 1).contiguous(), torch.arange(B, dtype=torch.int32, device="cuda"),
                                cache)
    ref = model.decode(q, g, cache, lens)
    out = torch.full_like(ref, float("nan"))
    st = _lib.gmla_decode_noalloc(model.cfg, model.w, q.data_ptr(), g.data_ptr(), cache.struct(),
                                  lens.data_ptr(), B, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    _lib.check(st, "gmla_decode_noalloc")
    torch.cuda.synchronize()
    model.sync_status()
    return out.float().cpu().numpy(), ref.float().cpu().numpy()


def test_noalloc_matches_workspace_decode_on_two_calls():
    # first call: the full batch-32 shape class with short caches
    a = small_decode("decode_b32", 32, np.random.default_rng(1).integers(1, 3000, 32).tolist())
    got, ref = _decode_both(a)
    assert_close(got, ref, BF16_TOL, "noalloc call 1")
    # second call: different batch and lengths, reusing the same static scratch
    b = small_decode("decode_paged_head", 5, [1, 64, 65, 700, 4000])
    got, ref = _decode_both(b)
    assert_close(got, ref, BF16_TOL, "noalloc call 2")


def test_noalloc_rejects_batches_beyond_its_scratch():
    from gated_mla_b200 import _lib
    a = small_decode("decode_b32", 2, [10, 20])
    model = make_model(a)
    cache = make_decode_cache(a)
    big_B = 4096
    assert _lib.gmla_decode_workspace_size(model.cfg, big_B) > 16 << 20
    st = _lib.gmla_decode_noalloc(model.cfg, model.w, None, None, cache.struct(), None, big_B, None,
                                  torch.cuda.current_stream().cuda_stream)
    assert st == _lib.GMLA_ERR_WORKSPACE
    assert b"16 MiB" in _lib.lib.gmla_last_error()
