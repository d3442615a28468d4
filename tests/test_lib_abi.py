"""The C-ABI library loads, exports every declared entry point and rejects bad
arguments before touching a GPU (these tests run without one)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gmla.h")


def declared_symbols():
    txt = open(HEADER, encoding="utf-8").read()
    return sorted(set(re.findall(r"GMLA_API\s+[\w\s\*]+?\b(gmla_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def L():
    from gated_mla_b200 import _lib
    return _lib


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for s in ("gmla_latent_project", "gmla_prefill", "gmla_decode", "gmla_gate_out"):
        assert s in syms
    assert len(syms) >= 13


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_status_strings_and_version(L):
    assert b"sm_100a" in L.lib.gmla_version()
    for s in range(7):
        assert L.lib.gmla_status_string(s)


def _cfg(L, **kw):
    c = L.gmla_config()
    c.d_model, c.n_heads, c.d_h, c.d_c, c.d_rope = 2048, 16, 128, 512, 0
    c.gate_mode, c.gate_bias, c.softmax_scale, c.rope_base, c.dtype = 0, 0, 128 ** -0.5, 1e4, 0
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_invalid_arguments_are_rejected_without_a_gpu(L):
    c = _cfg(L)
    w = L.gmla_weights()
    k = L.gmla_cache()
    # null config
    assert L.lib.gmla_decode(None, ctypes.byref(w), None, None, ctypes.byref(k), None, 1, None, None, 0,
                             None) == L.GMLA_ERR_INVALID_ARG
    # bad config values
    for bad in (dict(d_h=0), dict(d_rope=3), dict(gate_mode=5), dict(softmax_scale=0.0), dict(dtype=9)):
        cb = _cfg(L, **bad)
        st = L.gmla_decode(cb, w, None, None, k, None, 1, None, None, 0, None)
        assert st == L.GMLA_ERR_INVALID_ARG, bad
    # missing cache data
    assert L.gmla_decode(c, w, None, None, k, None, 1, None, None, 0, None) == L.GMLA_ERR_INVALID_ARG
    assert b"cache" in L.lib.gmla_last_error()
    # misaligned pointer
    k.data = 0x1001
    k.batch, k.capacity = 1, 16
    assert L.gmla_decode(c, w, None, None, k, None, 1, None, None, 0, None) == L.GMLA_ERR_INVALID_ARG
    assert b"aligned" in L.lib.gmla_last_error()
    # workspace too small
    k.data = 0x1000
    assert L.gmla_decode(c, w, None, None, k, None, 1, None, 0x2000, 16, None) == L.GMLA_ERR_WORKSPACE
    # unsupported page size
    k.paged, k.block_table, k.page_size, k.num_pages, k.max_pages_per_seq = 1, 0x3000, 48, 4, 4
    assert L.gmla_decode(c, w, None, None, k, None, 1, None, None, 0, None) == L.GMLA_ERR_UNSUPPORTED


def test_workspace_sizes_are_positive_and_aligned(L):
    c = _cfg(L)
    for B in (0, 1, 32, 1000):
        n = L.gmla_decode_workspace_size(c, B)
        assert n >= 256 and n % 256 == 0
    assert L.gmla_prefill_workspace_size(c, 16384, 4) >= 2 * 16384 * 16 * 128 * 2
    assert L.gmla_gate_out_workspace_size(c, 8) >= 256


def test_binding_names_match_the_c_abi(L):
    for s in declared_symbols():
        if s in ("gmla_status_string", "gmla_last_error", "gmla_version"):
            continue
        assert hasattr(L, s), s


def test_bad_config_never_reaches_a_size_computation(L):
    """n_heads = 0 (or another invalid config) must not crash a size query or
    the no-allocation decode: the queries answer 256 and the call returns
    GMLA_ERR_INVALID_ARG before any device work."""
    w = L.gmla_weights()
    k = L.gmla_cache()
    for bad in (dict(n_heads=0), dict(d_h=-1), dict(d_c=0), dict(dtype=7)):
        cb = _cfg(L, **bad)
        assert L.gmla_decode_workspace_size(cb, 32) == 256, bad
        assert L.gmla_prefill_workspace_size(cb, 64, 1) == 256, bad
        assert L.gmla_latent_project_workspace_size(cb, 8) == 256, bad
        assert L.gmla_gate_out_workspace_size(cb, 8) == 256, bad
        st = L.gmla_decode_noalloc(cb, w, None, None, k, None, 4, None, None)
        assert st == L.GMLA_ERR_INVALID_ARG, bad
    st = L.gmla_decode_noalloc(_cfg(L), w, None, None, k, None, -1, None, None)
    assert st == L.GMLA_ERR_INVALID_ARG
    assert b"B < 0" in L.lib.gmla_last_error()
