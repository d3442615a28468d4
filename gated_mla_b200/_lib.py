"""ctypes binding of libgmla.so: the C ABI of include/gmla.h, same names.

Argument marshalling only. Every compute step runs in the library's CUDA
kernels; if the library is missing this module raises at import.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("GMLA_LIB", os.path.join(_HERE, "libgmla.so"))

GMLA_OK = 0
GMLA_ERR_INVALID_ARG = 1
GMLA_ERR_UNSUPPORTED = 2
GMLA_ERR_WORKSPACE = 3
GMLA_ERR_CUDA = 4
GMLA_ERR_TIMEOUT = 5
GMLA_ERR_DEVICE_RANGE = 6

GMLA_BF16 = 0
GMLA_FP32 = 1
GMLA_CACHE_SAME = 0
GMLA_CACHE_FP8_E4M3 = 1
GMLA_GATE_CHANNEL = 0
GMLA_GATE_HEAD = 1
GMLA_GATE_HEAD_TOPK = 2
GMLA_GATE_HEAD_BINARY = 3
GMLA_GATE_HEAD_TERNARY = 4


class gmla_config(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("d_h", ctypes.c_int32),
        ("d_c", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("gate_mode", ctypes.c_int32),
        ("gate_bias", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("rope_base", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("d_cq", ctypes.c_int32),
        ("gate_topk", ctypes.c_int32),
        ("cache_dtype", ctypes.c_int32),
        ("cache_scale", ctypes.c_float),
    ]


class gmla_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("W_c", "W_kr", "W_q", "W_qr", "W_k", "W_v", "W_g", "b_g", "W_o", "W_dq", "W_uq")]


class gmla_cache(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("paged", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
    ]


class GmlaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({message})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libgmla.so not found at {LIB_PATH}; build it with `python -m gated_mla_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int32
    S = ctypes.c_size_t
    st = ctypes.c_int
    cfgp = ctypes.POINTER(gmla_config)
    wp = ctypes.POINTER(gmla_weights)
    cp = ctypes.POINTER(gmla_cache)
    sig = {
        "gmla_latent_project": (st, [cfgp, wp, P, I, P, P, cp, P, P, P, S, P]),
        "gmla_decode": (st, [cfgp, wp, P, P, cp, P, I, P, P, S, P]),
        "gmla_decode_noalloc": (st, [cfgp, wp, P, P, cp, P, I, P, P]),
        "gmla_decode_partial": (st, [cfgp, wp, P, P, cp, P, P, I, P, P, S, P]),
        "gmla_decode_merge": (st, [cfgp, wp, P, I, P, I, P, P, S, P]),
        "gmla_decode_merge_workspace_size": (S, [cfgp, I]),
        "gmla_prefill": (st, [cfgp, wp, P, P, cp, P, I, I, I, P, P, S, P]),
        "gmla_gate_out": (st, [cfgp, wp, P, I, P, P, P, S, P]),
        "gmla_latent_project_workspace_size": (S, [cfgp, I]),
        "gmla_decode_workspace_size": (S, [cfgp, I]),
        "gmla_prefill_workspace_size": (S, [cfgp, I, I]),
        "gmla_gate_out_workspace_size": (S, [cfgp, I]),
        "gmla_clear_status": (st, [P, P]),
        "gmla_sync_status": (st, [P, P]),
        "gmla_status_string": (ctypes.c_char_p, [st]),
        "gmla_last_error": (ctypes.c_char_p, []),
        "gmla_version": (ctypes.c_char_p, []),
        "gmla_launch_count": (ctypes.c_uint64, []),
        "gmla_test_stall_next_decode": (st, [I]),
        "gmla_profile_enable": (st, [I]),
        "gmla_profile_count": (I, []),
        "gmla_profile_get": (st, [I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def check(status: int, where: str) -> None:
    if status != GMLA_OK:
        msg = lib.gmla_last_error().decode() or lib.gmla_status_string(status).decode()
        raise GmlaError(status, where, msg)


# Thin wrappers with the C names (pointers are ints or None).
def gmla_latent_project(cfg, w, x, T, positions, seq_ids, cache, q_out, gate_logits, ws, ws_bytes, stream):
    return lib.gmla_latent_project(ctypes.byref(cfg), ctypes.byref(w), x, T, positions, seq_ids,
                                   ctypes.byref(cache), q_out, gate_logits, ws, ws_bytes, stream)


def gmla_decode(cfg, w, q, gate_logits, cache, seq_lens, B, o, ws, ws_bytes, stream):
    return lib.gmla_decode(ctypes.byref(cfg), ctypes.byref(w), q, gate_logits, ctypes.byref(cache),
                           seq_lens, B, o, ws, ws_bytes, stream)


def gmla_decode_noalloc(cfg, w, q, gate_logits, cache, seq_lens, B, o, stream):
    return lib.gmla_decode_noalloc(ctypes.byref(cfg), ctypes.byref(w), q, gate_logits, ctypes.byref(cache),
                                   seq_lens, B, o, stream)


def gmla_decode_partial(cfg, w, q, gate_logits, cache, seq_starts, seq_ends, B, partial, ws, ws_bytes, stream):
    return lib.gmla_decode_partial(ctypes.byref(cfg), ctypes.byref(w), q, gate_logits, ctypes.byref(cache),
                                   seq_starts, seq_ends, B, partial, ws, ws_bytes, stream)


def gmla_decode_merge(cfg, w, partials, R, gate_logits, B, o, ws, ws_bytes, stream):
    return lib.gmla_decode_merge(ctypes.byref(cfg), ctypes.byref(w), partials, R, gate_logits, B, o, ws, ws_bytes,
                                 stream)


def gmla_decode_merge_workspace_size(cfg, B):
    return lib.gmla_decode_merge_workspace_size(ctypes.byref(cfg), B)


def gmla_prefill(cfg, w, q, gate_logits, cache, cu_seqlens, B, T, max_seqlen, o, ws, ws_bytes, stream):
    return lib.gmla_prefill(ctypes.byref(cfg), ctypes.byref(w), q, gate_logits, ctypes.byref(cache),
                            cu_seqlens, B, T, max_seqlen, o, ws, ws_bytes, stream)


def gmla_gate_out(cfg, w, o, T, gate_logits, y, ws, ws_bytes, stream):
    return lib.gmla_gate_out(ctypes.byref(cfg), ctypes.byref(w), o, T, gate_logits, y, ws, ws_bytes, stream)


def gmla_decode_workspace_size(cfg, B):
    return lib.gmla_decode_workspace_size(ctypes.byref(cfg), B)


def gmla_prefill_workspace_size(cfg, T, B):
    return lib.gmla_prefill_workspace_size(ctypes.byref(cfg), T, B)


def gmla_latent_project_workspace_size(cfg, T):
    return lib.gmla_latent_project_workspace_size(ctypes.byref(cfg), T)


def gmla_gate_out_workspace_size(cfg, T):
    return lib.gmla_gate_out_workspace_size(ctypes.byref(cfg), T)


def gmla_clear_status(ws, stream):
    return lib.gmla_clear_status(ws, stream)


def gmla_sync_status(ws, stream):
    return lib.gmla_sync_status(ws, stream)


def gmla_test_stall_next_decode(enable):
    return lib.gmla_test_stall_next_decode(1 if enable else 0)


def gmla_launch_count():
    return lib.gmla_launch_count()


def gmla_profile_enable(enable):
    return lib.gmla_profile_enable(1 if enable else 0)


def gmla_profile_count():
    return lib.gmla_profile_count()


def gmla_profile_get(i):
    """Returns (name, ms) of record i."""
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    check(lib.gmla_profile_get(i, ctypes.byref(name), ctypes.byref(ms)), "gmla_profile_get")
    return name.value.decode(), ms.value


def profile_records():
    return [gmla_profile_get(i) for i in range(gmla_profile_count())]
