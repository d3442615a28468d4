"""Torch-facing marshalling over the C ABI (device memory and streams only).

``GatedMLA`` holds a configuration and device weight tensors and exposes the
four library calls. Outputs and workspaces are torch allocations; every
computation happens inside libgmla.so on the current CUDA stream.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

from . import _lib as L

_DT = {torch.bfloat16: L.GMLA_BF16, torch.float32: L.GMLA_FP32}
_GATE = {"channel": L.GMLA_GATE_CHANNEL, "head": L.GMLA_GATE_HEAD, "head_topk": L.GMLA_GATE_HEAD_TOPK,
         "head_binary": L.GMLA_GATE_HEAD_BINARY, "head_ternary": L.GMLA_GATE_HEAD_TERNARY}


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gated_mla_b200 takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


@dataclasses.dataclass
class LatentCache:
    """Latent cache rows [c | k^R] (contiguous [B, cap, row] or paged [pages, page, row])."""
    data: torch.Tensor
    block_table: Optional[torch.Tensor] = None   # int32 [B, max_pages_per_seq] for paged
    batch: int = 0

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def struct(self) -> L.gmla_cache:
        c = L.gmla_cache()
        c.data = _p(self.data)
        c.paged = 1 if self.paged else 0
        if self.paged:
            c.batch = self.block_table.shape[0]
            c.page_size = self.data.shape[1]
            c.num_pages = self.data.shape[0]
            c.max_pages_per_seq = self.block_table.shape[1]
            c.block_table = _p(self.block_table)
            c.capacity = c.max_pages_per_seq * c.page_size
        else:
            c.batch = self.data.shape[0]
            c.capacity = self.data.shape[1]
        return c


class GatedMLA:
    def __init__(self, *, d_model: int, n_heads: int, d_h: int, d_c: int, d_rope: int = 0,
                 gate_mode: str = "channel", softmax_scale: Optional[float] = None,
                 rope_base: float = 10000.0, dtype: torch.dtype = torch.bfloat16,
                 weights: dict, d_cq: int = 0, gate_topk: int = 0, cache_fp8: bool = False,
                 cache_scale: float = 1.0):
        self.dtype = dtype
        self.cfg = L.gmla_config()
        self.cfg.d_model, self.cfg.n_heads, self.cfg.d_h, self.cfg.d_c, self.cfg.d_rope = (
            d_model, n_heads, d_h, d_c, d_rope)
        self.cfg.gate_mode = _GATE[gate_mode]
        self.cfg.gate_topk = gate_topk
        self.cfg.gate_bias = 1 if weights.get("b_g") is not None else 0
        self.cfg.softmax_scale = softmax_scale if softmax_scale else 1.0 / math.sqrt(d_h + d_rope)
        self.cfg.rope_base = rope_base
        self.cfg.dtype = _DT[dtype]
        self.cfg.d_cq = d_cq
        self.cfg.cache_dtype = L.GMLA_CACHE_FP8_E4M3 if cache_fp8 else L.GMLA_CACHE_SAME
        self.cfg.cache_scale = cache_scale
        self.weights = dict(weights)
        self.w = L.gmla_weights()
        for k in ("W_c", "W_kr", "W_q", "W_qr", "W_k", "W_v", "W_g", "b_g", "W_o", "W_dq", "W_uq"):
            setattr(self.w, k, _p(self.weights.get(k)))
        self._ws = {}

    # -- sizes
    @property
    def G(self) -> int:
        return self.cfg.n_heads * self.cfg.d_h if self.cfg.gate_mode == L.GMLA_GATE_CHANNEL else self.cfg.n_heads

    @property
    def row(self) -> int:
        return self.cfg.d_c + self.cfg.d_rope

    def workspace(self, key: str, nbytes: int, device) -> torch.Tensor:
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            self._ws[key] = ws
            L.check(L.gmla_clear_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream), "clear_status")
        return ws

    @staticmethod
    def _stream() -> int:
        return torch.cuda.current_stream().cuda_stream

    # -- the four calls
    def latent_project(self, x, positions, seq_ids, cache: LatentCache, q_out=None, gate_logits=None):
        T = x.shape[0]
        c = self.cfg
        if q_out is None:
            q_out = torch.empty(T, c.n_heads, c.d_h + c.d_rope, dtype=self.dtype, device=x.device)
        if gate_logits is None:
            gate_logits = torch.empty(T, self.G, dtype=torch.float32, device=x.device)
        nb = L.gmla_latent_project_workspace_size(c, T)
        ws = self.workspace("project", nb, x.device)
        L.check(L.gmla_latent_project(c, self.w, _p(x), T, _p(positions), _p(seq_ids), cache.struct(),
                                      _p(q_out), _p(gate_logits), ws.data_ptr(), ws.numel(), self._stream()),
                "gmla_latent_project")
        return q_out, gate_logits

    def decode(self, q, gate_logits, cache: LatentCache, seq_lens, o_out=None, ws=None):
        B = q.shape[0]
        c = self.cfg
        if o_out is None:
            o_out = torch.empty(B, c.n_heads * c.d_h, dtype=self.dtype, device=q.device)
        nb = L.gmla_decode_workspace_size(c, B)
        if ws is None:
            ws = self.workspace("decode", nb, q.device)
        L.check(L.gmla_decode(c, self.w, _p(q), _p(gate_logits), cache.struct(), _p(seq_lens), B,
                              _p(o_out), ws.data_ptr(), ws.numel(), self._stream()), "gmla_decode")
        return o_out

    def prefill(self, q, gate_logits, cache: LatentCache, cu_seqlens, max_seqlen: int, o_out=None):
        T = q.shape[0]
        B = cu_seqlens.shape[0] - 1
        c = self.cfg
        if o_out is None:
            o_out = torch.empty(T, c.n_heads * c.d_h, dtype=self.dtype, device=q.device)
        nb = L.gmla_prefill_workspace_size(c, T, B)
        ws = self.workspace("prefill", nb, q.device)
        L.check(L.gmla_prefill(c, self.w, _p(q), _p(gate_logits), cache.struct(), _p(cu_seqlens), B, T,
                               int(max_seqlen), _p(o_out), ws.data_ptr(), ws.numel(), self._stream()),
                "gmla_prefill")
        return o_out

    def gate_out(self, o, gate_logits=None, y_out=None):
        T = o.shape[0]
        c = self.cfg
        if y_out is None:
            y_out = torch.empty(T, c.d_model, dtype=self.dtype, device=o.device)
        nb = L.gmla_gate_out_workspace_size(c, T)
        ws = self.workspace("gate_out", nb, o.device)
        L.check(L.gmla_gate_out(c, self.w, _p(o), T, _p(gate_logits), _p(y_out), ws.data_ptr(), ws.numel(),
                                self._stream()), "gmla_gate_out")
        return y_out

    def sync_status(self):
        """Synchronise and raise if any kernel reported a device-side fault."""
        for key, ws in self._ws.items():
            L.check(L.gmla_sync_status(ws.data_ptr(), self._stream()), f"device status ({key})")

    # -- whole steps
    def decode_step(self, x, cache: LatentCache, seq_lens, positions, seq_ids):
        """One decode step: project (writing each new latent row), attend, gate, W_o."""
        q, g = self.latent_project(x, positions, seq_ids, cache)
        o = self.decode(q, g, cache, seq_lens)
        return self.gate_out(o)

    def prefill_step(self, x, cache: LatentCache, cu_seqlens, max_seqlen, positions, seq_ids):
        q, g = self.latent_project(x, positions, seq_ids, cache)
        o = self.prefill(q, g, cache, cu_seqlens, max_seqlen)
        return self.gate_out(o)
