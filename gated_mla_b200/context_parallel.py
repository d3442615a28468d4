"""Context-parallel decode: one sequence's latent cache split across ranks.

Each rank holds the cached rows of a contiguous range of positions of every
sequence. The causal softmax over all L rows ("Gated MLA 计算公式" §二)
decomposes over disjoint ranges: rank r computes, for its range, the
normalised latent output O_r and its log-sum-exp lse_r (gmla_decode_partial);
the partials of all ranks are gathered with one all-gather of
R x B x H x (d_c + 4) floats; gmla_decode_merge then weights them by
2^(lse_r - max lse) and applies W_v and the gate as gmla_decode does.

The collective is torch.distributed's (NCCL between GPUs); everything else
runs in libgmla.so. Ranges are cut on 128-token tile boundaries, and the last
rank's range ends at the sequence's length (it holds the newest token).
"""
from __future__ import annotations

from typing import List, Tuple

import torch

from . import _lib as L
from .api import GatedMLA, LatentCache, _p

TILE = 128
PARTIAL_PAD = 4   # floats after the d_c values of one partial row


def shard_ranges(length: int, world: int, rank: int, tile: int = TILE) -> Tuple[int, int]:
    """[start, end) positions of a length-`length` sequence held by `rank` of `world`:
    contiguous ranges of whole tiles, as equal as the tiles allow, the last
    rank ending at `length`. Ranges of different ranks are disjoint and cover
    [0, length); a rank may hold an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    tiles = (length + tile - 1) // tile
    lo_t = tiles * rank // world
    hi_t = tiles * (rank + 1) // world
    start = min(lo_t * tile, length)
    end = length if rank == world - 1 else min(hi_t * tile, length)
    return start, max(start, end)


def shard_table(lengths: List[int], world: int, rank: int):
    """Per-sequence (starts, ends) of one rank as two int32 CPU tensors."""
    se = [shard_ranges(int(n), world, rank) for n in lengths]
    return (torch.tensor([s for s, _ in se], dtype=torch.int32),
            torch.tensor([e for _, e in se], dtype=torch.int32))


def partial_width(model: GatedMLA) -> int:
    return model.cfg.d_c + PARTIAL_PAD


def decode_partial(model: GatedMLA, q, gate_logits, cache: LatentCache, seq_starts, seq_ends, out=None):
    """This rank's partial [B, H, d_c + 4] fp32 over its positions."""
    B = q.shape[0]
    c = model.cfg
    if out is None:
        out = torch.empty(B, c.n_heads, partial_width(model), dtype=torch.float32, device=q.device)
    ws = model.workspace("decode", L.gmla_decode_workspace_size(c, B), q.device)
    L.check(L.gmla_decode_partial(c, model.w, _p(q), _p(gate_logits), cache.struct(), _p(seq_starts),
                                  _p(seq_ends), B, _p(out), ws.data_ptr(), ws.numel(), model._stream()),
            "gmla_decode_partial")
    return out


def decode_merge(model: GatedMLA, partials, gate_logits, out=None):
    """o_gated [B, H*d_h] from the gathered partials [R, B, H, d_c + 4]."""
    R, B = partials.shape[0], partials.shape[1]
    c = model.cfg
    if out is None:
        out = torch.empty(B, c.n_heads * c.d_h, dtype=model.dtype, device=partials.device)
    ws = model.workspace("decode_merge", L.gmla_decode_merge_workspace_size(c, B), partials.device)
    L.check(L.gmla_decode_merge(c, model.w, _p(partials), R, _p(gate_logits), B, _p(out), ws.data_ptr(),
                                ws.numel(), model._stream()), "gmla_decode_merge")
    return out


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's partial into [R, ...] in rank order (one
    collective: all_gather_into_tensor on NCCL, a list all-gather elsewhere)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(partial.shape), dtype=partial.dtype, device=partial.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, partial.contiguous(), group=group)
    else:
        parts = list(out.unbind(0))
        dist.all_gather(parts, partial.contiguous(), group=group)
        out = torch.stack(parts)
    return out


def decode_step(model: GatedMLA, q, gate_logits, cache: LatentCache, seq_starts, seq_ends, group=None):
    """One context-parallel decode of the calling rank: its partial, the
    all-gather, and the merge (every rank gets the full o_gated)."""
    part = decode_partial(model, q, gate_logits, cache, seq_starts, seq_ends)
    return decode_merge(model, gather_partials(part, group), gate_logits)
