"""Gated Multi-head Latent Attention hot path for B200 (sm_100a).

The compute lives in ``libgmla.so`` (C ABI in include/gmla.h): tcgen05/TMA
kernels for bf16 and CUDA-core kernels for fp32. This package only marshals
torch tensors into those calls; importing it fails if the library is missing.
"""
from . import _lib  # noqa: F401  (raises ImportError when libgmla.so is absent)
from .api import GatedMLA, LatentCache  # noqa: F401

__all__ = ["GatedMLA", "LatentCache", "_lib"]
