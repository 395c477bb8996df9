"""Selective quantisation rule (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

The B200 MXFP8/NVFP4 diffusion article, "Detailed by section" (selective
quantisation paragraph): a layer whose GEMM is too small for quantisation to
pay - min(M, K, N) < 1024 - or that is an accuracy-sensitive embedding stays
in bf16; everything else is quantised.  Reading: "< 1024" is strict, so a
dimension of exactly 1024 is quantised; the embedding exclusion is a per-weight
``keep_bf16`` flag set by the caller.
"""

from __future__ import annotations

__all__ = ["use_bf16", "DEFAULT_MIN_DIM"]

DEFAULT_MIN_DIM = 1024


def use_bf16(M: int, K: int, N: int, keep_bf16: bool = False,
             min_dim: int = DEFAULT_MIN_DIM) -> bool:
    """True when the layer runs as a plain bf16 GEMM."""
    return bool(keep_bf16) or min(M, K, N) < min_dim
