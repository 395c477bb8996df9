"""Seeded synthetic inputs for the microscaled linear layer.

This module only draws random numbers and shapes them into bf16 tensors.  It
holds none of the quantisation or GEMM arithmetic, and it is the one piece of
code that both the CPU oracle and the CUDA path consume: the same bytes feed
both sides.

Every configuration uses its own CPU ``torch.Generator`` seeded with 0 and
draws its tensors in the order listed in its docstring.  Values are sampled in
fp32 and rounded to bf16 (round to nearest even) at the end.

The shapes are FLUX-shaped stand-ins for the Flux.1-Dev workload of the B200
MXFP8/NVFP4 diffusion article ("Benchmark Results - Flux.1-Dev" table); no
dataset or trained weight is involved.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

__all__ = [
    "LinearCase",
    "c1_nvfp4_small",
    "c2_mxfp8_qkv",
    "c3_nvfp4_mlp_up",
    "c4_nvfp4_mlp_down",
    "make_case",
    "random_case",
    "flux_linear_stack",
    "flux_attention",
    "CONFIG_NAMES",
]


@dataclass
class LinearCase:
    """One linear layer: activations A [M,K], weights W [N,K], optional bias [N]."""

    name: str
    fmt: str  # "nvfp4" | "mxfp8" | "bf16"
    A: torch.Tensor  # bf16 [M, K], CPU
    W: torch.Tensor  # bf16 [N, K], CPU
    bias: Optional[torch.Tensor] = None  # bf16 [N], CPU
    meta: dict = field(default_factory=dict)

    @property
    def M(self) -> int:
        return self.A.shape[0]

    @property
    def K(self) -> int:
        return self.A.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[0]


def _gen(seed: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def c1_nvfp4_small(seed: int = 0) -> LinearCase:
    """NVFP4 W4A4 single GEMM, M=256, K=1024, N=1024, no bias.

    Draw order: A ~ N(0,1) [256,1024]; W ~ N(0,0.02) [1024,1024];
    U ~ U[0,1) [1024,1024]; entries of W with U < 0.01 are multiplied by 20.
    """
    g = _gen(seed)
    M, K, N = 256, 1024, 1024
    A = torch.randn(M, K, generator=g)
    W = torch.randn(N, K, generator=g) * 0.02
    U = torch.rand(N, K, generator=g)
    W = torch.where(U < 0.01, W * 20.0, W)
    return LinearCase("c1_nvfp4_256x1024x1024", "nvfp4", A.bfloat16(), W.bfloat16())


def c2_mxfp8_qkv(seed: int = 0, M: int = 4608) -> LinearCase:
    """MXFP8 QKV projection, M=4608 (4096 image + 512 text), K=3072, N=9216.

    Draw order: A0 ~ N(0,1) [M,3072]; z ~ N(0,1) [3072], s = exp(z)
    (LogNormal(0,1) per K channel); A = A0 * s; W ~ N(0,0.02) [9216,3072].
    No bias.
    """
    g = _gen(seed)
    K, N = 3072, 9216
    A = torch.randn(M, K, generator=g)
    s = torch.exp(torch.randn(K, generator=g))
    A = A * s[None, :]
    W = torch.randn(N, K, generator=g) * 0.02
    return LinearCase(f"c2_mxfp8_{M}x{K}x{N}", "mxfp8", A.bfloat16(), W.bfloat16())


def c3_nvfp4_mlp_up(seed: int = 0, M: int = 4608) -> LinearCase:
    """NVFP4 MLP-up, M=4608, K=3072, N=12288, bias in the epilogue.

    Draw order: A ~ N(0,1) [M,3072]; p = randperm(3072), the first
    round(0.001*3072) = 3 channels of p are multiplied by 50;
    W ~ N(0,0.02) [12288,3072]; bias ~ N(0,0.02) [12288].
    """
    g = _gen(seed)
    K, N = 3072, 12288
    A = torch.randn(M, K, generator=g)
    n_out = int(round(0.001 * K))
    chans = torch.randperm(K, generator=g)[:n_out]
    A[:, chans] *= 50.0
    W = torch.randn(N, K, generator=g) * 0.02
    bias = torch.randn(N, generator=g) * 0.02
    return LinearCase(
        f"c3_nvfp4_{M}x{K}x{N}", "nvfp4", A.bfloat16(), W.bfloat16(), bias.bfloat16(),
        meta={"outlier_channels": chans.tolist()},
    )


def _gelu_erf(x: torch.Tensor) -> torch.Tensor:
    # exact-erf GELU in fp32: x * 0.5 * (1 + erf(x / sqrt(2)))
    return x * 0.5 * (1.0 + torch.erf(x * (1.0 / math.sqrt(2.0))))


def c4_nvfp4_mlp_down(seed: int = 0, M: int = 16896) -> LinearCase:
    """NVFP4 MLP-down at 2048x2048 resolution: M=16896, K=12288, N=3072.

    Draw order: Z ~ N(0,1) [M,12288], A = GELU(Z) (exact erf, fp32);
    W ~ N(0,0.01) [3072,12288].  No bias.
    """
    g = _gen(seed)
    K, N = 12288, 3072
    A = _gelu_erf(torch.randn(M, K, generator=g))
    W = torch.randn(N, K, generator=g) * 0.01
    return LinearCase(f"c4_nvfp4_{M}x{K}x{N}", "nvfp4", A.bfloat16(), W.bfloat16())


CONFIG_NAMES = {
    "c1": c1_nvfp4_small,
    "c2": c2_mxfp8_qkv,
    "c3": c3_nvfp4_mlp_up,
    "c4": c4_nvfp4_mlp_down,
}


CASE_NAMES = {
    "c1": "c1_nvfp4_256x1024x1024",
    "c2": "c2_mxfp8_4608x3072x9216",
    "c3": "c3_nvfp4_4608x3072x12288",
    "c4": "c4_nvfp4_16896x12288x3072",
}


def make_case(name: str, **kw) -> LinearCase:
    return CONFIG_NAMES[name](**kw)


def random_case(M: int, K: int, N: int, fmt: str, seed: int = 0, bias: bool = True,
                a_std: float = 1.0, w_std: float = 0.02) -> LinearCase:
    """A small seeded case of any shape (ragged tiles, edge sizes).

    Draw order: A ~ N(0, a_std) [M,K]; W ~ N(0, w_std) [N,K]; bias ~ N(0,0.02) [N].
    """
    g = _gen(seed)
    A = torch.randn(M, K, generator=g) * a_std
    W = torch.randn(N, K, generator=g) * w_std
    b = (torch.randn(N, generator=g) * 0.02).bfloat16() if bias else None
    return LinearCase(f"rand_{fmt}_{M}x{K}x{N}", fmt, A.bfloat16(), W.bfloat16(), b)


def flux_linear_stack(batch: int = 1, n_double: int = 19, n_single: int = 38,
                      hidden: int = 3072, mlp: int = 12288, img_tokens: int = 4096,
                      txt_tokens: int = 512):
    """The linear layers of a FLUX-shaped DiT in forward order.

    Returns a list of dicts {name, M, K, N}.  Per double-stream block and per
    stream (image M=4096*B, text M=512*B): mod 3072->18432 (M=B), qkv
    3072->9216, proj 3072->3072, mlp_up 3072->12288, mlp_down 12288->3072.
    Per single-stream block (M=4608*B): mod 3072->9216 (M=B), linear1
    3072->21504, linear2 15360->3072.  Embedders and the final layer are left
    out (tiny, and kept in bf16 by the selection rule anyway).
    """
    layers = []
    B = batch
    for b in range(n_double):
        for stream, toks in (("img", img_tokens), ("txt", txt_tokens)):
            Ms = toks * B
            layers += [
                dict(name=f"d{b}.{stream}.mod", M=B, K=hidden, N=6 * hidden),
                dict(name=f"d{b}.{stream}.qkv", M=Ms, K=hidden, N=3 * hidden),
                dict(name=f"d{b}.{stream}.proj", M=Ms, K=hidden, N=hidden),
                dict(name=f"d{b}.{stream}.mlp_up", M=Ms, K=hidden, N=mlp),
                dict(name=f"d{b}.{stream}.mlp_down", M=Ms, K=mlp, N=hidden),
            ]
    Ms = (img_tokens + txt_tokens) * B
    for b in range(n_single):
        layers += [
            dict(name=f"s{b}.mod", M=B, K=hidden, N=3 * hidden),
            dict(name=f"s{b}.linear1", M=Ms, K=hidden, N=3 * hidden + mlp),
            dict(name=f"s{b}.linear2", M=Ms, K=hidden + mlp, N=hidden),
        ]
    return layers


def flux_attention(heads: int = 24, tokens: int = 4608, d: int = 128, seed: int = 0):
    """Q, K, V [heads, tokens, d] bf16 of one FLUX-shaped attention (24 heads of
    128 channels over 4096 image + 512 text tokens at 1024 x 1024).

    Draw order: Q, K, V ~ N(0, 1) (the queries and keys of a FLUX block are
    RMS-normalised, so unit-scale entries are the plain stand-in).
    """
    g = _gen(seed)
    Q = torch.randn(heads, tokens, d, generator=g)
    K = torch.randn(heads, tokens, d, generator=g)
    V = torch.randn(heads, tokens, d, generator=g)
    return Q.bfloat16(), K.bfloat16(), V.bfloat16()
