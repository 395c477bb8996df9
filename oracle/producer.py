"""Activation epilogue of a quantised linear layer (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

Source passages: the devin.kr page on Blackwell FLUX image generation
("엔비디아 블랙웰 기반 플럭스 3 이미지 생성 4.45배 가속"), section "연산 효율화와
가속 기술" (compute efficiency and acceleration): its custom matrix-multiply
kernels have the activation functions (and the rotary position embedding)
fused into them; and the WaveSpeedAI B200 article ("WaveSpeedAI X DataCrunch:
B200에서 FLUX 실시간 이미지 추론"), section "WaveSpeedAI의 독점 추론 프레임워크"
(its proprietary inference framework): custom CUDA kernels and kernel fusion.
In a FLUX-shaped block the MLP's first linear layer is followed by GELU, whose
output is the next linear layer's input; fused, the GEMM's epilogue applies
the activation before the bf16 rounding:

    Y[m, n] = GELU( sum_k deq(A)[m, k] * deq(W)[n, k] + bias[n] )

Reading (the pages name no variant): GELU with the exact error function,
GELU(x) = x * Phi(x) = 0.5 * x * (1 + erf(x / sqrt(2))).

Error scale.  GELU is Lipschitz with constant
    max_x GELU'(x) = GELU'(sqrt(2)) = Phi(sqrt(2)) + exp(-1) / sqrt(pi) = 1.1289...
(GELU'' = phi(x) (2 - x^2) vanishes at sqrt(2)), so an accumulation error e
before the activation is at most 1.1289 e after it, and |GELU(y)| <= |y|
keeps the bf16 rounding of the output inside the same budget.  The
activation's error scale is therefore GELU_MAX_SLOPE * T with T the plain
layer's sum_k |a_k b_k|, under the plain layer's 2e-3 * T + 1e-6 rule.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

from .gemm import linear_ref

__all__ = ["gelu", "gelu_slope", "GELU_MAX_SLOPE", "linear_gelu_ref"]

# Phi(sqrt(2)) + exp(-1) / sqrt(pi) = 1.1289041..., rounded up
GELU_MAX_SLOPE = 1.12891


def gelu(x) -> np.ndarray:
    """x * Phi(x) with the exact error function, float64."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def gelu_slope(x) -> np.ndarray:
    """d/dx GELU(x) = Phi(x) + x phi(x), float64."""
    x = np.asarray(x, dtype=np.float64)
    phi = np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    return 0.5 * (1.0 + _erf(x / math.sqrt(2.0))) + x * phi


def linear_gelu_ref(Adeq, Wdeq, bias=None):
    """(Y, T_act): Y = GELU(Adeq Wdeq^T + bias) and its error scale, float64."""
    Y, T = linear_ref(Adeq, Wdeq, bias)
    return gelu(Y), GELU_MAX_SLOPE * T
