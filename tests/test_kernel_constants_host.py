"""The kernels' own approximations, checked on the CPU against the
mathematics (no GPU): the coefficients are read from the CUDA headers, so a
changed constant fails here.

- 2^x on the FMA pipe (attention.cuh, exp2_poly): degree-5 polynomial on the
  nearest-integer reduction, evaluated in float32 as the kernel does; relative
  error <= 3e-7 against 2^x over [-20, 9];
- GELU of the producer epilogue (gemm_pair.cuh, gelu_erf): erf by Abramowitz
  and Stegun 7.1.26, evaluated in float32; absolute error <= 3e-7 (1 + |x|)
  against x * Phi(x) with the exact error function (math.erf).
"""

import math
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "fp8_gemm_diffusion_b200", "csrc")


def _function_body(path, name):
    src = open(os.path.join(CSRC, path)).read()
    i = src.index(f" {name}(")
    j = src.index("\n}\n", i)
    return src[i:j]


def _floats(body):
    return [float(v.rstrip("f")) for v in re.findall(r"-?\d+\.\d+(?:e-?\d+)?f", body)]


def test_exp2_polynomial_constants():
    body = _function_body("attention.cuh", "exp2_poly")
    lits = _floats(body)
    # clamp, the rounding constant (twice), then the six coefficients, highest first
    assert lits[0] == -20.0 and lits[1] == 12582912.0 and lits[2] == 12582912.0
    coef = np.array(lits[3:9], dtype=np.float32)
    x = np.linspace(-20.0, 9.0, 400001).astype(np.float32)
    y = (x + np.float32(12582912.0)).astype(np.float32)
    j = (y.view(np.int32) - np.int32(0x4B400000)).astype(np.int32)
    f = (x - (y - np.float32(12582912.0))).astype(np.float32)
    p = np.full_like(f, coef[0])
    for c in coef[1:]:
        p = (p * f + c).astype(np.float32)  # one rounding per step, like fmaf up to the fused product
    r = (p.view(np.int32) + (j << 23)).view(np.float32)
    rel = np.abs(r.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 3e-7, rel.max()


def test_gelu_constants():
    body = _function_body("gemm_pair.cuh", "gelu_erf")
    lits = _floats(body)
    p, inv_sqrt2, a5, a4, a3, a2, a1 = lits[0], lits[1], lits[3], lits[4], lits[5], lits[6], lits[7]
    half_log2e = -lits[8]  # the kernel multiplies by its negative
    assert (p, a1, a2, a3, a4, a5) == (0.3275911, 0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429)
    assert abs(inv_sqrt2 - 1 / math.sqrt(2)) < 1e-15 and abs(half_log2e - math.log2(math.e) / 2) < 1e-15
    xs = np.linspace(-10.0, 10.0, 200001)
    f32 = np.float32
    worst = 0.0
    for x in xs[::7]:
        xf = f32(x)
        t = f32(1.0) / (f32(p * inv_sqrt2) * abs(xf) + f32(1.0))
        q = f32(a5)
        for a in (a4, a3, a2, a1):
            q = f32(q * t + f32(a))
        e = f32(2.0 ** float(f32(-half_log2e) * xf * xf))
        hq = f32(0.5) * xf * (q * t) * e
        g = xf - hq if xf >= 0 else hq
        exact = float(xf) * 0.5 * (1.0 + math.erf(float(xf) / math.sqrt(2.0)))
        worst = max(worst, abs(float(g) - exact) / (1.0 + abs(float(xf))))
    assert worst <= 3e-7, worst
