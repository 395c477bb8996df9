"""Pins of the activation-epilogue oracle (GELU with the exact error function)
against facts other than itself: standard-normal CDF table values, the odd-part
identity GELU(x) - GELU(-x) = x, the asymptotes, the closed-form maximum
slope, the C library's erf element by element, and the Lipschitz bound the
tolerance rests on."""

import math

import numpy as np

from oracle import gemm as G
from oracle import producer as P


def test_gelu_textbook_values():
    # GELU(x) = x * Phi(x); Phi from the standard normal table
    table = {1.0: 0.8413447460685429, 2.0: 0.9772498680518208, -1.0: 0.15865525393145707,
             0.5: 0.6914624612740131, -2.0: 0.022750131948179195}
    for x, phi in table.items():
        assert abs(P.gelu(x) - x * phi) < 1e-15, x
    assert P.gelu(0.0) == 0.0


def test_gelu_odd_part_and_asymptotes():
    x = np.linspace(-12, 12, 4801)
    assert np.allclose(P.gelu(x) - P.gelu(-x), x, rtol=0, atol=1e-13)
    assert abs(P.gelu(10.0) - 10.0) < 1e-14
    assert abs(P.gelu(-10.0)) < 1e-20
    assert np.all(np.abs(P.gelu(x)) <= np.abs(x))


def test_gelu_slope_closed_form_and_maximum():
    exact = 0.5 * (1 + math.erf(1.0)) + math.exp(-1.0) / math.sqrt(math.pi)  # Phi(sqrt 2) + e^-1/sqrt(pi)
    assert exact <= P.GELU_MAX_SLOPE < exact + 1e-5
    assert abs(P.gelu_slope(math.sqrt(2.0)) - exact) < 1e-14
    x = np.linspace(-8, 8, 160001)
    fd = np.diff(P.gelu(x)) / np.diff(x)
    assert fd.max() <= P.GELU_MAX_SLOPE
    assert np.allclose(P.gelu_slope(0.5 * (x[1:] + x[:-1])), fd, rtol=0, atol=1e-8)


def test_linear_gelu_ref_against_libm_erf():
    rng = np.random.default_rng(5)
    A = rng.integers(-3, 4, size=(5, 24)).astype(np.float64) * 0.25
    W = rng.integers(-3, 4, size=(7, 24)).astype(np.float64) * 0.125
    b = (rng.integers(-4, 5, size=7) * 0.0625).astype(np.float32)
    Y, T = P.linear_gelu_ref(A, W, b)
    for m in range(5):
        for n in range(7):
            y = sum(A[m, k] * W[n, k] for k in range(24)) + float(b[n])
            assert abs(Y[m, n] - 0.5 * y * (1 + math.erf(y / math.sqrt(2)))) < 1e-14
            t = sum(abs(A[m, k] * W[n, k]) for k in range(24))
            assert abs(T[m, n] - P.GELU_MAX_SLOPE * t) < 1e-12


def test_activation_tolerance_is_sound():
    # an accumulation error within the plain layer's bound stays within the
    # activation's bound after GELU
    rng = np.random.default_rng(6)
    A = rng.standard_normal((64, 256))
    W = rng.standard_normal((48, 256)) * 0.05
    Y0, T = G.linear_ref(A, W)
    e = (rng.random(Y0.shape) * 2 - 1) * G.RTOL * T
    Yg, Tg = P.linear_gelu_ref(A, W)
    assert np.all(np.abs(P.gelu(Y0 + e) - Yg) <= G.RTOL * Tg + G.ATOL)
