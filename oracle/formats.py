"""Element and scale codecs of the microscaling formats (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

Formats (the B200 MXFP8/NVFP4 diffusion article, "Glossary" entries
"Microscaling Formats", "MXFP8" and "NVFP4", name the formats; their bit-level
definitions are the public OCP Microscaling v1.0 specification and NVIDIA's
published NVFP4 description, which the article points to):

* E2M1  (FP4 element): sign, 2 exponent bits, 1 mantissa bit, bias 1.
  Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no Inf, no NaN.
* E4M3  (FP8 element, and NVFP4 block scale): sign, 4 exponent bits,
  3 mantissa bits, bias 7.  Largest finite 448 (0x7E); 0x7F / 0xFF are NaN;
  no Inf; smallest subnormal 2^-9.
* E8M0  (MX block scale): unsigned exponent only, code c -> 2^(c-127);
  0xFF is NaN.

Encoders round to nearest, ties to the even code (the code's least
significant bit, which is the mantissa LSB), and saturate finite values that
lie beyond the largest finite magnitude to that magnitude.  The sign is kept,
so a negative input that rounds to zero encodes as the negative-zero code.

The encoders are written as the definition: the result is the representable
value nearest to the input, found by searching the full table of decoded
codes; no bit tricks are used, so this file is independent of how a GPU
converts.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_BITS", "E4M3_BITS",
    "e2m1_decode", "e4m3_decode", "e8m0_decode",
    "e2m1_encode", "e4m3_encode",
    "E2M1_MAX", "E4M3_MAX",
]

E2M1_BITS = 4
E4M3_BITS = 8
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _e2m1_value(code: int) -> float:
    s = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = (m / 2.0) * 2.0 ** (1 - 1)  # subnormal: 0.m x 2^(1-bias)
    else:
        mag = (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return s * mag


def _e4m3_value(code: int) -> float:
    s = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - 7)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return s * mag


# Decode tables over every code (exact in float64).
_E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
_E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
_E8M0_TABLE = np.array(
    [np.ldexp(1.0, c - 127) if c != 255 else np.nan for c in range(256)], dtype=np.float64)

# Non-negative finite magnitudes, in code order (which is value order).
_E2M1_POS_CODES = np.arange(0, 8, dtype=np.int64)
_E2M1_POS_VALS = _E2M1_TABLE[:8].copy()
_E4M3_POS_CODES = np.arange(0, 0x7F, dtype=np.int64)  # 0x00..0x7E
_E4M3_POS_VALS = _E4M3_TABLE[:0x7F].copy()


def e2m1_decode(codes) -> np.ndarray:
    """E2M1 codes (low 4 bits used) -> float64 values."""
    return _E2M1_TABLE[np.asarray(codes, dtype=np.int64) & 0xF]


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 codes -> float64 values (NaN for 0x7F/0xFF)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.int64) & 0xFF]


def e8m0_decode(codes) -> np.ndarray:
    """E8M0 codes -> float64 values 2^(c-127) (NaN for 0xFF)."""
    return _E8M0_TABLE[np.asarray(codes, dtype=np.int64) & 0xFF]


def _encode_nearest_even(x, pos_vals: np.ndarray, pos_codes: np.ndarray,
                         sign_bit: int) -> np.ndarray:
    """Round-to-nearest-even with saturation, by table search.

    For each |x|: lo = largest representable magnitude <= |x|.  If lo is the
    largest finite magnitude the result saturates to it.  Otherwise hi is the
    next magnitude up, mid = (lo+hi)/2 (exact in float64 for these formats),
    and the result is lo if |x| < mid, hi if |x| > mid, and on a tie the one
    with the even code.
    """
    x = np.asarray(x)
    if x.dtype != np.float32:
        raise TypeError("encoders take float32 inputs (the precision the method computes in)")
    if np.isnan(x).any():
        raise ValueError("NaN input: the formats' conversion of NaN is outside the oracle's domain")
    a = np.abs(x.astype(np.float64))  # exact
    neg = np.signbit(x)
    idx = np.searchsorted(pos_vals, a, side="right") - 1  # lo index, >= 0 since vals[0] == 0
    last = len(pos_vals) - 1
    sat = idx >= last
    idx_c = np.minimum(idx, last - 1)
    lo = pos_vals[idx_c]
    hi = pos_vals[idx_c + 1]
    mid = (lo + hi) * 0.5
    lo_code = pos_codes[idx_c]
    hi_code = pos_codes[idx_c + 1]
    pick_hi = (a > mid) | ((a == mid) & ((hi_code & 1) == 0))
    code = np.where(pick_hi, hi_code, lo_code)
    code = np.where(sat, pos_codes[last], code)
    code = code | (neg.astype(np.int64) << sign_bit)
    return code.astype(np.uint8)


def e2m1_encode(x) -> np.ndarray:
    """float32 -> E2M1 code (uint8 holding 4 bits), RNE, saturating to +-6."""
    return _encode_nearest_even(x, _E2M1_POS_VALS, _E2M1_POS_CODES, 3)


def e4m3_encode(x) -> np.ndarray:
    """float32 -> E4M3 code, RNE, saturating to +-448 (never NaN for finite x)."""
    return _encode_nearest_even(x, _E4M3_POS_VALS, _E4M3_POS_CODES, 7)
