"""Pins for the oracle's element codecs (CPU only).

Each test checks the oracle against something other than itself: the format
tables of the public specifications (fixtures under tests/golden/), the
IEEE round-ties-to-even rule on hand-picked midpoints, a brute-force nearest
search written independently here, and torch's own float8_e4m3fn cast.
"""

import math

import numpy as np
import pytest
import torch

from oracle import formats as F
from tests._golden import code_table, rounding_cases


def _same_value(a, b):
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_e2m1_table_matches_spec():
    for code, val in code_table("e2m1_codes.txt"):
        assert _same_value(float(F.e2m1_decode(code)), val), hex(code)


def test_e4m3_points_match_spec():
    for code, val in code_table("e4m3_points.txt"):
        assert _same_value(float(F.e4m3_decode(code)), val), hex(code)


def test_e4m3_closed_form_all_codes():
    # value = (-1)^s * 2^(e-7) * (1 + m/8) for e > 0, 2^-6 * m/8 for e == 0
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        v = float(F.e4m3_decode(c))
        if e == 15 and m == 7:
            assert math.isnan(v)
            continue
        mag = (2.0 ** (e - 7)) * (1 + m / 8) if e else (2.0 ** -6) * (m / 8)
        assert _same_value(v, -mag if s else mag), hex(c)


def test_e8m0_all_codes():
    for c in range(255):
        assert F.e8m0_decode(c) == 2.0 ** (c - 127)
    assert math.isnan(F.e8m0_decode(255))


def test_roundtrip_all_e2m1_codes():
    vals = F.e2m1_decode(np.arange(16)).astype(np.float32)
    assert list(F.e2m1_encode(vals)) == list(range(16))  # +-0 stay distinct


def test_roundtrip_all_e4m3_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    vals = F.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(F.e4m3_encode(vals), codes.astype(np.uint8))


@pytest.mark.parametrize("case", rounding_cases(), ids=lambda c: f"{c[0]}:{c[1]!r}")
def test_rounding_cases(case):
    fmt, x, code = case
    enc = F.e2m1_encode if fmt == "e2m1" else F.e4m3_encode
    assert int(enc(np.array([x], dtype=np.float32))[0]) == code


def _brute_nearest_even(x, table_codes):
    """Independent brute force: scan every finite code, keep the nearest value;
    on equal distance keep the even code; beyond the largest magnitude the
    largest magnitude is nearest by construction of the scan."""
    best = None
    for c in table_codes:
        v = table_codes[c]
        if math.copysign(1.0, v) != math.copysign(1.0, x):
            continue
        d = abs(float(x) - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0 and best[1] % 2 == 1):
            best = (d, c)
    return best[1]


def _table(decode, codes):
    out = {}
    for c in codes:
        v = float(decode(c))
        if not math.isnan(v):
            out[c] = v
    return out


def test_e2m1_vs_brute_force():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        rng.normal(0, 3, 4000), rng.uniform(-8, 8, 4000),
        np.arange(-7.0, 7.01, 0.125),  # includes every midpoint
    ]).astype(np.float32)
    tab = _table(F.e2m1_decode, range(16))
    got = F.e2m1_encode(xs)
    for x, g in zip(xs, got):
        assert g == _brute_nearest_even(x, tab), (x, g)


def test_e4m3_vs_brute_force_sample():
    rng = np.random.default_rng(2)
    xs = np.concatenate([
        rng.normal(0, 50, 1500), rng.uniform(-470, 470, 500),
        np.exp(rng.uniform(-14, 6.2, 1000)) * rng.choice([-1, 1], 1000),
    ]).astype(np.float32)
    tab = _table(F.e4m3_decode, range(256))
    got = F.e4m3_encode(xs)
    for x, g in zip(xs, got):
        assert g == _brute_nearest_even(x, tab), (x, g)


def test_e4m3_vs_torch_cast():
    # torch's float8_e4m3fn cast is an independent RNE implementation; it
    # returns NaN instead of saturating above 464, so compare below that.
    rng = np.random.default_rng(3)
    vals = F.e4m3_decode(np.arange(0, 0x7E)).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2  # every tie point
    xs = np.concatenate([
        rng.normal(0, 30, 200000), np.exp(rng.uniform(-16, 6.1, 200000)),
        mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
    ])
    xs = np.concatenate([xs, -xs]).astype(np.float32)
    xs = xs[np.abs(xs) <= 464]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(xs), ref)


def test_saturation_and_sign():
    assert F.e4m3_encode(np.array([np.float32(3e38)]))[0] == 0x7E
    assert F.e4m3_encode(np.array([np.float32(-3e38)]))[0] == 0xFE
    assert F.e2m1_encode(np.array([np.float32(-1e-30)]))[0] == 0x8
    assert F.e4m3_encode(np.array([np.float32(-0.0)]))[0] == 0x80


def test_encoders_reject_nan_and_non_float32():
    with pytest.raises(ValueError):
        F.e2m1_encode(np.array([np.nan], dtype=np.float32))
    with pytest.raises(TypeError):
        F.e4m3_encode(np.array([1.0]))
