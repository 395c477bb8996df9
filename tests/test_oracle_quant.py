"""Pins for the oracle's NVFP4 / MXFP8 quantisers (CPU only).

Pinned against: hand-worked examples (tests/golden/*_worked_example.txt),
blocks built from exactly representable values that must reproduce exactly,
closed forms for the shared-exponent rule, and invariants of the definitions
(scale invariance by powers of two, sign symmetry, zero blocks).
"""

import math

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import quant as Q
from tests._golden import _lines, keyed

f32 = np.float32


def _bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).bfloat16()


def test_nvfp4_worked_example():
    d = keyed("nvfp4_worked_example.txt")
    x = np.array([[float(v) for v in d["x0"]], [float(v) for v in d["x1"]]], dtype=np.float32)
    q = Q.quantize_nvfp4(_bf16(x))
    assert q["amax"] == 15.0
    assert q["g"] == f32(15.0) / f32(2688.0)
    assert list(q["sf"][:, 0]) == [int(d["sf0"][0], 16), int(d["sf1"][0], 16)]
    assert list(q["codes"][0]) == [int(c, 16) for c in d["codes0"]]
    assert list(q["codes"][1]) == [int(c, 16) for c in d["codes1"]]


def test_mxfp8_worked_example():
    d = keyed("mxfp8_worked_example.txt")
    x = np.array([[float(v) for v in d["x"]]], dtype=np.float32)
    q = Q.quantize_mxfp8(_bf16(x))
    assert q["sf"][0, 0] == int(d["sf"][0], 16)
    assert list(q["codes"][0]) == [int(c, 16) for c in d["codes"]]


def _exact_nvfp4_tensor(rng, R, K, j):
    """Blocks c_i * e * 2^j with e an E4M3 value, c_i E2M1 values, one |c|=6
    per block, plus one block whose amax is 2688 * 2^j (so g = 2^j exactly)."""
    e2 = F.e2m1_decode(np.arange(16))
    e4 = F.e4m3_decode(np.arange(1, 0x7F))  # positive finite scales
    X = np.zeros((R, K))
    codes = rng.integers(0, 16, size=(R, K))
    nb = K // 16
    scales = rng.choice(e4[e4 >= 2.0 ** -6], size=(R, nb))  # keep 1/s finite and exact-ish
    for r in range(R):
        for b in range(nb):
            cs = codes[r, b * 16:(b + 1) * 16]
            cs[rng.integers(0, 16)] = rng.choice([7, 15])  # +-6 present
            X[r, b * 16:(b + 1) * 16] = e2[cs] * scales[r, b] * 2.0 ** j
    scales[0, 0] = 448.0
    X[0, 0:16] = e2[codes[0, 0:16]] * 448.0 * 2.0 ** j
    X[0, 0] = 6 * 448.0 * 2.0 ** j
    return X.astype(np.float32)


@pytest.mark.parametrize("j", [-12, -3, 0, 2])
def test_nvfp4_exact_blocks_reproduce(j):
    rng = np.random.default_rng(100 + j)
    X = _exact_nvfp4_tensor(rng, 5, 64, j)
    xb = _bf16(X)
    assert np.array_equal(xb.float().numpy(), X), "fixture values must be bf16-exact"
    q = Q.quantize_nvfp4(xb)
    assert q["g"] == f32(2.0 ** j)
    deq = Q.dequant_nvfp4(q["codes"], q["sf"], q["g"])
    assert np.array_equal(deq, X.astype(np.float64))


def test_nvfp4_without_tensor_scale_exact_blocks():
    # g = 1: blocks c_i * e (e an E4M3 value, one |c_i| = 6) give sf = e and
    # codes c_i, so the dequantised tensor is the input, bit for bit
    rng = np.random.default_rng(7)
    e2 = F.e2m1_decode(np.arange(16))
    e4 = F.e4m3_decode(np.arange(1, 0x7F))
    R, K = 6, 96
    codes = rng.integers(0, 16, size=(R, K))
    scales = rng.choice(e4[e4 >= 2.0 ** -6], size=(R, K // 16))
    X = np.zeros((R, K))
    for r in range(R):
        for b in range(K // 16):
            cs = codes[r, b * 16:(b + 1) * 16]
            cs[rng.integers(0, 16)] = rng.choice([7, 15])
            X[r, b * 16:(b + 1) * 16] = e2[cs] * scales[r, b]
    X = X.astype(np.float32)
    xb = _bf16(X)
    assert np.array_equal(xb.float().numpy(), X), "fixture values must be bf16-exact"
    q = Q.quantize_nvfp4(xb, tensor_scale=False)
    assert q["g"] == f32(1.0) and q["amax"] == f32(0.0)
    assert np.array_equal(F.e4m3_decode(q["sf"]), scales)
    assert np.array_equal(Q.dequant_nvfp4(q["codes"], q["sf"], q["g"]), X.astype(np.float64))


def test_nvfp4_without_tensor_scale_saturation_and_underflow():
    x = np.zeros((3, 16), dtype=np.float32)
    # bamax / 6 = 1024 > 448: the scale saturates at 448 (0x7E); then
    # 6144 / 448 = 13.7 saturates to +6, -700 / 448 = -1.5625 rounds to -1.5,
    # 448 / 448 = 1
    x[0, 0], x[0, 1], x[0, 2] = 6144.0, -700.0, 448.0
    # bamax / 6 = 2^-10: half of E4M3's smallest subnormal 2^-9, a tie -> 0,
    # so the block's scale and codes are 0
    x[1, 0] = 6 * 2.0 ** -10
    # bamax / 6 = 3 * 2^-10: a tie between 2^-9 (code 1) and 2^-8 (code 2) -> 2^-8
    x[2, 0] = 6 * 3 * 2.0 ** -10
    q = Q.quantize_nvfp4(x, tensor_scale=False)
    assert list(q["sf"][:, 0]) == [0x7E, 0x00, 0x02]
    c = Q.unpack_fp4(q["codes"])
    assert list(c[0, :3]) == [0x7, 0xB, 0x2]          # +6, -1.5, +1
    assert np.all(c[1] == 0)
    # row 2: x / 2^-8 = 4.5 -> E2M1 tie between 4 and 6 -> 4 (even mantissa)
    assert c[2, 0] == 0x6


def test_nvfp4_without_tensor_scale_is_unit_g():
    # g = amax / 2688 is exactly 1 for amax = 2688, so the variant equals the
    # general recipe with that amax
    x = torch.randn(40, 128, generator=torch.Generator().manual_seed(12)) * 5
    x[3, 7] = 9000.0
    a = Q.quantize_nvfp4(x.bfloat16(), tensor_scale=False)
    b = Q.quantize_nvfp4(x.bfloat16(), global_amax=np.float32(2688.0))
    assert b["g"] == f32(1.0)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["sf"], b["sf"])
    with pytest.raises(ValueError):
        Q.quantize_nvfp4(x, global_amax=1.0, tensor_scale=False)


@pytest.mark.parametrize("k", [-20, -5, 0, 7])
def test_mxfp8_exact_blocks_reproduce(k):
    rng = np.random.default_rng(100 + k)
    vals = F.e4m3_decode(np.arange(0, 0x7F))
    R, K = 4, 96
    X = rng.choice(vals, size=(R, K)) * rng.choice([-1, 1], size=(R, K))
    X = X.reshape(R, K // 32, 32)
    X[:, :, 0] = rng.choice(vals[(vals >= 256) & (vals <= 448)], size=(R, K // 32))
    X = (X.reshape(R, K) * 2.0 ** k)
    # keep every element bf16-exact: E4M3 values have <= 4 significant bits
    q = Q.quantize_mxfp8(_bf16(X.astype(np.float32)))
    assert np.all(q["sf"] == 127 + k)
    assert np.array_equal(Q.dequant_mxfp8(q["codes"], q["sf"]), X)


def test_mxfp8_scale_closed_form():
    # one element per block, |x| = 2^p * (1 + f): scale code = p - 8 + 127
    for p in range(-125, 127, 7):
        for f in (0.0, 0.5, 0.99):
            x = np.zeros((1, 32), dtype=np.float32)
            x[0, 3] = f32(2.0 ** p * (1 + f))
            q = Q.quantize_mxfp8(x)
            assert q["sf"][0, 0] == max(p - 8, -127) + 127, (p, f)


def test_mxfp8_subnormal_block_scale():
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = np.float32(2.0 ** -140)  # fp32 subnormal: floor(log2) = -140 -> clamp
    q = Q.quantize_mxfp8(x)
    assert q["sf"][0, 0] == 0
    # 2^-140 * 2^127 = 2^-13 -> below half of E4M3's smallest subnormal -> 0
    assert q["codes"][0, 0] == 0


def test_zero_tensor():
    x = np.zeros((3, 64), dtype=np.float32)
    q = Q.quantize_nvfp4(x)
    assert q["g"] == 1.0 and q["amax"] == 0.0
    assert not q["sf"].any() and not q["codes"].any()
    m = Q.quantize_mxfp8(x)
    assert not m["sf"].any() and not m["codes"].any()


def test_zero_block_inside_nonzero_tensor():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(2, 64)).astype(np.float32)
    x[1, 16:32] = 0
    x[1, 20] = -0.0
    q = Q.quantize_nvfp4(x)
    assert q["sf"][1, 1] == 0
    codes = Q.unpack_fp4(q["codes"])
    assert list(codes[1, 16:32]) == [0x8 if i == 4 else 0 for i in range(16)]


def test_power_of_two_scale_invariance():
    # scaling the whole tensor by 2^k leaves NVFP4 codes/scales unchanged
    # (g scales with it) and shifts every MXFP8 scale code by k
    rng = np.random.default_rng(5)
    x = torch.randn(8, 128, generator=torch.Generator().manual_seed(5)).bfloat16()
    for k in (-6, 3):
        xs = (x.float() * 2.0 ** k).bfloat16()
        a, b = Q.quantize_nvfp4(x), Q.quantize_nvfp4(xs)
        assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["sf"], b["sf"])
        assert b["g"] == a["g"] * f32(2.0 ** k)
        a, b = Q.quantize_mxfp8(x), Q.quantize_mxfp8(xs)
        assert np.array_equal(a["codes"], b["codes"])
        assert np.array_equal(b["sf"].astype(int), a["sf"].astype(int) + k)


def test_sign_symmetry():
    x = torch.randn(4, 64, generator=torch.Generator().manual_seed(6)).bfloat16()
    a, b = Q.quantize_nvfp4(x), Q.quantize_nvfp4(-x)
    assert np.array_equal(Q.unpack_fp4(a["codes"]) ^ 0x8, Q.unpack_fp4(b["codes"]))
    a, b = Q.quantize_mxfp8(x), Q.quantize_mxfp8(-x)
    assert np.array_equal(a["codes"] ^ 0x80, b["codes"])


def test_nvfp4_error_bound():
    # each element is within half an E2M1 step (<= 1 at the top of [4,6]) of
    # its block scale, after clamping at 6: |x - deq| <= s * 1 (plus the E4M3
    # rounding of the scale, which at most grows |x/s| to 6 * 1.0625)
    x = torch.randn(16, 256, generator=torch.Generator().manual_seed(7)).bfloat16()
    q = Q.quantize_nvfp4(x)
    deq = Q.dequant_nvfp4(q["codes"], q["sf"], q["g"])
    s = F.e4m3_decode(q["sf"]) * float(q["g"])
    err = np.abs(deq - x.float().numpy()).reshape(16, 16, 16)
    assert np.all(err <= s[:, :, None] * 1.0 + 1e-12)


def _sf_layout_fixture():
    """(r, c, C, offset) entries and (rows, C, size) entries of sf_layout.txt."""
    entries, sizes = [], []
    for parts in _lines("sf_layout.txt"):
        if parts[0] == "size":
            sizes.append(tuple(int(v) for v in parts[1:4]))
        else:
            entries.append(tuple(int(v) for v in parts[:4]))
    return entries, sizes


def test_swizzle_matches_hand_worked_layout():
    # each scale alone in an otherwise empty matrix must land at the byte the
    # published layout gives (a swapped or dropped term moves it)
    entries, sizes = _sf_layout_fixture()
    assert len(entries) >= 12
    for r, c, C, off in entries:
        R = r + 1
        sf = np.zeros((R, C), dtype=np.uint8)
        sf[r, c] = 0xA5
        swz = Q.swizzle_sf(sf)
        assert swz.size == Q.sf_bytes(R, C * 16, 16)
        assert np.flatnonzero(swz).tolist() == [off], (r, c, C, off, np.flatnonzero(swz))
        # and the inverse reads the byte at that offset back to (r, c)
        flat = np.zeros(swz.size, dtype=np.uint8)
        flat[off] = 0x5A
        back = Q.unswizzle_sf(flat, R, C)
        assert back[r, c] == 0x5A and np.count_nonzero(back) == 1, (r, c, C, off)
    for rows, C, size in sizes:
        assert Q.sf_bytes(rows, C * 16, 16) == size
        assert Q.sf_bytes(rows, C * 32, 32) == size
        assert Q.swizzle_sf(np.ones((rows, C), dtype=np.uint8)).size == size


def test_swizzle_roundtrip_and_padding():
    rng = np.random.default_rng(8)
    for R, C in [(1, 4), (130, 8), (256, 12), (77, 4)]:
        sf = rng.integers(1, 255, size=(R, C)).astype(np.uint8)
        swz = Q.swizzle_sf(sf)
        assert swz.size == Q.sf_bytes(R, C * 16, 16)
        assert np.array_equal(Q.unswizzle_sf(swz, R, C), sf)
        assert np.count_nonzero(swz) == np.count_nonzero(sf)  # padding is zero


def test_pack_unpack_fp4():
    c = np.arange(32, dtype=np.uint8).reshape(2, 16) & 0xF
    p = Q.pack_fp4(c)
    assert p[0, 0] == (c[0, 0] | (c[0, 1] << 4))
    assert np.array_equal(Q.unpack_fp4(p), c)


def test_mxfp8_rceil_scale_closed_form():
    # one element per block, |x| = 2^p * (1 + f): the ceiling rule adds one to
    # the floor rule's exponent exactly when 1 + f > 448 / 256 = 1.75
    for p in range(-120, 120, 9):
        for f in (0.0, 0.5, 0.75, 0.7578125, 0.99):
            x = np.zeros((1, 32), dtype=np.float32)
            x[0, 5] = f32(2.0 ** p * (1 + f))
            qf = Q.quantize_mxfp8(x)
            qc = Q.quantize_mxfp8(x, scale_rule="rceil")
            want = max(p - 8 + (1 if 1 + f > 1.75 else 0), -127) + 127
            assert qc["sf"][0, 0] == want, (p, f)
            assert qf["sf"][0, 0] == max(p - 8, -127) + 127


def test_mxfp8_rceil_never_saturates():
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, size=(64, 1)))).astype(np.float32)
    q = Q.quantize_mxfp8(x, scale_rule="rceil")
    X = q["sf"].astype(np.int64) - 127
    bamax = np.abs(x).reshape(64, 8, 32).max(axis=2).astype(np.float64)
    scaled = bamax * np.ldexp(1.0, -X)
    # the block maximum lands in the top binade (224, 448] and so encodes
    # without saturating
    assert np.all((scaled > 224) & (scaled <= 448))
    deq = Q.dequant_mxfp8(q["codes"], q["sf"])
    assert np.all(np.abs(deq).reshape(64, 8, 32).max(axis=2) <= 448.0 * np.ldexp(1.0, X))
    with pytest.raises(ValueError):
        Q.quantize_mxfp8(x, scale_rule="ceil")
