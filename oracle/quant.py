"""Dynamic quantisation to NVFP4 and MXFP8 (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

Source passages (B200 MXFP8/NVFP4 diffusion article):

* "Glossary - Microscaling Formats": a small block of 16-32 elements shares
  one higher-precision scale factor.
* "Glossary - MXFP8": the OCP-standard 8-bit MX format -> E4M3 elements,
  32-element blocks, E8M0 power-of-two scale (OCP MX v1.0 conversion).
* "Glossary - NVFP4": NVIDIA's Blackwell 4-bit float -> E2M1 elements,
  16-element blocks, E4M3 block scale.
* "Detailed by section" (the TorchAO configuration listing):
  ``use_dynamic_per_tensor_scale=True`` -> an fp32 per-tensor scale computed
  on every call from the tensor's global amax; activations are quantised
  dynamically, weights once, in the same format.

The pages fix no constant, order of operations or rounding rule.  The readings
used here (all arithmetic in IEEE fp32 with round-to-nearest-even and
subnormals kept, the precision the kernels decide codes in):

NVFP4, tensor X [R, K]:
  1. amax = max |x|;  g = amax / 2688 (2688 = 6 * 448, the largest E2M1
     magnitude times the largest E4M3 magnitude); g = 1 when amax == 0.
  2. per row and 16-element block: bamax = max |x_i|;
     sf = E4M3(bamax / (6 * g))   (6 * g rounded to fp32 first).
  3. s = value(sf) * g;  inv = 1 / s, or 0 when s == 0.
  4. code_i = E2M1(x_i * inv).  Element 2j goes in the low nibble of byte j.
  5. Dequantised value = value(code) * value(sf) * g.
  Without the per-tensor scale (the listing's flag switched off; reading: the
  block scale then carries the whole range) g = 1 in every step above, so
  sf = E4M3(bamax / 6), saturating at 448, and no amax is taken.

MXFP8, tensor X [R, K] (OCP MX v1.0, scale from floor(log2 amax)):
  1. per row and 32-element block: e = floor(log2(bamax)), exact;
     X = clamp(e - 8, -127, 127) (8 = E4M3's largest exponent); sf = X + 127;
     a zero block gets sf = 0 (X = -127).
  2. code_i = E4M3(x_i * 2^-X)  (exact power-of-two multiply in fp32).
  3. Dequantised value = value(code) * 2^(sf - 127).

Scale-factor layout handed to the tensor cores (the pages are silent; this is
the public Blackwell block-scaling layout): tiles of 128 rows x 4 scale
columns = 512 bytes; inside a tile byte (r % 32) * 16 + ((r // 32) % 4) * 4
+ (c % 4); tiles ordered row-block-major, tile = (r // 128) * ceil(C / 4) +
c // 4; rows padded to 128 and columns to 4 with zero bytes.
"""

from __future__ import annotations

import numpy as np

from .formats import e2m1_encode, e4m3_encode, e4m3_decode, e2m1_decode, e8m0_decode

__all__ = [
    "amax", "nvfp4_global_scale", "quantize_nvfp4", "quantize_mxfp8",
    "swizzle_sf", "unswizzle_sf", "sf_bytes", "pack_fp4", "unpack_fp4",
    "dequant_nvfp4", "dequant_mxfp8",
    "NVFP4_BLOCK", "MXFP8_BLOCK",
]

NVFP4_BLOCK = 16
MXFP8_BLOCK = 32
_F32 = np.float32


def _as_f32(x) -> np.ndarray:
    """bf16 tensor / float array -> float32 numpy (bf16 -> fp32 is exact)."""
    try:
        import torch  # only for accepting torch tensors as input
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").float().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype != np.float32:
        raise TypeError("expected float32 values (or a torch bf16 tensor)")
    return x


def amax(x) -> np.float32:
    """Global max |x| of a tensor (exact)."""
    x = _as_f32(x)
    if x.size == 0:
        return _F32(0.0)
    return _F32(np.max(np.abs(x)))


def nvfp4_global_scale(a: np.float32) -> np.float32:
    """g = amax / (6 * 448) in fp32, and 1 for an all-zero tensor."""
    a = _F32(a)
    if a == 0:
        return _F32(1.0)
    return _F32(a / _F32(2688.0))


def pad_to(n: int, m: int) -> int:
    return (n + m - 1) // m * m


def sf_bytes(rows: int, k: int, block: int) -> int:
    """Size of the swizzled scale-factor array: pad128(rows) * pad4(k / block)."""
    return pad_to(rows, 128) * pad_to(k // block, 4)


def swizzle_sf(sf_plain: np.ndarray) -> np.ndarray:
    """[R, C] scale bytes -> flat swizzled array (zero padded)."""
    R, C = sf_plain.shape
    Rp, Cp = pad_to(R, 128), pad_to(C, 4)
    out = np.zeros(Rp * Cp, dtype=np.uint8)
    r = np.arange(R)[:, None]
    c = np.arange(C)[None, :]
    tile = (r // 128) * (Cp // 4) + c // 4
    off = tile * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)
    out[off] = sf_plain
    return out


def unswizzle_sf(sf_swz: np.ndarray, R: int, C: int) -> np.ndarray:
    """Inverse of swizzle_sf for the first R rows and C columns."""
    Cp = pad_to(C, 4)
    r = np.arange(R)[:, None]
    c = np.arange(C)[None, :]
    tile = (r // 128) * (Cp // 4) + c // 4
    off = tile * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)
    return np.asarray(sf_swz)[off]


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes, element 2j in the low nibble."""
    codes = codes.astype(np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """[R, K/2] bytes -> [R, K] 4-bit codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    R, H = packed.shape
    out = np.empty((R, 2 * H), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def quantize_nvfp4(x, global_amax=None, tensor_scale=True):
    """NVFP4 quantisation of X [R, K] (K a multiple of 16).

    Returns dict(codes=[R, K/2] uint8 packed, sf=[R, K/16] uint8 (E4M3),
    sf_swz=flat swizzled scale array, g=float32 per-tensor scale,
    amax=float32).  ``global_amax`` overrides the tensor's own amax (used when
    the amax comes from elsewhere, e.g. a reduction across shards).
    ``tensor_scale=False``: no per-tensor scale, g = 1 and no amax is taken
    (amax is reported as 0).
    """
    x = _as_f32(x)
    R, K = x.shape
    if K % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    if tensor_scale:
        a = amax(x) if global_amax is None else _F32(global_amax)
        g = nvfp4_global_scale(a)
    else:
        if global_amax is not None:
            raise ValueError("global_amax needs the per-tensor scale")
        a, g = _F32(0.0), _F32(1.0)
    blocks = x.reshape(R, K // NVFP4_BLOCK, NVFP4_BLOCK)
    bamax = np.max(np.abs(blocks), axis=2) if K else np.zeros((R, 0), _F32)
    denom = _F32(_F32(6.0) * g)
    sf = e4m3_encode((bamax / denom).astype(_F32))
    s = (e4m3_decode(sf).astype(_F32) * g).astype(_F32)
    with np.errstate(divide="ignore"):
        inv = np.where(s == 0, _F32(0.0), _F32(1.0) / np.where(s == 0, _F32(1.0), s)).astype(_F32)
    q = (blocks * inv[:, :, None]).astype(_F32)
    codes = e2m1_encode(q).reshape(R, K)
    return dict(codes=pack_fp4(codes), sf=sf, sf_swz=swizzle_sf(sf), g=g, amax=a)


def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for positive float32 values, exactly (frexp is exact)."""
    _, e = np.frexp(a.astype(np.float64))  # a = f * 2^e, f in [0.5, 1)
    return e.astype(np.int64) - 1


def quantize_mxfp8(x, scale_rule="floor"):
    """MXFP8 quantisation of X [R, K] (K a multiple of 32).

    Returns dict(codes=[R, K] uint8 (E4M3), sf=[R, K/32] uint8 (E8M0),
    sf_swz=flat swizzled scale array).

    scale_rule "floor" is the OCP rule above.  "rceil" (TorchAO's ceiling
    mode; the pages name only the OCP standard) takes the smallest X with
    bamax <= 448 * 2^X, so no element saturates; since 2^e <= bamax < 2^(e+1)
    that X is e - 8 or e - 7, decided by one exact comparison.
    """
    if scale_rule not in ("floor", "rceil"):
        raise ValueError(scale_rule)
    x = _as_f32(x)
    R, K = x.shape
    if K % MXFP8_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(R, K // MXFP8_BLOCK, MXFP8_BLOCK)
    bamax = np.max(np.abs(blocks), axis=2) if K else np.zeros((R, 0), _F32)
    pos = bamax > 0
    e = np.where(pos, _floor_log2(np.where(pos, bamax, _F32(1.0))), -(1 << 20))
    X = e - 8
    if scale_rule == "rceil":
        over = bamax.astype(np.float64) > 448.0 * np.ldexp(1.0, np.maximum(X, -1000))
        X = np.where(pos & over, X + 1, X)
    X = np.clip(X, -127, 127)
    sf = (X + 127).astype(np.uint8)
    mult = np.ldexp(np.ones_like(X, dtype=np.float64), -X).astype(_F32)  # 2^-X, exact in fp32
    q = (blocks * mult[:, :, None]).astype(_F32)
    codes = e4m3_encode(q).reshape(R, K)
    return dict(codes=codes, sf=sf, sf_swz=swizzle_sf(sf))


def dequant_nvfp4(codes: np.ndarray, sf: np.ndarray, g) -> np.ndarray:
    """[R, K/2] packed codes, [R, K/16] scales, per-tensor g -> float64 [R, K]."""
    vals = e2m1_decode(unpack_fp4(codes))
    R, K = vals.shape
    scale = e4m3_decode(sf) * np.float64(g)
    return (vals.reshape(R, K // NVFP4_BLOCK, NVFP4_BLOCK) * scale[:, :, None]).reshape(R, K)


def dequant_mxfp8(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """[R, K] E4M3 codes, [R, K/32] E8M0 scales -> float64 [R, K]."""
    vals = e4m3_decode(codes)
    R, K = vals.shape
    scale = e8m0_decode(sf)
    return (vals.reshape(R, K // MXFP8_BLOCK, MXFP8_BLOCK) * scale[:, :, None]).reshape(R, K)
