"""GPU parity of the quantisation kernels (amax, NVFP4, MXFP8) and of the
device conversion routines: bit-exact against the oracle, padding included."""

import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import quant as Q
from tests._gpu import (DEV, assert_mxfp8_equal, assert_nvfp4_equal, gpu_quant_mxfp8,
                        gpu_quant_nvfp4)

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu


def _gpu_convert(xs: np.ndarray, fmt: int) -> np.ndarray:
    xin = torch.from_numpy(xs).to(DEV)
    out = torch.empty(xs.size, dtype=torch.uint8, device=DEV)
    mxq.convert_f32(xin, xs.size, fmt, out)
    return out.cpu().numpy()


def _window(e_lo, e_hi):
    """Every positive float32 with exponent field in [e_lo, e_hi] (all mantissas)."""
    for e in range(e_lo, e_hi + 1):
        bits = (np.uint32(e) << np.uint32(23)) | np.arange(1 << 23, dtype=np.uint32)
        yield bits.view(np.float32)


def test_e2m1_conversion_exhaustive_window():
    # every fp32 in [2^-4, 2^4) (all mantissas): every rounding decision of
    # E2M1 happens in here; below rounds to 0, above saturates (checked next)
    for xs in _window(127 - 4, 127 + 3):
        assert np.array_equal(_gpu_convert(xs, 1), F.e2m1_encode(xs))
        neg = -xs[::97]
        assert np.array_equal(_gpu_convert(neg, 1), F.e2m1_encode(neg))


def test_e4m3_conversion_exhaustive_window():
    # every fp32 in [2^-12, 2^10): all E4M3 normal / subnormal / saturation decisions
    for xs in _window(127 - 12, 127 + 9):
        assert np.array_equal(_gpu_convert(xs, 2), F.e4m3_encode(xs))
        neg = -xs[::97]
        assert np.array_equal(_gpu_convert(neg, 2), F.e4m3_encode(neg))


def test_conversion_outside_window_and_zeros():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 0x7F800000, size=1 << 22, dtype=np.uint32)  # all finite positives
    xs = np.concatenate([bits.view(np.float32), np.array([0.0, -0.0, 3.4e38, -3.4e38,
                                                         1e-45, -1e-45], dtype=np.float32)])
    xs = np.concatenate([xs, -xs[: 1 << 20]])
    assert np.array_equal(_gpu_convert(xs, 1), F.e2m1_encode(xs))
    assert np.array_equal(_gpu_convert(xs, 2), F.e4m3_encode(xs))


NVFP4_CASES = [
    ("c1_A", lambda: workloads.c1_nvfp4_small().A),
    ("c1_W", lambda: workloads.c1_nvfp4_small().W),
    ("c3_A", lambda: workloads.c3_nvfp4_mlp_up().A),
    ("rows1_k64", lambda: workloads.random_case(1, 64, 8, "nvfp4", seed=1).A),
    ("rows77_k192", lambda: workloads.random_case(77, 192, 8, "nvfp4", seed=2).A),
    ("rows130_k320", lambda: workloads.random_case(130, 320, 8, "nvfp4", seed=3).A),
    ("rows257_k1024", lambda: workloads.random_case(257, 1024, 8, "nvfp4", seed=4, a_std=1e-3).A),
    # the two-pass kernels deal row chunks to warps (1024 elements for the
    # amax, 2048 for the encode pass): K = 5184 ends both on a partial chunk,
    # and 3000 rows give more chunks than warps, so a warp's walk carries
    # from one row's chunks into the next row's
    ("rows3000_k5184", lambda: workloads.random_case(3000, 5184, 8, "nvfp4", seed=7).A),
]


@pytest.mark.parametrize("name,make", NVFP4_CASES, ids=[c[0] for c in NVFP4_CASES])
def test_nvfp4_quantize_bit_exact(name, make):
    x = make()
    rows, k = x.shape
    assert_nvfp4_equal(gpu_quant_nvfp4(x.to(DEV)), Q.quantize_nvfp4(x), rows, k)


def test_nvfp4_special_values():
    g = torch.Generator().manual_seed(9)
    x = torch.randn(160, 256, generator=g)
    x[0, :16] = 0.0                         # zero block
    x[1, :16] = -0.0                        # negative-zero block
    x[2, 16:32] = 1e-38                     # tiny block next to normal ones
    x[3, :] = torch.linspace(-6, 6, 256)    # exact grid values
    x[5, ::7] = -x[5, ::7] * 1e4
    x = x.bfloat16()
    assert_nvfp4_equal(gpu_quant_nvfp4(x.to(DEV)), Q.quantize_nvfp4(x), 160, 256)


def test_nvfp4_huge_amax():
    x = torch.randn(128, 128, generator=torch.Generator().manual_seed(10))
    x[4, 5] = 3.0e38  # near the bf16 maximum: most blocks get a zero scale
    x[7, :16] = 1e36
    x = x.bfloat16()
    assert_nvfp4_equal(gpu_quant_nvfp4(x.to(DEV)), Q.quantize_nvfp4(x), 128, 128)


def test_nvfp4_zero_tensor_and_external_amax():
    x = torch.zeros(129, 128, dtype=torch.bfloat16)
    assert_nvfp4_equal(gpu_quant_nvfp4(x.to(DEV)), Q.quantize_nvfp4(x), 129, 128)
    # amax supplied by the caller (e.g. reduced over shards): larger than the tensor's own
    y = torch.randn(64, 128, generator=torch.Generator().manual_seed(3)).bfloat16()
    amax = torch.tensor([40.0], device=DEV)
    gq = gpu_quant_nvfp4(y.to(DEV), amax_dev=amax)
    oq = Q.quantize_nvfp4(y, global_amax=np.float32(40.0))
    assert_nvfp4_equal(gq, oq, 64, 128)


def test_nvfp4_strided_rows():
    base = torch.randn(96, 512, generator=torch.Generator().manual_seed(4)).bfloat16()
    view = base.to(DEV)[:, 64:320]  # ld = 512, k = 256
    gq = gpu_quant_nvfp4(view)
    assert_nvfp4_equal(gq, Q.quantize_nvfp4(base[:, 64:320].contiguous()), 96, 256)


def test_nvfp4_full_size_c4_sampled_rows():
    c = workloads.c4_nvfp4_mlp_down()
    rows, k = c.A.shape
    gq = gpu_quant_nvfp4(c.A.to(DEV))
    amax = Q.amax(c.A)
    assert float(gq["amax"].item()) == float(amax)
    sample = np.unique(np.concatenate([np.arange(0, 64), np.arange(rows - 200, rows),
                                       np.random.default_rng(0).integers(0, rows, 256)]))
    oq = Q.quantize_nvfp4(c.A[sample], global_amax=amax)
    codes = gq["codes"].cpu().numpy().reshape(rows, k // 2)[sample]
    assert np.array_equal(codes, oq["codes"])
    sf = Q.unswizzle_sf(gq["sf"].cpu().numpy(), rows, k // 16)[sample]
    assert np.array_equal(sf, oq["sf"])
    assert np.float32(gq["g"].item()) == oq["g"]


MXFP8_CASES = [
    ("c2_A", lambda: workloads.c2_mxfp8_qkv().A),
    ("c2_W", lambda: workloads.c2_mxfp8_qkv().W),
    ("rows1_k128", lambda: workloads.random_case(1, 128, 8, "mxfp8", seed=5).A),
    ("rows200_k384", lambda: workloads.random_case(200, 384, 8, "mxfp8", seed=6, a_std=300.0).A),
]


@pytest.mark.parametrize("name,make", MXFP8_CASES, ids=[c[0] for c in MXFP8_CASES])
def test_mxfp8_quantize_bit_exact(name, make):
    x = make()
    rows, k = x.shape
    assert_mxfp8_equal(gpu_quant_mxfp8(x.to(DEV)), Q.quantize_mxfp8(x), rows, k)


def test_mxfp8_special_values():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(130, 256, generator=g)
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    x[2, :32] = 1e-39          # bf16 subnormal block
    x[3, :32] = 3.0e38
    x[4, :] = torch.arange(256) * 2.0 - 200.0
    x = x.bfloat16()
    assert_mxfp8_equal(gpu_quant_mxfp8(x.to(DEV)), Q.quantize_mxfp8(x), 130, 256)


def test_empty_inputs_are_noops():
    x = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros(16, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(16, dtype=torch.uint8, device=DEV)
    mxq.quantize_mxfp8(x, codes, sf, rows=0, k=128, ld=128)
    amax = torch.full((1,), 7.0, device=DEV)
    mxq.amax(x, amax, rows=0, k=128, ld=128)
    torch.cuda.synchronize()
    assert amax.item() == 0.0 and not codes.any()
    assert mxq.get_device_error() == mxq.OK
