"""GPU parity of NVFP4 without a per-tensor scale (g = 1): the quantiser with a
NULL amax, bit-exact against the oracle's tensor_scale=False reading, and
mxq_linear with a weight prepared with MXQ_WEIGHT_NO_TENSOR_SCALE, within
|gpu - oracle| <= 2e-3 * sum_k |a_k b_k| + 1e-6."""

import numpy as np
import pytest
import torch

from oracle import gemm as G
from oracle import quant as Q
from tests._gpu import DEV, assert_nvfp4_equal, assert_within_tol

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu


def _gpu_quant_unit_g(x_dev):
    rows, k = x_dev.shape
    codes = torch.full((max(mxq.codes_bytes(rows, k, "nvfp4"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    sf = torch.full((max(mxq.sf_bytes(rows, k, "nvfp4"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    g = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    mxq.quantize_nvfp4(x_dev, None, codes, sf, g)
    torch.cuda.synchronize()
    return dict(amax=torch.zeros(1), codes=codes, sf=sf, g=g)


def _case(rows, k, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, k, generator=g) * scale
    if rows > 3:
        x[1, :16] = 0.0                 # zero block
        x[2, 5] = 7.0e4                 # bamax / 6 above 448: saturated block scale
        x[3, 16:32] = 3.0e-3            # scale in E4M3's subnormal range
    return x.bfloat16()


@pytest.mark.parametrize("rows,k,seed,scale", [(200, 320, 1, 1.0), (1, 64, 2, 1.0), (129, 128, 3, 300.0),
                                               (640, 1024, 4, 0.01)])
def test_quantize_unit_g_bit_exact(rows, k, seed, scale):
    x = _case(rows, k, seed, scale)
    gq = _gpu_quant_unit_g(x.to(DEV))
    assert float(gq["g"].item()) == 1.0
    assert_nvfp4_equal(gq, Q.quantize_nvfp4(x, tensor_scale=False), rows, k)


@pytest.mark.parametrize("M,K,N", [(1280, 1024, 1536), (4608, 3072, 1024)])
def test_linear_unit_g(M, K, N):
    g = torch.Generator().manual_seed(M + N)
    W = (torch.randn(N, K, generator=g) * 0.02).bfloat16()
    b = (torch.randn(N, generator=g) * 0.02).bfloat16()
    A = (torch.randn(M, K, generator=g) * 3.0).bfloat16()
    layer = mxq.Weight(W.to(DEV), b.to(DEV), fmt="nvfp4", tensor_scale=False)
    assert layer.handle.flags == mxq.WEIGHT_NO_TENSOR_SCALE
    assert mxq.linear_path(layer.handle, M) == mxq.NVFP4
    assert mxq.linear_kernel_count(layer.handle, M) == 2
    y = mxq.linear_forward(layer, A.to(DEV))
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    # the weight's amax slot holds 0 and its per-tensor scale 1 (offsets 0 and 4
    # of the storage; the handle points there)
    assert layer.handle.amax_dev == layer.storage.data_ptr()
    assert layer.handle.g_dev == layer.storage.data_ptr() + 4
    assert layer.storage[:8].view(torch.float32).tolist() == [0.0, 1.0]
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(M - 8, M),
                                     np.random.default_rng(M).integers(0, M, 40)]))
    qa = Q.quantize_nvfp4(A[torch.as_tensor(rows)], tensor_scale=False)  # row-local: g = 1
    qw = Q.quantize_nvfp4(W, tensor_scale=False)
    Y, T = G.linear_ref(Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"]),
                        Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"]), b)
    assert_within_tol(y[torch.as_tensor(rows, device=DEV)], Y, T, f"unit-g linear {M}x{K}x{N}")
