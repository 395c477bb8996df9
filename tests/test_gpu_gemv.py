"""GPU parity of the bf16 layer at M <= 8 rows (the CUDA-core weight-stream
kernel that mxq_gemm_blockscaled and mxq_linear's bf16 branch use there):
every output within |gpu - oracle| <= 2e-3 * sum_k |a_k b_k| + 1e-6 of the
float64 product of the same bf16 operands (or equal to it rounded to bf16);
columns past N and rows past M of a padded output left untouched."""

import numpy as np
import pytest
import torch

import workloads
from oracle import gemm as G
from tests._gpu import DEV, assert_within_tol

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu


def _gemv(A, W, bias):
    """The bf16 layer through mxq_gemm_blockscaled with the output's leading
    dimension rounded up to 8 (16-byte rows), so that any N is allowed."""
    M, K = A.shape
    N = W.shape[0]
    ldy = (N + 7) // 8 * 8
    y = torch.full((M, ldy), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxq.gemm_blockscaled("bf16", M, N, K, A.to(DEV), None, None, W.to(DEV), None, None,
                         None if bias is None else bias.to(DEV), y, ldy=ldy)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    return y[:, :N]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("K,N", [(72, 1000), (3080, 37), (3072, 9216), (8, 5), (1032, 4099)])
def test_gemv_matches_oracle(M, K, N):
    # N % 4 != 0: the last warp task holds fewer than four rows of W;
    # K % 256 != 0: the last step covers part of a warp
    c = workloads.random_case(M, K, N, "bf16", seed=M * 131 + K + N)
    y = _gemv(c.A, c.W, c.bias)
    Y, T, _, _ = G.linear_ref_quantized("bf16", c.A, c.W, c.bias)
    assert_within_tol(y, Y, T, f"bf16 {M}x{K}x{N}")


def test_gemv_no_bias_and_padded_output():
    M, K, N, ldy = 3, 264, 300, 320
    c = workloads.random_case(M, K, N, "bf16", seed=5)
    A, W = c.A.to(DEV), c.W.to(DEV)
    y = torch.full((M + 1, ldy), 7.0, dtype=torch.bfloat16, device=DEV)
    mxq.gemm_blockscaled("bf16", M, N, K, A, None, None, W, None, None, None, y, ldy=ldy)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    Y, T, _, _ = G.linear_ref_quantized("bf16", c.A, c.W, None)
    assert_within_tol(y[:M, :N], Y, T, "bf16 no bias, ldy > N")
    assert torch.all(y[:M, N:] == 7.0) and torch.all(y[M] == 7.0)


def test_gemv_through_linear_on_the_flux_modulation_shape():
    # the FLUX modulation layer (3072 -> 18432) at batch 1 and 4 through the
    # dispatcher's bf16 branch; sampled columns against the oracle
    K, N = 3072, 18432
    for M in (1, 4):
        c = workloads.random_case(M, K, N, "bf16", seed=M)
        w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt="nvfp4")
        assert mxq.linear_path(w.handle, M) == mxq.BF16
        y = mxq.linear_forward(w, c.A.to(DEV))
        torch.cuda.synchronize()
        cols = np.unique(np.r_[0, 1, N - 1, np.random.default_rng(M).integers(0, N, 200)])
        ci = torch.as_tensor(cols)
        Y, T = G.linear_ref(c.A.float().numpy().astype(np.float64), c.W.float()[ci].numpy().astype(np.float64),
                            c.bias[ci])
        assert_within_tol(y[:, torch.as_tensor(cols, device=DEV)], Y, T, f"linear bf16 M={M}")
