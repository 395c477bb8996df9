"""GPU parity of the tcgen05 GEMMs (NVFP4, MXFP8, bf16) and of mxq_linear:
every output element within |gpu - oracle| <= 2e-3 * sum_k |a_k b_k| + 1e-6,
the oracle accumulating in float64 over its own quantisation of the same
seeded inputs (so the whole chain, quantiser included, is checked)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import gemm as G
from oracle import quant as Q
from tests._gpu import DEV, assert_within_tol, run_gemm

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu

SHAPES = [
    # (M, K, N): one tile, several tiles, ragged M/N, partial last k-stage
    (128, 256, 128),
    (128, 256, 192),
    (256, 512, 384),
    (200, 320, 200),
    (1, 64, 136),
    (333, 1024, 520),
    (640, 768, 1152),
    # CTA-pair kernel edges: just above one CTA, a pair whose second CTA is
    # entirely out of range, a 128-wide pair tile, ragged N on a 256-wide tile
    (129, 256, 384),
    (300, 512, 128),
    (520, 1024, 136),
]


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8", "bf16"])
@pytest.mark.parametrize("M,K,N", SHAPES)
def test_gemm_small_shapes(fmt, M, K, N):
    if fmt == "mxfp8" and K % 128:
        K = (K + 127) // 128 * 128
    c = workloads.random_case(M, K, N, fmt, seed=M * 7 + N)
    y = run_gemm(fmt, c.A, c.W, c.bias)
    Y, T, _, _ = G.linear_ref_quantized(fmt, c.A, c.W, c.bias)
    assert_within_tol(y, Y, T, f"{fmt} {M}x{K}x{N}")


def test_gemm_nvfp4_c1():
    c = workloads.c1_nvfp4_small()
    y = run_gemm("nvfp4", c.A, c.W)
    Y, T, _, _ = G.linear_ref_quantized("nvfp4", c.A, c.W)
    assert_within_tol(y, Y, T, "c1")


def _sample_rows(M, seed=0, n=192):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.arange(0, 32), np.arange(M - 160, M), rng.integers(0, M, n)]))


@pytest.mark.parametrize("cfg", ["c2", "c3"])
def test_gemm_full_size_sampled_rows(cfg):
    c = workloads.make_case(cfg)
    y = run_gemm(c.fmt, c.A, c.W, c.bias)
    rows = _sample_rows(c.M)
    Y, T, _, _ = G.linear_ref_quantized(c.fmt, c.A, c.W, c.bias, rows=rows)
    assert_within_tol(y[torch.from_numpy(rows).to(DEV)], Y, T, cfg)


def test_gemm_full_size_c4_sampled_rows():
    c = workloads.c4_nvfp4_mlp_down()
    y = run_gemm("nvfp4", c.A, c.W)
    rows = _sample_rows(c.M, n=96)
    amax = Q.amax(c.A)
    qa = Q.quantize_nvfp4(c.A[rows], global_amax=amax)
    qw = Q.quantize_nvfp4(c.W)
    Y, T = G.linear_ref(Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"]),
                        Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"]))
    assert_within_tol(y[torch.from_numpy(rows).to(DEV)], Y, T, "c4")


def test_gemm_zero_activation_gives_bias():
    c = workloads.random_case(256, 512, 384, "nvfp4", seed=3)
    A = torch.zeros_like(c.A)
    y = run_gemm("nvfp4", A, c.W, c.bias)
    expect = c.bias.to(DEV)[None, :].expand(256, 384)
    assert torch.equal(y, expect)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_linear_dispatch(fmt):
    M, K, N = 1024, 1024, 1152
    c = workloads.random_case(M, K, N, fmt, seed=12)
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt=fmt)
    x = c.A.to(DEV)
    y = mxq.linear_forward(w, x)  # quantised path (min dim == 1024)
    Y, T, _, _ = G.linear_ref_quantized(fmt, c.A, c.W, c.bias)
    assert_within_tol(y, Y, T, "linear quantised")
    y2 = mxq.linear_forward(w, x[:512].contiguous())  # M = 512 -> bf16 path
    Yb, Tb, _, _ = G.linear_ref_quantized("bf16", c.A[:512], c.W, c.bias)
    assert_within_tol(y2, Yb, Tb, "linear bf16")
    wk = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt=fmt, keep_bf16=True)
    y3 = mxq.linear_forward(wk, x)
    Yk, Tk, _, _ = G.linear_ref_quantized("bf16", c.A, c.W, c.bias)
    assert_within_tol(y3, Yk, Tk, "linear keep_bf16")
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK


def test_weight_prepare_matches_oracle():
    c = workloads.c3_nvfp4_mlp_up()
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt="nvfp4")
    torch.cuda.synchronize()
    N, K = c.W.shape
    oq = Q.quantize_nvfp4(c.W)
    st = w.storage.cpu().numpy()
    off = 256
    codes = st[off: off + N * K // 2].reshape(N, K // 2)
    assert np.array_equal(codes, oq["codes"])
    sf_off = off + (N * K // 2 + 255) // 256 * 256
    assert np.array_equal(st[sf_off: sf_off + Q.sf_bytes(N, K, 16)], oq["sf_swz"])
    assert np.frombuffer(st[4:8].tobytes(), np.float32)[0] == oq["g"]
