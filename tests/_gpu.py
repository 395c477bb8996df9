"""Helpers of the GPU parity tests: run the CUDA path through the C-ABI
binding on seeded inputs, and compare with the oracle."""

import numpy as np
import torch

import fp8_gemm_diffusion_b200 as mxq
from oracle import quant as Q
from oracle import gemm as G

DEV = "cuda"


def gpu_quant_nvfp4(x_dev, amax_dev=None):
    """Run mxq_amax (unless an amax is given) + mxq_quantize_nvfp4."""
    rows, k = x_dev.shape
    if amax_dev is None:
        amax_dev = torch.full((1,), 123.0, dtype=torch.float32, device=DEV)  # overwritten
        mxq.amax(x_dev, amax_dev)
    codes = torch.full((max(mxq.codes_bytes(rows, k, "nvfp4"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    sf = torch.full((max(mxq.sf_bytes(rows, k, "nvfp4"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    g = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    mxq.quantize_nvfp4(x_dev, amax_dev, codes, sf, g)
    torch.cuda.synchronize()
    return dict(amax=amax_dev, codes=codes, sf=sf, g=g)


def gpu_quant_mxfp8(x_dev):
    rows, k = x_dev.shape
    codes = torch.full((max(mxq.codes_bytes(rows, k, "mxfp8"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    sf = torch.full((max(mxq.sf_bytes(rows, k, "mxfp8"), 1),), 0xEE, dtype=torch.uint8, device=DEV)
    mxq.quantize_mxfp8(x_dev, codes, sf)
    torch.cuda.synchronize()
    return dict(codes=codes, sf=sf)


def assert_nvfp4_equal(gq, oq, rows, k):
    codes = gq["codes"].cpu().numpy()[: rows * k // 2].reshape(rows, k // 2)
    sf = gq["sf"].cpu().numpy()
    assert float(gq["amax"].item()) == float(oq["amax"]), "amax"
    assert np.float32(gq["g"].item()) == oq["g"], "per-tensor scale g"
    bad = np.argwhere(codes != oq["codes"])
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    bad = np.flatnonzero(sf != oq["sf_swz"])
    assert bad.size == 0, f"{len(bad)} scale bytes differ, first at {bad[:4].tolist()}"


def assert_mxfp8_equal(gq, oq, rows, k):
    codes = gq["codes"].cpu().numpy()[: rows * k].reshape(rows, k)
    sf = gq["sf"].cpu().numpy()
    bad = np.argwhere(codes != oq["codes"])
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:4].tolist()}"
    bad = np.flatnonzero(sf != oq["sf_swz"])
    assert bad.size == 0, f"{len(bad)} scale bytes differ, first at {bad[:4].tolist()}"


def assert_within_tol(Y_gpu, Y_ref, T, what=""):
    Yg = Y_gpu.float().cpu().numpy().astype(np.float64) if isinstance(Y_gpu, torch.Tensor) else Y_gpu
    ok = G.within_tol(Yg, Y_ref, T)
    if not ok.all():
        idx = np.argwhere(~ok)
        i, j = idx[0]
        raise AssertionError(
            f"{what}: {len(idx)} of {ok.size} outputs out of tolerance; first ({i},{j}): "
            f"gpu={Yg[i, j]!r} ref={Y_ref[i, j]!r} T={T[i, j]!r}")


def run_gemm(fmt, A, W, bias=None):
    """Quantise A and W on the GPU (through the C-ABI), run the GEMM, return
    Y (bf16 on the device)."""
    M, K = A.shape
    N = W.shape[0]
    Ad, Wd = A.to(DEV), W.to(DEV)
    bd = bias.to(DEV) if bias is not None else None
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    if fmt == "bf16":
        mxq.gemm_blockscaled("bf16", M, N, K, Ad, None, None, Wd, None, None, bd, y)
    elif fmt == "nvfp4":
        qa, qw = gpu_quant_nvfp4(Ad), gpu_quant_nvfp4(Wd)
        mxq.gemm_blockscaled("nvfp4", M, N, K, qa["codes"], qa["sf"], qa["g"], qw["codes"],
                             qw["sf"], qw["g"], bd, y)
    else:
        qa, qw = gpu_quant_mxfp8(Ad), gpu_quant_mxfp8(Wd)
        mxq.gemm_blockscaled("mxfp8", M, N, K, qa["codes"], qa["sf"], None, qw["codes"],
                             qw["sf"], None, bd, y)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    return y
