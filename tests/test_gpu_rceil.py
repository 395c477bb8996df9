"""GPU parity of the MXFP8 ceiling scale rule (RCEIL).

The ceiling rule picks the smallest shared exponent X with bamax <= 448 * 2^X,
so no element of a block saturates (the OCP floor rule, the default, lets
values in [448, 512) * 2^X saturate).  It differs from the floor rule exactly
when the block maximum's significand exceeds 1.75 (448 = 1.75 * 2^8).  Codes
and swizzled scales must match the oracle (quantize_mxfp8(scale_rule="rceil"))
bit for bit, padding included.
"""

import numpy as np
import pytest
import torch

import fp8_gemm_diffusion_b200 as mxq
import workloads
from oracle import gemm as G
from oracle import quant as Q

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(rows, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, k, generator=g) * torch.exp(torch.empty(rows, 1).uniform_(-30, 30, generator=g))
    # block maxima at, just under and just over 1.75 * 2^e (bf16 neighbours of
    # 1.75 are 1.75 -/+ 2^-7), at the largest significand, and a subnormal block
    edge = [1.75, 1.7421875, 1.7578125, 1.9921875, 1.0]
    for i, f in enumerate(edge):
        if 32 * (i + 1) <= k:
            # every other element below the planted maximum in magnitude
            x[0, 32 * i:32 * (i + 1)] = torch.linspace(-0.9, 0.9, 32) * (f * 2.0 ** 5)
            x[0, 32 * i] = f * 2.0 ** 5
    if rows > 1:
        x[1, :32] = 1e-39
        x[1, 32:64] = -3.5 * 2.0 ** -130
    return x.bfloat16()


@pytest.mark.parametrize("rows,k,seed", [(130, 256, 1), (1, 128, 2), (2, 256, 4), (257, 384, 3)])
def test_mxfp8_rceil_bit_exact(rows, k, seed):
    x = _case(rows, k, seed)
    codes = torch.full((rows * k,), 0xEE, dtype=torch.uint8, device=DEV)
    sf = torch.full((mxq.sf_bytes(rows, k, "mxfp8"),), 0xEE, dtype=torch.uint8, device=DEV)
    mxq.quantize_mxfp8(x.to(DEV), codes, sf, scale_rule=mxq.SCALE_RCEIL)
    torch.cuda.synchronize()
    o = Q.quantize_mxfp8(x, scale_rule="rceil")
    assert np.array_equal(codes.cpu().numpy().reshape(rows, k), o["codes"])
    assert np.array_equal(sf.cpu().numpy(), o["sf_swz"])


def test_linear_rceil():
    M, K, N = 1280, 1024, 1536
    g = torch.Generator().manual_seed(8)
    W = (torch.randn(N, K, generator=g) * 0.02).bfloat16()
    b = (torch.randn(N, generator=g) * 0.02).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    layer = mxq.Weight(W.to(DEV), b.to(DEV), fmt="mxfp8", mxfp8_rceil=True)
    assert layer.handle.flags == mxq.WEIGHT_MXFP8_RCEIL
    y = mxq.linear_forward(layer, A.to(DEV))
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    rows = np.unique(np.random.default_rng(1).integers(0, M, 48))
    qa = Q.quantize_mxfp8(A[torch.as_tensor(rows)], scale_rule="rceil")
    qw = Q.quantize_mxfp8(W, scale_rule="rceil")
    Y, T = G.linear_ref(Q.dequant_mxfp8(qa["codes"], qa["sf"]), Q.dequant_mxfp8(qw["codes"], qw["sf"]), b)
    Yg = y[torch.as_tensor(rows, device=DEV)].float().cpu().numpy().astype(np.float64)
    assert G.within_tol(Yg, Y, T).all()


def test_mxfp8_rceil_c2_activation_bit_exact():
    A = workloads.make_case("c2").A
    rows, k = A.shape
    codes = torch.empty(rows * k, dtype=torch.uint8, device=DEV)
    sf = torch.full((mxq.sf_bytes(rows, k, "mxfp8"),), 0xEE, dtype=torch.uint8, device=DEV)
    mxq.quantize_mxfp8(A.to(DEV), codes, sf, scale_rule=mxq.SCALE_RCEIL)
    torch.cuda.synchronize()
    o = Q.quantize_mxfp8(A, scale_rule="rceil")
    assert np.array_equal(sf.cpu().numpy(), o["sf_swz"])
    assert np.array_equal(codes.cpu().numpy().reshape(rows, k), o["codes"])
    # the ceiling rule moved some blocks of this activation (else the case pins nothing)
    floor = Q.quantize_mxfp8(A[:256])
    assert (o["sf"][:256] != floor["sf"]).any()
