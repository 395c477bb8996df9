"""GPU parity over the linear stack of a FLUX-shaped DiT (19 double-stream +
38 single-stream blocks, hidden 3072, MLP 12288, 4608 tokens; batch 1 and 4):
every distinct layer shape runs once through mxq_linear with the selective
rule (bf16 when min(M, K, N) < 1024, NVFP4 otherwise), on seeded random
weights and activations.  Sampled output rows are compared with the oracle
within |gpu - oracle| <= 2e-3 * sum_k |a_k b_k| + 1e-6.

For the oracle side of the NVFP4 layers the per-tensor amax is taken over the
whole activation and only the sampled rows are quantised with it (block
scales depend only on their block and the per-tensor scale, so this equals
quantising everything and then selecting rows)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import dispatch as D
from oracle import gemm as G
from oracle import quant as Q
from tests._gpu import DEV, assert_within_tol

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu


def _shapes():
    out = []
    for B in (1, 4):
        seen = set()
        for l in workloads.flux_linear_stack(batch=B):
            key = (l["M"], l["K"], l["N"])
            if key not in seen:
                seen.add(key)
                out.append((B, l["name"], *key))
    return out


SHAPES = _shapes()
_W = {}


def _weight(N, K):
    """One seeded weight, bias and oracle quantisation per (N, K), shared by the layers."""
    if (N, K) not in _W:
        g = torch.Generator().manual_seed(1000 + N + 7 * K)
        W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
        b = (torch.randn(N, generator=g) * 0.02).to(torch.bfloat16)
        _W[(N, K)] = dict(W=W, b=b, qw=None)
    return _W[(N, K)]


def _rows(M, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.arange(0, min(M, 8)), np.arange(max(M - 8, 0), M),
                                     rng.integers(0, M, 32)]))


@pytest.mark.parametrize("B,name,M,K,N", SHAPES, ids=[f"b{s[0]}-{s[1]}-{s[2]}x{s[3]}x{s[4]}" for s in SHAPES])
def test_flux_layer(B, name, M, K, N):
    w = _weight(N, K)
    g = torch.Generator().manual_seed(M * 31 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    layer = mxq.Weight(w["W"].to(DEV), w["b"].to(DEV), fmt="nvfp4")
    path = mxq.linear_path(layer.handle, M)
    want = mxq.BF16 if D.use_bf16(M, K, N) else mxq.NVFP4
    assert path == want
    y = mxq.linear_forward(layer, A.to(DEV))
    torch.cuda.synchronize()
    rows = _rows(M, seed=M + N)
    if path == mxq.BF16:
        Y, T, _, _ = G.linear_ref_quantized("bf16", A, w["W"], w["b"], rows=rows)
    else:
        if w["qw"] is None:
            w["qw"] = Q.quantize_nvfp4(w["W"])
        qw = w["qw"]
        qa = Q.quantize_nvfp4(A[torch.as_tensor(rows)], global_amax=Q.amax(A))
        Ad = Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"])
        Wd = Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"])
        Y, T = G.linear_ref(Ad, Wd, w["b"])
    assert_within_tol(y[torch.as_tensor(rows, device=DEV)], Y, T, f"{name} {M}x{K}x{N}")
    assert mxq.get_device_error() == mxq.OK
    del y, layer
