"""mxq_linear_noalloc: the linear layer for callers that cannot allocate
device memory (a fixed device-memory budget, or no cudaMalloc allowed in a
latency-critical loop).  It must give the same result as mxq_linear with a
caller-allocated workspace, call after call, although every call reuses one
static device scratch array that keeps the previous call's contents.

This file is collected last on purpose, and passes both alone in a fresh
process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import gemm as G

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_noalloc_matches_linear_on_two_calls_in_a_row(fmt):
    M, K, N = 1024, 1024, 1152
    c = workloads.random_case(M, K, N, fmt, seed=31)
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt=fmt)
    # two different activations: the second has a much smaller amax, so a
    # stale amax or scale left in the scratch by the first call would show
    inputs = [c.A, (c.A.float() * 1e-3).bfloat16()]
    outs = []
    for a in inputs:
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        mxq.linear_noalloc(w.handle, a.to(DEV), M, y)
        outs.append(y)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    for a, y in zip(inputs, outs):
        ref = mxq.linear_forward(w, a.to(DEV))  # existing entry point, own workspace
        torch.cuda.synchronize()
        _, T, _, _ = G.linear_ref_quantized(fmt, a, c.W, c.bias)
        ok = G.within_tol(y.float().cpu().numpy(), ref.float().cpu().numpy(), T)
        assert ok.all(), f"{np.count_nonzero(~ok)} outputs differ from mxq_linear"


def test_noalloc_bf16_path_and_size_limit():
    # bf16 path (min dimension < 1024): no scratch involved
    M, K, N = 256, 512, 384
    c = workloads.random_case(M, K, N, "bf16", seed=32)
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt="nvfp4")
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    mxq.linear_noalloc(w.handle, c.A.to(DEV), M, y)
    ref = mxq.linear_forward(w, c.A.to(DEV))
    torch.cuda.synchronize()
    _, T, _, _ = G.linear_ref_quantized("bf16", c.A, c.W, c.bias)
    assert G.within_tol(y.float().cpu().numpy(), ref.float().cpu().numpy(), T).all()
    # a quantised layer whose workspace exceeds the static scratch is refused
    # before anything is enqueued
    big = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=3072, K=12288, w_bf16=1 << 20,
                         codes=1 << 20, sf=1 << 20, g_dev=1 << 20)
    M_big = 16896
    assert mxq.linear_workspace_bytes(M_big, 12288, "nvfp4") > mxq.NOALLOC_SCRATCH_BYTES
    with pytest.raises(mxq.MxqError) as e:
        mxq.linear_noalloc(big, 1 << 20, M_big, 1 << 20)
    assert e.value.status == mxq.ERR_WORKSPACE
