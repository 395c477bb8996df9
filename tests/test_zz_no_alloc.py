"""mxq_linear_noalloc: the linear layer for callers that cannot allocate
device memory (a fixed device-memory budget, or no cudaMalloc allowed in a
latency-critical loop).  Every call reuses one static device scratch array
that keeps the previous call's contents, so each call is checked twice: its
output must be within the oracle's tolerance, and it must equal, bit for bit,
the output of mxq_linear with a caller-allocated workspace (the same kernels
on the same quantised operands).  A stale amax, scale or barrier word left in
the scratch by an earlier call would break the second check.

This file is collected last on purpose, and passes both alone in a fresh
process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import gemm as G
from oracle import quant as Q

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_rows(fmt, A, W, bias, rows):
    """Oracle Y and T on the given output rows (the per-tensor amax of the
    whole activation, as the layer uses it)."""
    if fmt == "nvfp4":
        qa = Q.quantize_nvfp4(A[torch.as_tensor(rows)], global_amax=Q.amax(A))
        qw = Q.quantize_nvfp4(W)
        Ad = Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"])
        Wd = Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"])
    else:
        qa = Q.quantize_mxfp8(A[torch.as_tensor(rows)])
        qw = Q.quantize_mxfp8(W)
        Ad = Q.dequant_mxfp8(qa["codes"], qa["sf"])
        Wd = Q.dequant_mxfp8(qw["codes"], qw["sf"])
    return G.linear_ref(Ad, Wd, bias)


def _check_call(w, fmt, a_cpu, y, M, bias, min_dim=None, rows=None):
    ref = torch.full_like(y, float("nan"))
    ws = torch.empty(mxq.linear_workspace_bytes(M, a_cpu.shape[1], fmt), dtype=torch.uint8, device=DEV)
    mxq.linear(w.handle, a_cpu.to(DEV), M, ref, ws, ws.numel(), min_dim=min_dim)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    assert torch.equal(y, ref), "no-alloc output differs from mxq_linear's"
    if rows is None:
        rows = np.arange(M)
    Y, T = _oracle_rows(fmt, a_cpu, w.W_cpu, bias, rows)
    Yg = y[torch.as_tensor(rows, device=DEV)].float().cpu().numpy()
    ok = G.within_tol(Yg, Y, T)
    assert ok.all(), f"{np.count_nonzero(~ok)} outputs out of the oracle's tolerance"


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_noalloc_matches_oracle_and_linear_on_two_calls_in_a_row(fmt):
    M, K, N = 1024, 1024, 1152
    c = workloads.random_case(M, K, N, fmt, seed=31)
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt=fmt)
    w.W_cpu = c.W
    # two different activations: the second is the first times 2^-4 (exact in
    # bf16), so its amax and every scale differ, and a stale amax or scale
    # left in the scratch by the first call would show.  (A much smaller
    # factor would make every output bias-dominated: the bf16 rounding of the
    # bias alone then exceeds 2e-3 * sum|a b|, whose scale leaves the bias out.)
    inputs = [c.A, (c.A.float() * 0.0625).bfloat16()]
    outs = []
    for a in inputs:
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        mxq.linear_noalloc(w.handle, a.to(DEV), M, y)
        outs.append(y)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    for a, y in zip(inputs, outs):
        _check_call(w, fmt, a, y, M, c.bias)


def test_noalloc_two_pass_after_single_pass():
    # An NVFP4 activation that fits in shared memory is quantised in one pass
    # (grid barrier state in the scratch); a larger one takes the amax-partials
    # pass first (partials region of the scratch).  Run the first, then the
    # second, so the second starts from what the first left behind.
    K, N = 1024, 256
    small = workloads.random_case(1024, K, N, "nvfp4", seed=33)
    w = mxq.Weight(small.W.to(DEV), small.bias.to(DEV), fmt="nvfp4")
    w.W_cpu = small.W
    y1 = torch.empty(1024, N, dtype=torch.bfloat16, device=DEV)
    mxq.linear_noalloc(w.handle, small.A.to(DEV), 1024, y1, min_dim=1)
    M2 = 16640  # rows of 1024 bf16: too large for the single-pass quantiser
    g = torch.Generator().manual_seed(34)
    A2 = (torch.randn(M2, K, generator=g) * 3.0).bfloat16()
    assert mxq.linear_kernel_count(w.handle, 1024, min_dim=1) == 2
    assert mxq.linear_kernel_count(w.handle, M2, min_dim=1) == 3
    assert mxq.linear_workspace_bytes(M2, K, "nvfp4") <= mxq.NOALLOC_SCRATCH_BYTES
    y2 = torch.full((M2, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxq.linear_noalloc(w.handle, A2.to(DEV), M2, y2, min_dim=1)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    _check_call(w, "nvfp4", small.A, y1, 1024, small.bias, min_dim=1)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(M2 - 8, M2),
                                     np.random.default_rng(35).integers(0, M2, 48)]))
    _check_call(w, "nvfp4", A2, y2, M2, small.bias, min_dim=1, rows=rows)


def test_noalloc_bf16_path_and_size_limit():
    # bf16 path (min dimension < 1024): no scratch involved
    M, K, N = 256, 512, 384
    c = workloads.random_case(M, K, N, "bf16", seed=32)
    w = mxq.Weight(c.W.to(DEV), c.bias.to(DEV), fmt="nvfp4")
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    mxq.linear_noalloc(w.handle, c.A.to(DEV), M, y)
    ref = mxq.linear_forward(w, c.A.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    Y, T, _, _ = G.linear_ref_quantized("bf16", c.A, c.W, c.bias)
    assert G.within_tol(y.float().cpu().numpy(), Y, T).all()
    # A quantised layer whose workspace exceeds the static scratch is refused
    # before anything is enqueued.  The buffers are real and of the stated
    # size, so the call could touch only valid memory even if it were not refused.
    M_big, K_big, N_big = 16896, 12288, 3072
    assert mxq.linear_workspace_bytes(M_big, K_big, "nvfp4") > mxq.NOALLOC_SCRATCH_BYTES
    g = torch.Generator(device=DEV).manual_seed(36)
    big = mxq.Weight((torch.randn(N_big, K_big, generator=g, device=DEV) * 0.02).bfloat16(), None,
                     fmt="nvfp4")
    x = torch.zeros(M_big, K_big, dtype=torch.bfloat16, device=DEV)
    y_big = torch.zeros(M_big, N_big, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mxq.MxqError) as e:
        mxq.linear_noalloc(big.handle, x, M_big, y_big)
    assert e.value.status == mxq.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(y_big)) == 0  # nothing was written
