"""GPU parity of the producer epilogue and of the consumer's known-amax path.

Kernel fusion of the activation into the producing GEMM (the devin.kr
Blackwell FLUX page, section "연산 효율화와 가속 기술": activation functions
fused into the custom GEMM): mxq_linear applies GELU (exact erf) to
alpha * acc + bias before the bf16 rounding and folds max |y| of the bf16
output into one device word; the next layer's NVFP4 quantisation takes that
amax (x_amax_dev) instead of its own pass over the activation.

Checks: GELU outputs within the oracle's epilogue tolerance (oracle/producer.py);
the folded amax equal to the max over the layer's own bf16 output; a layer fed
the known amax gives exactly the output of the same layer with its own amax pass.
"""

import numpy as np
import pytest
import torch

import fp8_gemm_diffusion_b200 as mxq
from oracle import gemm as G
from oracle import producer as P
from oracle import quant as Q

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _deq(fmt, x, rows=None, amax=None):
    xs = x if rows is None else x[torch.as_tensor(rows)]
    if fmt == "nvfp4":
        q = Q.quantize_nvfp4(xs, global_amax=Q.amax(x) if amax is None else amax)
        return Q.dequant_nvfp4(q["codes"], q["sf"], q["g"])
    if fmt == "mxfp8":
        q = Q.quantize_mxfp8(xs)
        return Q.dequant_mxfp8(q["codes"], q["sf"])
    return np.asarray(xs.float().numpy(), dtype=np.float64)


@pytest.mark.parametrize("fmt,M,K,N", [("nvfp4", 1280, 1024, 1536), ("mxfp8", 1280, 1024, 1536),
                                       ("nvfp4", 300, 1024, 1096), ("bf16", 640, 512, 640)])
def test_producer_gelu_and_amax(fmt, M, K, N):
    g = torch.Generator().manual_seed(M + N + K)
    W = (torch.randn(N, K, generator=g) * 0.03).bfloat16()
    b = (torch.randn(N, generator=g) * 0.05).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    layer = mxq.Weight(W.to(DEV), b.to(DEV), fmt="nvfp4" if fmt == "bf16" else fmt, keep_bf16=fmt == "bf16")
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    ymax = torch.full((1,), -5.0, device=DEV)
    nbytes = mxq.linear_workspace_bytes(M, K, "nvfp4" if fmt == "bf16" else fmt)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=DEV)
    mxq.linear(layer.handle, A.to(DEV), M, y, ws, ws.numel(), min_dim=1,
               activation=mxq.ACT_GELU, y_amax=ymax)
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    # the amax is exactly the max over the layer's own bf16 output
    assert float(ymax.item()) == float(y.float().abs().max().item())
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(M - 8, M),
                                     np.random.default_rng(M).integers(0, M, 40)]))
    Ad = _deq(fmt, A, rows)
    Wd = _deq(fmt, W)
    Y, T = P.linear_gelu_ref(Ad, Wd, b)
    Yg = y[torch.as_tensor(rows, device=DEV)].float().cpu().numpy().astype(np.float64)
    ok = G.within_tol(Yg, Y, T)
    assert ok.all(), f"{(~ok).sum()} outputs out of tolerance, worst {np.abs(Yg - Y)[~ok].max()}"


def test_consumer_known_amax_matches_and_chains():
    M, K, N = 1536, 1024, 2048
    g = torch.Generator().manual_seed(3)
    W1 = (torch.randn(K, K, generator=g) * 0.03).bfloat16().to(DEV)
    W2 = (torch.randn(N, K, generator=g) * 0.03).bfloat16().to(DEV)
    A = torch.randn(M, K, generator=g).bfloat16().to(DEV)
    l1 = mxq.Weight(W1, None, fmt="nvfp4")
    l2 = mxq.Weight(W2, None, fmt="nvfp4")
    ws = torch.empty(mxq.linear_workspace_bytes(M, K, "nvfp4"), dtype=torch.uint8, device=DEV)
    h = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    hmax = torch.empty(1, device=DEV)
    mxq.linear(l1.handle, A, M, h, ws, ws.numel(), activation=mxq.ACT_GELU, y_amax=hmax)
    y_known = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    assert mxq.linear_kernel_count(l2.handle, M, x_amax=hmax) == 2
    mxq.linear(l2.handle, h, M, y_known, ws, ws.numel(), x_amax=hmax)
    y_plain = torch.empty_like(y_known)
    mxq.linear(l2.handle, h, M, y_plain, ws, ws.numel())
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    assert float(hmax.item()) == float(h.float().abs().max().item())
    # same amax -> same codes and scales -> identical outputs
    assert torch.equal(y_known, y_plain)


def test_producer_rejected_on_small_m():
    W = torch.randn(1024, 1024, device=DEV).bfloat16()
    l = mxq.Weight(W, None, fmt="nvfp4")
    x = torch.randn(64, 1024, device=DEV).bfloat16()
    y = torch.empty(64, 1024, dtype=torch.bfloat16, device=DEV)
    st = mxq._linear(mxq.ctypes.byref(l.handle), x.data_ptr(), 64, y.data_ptr(), None, 0,
                     mxq._opts(None, activation=mxq.ACT_GELU), mxq._stream(None))
    assert st == mxq.ERR_UNSUPPORTED_SHAPE
