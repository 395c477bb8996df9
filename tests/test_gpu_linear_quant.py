"""GPU parity of the activation quantisation inside mxq_linear (NVFP4): the
amax, g, E2M1 codes and E4M3 block scales it leaves in the workspace equal
the oracle's bit for bit, on both of its paths:

- single pass (the activation fits in the grid's shared memory): rows are
  held on chip, the per-tensor amax goes through a grid-wide barrier whose
  state lives in the workspace header;
- two passes (larger activations): amax partials, then the quantiser.

The barrier state starts from whatever the workspace holds, so the cases run
on zero-filled and 0xFF-filled workspaces, and reuse one workspace for a
second input whose amax differs (a stale barrier would hand back the first
input's amax)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import quant as Q
from tests._gpu import DEV

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu

SMEM_LIMIT = 227 * 1024 - 1024


def _pad256(n):
    return (n + 255) // 256 * 256


def _header(M, K):
    """Bytes before the codes in the workspace (amax, g, amax partials,
    barrier state): the workspace is header + codes + scales, each part
    padded to 256 bytes."""
    return (mxq.linear_workspace_bytes(M, K, "nvfp4") - _pad256(M * K // 2)
            - _pad256(Q.sf_bytes(M, K, 16)))


def _single_pass(M, K):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rpc = -(-M // sms)
    return rpc * K * 2 + 8 * rpc <= SMEM_LIMIT


def _weight(K, N=128, seed=5):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    return mxq.Weight(W.to(DEV), None, fmt="nvfp4")


def _run(w, A, fill):
    M, K = A.shape
    nbytes = mxq.linear_workspace_bytes(M, K, "nvfp4")
    ws = torch.full((nbytes,), fill, dtype=torch.uint8, device=DEV)
    mxq.linear_forward(w, A.to(DEV), ws=ws, min_dim=1)
    torch.cuda.synchronize()
    return ws


def _check(ws, A):
    M, K = A.shape
    oq = Q.quantize_nvfp4(A)
    st = ws.cpu().numpy()
    amax = np.frombuffer(st[0:4].tobytes(), np.float32)[0]
    g = np.frombuffer(st[4:8].tobytes(), np.float32)[0]
    assert float(amax) == float(oq["amax"]), "amax"
    assert g == oq["g"], "per-tensor scale g"
    nc = M * K // 2
    HEADER = _header(M, K)
    assert HEADER % 256 == 0 and HEADER >= 8
    codes = st[HEADER: HEADER + nc].reshape(M, K // 2)
    bad = np.argwhere(codes != oq["codes"])
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    sf_off = HEADER + (nc + 255) // 256 * 256
    sf = st[sf_off: sf_off + Q.sf_bytes(M, K, 16)]
    bad = np.flatnonzero(sf != oq["sf_swz"])
    assert bad.size == 0, f"{len(bad)} scale bytes differ, first at {bad[:4].tolist()}"


def test_single_pass_c3_activation():
    c = workloads.c3_nvfp4_mlp_up()
    assert _single_pass(*c.A.shape)
    ws = _run(_weight(c.A.shape[1]), c.A, 0x00)
    _check(ws, c.A)
    assert mxq.get_device_error() == mxq.OK


@pytest.mark.parametrize("M,K", [(1, 64), (37, 192), (1000, 1024), (4607, 3072)])
@pytest.mark.parametrize("fill", [0x00, 0xFF])
def test_single_pass_shapes(M, K, fill):
    assert _single_pass(M, K)
    c = workloads.random_case(M, K, 8, "nvfp4", seed=M + K)
    ws = _run(_weight(K), c.A, fill)
    _check(ws, c.A)
    assert mxq.get_device_error() == mxq.OK


def test_single_pass_reused_workspace():
    M, K = 2000, 1024
    w = _weight(K)
    nbytes = mxq.linear_workspace_bytes(M, K, "nvfp4")
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device=DEV)
    for i, scale in enumerate((1.0, 7.5, 0.01)):
        A = (workloads.random_case(M, K, 8, "nvfp4", seed=40 + i).A.float() * scale).to(torch.bfloat16)
        mxq.linear_forward(w, A.to(DEV), ws=ws, min_dim=1)
        torch.cuda.synchronize()
        _check(ws, A)
    assert mxq.get_device_error() == mxq.OK


def test_single_pass_zero_activation():
    A = torch.zeros(256, 512, dtype=torch.bfloat16)
    ws = _run(_weight(512), A, 0xFF)
    _check(ws, A)  # amax 0 -> g = 1, every code and scale 0


def test_two_pass_large_activation():
    M, K = 4608, 4096  # 37.7 MB of bf16: more than the grid's shared memory holds
    assert not _single_pass(M, K)
    c = workloads.random_case(M, K, 8, "nvfp4", seed=77)
    ws = _run(_weight(K), c.A, 0xFF)
    _check(ws, c.A)
    assert mxq.get_device_error() == mxq.OK


def test_single_pass_wide_dynamic_range():
    # every 16-element block scaled by 2^-e, e in [0, 30]: block scales reach
    # the E4M3 subnormals and zero, codes reach every E2M1 magnitude
    M, K = 512, 2048
    g = torch.Generator().manual_seed(9)
    A = torch.randn(M, K, generator=g)
    e = torch.randint(0, 31, (M, K // 16), generator=g).float()
    A = (A.view(M, K // 16, 16) * torch.exp2(-e)[..., None]).view(M, K).to(torch.bfloat16)
    assert _single_pass(M, K)
    ws = _run(_weight(K), A, 0xFF)
    _check(ws, A)
    assert mxq.get_device_error() == mxq.OK


def test_kernel_count_matches_the_path_taken():
    w = _weight(3072)
    assert mxq.linear_kernel_count(w.handle, 4608, min_dim=1) == 2   # single pass + GEMM
    w = _weight(4096)
    assert mxq.linear_kernel_count(w.handle, 4608, min_dim=1) == 3   # amax + quantise + GEMM


def test_gemm_events_bracket_the_gemm():
    # the optional event pair of mxq_linear_opts brackets the GEMM launch: its
    # interval is positive and inside the interval of the whole call
    w = _weight(3072, N=1024)
    A = workloads.random_case(4608, 3072, 8, "nvfp4", seed=3).A.to(DEV)
    nbytes = mxq.linear_workspace_bytes(4608, 3072, "nvfp4")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    y = torch.empty(4608, 1024, dtype=torch.bfloat16, device=DEV)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    ev[0].record()
    mxq.linear(w.handle, A, 4608, y, ws, nbytes, min_dim=1, gemm_events=(ev[1], ev[2]))
    ev[3].record()
    torch.cuda.synchronize()
    gemm = ev[1].elapsed_time(ev[2])
    assert 0.0 < gemm <= ev[0].elapsed_time(ev[3])
    assert mxq.get_device_error() == mxq.OK
