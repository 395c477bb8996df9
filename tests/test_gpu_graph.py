"""A reduced FLUX-shaped linear stack captured into one CUDA graph and replayed.

CUDA graphs remove the host's launch gaps at batch 1 (B200 MXFP8/NVFP4
diffusion article, "Technical Considerations - Improving CPU Overhead with
CUDA Graphs").  mxq_linear never synchronises the host, so a pass over several
layers can be captured whole; the graph then holds the single-pass NVFP4
quantiser (a cooperative launch whose grid barrier lives in the workspace),
the amax + quantiser pair of the two-pass path, the block-scaled and bf16
GEMMs, all with programmatic stream serialisation.

Checks: every replay equals the eager pass bit for bit (same kernels, same
operands), and sampled rows of every layer whose input is not itself a GPU
output are within the oracle's tolerance.
"""

import numpy as np
import pytest
import torch

from oracle import gemm as G
from oracle import quant as Q

import fp8_gemm_diffusion_b200 as mxq

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (name, M, K, N, input): input "x" = its own seeded activation, or the name
# of the layer whose output it consumes
LAYERS = [
    ("proj_nvfp4_single_pass", 4608, 3072, 3072, "x"),     # 28 MB activation: one pass
    ("chained_nvfp4", 4608, 3072, 1024, "proj_nvfp4_single_pass"),
    ("wide_nvfp4_two_pass", 12288, 3072, 1024, "x"),       # 75 MB activation: amax pass + quantiser
    ("txt_bf16", 512, 3072, 3072, "x"),                    # min dim 512 < 1024: bf16
    ("mod_bf16_m1", 1, 3072, 9216, "x"),                   # one row: bf16, single-CTA kernel
]


def _oracle_rows(path, A, W, bias, rows):
    if path == mxq.BF16:
        Y, T, _, _ = G.linear_ref_quantized("bf16", A, W, bias, rows=rows)
        return Y, T
    qa = Q.quantize_nvfp4(A[torch.as_tensor(rows)], global_amax=Q.amax(A))
    qw = Q.quantize_nvfp4(W)
    return G.linear_ref(Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"]),
                        Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"]), bias)


def test_graph_replay_matches_eager_and_oracle():
    g = torch.Generator().manual_seed(41)
    layers, outs, ins, ws_bytes = [], {}, {}, 256
    for name, M, K, N, src in LAYERS:
        W = (torch.randn(N, K, generator=g) * 0.02).bfloat16()
        b = (torch.randn(N, generator=g) * 0.02).bfloat16()
        A = torch.randn(M, K, generator=g).bfloat16() if src == "x" else None
        w = mxq.Weight(W.to(DEV), b.to(DEV), fmt="nvfp4")
        path = mxq.linear_path(w.handle, M)
        if path != mxq.BF16:
            ws_bytes = max(ws_bytes, mxq.linear_workspace_bytes(M, K, path))
        x = A.to(DEV) if A is not None else outs[src]
        outs[name] = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
        ins[name] = A
        layers.append((name, M, K, N, w, W, b, x, path))
    paths = {name: path for name, _, _, _, _, _, _, _, path in layers}
    assert paths["proj_nvfp4_single_pass"] == mxq.NVFP4 and paths["txt_bf16"] == mxq.BF16
    assert mxq.linear_kernel_count(layers[0][4].handle, 4608) == 2   # single pass + GEMM
    assert mxq.linear_kernel_count(layers[2][4].handle, 12288) == 3  # amax + quantise + GEMM
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)

    def one_pass():
        for name, M, K, N, w, _, _, x, _ in layers:
            mxq.linear(w.handle, x, M, outs[name], ws, ws_bytes)

    # eager pass (also sets the kernels' shared-memory attributes before capture)
    one_pass()
    torch.cuda.synchronize()
    assert mxq.get_device_error() == mxq.OK
    eager = {k: v.clone() for k, v in outs.items()}

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        one_pass()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        one_pass()
    for rep in range(2):
        for v in outs.values():
            v.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert mxq.get_device_error() == mxq.OK
        for name in outs:
            assert torch.equal(outs[name], eager[name]), f"replay {rep}: {name} differs from eager"
    del graph

    for name, M, K, N, w, W, b, x, path in layers:
        A = ins[name]
        if A is None:
            continue  # input is a GPU output: covered by the bit-equality above
        rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M + N).integers(0, M, 24)]))
        Y, T = _oracle_rows(path, A, W, b, rows)
        Yg = eager[name][torch.as_tensor(rows, device=DEV)].float().cpu().numpy()
        ok = G.within_tol(Yg, Y, T)
        assert ok.all(), f"{name}: {np.count_nonzero(~ok)} outputs out of the oracle's tolerance"
