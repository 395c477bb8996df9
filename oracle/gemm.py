"""Reference linear layer Y = X W^T + bias on quantised operands (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

The B200 MXFP8/NVFP4 diffusion article quantises the ``nn.Linear`` layers of
the transformer ("Detailed by section", the TorchAO/Diffusers listing):
activations dynamically, weights once, and the layer then multiplies the two
quantised operands with bf16 output.  What the quantised linear computes,
written out:

    Y[m, n] = sum_k deq(A)[m, k] * deq(W)[n, k] + bias[n]

with deq() the dequantised values (for NVFP4 including the per-tensor scales
g_A and g_W).  The oracle evaluates it in float64 (every dequantised value and
every product is exact in float64; only the order of the float64 sum is left
to the library matmul), together with the error scale

    T[m, n] = sum_k |deq(A)[m, k] * deq(W)[n, k]|

A GPU result passes when |Y_gpu - Y| <= 2e-3 * T + 1e-6 element by element
(the error bound the kernels are held to: fp32 accumulation plus one bf16
rounding of the output), or when it is exactly Y rounded to bf16 (to
nearest, ties to even).  The second clause covers what the first cannot: a
bf16 rounding moves a value by up to 2^-8 of itself (half an ulp at the
bottom of a binade), which exceeds 2e-3 * T wherever |Y| is above about half
of T -- short sums (K of a few dozen), or a bias that dominates the product;
no bf16 output can do better than the correctly rounded value.
"""

from __future__ import annotations

import numpy as np

from .quant import dequant_mxfp8, dequant_nvfp4, quantize_mxfp8, quantize_nvfp4, _as_f32

__all__ = ["linear_ref", "linear_ref_quantized", "within_tol", "tol_bound", "RTOL", "ATOL",
           "gemm_triple_loop", "bf16_rne"]

RTOL = 2e-3
ATOL = 1e-6


def linear_ref(Adeq: np.ndarray, Wdeq: np.ndarray, bias=None):
    """Y = Adeq Wdeq^T + bias and T = |Adeq| |Wdeq|^T, both float64."""
    A = np.asarray(Adeq, dtype=np.float64)
    W = np.asarray(Wdeq, dtype=np.float64)
    Y = A @ W.T
    T = np.abs(A) @ np.abs(W).T
    if bias is not None:
        Y = Y + np.asarray(_as_f32(bias), dtype=np.float64)[None, :]
    return Y, T


def linear_ref_quantized(fmt: str, A, W, bias=None, rows=None):
    """Quantise A and W the way the layer does, then the float64 reference.

    fmt: "nvfp4" | "mxfp8" | "bf16".  ``rows`` optionally restricts Y to a
    subset of output rows (the whole of A is still used for the NVFP4
    per-tensor amax, as the method prescribes).
    Returns (Y, T, qa, qw) where qa / qw are the quantiser outputs (None for bf16).
    """
    if fmt == "bf16":
        Af = np.asarray(_as_f32(A), dtype=np.float64)
        Wf = np.asarray(_as_f32(W), dtype=np.float64)
        if rows is not None:
            Af = Af[rows]
        Y, T = linear_ref(Af, Wf, bias)
        return Y, T, None, None
    if fmt == "nvfp4":
        qa = quantize_nvfp4(A)
        qw = quantize_nvfp4(W)
        Ad = dequant_nvfp4(qa["codes"] if rows is None else qa["codes"][rows],
                           qa["sf"] if rows is None else qa["sf"][rows], qa["g"])
        Wd = dequant_nvfp4(qw["codes"], qw["sf"], qw["g"])
    elif fmt == "mxfp8":
        qa = quantize_mxfp8(A)
        qw = quantize_mxfp8(W)
        Ad = dequant_mxfp8(qa["codes"] if rows is None else qa["codes"][rows],
                           qa["sf"] if rows is None else qa["sf"][rows])
        Wd = dequant_mxfp8(qw["codes"], qw["sf"])
    else:
        raise ValueError(fmt)
    Y, T = linear_ref(Ad, Wd, bias)
    return Y, T, qa, qw


def tol_bound(T: np.ndarray) -> np.ndarray:
    return RTOL * np.asarray(T, dtype=np.float64) + ATOL


def bf16_rne(x) -> np.ndarray:
    """float64 -> the nearest bf16 value (8 significant bits, ties to the even
    significand), returned as float64; exact (no intermediate float32), for
    normal-range values and zero.  With |x| = s * 2^e, 1 <= s < 2, the bf16
    neighbours are multiples of 2^(e - 7)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    ulp = np.exp2(e - 7)
    out[nz] = np.round(x[nz] / ulp) * ulp  # x / ulp is exact; np.round rounds half to even
    return out


def within_tol(Y_test, Y_ref, T) -> np.ndarray:
    """Element-wise pass mask: |Y_test - Y_ref| <= 2e-3 * T + 1e-6, or Y_test
    equal to Y_ref rounded to bf16 (see the module header)."""
    Y_test = np.asarray(Y_test, dtype=np.float64)
    Y_ref = np.asarray(Y_ref, dtype=np.float64)
    return (np.abs(Y_test - Y_ref) <= tol_bound(T)) | (Y_test == bf16_rne(Y_ref))


def gemm_triple_loop(Adeq, Wdeq, bias=None):
    """Plain triple loop (tiny shapes only): the definition with no library call."""
    A = np.asarray(Adeq, dtype=np.float64)
    W = np.asarray(Wdeq, dtype=np.float64)
    M, K = A.shape
    N = W.shape[0]
    Y = np.zeros((M, N))
    T = np.zeros((M, N))
    b = None if bias is None else np.asarray(_as_f32(bias), dtype=np.float64)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            tacc = 0.0
            for k in range(K):
                p = A[m, k] * W[n, k]
                acc += p
                tacc += abs(p)
            Y[m, n] = acc + (b[n] if b is not None else 0.0)
            T[m, n] = tacc
    return Y, T
