"""8-bit (MXFP8) attention with per-token scales (CPU oracle).

TEST INFRASTRUCTURE ONLY: nothing in the product path may import this module.

Source passage: the devin.kr page on Blackwell FLUX image generation
("엔비디아 블랙웰 기반 플럭스 3 이미지 생성 4.45배 가속"), section "연산 효율화와
가속 기술" (compute efficiency and acceleration): attention is run through a
dedicated 8-bit floating-point path that corrects the quantisation error
token by token (1.16-1.18x).  The page gives no formula.  Reading, in the
terms of the rest of this library (the MXFP8 quantiser of "Glossary -
MXFP8" on the B200 MXFP8/NVFP4 diffusion article):

  per head, Q, K, V in R^{T x d} (T tokens, d = head dimension):
  1. Qq = MXFP8(Q), Kq = MXFP8(K): E4M3 codes with one power-of-two scale
     per token and per 32 channels -- every token carries its own scales,
     and the tensor cores apply them inside the product (the per-token
     correction);
  2. Vq = MXFP8(V^T): scales per channel and per 32 tokens, so that the
     second product's contraction (over tokens) sees one scale per 32 terms;
  3. S = tau * deq(Qq) deq(Kq)^T, tau = 1 / sqrt(d);
  4. P = softmax(S) along keys (exact: maximum subtracted, normalised);
  5. the kernel quantises the unnormalised weights E = exp(S - rowmax(S)),
     in [0, 1] and in fp32, to MXFP8 along keys with the ceiling scale rule
     (the smallest shared exponent with no saturation: under the floor rule
     a block maximum in [448, 512) * 2^X would be clipped to 448, up to
     12.5 % off), computes deq(Eq) deq(Vq)^T with fp32 accumulation and
     divides by the row sum of E (fp32); bf16 output.

The oracle evaluates steps 1-4 exactly (float64 after the quantisers) and
O_ref = P deq(Vq)^T without rounding P.  The error of step 5 is bounded by
the rounding of E (relative errors carry over to P = E / sum E): E4M3 keeps
3 fraction bits, so a normal value moves by at most 2^-4 of itself (nothing
saturates under the ceiling rule); values below the block's normal range
(E4M3 subnormals and zero) move by at most 2^-10 of the block scale, i.e. at
most 2^-17 of the block maximum (the ceiling rule puts the maximum at
224 * 2^X or above), which is at most the block's sum.  With the error scale

  T[i, c] = sum_j P[i, j] |deq(Vq)^T[j, c]|      (T >= |O[i, c]|)

the normal-range rounding contributes at most 2^-4 T; the underflowed
weights at most 32 * 2^-17 of each block's sum times that block's largest
|V|, in all at most 2^-12 max_j |V[j, c]|; the bf16 output 2^-9 T; fp32
accumulation and the fp32 exponential far less.  So every element satisfies

  |O_gpu - O_ref| <= ATT_RTOL * T + 2^-12 * max_j |V[j, c]| + ATT_ATOL,
  ATT_RTOL = 0.07, ATT_ATOL = 1e-6                       (within_att_tol)

This worst case is loose when the weights are spread over many keys.  The
sharp check is against O_q, step 5 done by the oracle: E rounded to fp32 and
quantised by its own MXFP8 quantiser (ceiling rule), the product in float64,
divided by the float64 row sum of E.  The kernel differs from it only where
its fp32 E falls on the other side of a rounding boundary (a weight moves by
one E4M3 step) and by fp32 accumulation and the bf16 output, so nearly every
element satisfies the GEMM's rule |O_gpu - O_q| <= 2e-3 T + 1e-6
(within_att_tight).
"""

from __future__ import annotations

import math

import numpy as np

from .quant import _as_f32, dequant_mxfp8, quantize_mxfp8

__all__ = ["softmax_rows", "attention_plain", "attention_ref", "ATT_RTOL", "ATT_ATOL", "within_att_tol",
           "within_att_tight"]

ATT_RTOL = 0.07
ATT_ATOL = 1e-6
KEY_BLOCK = 32


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Row-wise softmax in float64, the row maximum subtracted first."""
    S = np.asarray(S, dtype=np.float64)
    m = np.max(S, axis=1, keepdims=True)
    e = np.exp(S - m)
    return e / np.sum(e, axis=1, keepdims=True)


def attention_plain(Q, K, V, tau=None) -> np.ndarray:
    """softmax(tau Q K^T) V in float64 on the given values (no quantisation)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if tau is None:
        tau = 1.0 / math.sqrt(Q.shape[1])
    return softmax_rows(tau * (Q @ K.T)) @ V


def attention_ref(Q, K, V, rows=None, tau=None):
    """One head of the 8-bit attention (steps 1-4 of the header).

    Q, K, V: [T, d] (torch bf16 tensors or float32 arrays), T and d multiples
    of 32.  rows: optional query rows to evaluate (the quantisation of K and
    V always uses every token).  Returns (O_ref, T_err, O_q, vmax): the
    first three [rows, d] float64, vmax [d] = max_j |deq(Vq)^T[j, c]|.
    """
    Qf, Kf, Vf = _as_f32(Q), _as_f32(K), _as_f32(V)
    T_, d = Qf.shape
    if tau is None:
        tau = 1.0 / math.sqrt(d)
    if rows is not None:
        Qf = Qf[np.asarray(rows)]
    qq = quantize_mxfp8(Qf)
    kq = quantize_mxfp8(Kf)
    vq = quantize_mxfp8(np.ascontiguousarray(Vf.T))
    Qd = dequant_mxfp8(qq["codes"], qq["sf"])
    Kd = dequant_mxfp8(kq["codes"], kq["sf"])
    Vd = dequant_mxfp8(vq["codes"], vq["sf"]).T          # [T, d]
    P = softmax_rows(tau * (Qd @ Kd.T))                   # [rows, T]
    O = P @ Vd
    T_err = P @ np.abs(Vd)
    vmax = np.abs(Vd).max(axis=0)
    S = tau * (Qd @ Kd.T)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    eq = quantize_mxfp8(E.astype(np.float32), scale_rule="rceil")
    Oq = (dequant_mxfp8(eq["codes"], eq["sf"]) @ Vd) / E.sum(axis=1, keepdims=True)
    return O, T_err, Oq, vmax


def within_att_tol(O_test, O_ref, T_err, vmax) -> np.ndarray:
    """Worst-case mask against the exact result:
    |O_test - O_ref| <= ATT_RTOL * T + 2^-12 * vmax + ATT_ATOL."""
    O_test = np.asarray(O_test, dtype=np.float64)
    bound = ATT_RTOL * np.asarray(T_err) + 2.0 ** -12 * np.asarray(vmax)[None, :] + ATT_ATOL
    return np.abs(O_test - np.asarray(O_ref, dtype=np.float64)) <= bound


def within_att_tight(O_test, O_q, T_err) -> np.ndarray:
    """Mask against the oracle's own rounding of the weights:
    |O_test - O_q| <= 2e-3 * T + 1e-6 (the GEMM's rule)."""
    O_test = np.asarray(O_test, dtype=np.float64)
    return np.abs(O_test - np.asarray(O_q, dtype=np.float64)) <= 2e-3 * np.asarray(T_err) + 1e-6
