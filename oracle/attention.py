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
  5. the kernel quantises P (in fp32) to MXFP8 along keys and computes
     O = deq(Pq) deq(Vq)^T with fp32 accumulation, bf16 output.

The oracle evaluates steps 1-4 exactly (float64 after the quantisers) and
O_ref = P deq(Vq)^T without rounding P.  The error of step 5 is bounded by
the rounding of P: E4M3 keeps 3 fraction bits, so a normal value moves by at
most 2^-4 of itself; values below the block's normal range (E4M3 subnormals
and zero) move by at most 2^-10 of the block scale, i.e. 2^-18 of the block
maximum, which is at most the block's sum.  With the block-wise error scale

  T[i, c] = sum_b ( sum_{j in b} P[i, j] ) * max_{j in b} |deq(Vq)^T[j, c]|

(b running over blocks of 32 keys; T >= sum_j P[i, j] |V[j, c]| >= |O[i, c]|)
the rounding of P contributes at most (2^-4 + 32 * 2^-18) T, the bf16
output 2^-9 T, fp32 accumulation and the fp32 exponential far less, so

  |O_gpu - O_ref| <= ATT_RTOL * T + ATT_ATOL,  ATT_RTOL = 0.07, ATT_ATOL = 1e-6.

``attention_ref`` also returns O_q, the product with P quantised by the
oracle's own MXFP8 quantiser (P rounded to fp32 first): the kernel differs
from it only where its fp32 P falls on the other side of a rounding boundary.
"""

from __future__ import annotations

import math

import numpy as np

from .quant import _as_f32, dequant_mxfp8, quantize_mxfp8

__all__ = ["softmax_rows", "attention_plain", "attention_ref", "ATT_RTOL", "ATT_ATOL", "within_att_tol"]

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
    V always uses every token).  Returns (O_ref, T_err, O_q), each [rows, d]
    float64.
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
    nb = T_ // KEY_BLOCK
    Pb = P.reshape(P.shape[0], nb, KEY_BLOCK).sum(axis=2)             # [rows, nb]
    Vb = np.abs(Vd).reshape(nb, KEY_BLOCK, d).max(axis=1)             # [nb, d]
    T_err = Pb @ Vb
    pq = quantize_mxfp8(P.astype(np.float32))
    Oq = dequant_mxfp8(pq["codes"], pq["sf"]) @ Vd
    return O, T_err, Oq


def within_att_tol(O_test, O_ref, T_err) -> np.ndarray:
    """Element-wise pass mask |O_test - O_ref| <= ATT_RTOL * T + ATT_ATOL."""
    O_test = np.asarray(O_test, dtype=np.float64)
    return np.abs(O_test - np.asarray(O_ref, dtype=np.float64)) <= ATT_RTOL * np.asarray(T_err) + ATT_ATOL
