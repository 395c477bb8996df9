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
  5. the kernel quantises the unnormalised weights, in fp32,
       E = 2^(t - m),  t = tau * log2(e) * S,  m = ceil(max_j t_j)  (an integer),
     to MXFP8 along keys with the ceiling scale rule (the smallest shared
     exponent with no saturation: under the floor rule a block maximum in
     [448, 512) * 2^X would be clipped to 448, up to 12.5 % off), computes
     deq(Eq) deq(Vq)^T with fp32 accumulation and divides each query row by
     the sum of its quantised weights, rowsum(deq(Eq)); bf16 output.  The
     division by the quantised sum is the per-token correction of the
     weights' own rounding: each row's weights sum to one again, so a
     constant V passes through unchanged.  Softmax does not depend on the
     constant taken out of the exponent; it is read here as a power of two
     because the MXFP8 codes then do not depend on it either: multiplying a
     block by 2^k moves its shared exponent by k and leaves every code (and
     the result) as it was, so a kernel may take the weights against any
     integer m -- a running maximum, for instance -- and quantise to the
     same codes.

The oracle evaluates steps 1-4 exactly (float64 after the quantisers) and
O_ref = P deq(Vq)^T without rounding P.  The error of step 5 comes from the
rounding of E: E4M3 keeps 3 fraction bits, so a normal value moves by at
most 2^-4 of itself (nothing saturates under the ceiling rule); values below
the block's normal range (E4M3 subnormals and zero) move by at most 2^-10 of
the block scale, i.e. at most 2^-17 of the block maximum (the ceiling rule
puts the maximum at 224 * 2^X or above), which is at most the block's sum.
With q_j = E_j (1 + e_j) the renormalised weights are
w'_j = P_j (1 + e_j) / (1 + ebar), ebar = sum_j P_j e_j, so

  O_q - O_ref = (sum_j P_j e_j V_j - ebar O_ref) / (1 + ebar),

and with the error scale

  T[i, c] = sum_j P[i, j] |deq(Vq)^T[j, c]|      (T >= |O[i, c]|)

the normal-range rounding contributes at most 2 * 2^-4 T / (1 - 2^-4)
= 0.1334 T; the underflowed weights at most 32 * 2^-17.8 = 2^-12.8 of each
block's sum times that block's largest |V|, once directly and once through
ebar, in all at most 2^-11 max_j |V[j, c]|; the bf16 output 2^-9 T; fp32
accumulation and the fp32 exponential far less.  So every element satisfies

  |O_gpu - O_ref| <= ATT_RTOL * T + 2^-11 * max_j |V[j, c]| + ATT_ATOL,
  ATT_RTOL = 0.14, ATT_ATOL = 1e-6                       (within_att_tol)

This worst case is loose when the weights are spread over many keys.  The
sharp check is against O_q, step 5 done by the oracle: E (against
m = ceil(max t)) rounded to fp32 and quantised by its own MXFP8 quantiser
(ceiling rule), the product in float64, divided by the float64 row sum of
the quantised weights.  The kernel differs from it only where
its fp32 E falls on the other side of a rounding boundary (a weight moves by
one E4M3 step; the tensor cores' error in S can move a large logit's E
across such a boundary), by fp32 accumulation, and by the bf16 output (up
to 2^-9 of |O|, which for a peaked row is nearly all of 2e-3 T); so nearly
every element satisfies
|O_gpu - O_q| <= 2^-9 |O_q| + 2e-3 T + 1e-6 (within_att_tight).
"""

from __future__ import annotations

import math

import numpy as np

from .quant import _as_f32, dequant_mxfp8, quantize_mxfp8

__all__ = ["softmax_rows", "attention_plain", "weights_pow2", "attention_ref", "ATT_RTOL", "ATT_ATOL", "within_att_tol",
           "within_att_tight"]

ATT_RTOL = 0.14
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


def weights_pow2(t: np.ndarray, shift: int = 0) -> np.ndarray:
    """Unnormalised softmax weights E = 2^(t - m) per row, m = ceil(max t) +
    shift (an integer; step 5 of the header), in float64."""
    t = np.asarray(t, dtype=np.float64)
    m = np.ceil(t.max(axis=1, keepdims=True)) + shift
    return np.exp2(t - m)


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
    t = (tau * math.log2(math.e)) * (Qd @ Kd.T)
    E = weights_pow2(t)
    eq = quantize_mxfp8(E.astype(np.float32), scale_rule="rceil")
    Ed = dequant_mxfp8(eq["codes"], eq["sf"])
    Oq = (Ed @ Vd) / Ed.sum(axis=1, keepdims=True)
    return O, T_err, Oq, vmax


def within_att_tol(O_test, O_ref, T_err, vmax) -> np.ndarray:
    """Worst-case mask against the exact result:
    |O_test - O_ref| <= ATT_RTOL * T + 2^-11 * vmax + ATT_ATOL."""
    O_test = np.asarray(O_test, dtype=np.float64)
    bound = ATT_RTOL * np.asarray(T_err) + 2.0 ** -11 * np.asarray(vmax)[None, :] + ATT_ATOL
    return np.abs(O_test - np.asarray(O_ref, dtype=np.float64)) <= bound


def within_att_tight(O_test, O_q, T_err) -> np.ndarray:
    """Mask against the oracle's own rounding of the weights:
    |O_test - O_q| <= 2^-9 |O_q| + 2e-3 * T + 1e-6: the bf16 rounding of the
    output (at most half an ulp, 2^-9 of the value) plus the GEMM's rule."""
    O_test = np.asarray(O_test, dtype=np.float64)
    O_q = np.asarray(O_q, dtype=np.float64)
    return np.abs(O_test - O_q) <= 2.0 ** -9 * np.abs(O_q) + 2e-3 * np.asarray(T_err) + 1e-6
