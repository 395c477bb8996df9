"""Pins for the 8-bit attention oracle (CPU only).

Pinned against: explicit loops with math.exp on tiny inputs (no numpy
softmax or matmul), softmax invariants, closed forms (equal keys give the
mean of the values, equal values pass through, two keys give the logistic
function), inputs that MXFP8 represents exactly (the quantised attention
must then equal the plain one), the power-of-two normaliser (explicit
loops; an integer shift of it leaves every code and the dequantised result
up to that power of two unchanged), and the derived error bound (it holds
for the rounding of the weights, and the sharp check rejects a planted
scale mistake and a dropped key block).
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import quant as Qz


def _bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).bfloat16()


def test_softmax_matches_explicit_loops():
    rng = np.random.default_rng(1)
    S = rng.normal(size=(3, 5)) * 4
    P = A.softmax_rows(S)
    for i in range(3):
        den = sum(math.exp(S[i, j]) for j in range(5))
        for j in range(5):
            assert abs(P[i, j] - math.exp(S[i, j]) / den) < 1e-15


def test_softmax_invariants():
    rng = np.random.default_rng(2)
    S = rng.normal(size=(4, 64)) * 10
    P = A.softmax_rows(S)
    assert np.allclose(P.sum(axis=1), 1.0, atol=1e-15)
    assert np.allclose(A.softmax_rows(S + rng.normal(size=(4, 1)) * 100), P, atol=1e-15)
    assert np.allclose(A.softmax_rows(np.zeros((2, 10))), 0.1)


def test_plain_attention_matches_explicit_loops():
    rng = np.random.default_rng(3)
    T, d = 4, 3
    Q, K, V = (rng.normal(size=(T, d)) for _ in range(3))
    tau = 1 / math.sqrt(d)
    O = A.attention_plain(Q, K, V)
    for i in range(T):
        s = [tau * sum(Q[i, c] * K[j, c] for c in range(d)) for j in range(T)]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        for c in range(d):
            assert abs(O[i, c] - sum(w[j] * V[j, c] for j in range(T)) / sum(w)) < 1e-14


def _exact_mx(rng, R, C):
    """[R, C] values MXFP8 represents exactly along rows AND along columns:
    integers in [-16, 16] (E4M3-exact) times 2^-8, and every 32 x 32 tile's
    diagonal set to 1 = 256 * 2^-8, so every 32-element block of every row
    and of every column has maximum exactly 1 (shared exponent -8)."""
    x = rng.integers(-16, 17, size=(R, C)).astype(np.float32)
    for i in range(R):
        x[i, (i % 32)::32] = 256.0
    return x * np.float32(2.0 ** -8)


def test_exactly_representable_inputs_give_the_plain_attention():
    rng = np.random.default_rng(4)
    T, d = 64, 64
    Q, K, V = (_exact_mx(rng, T, d) for _ in range(3))
    O, Terr, Oq, vmax = A.attention_ref(_bf16(Q), _bf16(K), _bf16(V))
    assert np.allclose(O, A.attention_plain(Q, K, V), rtol=0, atol=1e-13)
    assert np.all(Terr + 1e-15 >= np.abs(O))
    # the rounding of the weights moves the result by less than the derived bound
    assert A.within_att_tol(Oq, O, Terr, vmax).all()


def test_equal_keys_average_the_values():
    rng = np.random.default_rng(5)
    T, d = 64, 32
    Q = _exact_mx(rng, T, d)
    K = np.tile(_exact_mx(rng, 1, d), (T, 1))
    V = _exact_mx(rng, T, d)
    O, _, _, _ = A.attention_ref(_bf16(Q), _bf16(K), _bf16(V))
    assert np.allclose(O, np.tile(V.astype(np.float64).mean(axis=0), (T, 1)), atol=1e-14)


def test_equal_values_pass_through():
    rng = np.random.default_rng(6)
    T, d = 64, 32
    Q, K = (rng.normal(size=(T, d)).astype(np.float32) for _ in range(2))
    v = np.float32(2.0 ** -3) * rng.integers(1, 8, size=d).astype(np.float32)
    V = np.tile(v, (T, 1))
    O, _, _, _ = A.attention_ref(_bf16(Q), _bf16(K), _bf16(V))
    assert np.allclose(O, np.tile(v.astype(np.float64), (T, 1)), atol=1e-14)


def test_quantised_weights_renormalise_a_constant_value_exactly():
    # the division by the sum of the quantised weights: with every key's value
    # equal (and exactly representable) the quantised path returns it exactly,
    # whatever the rounding of the weights; a division by the unquantised sum
    # would be off by the weights' mean rounding error
    rng = np.random.default_rng(9)
    T, d = 96, 32
    Q, K = (rng.normal(size=(T, d)).astype(np.float32) * 2 for _ in range(2))
    v = np.float32(2.0 ** -3) * rng.integers(-7, 8, size=d).astype(np.float32)
    V = np.tile(v, (T, 1))
    _, _, Oq, _ = A.attention_ref(_bf16(Q), _bf16(K), _bf16(V))
    assert np.array_equal(Oq, np.tile(v.astype(np.float64), (T, 1)))


def test_two_key_closed_form():
    # plain attention, two keys: p = sigmoid(tau (s0 - s1))
    Q = np.array([[1.0, 2.0]])
    K = np.array([[0.5, -1.0], [2.0, 1.0]])
    V = np.array([[3.0, -1.0], [-2.0, 5.0]])
    tau = 1 / math.sqrt(2)
    d0, d1 = Q[0] @ K[0], Q[0] @ K[1]
    p = 1 / (1 + math.exp(-tau * (d0 - d1)))
    want = p * V[0] + (1 - p) * V[1]
    assert np.allclose(A.attention_plain(Q, K, V)[0], want, atol=1e-14)


def test_pow2_weights_match_explicit_loops():
    t = np.array([[0.25, 3.5, -1.0], [-7.75, -7.5, -9.0]])
    E = A.weights_pow2(t)
    for i in range(2):
        m = math.ceil(max(t[i]))
        for j in range(3):
            assert E[i, j] == 2.0 ** (t[i, j] - m)
    # the largest weight of a row lies in (1/2, 1]
    rng = np.random.default_rng(7)
    E = A.weights_pow2(rng.normal(size=(16, 64)) * 5)
    assert np.all(E.max(axis=1) <= 1.0) and np.all(E.max(axis=1) > 0.5)


def test_power_of_two_normaliser_leaves_codes_and_result_unchanged():
    # the reading's claim: shifting m by an integer k scales every block by
    # 2^-k, moves each ceiling-rule shared exponent by -k and keeps every code
    rng = np.random.default_rng(8)
    t = rng.normal(size=(8, 256)) * 3
    E0 = A.weights_pow2(t).astype(np.float32)
    for k in (-8, -3, 5):
        Ek = A.weights_pow2(t, shift=k).astype(np.float32)
        q0 = Qz.quantize_mxfp8(E0, scale_rule="rceil")
        qk = Qz.quantize_mxfp8(Ek, scale_rule="rceil")
        assert np.array_equal(q0["codes"], qk["codes"])
        d0 = Qz.dequant_mxfp8(q0["codes"], q0["sf"])
        dk = Qz.dequant_mxfp8(qk["codes"], qk["sf"])
        assert np.array_equal(dk, d0 * 2.0 ** -k)


def test_bounds_hold_for_the_weight_rounding_and_reject_planted_mistakes():
    T, d = 256, 128
    Q, K, V = (torch.randn(T, d, generator=torch.Generator().manual_seed(s)).bfloat16() for s in (1, 2, 3))
    O, Terr, Oq, vmax = A.attention_ref(Q, K, V)
    assert A.within_att_tol(Oq, O, Terr, vmax).all()
    assert np.all(Terr + 1e-15 >= np.abs(O))
    # a kernel that forgot the 1/sqrt(d) softmax scale fails both checks
    Obad, _, _, _ = A.attention_ref(Q, K, V, tau=1.0)
    assert not A.within_att_tol(Obad, O, Terr, vmax).all()
    assert A.within_att_tight(Obad, Oq, Terr).mean() < 0.5
    # so does one that left the weights unrounded ... only for a few elements:
    # the sharp check separates O from O_q on most of them
    assert A.within_att_tight(O, Oq, Terr).mean() < 0.9
    # a kernel that dropped the last key block fails the sharp check
    Od, _, _, _ = A.attention_ref(Q[:, :], K[: T - 32], V[: T - 32])
    assert A.within_att_tight(Od, Oq, Terr).mean() < 0.5
    # rows restrict the queries only
    rows = np.array([0, 5, 255])
    O2, T2, Oq2, v2 = A.attention_ref(Q, K, V, rows=rows)
    assert np.allclose(O2, O[rows], atol=1e-15) and np.allclose(T2, Terr[rows], atol=1e-15)
    assert np.allclose(Oq2, Oq[rows], atol=1e-15) and np.array_equal(v2, vmax)
