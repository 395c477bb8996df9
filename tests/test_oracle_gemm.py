"""Pins for the oracle's float64 linear reference and its tolerance (CPU only).

Pinned against: a plain triple loop written with no library call (tiny,
non-square shapes, so a transposed operand fails), closed forms for rank-one
integer operands, one-hot weight rows that select activation columns, an
all-zero activation (Y = bias exactly), and lossless quantisation of exactly
representable operands (the quantised path must then equal the bf16 product).
"""

import numpy as np
import pytest
import torch

from oracle import gemm as G
from oracle import quant as Q
from oracle import dispatch as D
import workloads


def test_triple_loop_matches_library_matmul():
    rng = np.random.default_rng(0)
    A = rng.normal(size=(5, 7))
    W = rng.normal(size=(3, 7))
    b = torch.tensor(rng.normal(size=3), dtype=torch.float32).bfloat16()
    Y1, T1 = G.gemm_triple_loop(A, W, b)
    Y2, T2 = G.linear_ref(A, W, b)
    assert np.allclose(Y1, Y2, rtol=1e-13, atol=1e-13)
    assert np.allclose(T1, T2, rtol=1e-13, atol=1e-13)


def test_rank_one_integer_closed_form():
    M, K, N = 6, 40, 9
    a = np.arange(1, M + 1) * (-1.0) ** np.arange(M)
    w = np.arange(N) - 4.0
    A = np.repeat(a[:, None], K, axis=1)
    W = np.repeat(w[:, None], K, axis=1)
    Y, T = G.linear_ref(A, W)
    assert np.array_equal(Y, K * np.outer(a, w))
    assert np.array_equal(T, K * np.outer(np.abs(a), np.abs(w)))


def test_one_hot_rows_select_columns():
    rng = np.random.default_rng(1)
    M, K, N = 4, 64, 10
    A = rng.normal(size=(M, K))
    perm = rng.permutation(K)[:N]
    W = np.zeros((N, K))
    W[np.arange(N), perm] = 1.0
    Y, _ = G.linear_ref(A, W)
    assert np.array_equal(Y, A[:, perm])


def test_zero_activation_gives_bias():
    c = workloads.random_case(8, 64, 16, "nvfp4", seed=3)
    A = torch.zeros_like(c.A)
    Y, T, _, _ = G.linear_ref_quantized("nvfp4", A, c.W, c.bias)
    assert np.array_equal(Y, np.broadcast_to(c.bias.float().numpy().astype(np.float64), Y.shape))
    assert not T.any()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_lossless_operands_equal_bf16_product(fmt):
    # operands whose quantisation is exact: the quantised reference must equal
    # the plain float64 product of the bf16 operands
    rng = np.random.default_rng(2)
    if fmt == "nvfp4":
        vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
        A = rng.choice(vals, size=(8, 64)) * rng.choice([-1, 1], size=(8, 64))
        W = rng.choice(vals, size=(5, 64)) * rng.choice([-1, 1], size=(5, 64))
        A[:, ::16] = 6.0  # every block's max is 6 -> block scale 448 * g = 1
        W[:, ::16] = -6.0
        A *= 448.0  # amax = 2688 -> g = 1 ... then scale e = 448 -> s = 448
        W *= 448.0
    else:
        vals = np.array([0, 0.25, 1, 1.5, 3, 5, 7, 12])
        A = rng.choice(vals, size=(8, 64)) * 16
        W = rng.choice(vals, size=(5, 64)) * 16
        A[:, ::32] = 256.0
        W[:, ::32] = 256.0
    At = torch.tensor(A, dtype=torch.float32).bfloat16()
    Wt = torch.tensor(W, dtype=torch.float32).bfloat16()
    Yq, Tq, _, _ = G.linear_ref_quantized(fmt, At, Wt)
    Yb, Tb, _, _ = G.linear_ref_quantized("bf16", At, Wt)
    assert np.array_equal(Yq, Yb) and np.array_equal(Tq, Tb)


def test_quantized_reference_rows_subset():
    c = workloads.random_case(40, 128, 24, "nvfp4", seed=4)
    Y, T, _, _ = G.linear_ref_quantized("nvfp4", c.A, c.W, c.bias)
    rows = np.array([0, 7, 39])
    Ys, Ts, _, _ = G.linear_ref_quantized("nvfp4", c.A, c.W, c.bias, rows=rows)
    assert np.array_equal(Ys, Y[rows]) and np.array_equal(Ts, T[rows])


def test_tolerance_rule():
    T = np.array([0.0, 1.0, 100.0])
    ok = G.within_tol(np.array([1e-6, 1.002, 100.2]), np.zeros(3) + [0, 1, 100], T)
    assert ok.all()
    bad = G.within_tol(np.array([2e-6, 1.0021, 100.21]), np.zeros(3) + [0, 1, 100], T)
    assert not bad.any()


def test_bf16_rounding_matches_hand_worked_ties_and_torch():
    # ties to the even significand, by hand: 1 + 2^-8 lies halfway between 1
    # and 1 + 2^-7 (odd) -> 1; 1 + 3 * 2^-8 halfway between 1 + 2^-7 (odd) and
    # 1 + 2^-6 (even) -> 1 + 2^-6; the sign is kept; 2^-9 above 1.5 rounds down
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1.5 + 2.0 ** -9, 0.0, 3.0])
    assert np.array_equal(G.bf16_rne(x), [1.0, 1 + 2.0 ** -6, -1.0, 1.5, 0.0, 3.0])
    # float32 inputs: the same as torch's float32 -> bf16 cast (a library routine)
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(100000) * np.exp2(rng.integers(-30, 30, 100000))).astype(np.float32)
    assert np.array_equal(G.bf16_rne(f.astype(np.float64)), torch.tensor(f).bfloat16().double().numpy())


def test_correctly_rounded_output_passes_and_one_ulp_off_does_not():
    # |Y| comparable to T: the bf16 rounding of Y exceeds 2e-3 T
    Y = np.array([[-0.5408780856523663]])
    T = np.array([[0.8773537517990917]])
    good = G.bf16_rne(Y)
    assert good[0, 0] == -0.5390625 and abs(good[0, 0] - Y[0, 0]) > 2e-3 * T[0, 0] + 1e-6
    assert G.within_tol(good, Y, T).all()
    assert not G.within_tol(good - 2.0 ** -8, Y, T).any()


def test_quantization_error_within_gemm_tolerance_is_not_vacuous():
    # the bf16 product of the raw operands differs from the quantised one by
    # far more than the tolerance: the tolerance pins the quantised operands
    c = workloads.random_case(32, 256, 32, "nvfp4", seed=5)
    Yq, Tq, _, _ = G.linear_ref_quantized("nvfp4", c.A, c.W)
    Yb, _, _, _ = G.linear_ref_quantized("bf16", c.A, c.W)
    assert not G.within_tol(Yb, Yq, Tq).all()


def test_dispatch_rule():
    assert D.use_bf16(1, 3072, 18432)
    assert D.use_bf16(512, 3072, 9216)
    assert not D.use_bf16(4096, 3072, 9216)
    assert not D.use_bf16(1024, 1024, 1024)  # exactly 1024 is quantised
    assert D.use_bf16(1023, 4096, 4096)
    assert D.use_bf16(4096, 4096, 4096, keep_bf16=True)
    assert D.use_bf16(4096, 4096, 4096, min_dim=8192)


def test_dispatch_on_flux_stack():
    for B, frac in ((1, 0.963), (4, 0.9999)):
        layers = workloads.flux_linear_stack(batch=B)
        assert len(layers) == 19 * 10 + 38 * 3
        tot = sum(2 * l["M"] * l["K"] * l["N"] for l in layers)
        q = sum(2 * l["M"] * l["K"] * l["N"] for l in layers
                if not D.use_bf16(l["M"], l["K"], l["N"]))
        assert abs(q / tot - frac) < 0.001
        kinds = {l["name"].split(".", 1)[1]: D.use_bf16(l["M"], l["K"], l["N"])
                 for l in layers if l["name"].startswith(("d0.", "s0."))}
        assert kinds["img.mod"] and kinds["txt.mod"] and kinds["mod"]
        assert kinds["txt.qkv"] == (B == 1)
        assert not kinds["img.mlp_up"] and not kinds["linear1"]
    # 12B-class parameter count (the first article's "12 billion parameters")
    p = sum(l["K"] * l["N"] for l in workloads.flux_linear_stack(batch=1))
    assert 11.5e9 < p < 12.5e9
