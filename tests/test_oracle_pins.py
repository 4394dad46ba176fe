"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each test compares the oracle with exact integer brute force, a closed form,
an invariant that determines the answer, or a library routine that computes the
exact result (math.fsum, fractions, decimal).  The cases are picked so that a
plausible slip in the oracle -- a dropped term, a wrong sign or index, a
transposed operand, eps outside the square root, swapped gate/up halves --
fails at least one of them; the `*_detects_*` tests show that on purpose by
feeding the oracle a planted mistake on the CPU.
"""
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


def golden(op, name):
    for c in GOLDEN["cases"]:
        if c["op"] == op and c["name"] == name:
            return c
    raise KeyError((op, name))


def bits(t):
    return inputs.bf16_bits(t)


def ints(t):
    return t.to(torch.float32).numpy().astype(np.int64)


def py_matmul(a, b):
    """Exact integer brute force: list-of-lists A[M][K] times B[K][N]."""
    M, K, N = len(a), len(b), len(b[0])
    return [[sum(a[i][k] * b[k][j] for k in range(K)) for j in range(N)] for i in range(M)]


# ----------------------------------------------------------------------------- matmul / addmm

@pytest.mark.parametrize("M,K,N", [(5, 11, 7), (1, 1, 1), (3, 16, 9), (17, 33, 2)])
def test_matmul_integer_brute_force_both_layouts(M, K, N):
    a = inputs.rows_int(1, 0, M, K)
    b = inputs.weight_int(2, (K, N))
    exact = py_matmul(ints(a).tolist(), ints(b).tolist())
    c_kn = oracle.matmul(bits(a), bits(b), "kn")
    c_nk = oracle.matmul(bits(a), bits(b.t().contiguous()), "nk")
    assert c_kn.tolist() == exact
    assert c_nk.tolist() == exact


@pytest.mark.parametrize("K", [256, 4096])
def test_matmul_integer_exact_large_k(K):
    M, N = 3, 24
    a = inputs.rows_int(3, 0, M, K)
    b = inputs.weight_int(4, (N, K))
    exact = ints(a) @ ints(b).T  # int64 arithmetic: exact
    c = oracle.matmul(bits(a), bits(b), "nk")
    assert np.array_equal(c, exact.astype(np.float64))


def test_matmul_leading_dimensions():
    M, K, N = 4, 12, 5
    big_a = inputs.rows_int(5, 0, M, K + 9)
    big_b = inputs.weight_int(6, (K, N + 3))
    a, b = big_a[:, 3:3 + K], big_b[:, 1:1 + N]
    exact = py_matmul(ints(a).tolist(), ints(b).tolist())
    a_np, b_np = bits(big_a)[:, 3:3 + K], bits(big_b)[:, 1:1 + N]
    assert oracle.matmul(a_np, b_np, "kn").tolist() == exact


def test_matmul_identity_and_one_hot():
    case = golden("matmul", "identity")
    for K in case["K"]:
        a = inputs.rows_normal(7, 0, 6, K)
        eye = torch.eye(K, dtype=torch.bfloat16)
        c = oracle.matmul(bits(a), bits(eye), "kn")
        assert np.array_equal(c, a.to(torch.float64).numpy())
    K, N = 10, 6
    b = inputs.weight_normal(8, (K, N))
    onehot = torch.zeros(K, K, dtype=torch.bfloat16)
    onehot[torch.arange(K), torch.arange(K).flip(0)] = 1
    c = oracle.matmul(bits(onehot), bits(b), "kn")
    assert np.array_equal(c, b.to(torch.float64).flip(0).numpy())


def test_matmul_fp64_sum_matches_fsum():
    """Real-valued case: every entry within a few ulps of the exactly rounded sum."""
    M, K, N = 3, 4096, 5
    a = inputs.rows_normal(9, 0, M, K)
    b = inputs.weight_normal(10, (N, K))
    c = oracle.matmul(bits(a), bits(b), "nk")
    ad, bd = a.double().numpy(), b.double().numpy()
    for i in range(M):
        for j in range(N):
            terms = ad[i] * bd[j]  # bf16 x bf16 products are exact in binary64
            ref = math.fsum(terms)
            bound = K * 2.0 ** -53 * np.abs(terms).sum()
            assert abs(c[i, j] - ref) <= bound


def test_matmul_pin_detects_transposed_operand():
    """Planted mistake: reading B with the other layout must fail the brute-force pin."""
    M, K, N = 4, 6, 6
    a = inputs.rows_int(11, 0, M, K)
    b = inputs.weight_int(12, (K, N))
    exact = py_matmul(ints(a).tolist(), ints(b).tolist())
    wrong = oracle.matmul(bits(a), bits(b), "nk")  # square B read as [N, K]
    assert wrong.tolist() != exact


def test_addmm_zero_lhs_gives_input():
    golden("addmm", "zero_lhs")
    M, K, N = 5, 32, 9
    zero = torch.zeros(M, K, dtype=torch.bfloat16)
    b = inputs.weight_normal(13, (N, K))
    bias = inputs.bias(14, N)
    resid = inputs.rows_normal(15, 0, M, N)
    c = oracle.addmm(bits(bias), bits(zero), bits(b), "nk")
    assert np.array_equal(c, np.broadcast_to(bias.double().numpy(), (M, N)))
    c = oracle.addmm(bits(resid), bits(zero), bits(b), "nk")
    assert np.array_equal(c, resid.double().numpy())


@pytest.mark.parametrize("full", [False, True])
def test_addmm_integer_brute_force(full):
    M, K, N = 6, 19, 8
    a = inputs.rows_int(16, 0, M, K)
    b = inputs.weight_int(17, (K, N))
    inp = inputs.rows_int(18, 0, M, N) if full else inputs.weight_int(19, (N,))
    prod = py_matmul(ints(a).tolist(), ints(b).tolist())
    add = ints(inp)
    exact = [[prod[i][j] + int(add[i, j] if full else add[j]) for j in range(N)] for i in range(M)]
    assert oracle.addmm(bits(inp), bits(a), bits(b), "kn").tolist() == exact
    assert oracle.addmm(bits(inp), bits(a), bits(b.t().contiguous()), "nk").tolist() == exact


# ----------------------------------------------------------------------------- rmsnorm

def test_rmsnorm_constant_rows_closed_form():
    case = golden("rmsnorm", "constant_row")
    eps = case["eps"]
    for H in case["H"]:
        w = inputs.gain(20, H)
        for cval in case["c"]:
            x = torch.full((1, H), cval, dtype=torch.bfloat16)
            y = oracle.rmsnorm(bits(x), bits(w), eps)
            cx = float(x[0, 0])
            expect = w.double().numpy() * cx / math.sqrt(cx * cx + eps)
            assert np.allclose(y[0], expect, rtol=1e-14, atol=0)


def test_rmsnorm_integer_rows_against_exact_sum_of_squares():
    getcontext().prec = 50
    M, H, eps = 4, 256, 1e-6
    x = inputs.rows_int(21, 0, M, H)
    w = inputs.gain(22, H)
    y = oracle.rmsnorm(bits(x), bits(w), eps)
    xi, wd = ints(x), w.double().numpy()
    for i in range(M):
        S = int((xi[i] ** 2).sum())  # exact
        r = float(1 / (Decimal(S) / Decimal(H) + Decimal(eps)).sqrt())
        expect = xi[i] * r * wd
        assert np.allclose(y[i], expect, rtol=1e-14, atol=1e-300)


def test_rmsnorm_invariants_and_eps_placement():
    """y_j / (x_j w_j) is one positive constant r per row, and mean((y/w)^2) = ms/(ms+eps)."""
    M, H, eps = 3, 4096, 1e-6
    x = inputs.rows_normal_outliers(23, 0, M, H, torch.bfloat16)
    tiny = torch.full((1, H), 2.0 ** -11, dtype=torch.bfloat16)  # ms ~ eps: eps placement matters
    x = torch.cat([x, tiny])
    w = inputs.gain(24, H)
    y = oracle.rmsnorm(bits(x), bits(w), eps)
    xd, wd = x.double().numpy(), w.double().numpy()
    for i in range(x.shape[0]):
        nz = xd[i] != 0
        ratio = y[i][nz] / (xd[i][nz] * wd[nz])
        assert np.all(ratio > 0)
        assert np.allclose(ratio, ratio[0], rtol=1e-14)
        ms = math.fsum(xd[i] ** 2) / H
        assert math.isclose(math.fsum((y[i] / wd) ** 2) / H, ms / (ms + eps), rel_tol=1e-12)


def test_rmsnorm_pin_detects_eps_outside_sqrt():
    """Planted mistake: r = 1/sqrt(ms) + eps instead of 1/sqrt(ms + eps) fails the tiny-row pin."""
    H, eps = 256, 1e-6
    c = 2.0 ** -11
    good = c / math.sqrt(c * c + eps)
    wrong = c * (1.0 / math.sqrt(c * c) + eps)
    x = torch.full((1, H), c, dtype=torch.bfloat16)
    w = torch.ones(H, dtype=torch.bfloat16)
    y = oracle.rmsnorm(bits(x), bits(w), eps)
    assert math.isclose(y[0, 0], good, rel_tol=1e-14)
    assert not math.isclose(wrong, good, rel_tol=1e-3)


# ----------------------------------------------------------------------------- mean

def test_mean_arithmetic_progression():
    for H in golden("mean", "arithmetic_progression")["H"]:
        x = np.arange(1, H + 1, dtype=np.float32)[None, :]
        assert oracle.mean(x)[0] == (H + 1) / 2


def test_mean_constant_rows():
    case = golden("mean", "constant_row")
    for H in case["H"]:
        for c in case["c"]:
            x = np.full((2, H), c, dtype=np.float32)
            y = oracle.mean(x)
            assert math.isclose(y[0], float(np.float32(c)), rel_tol=1e-15)


@pytest.mark.parametrize("H", [256, 4096])
def test_mean_integer_exact(H):
    x = inputs.rows_int(25, 0, 5, H, dtype=torch.float32).numpy()
    y = oracle.mean(x)
    for i in range(5):
        assert Fraction(y[i]) == Fraction(int(x[i].astype(np.int64).sum()), H)


def test_mean_against_fsum_with_outliers():
    M, H = 4, 4096
    x = inputs.rows_normal_outliers(26, 0, M, H, torch.float32).numpy()
    y = oracle.mean(x)
    for i in range(M):
        ref = math.fsum(x[i].astype(np.float64)) / H
        assert abs(y[i] - ref) <= H * 2.0 ** -53 * np.abs(x[i]).sum() / H + 1e-300


# ----------------------------------------------------------------------------- log_softmax

def _check_log_softmax_invariants(x64, y, tol_sum=1e-13, tol_shift=1e-12):
    for i in range(x64.shape[0]):
        # sum_j exp(y_j) = 1 ...
        assert abs(math.fsum(np.exp(y[i])) - 1.0) <= tol_sum
        # ... and y - x is the same constant in every column: together they fix y uniquely.
        d = y[i] - x64[i]
        assert np.max(d) - np.min(d) <= tol_shift * max(1.0, np.max(np.abs(x64[i])))


def test_log_softmax_constant_rows():
    case = golden("log_softmax", "constant_row")
    for V in case["V"]:
        for c in case["c"]:
            x = np.full((1, V), c, dtype=np.float32)
            y = oracle.log_softmax(x)
            assert np.allclose(y, -math.log(V), rtol=0, atol=1e-12)


def test_log_softmax_two_entries():
    for row in golden("log_softmax", "two_entries")["x"]:
        x = np.array([row], dtype=np.float32)
        hi, lo = max(row), min(row)
        lse = hi + math.log1p(math.exp(lo - hi))
        assert np.allclose(oracle.log_softmax(x)[0], np.array(row) - lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("V", [1000, 151936])
def test_log_softmax_invariants(V):
    x = inputs.rows_normal(27, 0, 3, V, std=1.3, dtype=torch.float32).numpy()
    y = oracle.log_softmax(x)
    _check_log_softmax_invariants(x.astype(np.float64), y)


def test_log_softmax_large_and_shifted():
    V = 1000
    x = inputs.rows_normal(28, 0, 2, V, dtype=torch.float32).numpy()
    y0 = oracle.log_softmax(x)
    big = (x + np.float32(1.0e4)).astype(np.float32)
    y1 = oracle.log_softmax(big)
    assert np.all(np.isfinite(y1))
    _check_log_softmax_invariants(big.astype(np.float64), y1, tol_shift=1e-15)
    # shift invariance (the shifted input is rounded to fp32, so compare loosely)
    assert np.allclose(y0, y1, atol=2e-3)


def test_log_softmax_bf16_equals_widened_fp32():
    x = inputs.rows_normal(29, 0, 2, 5000, std=1.3)
    y_b = oracle.log_softmax(bits(x))
    y_f = oracle.log_softmax(x.to(torch.float32).numpy())
    assert np.array_equal(y_b, y_f)


def test_log_softmax_pin_detects_missing_max_shift_sign():
    """Planted mistake: y = x + m - log s (sign slip) breaks the exp-sum invariant."""
    x = inputs.rows_normal(30, 0, 1, 1000, dtype=torch.float32).numpy().astype(np.float64)
    m = x.max()
    s = np.exp(x - m).sum()
    wrong = (x + m) - math.log(s)
    assert abs(math.fsum(np.exp(wrong[0])) - 1.0) > 1e-6


# ----------------------------------------------------------------------------- silu_mul

def test_silu_mul_fixed_points_and_odd_identity():
    gs = golden("silu_mul", "fixed_points")["g"]
    g = torch.tensor(gs, dtype=torch.bfloat16)
    gu = torch.cat([g, torch.ones_like(g)])[None, :]
    h = oracle.silu_mul(bits(gu))[0]
    gd = g.double().numpy()
    for k, gv in enumerate(gd):
        ref = float(Decimal(gv) / (1 + (-Decimal(gv)).exp()))
        assert math.isclose(h[k], ref, rel_tol=1e-15, abs_tol=1e-300)
    assert h[0] == 0.0
    gm = torch.cat([-g, torch.ones_like(g)])[None, :]
    hm = oracle.silu_mul(bits(gm))[0]
    assert np.allclose(h - hm, gd, rtol=1e-15, atol=1e-15)


def test_silu_mul_halves_and_linearity_in_up():
    M, F = 3, 64
    g = inputs.rows_normal(31, 0, M, F)
    u = inputs.rows_int(32, 0, M, F)
    gu = torch.cat([g, u], dim=1)
    h = oracle.silu_mul(bits(gu))
    ones = torch.cat([g, torch.ones_like(u)], dim=1)
    s = oracle.silu_mul(bits(ones))
    assert np.array_equal(h, s * ints(u))  # multiplying by a small integer is exact
    swapped = oracle.silu_mul(bits(torch.cat([u, g], dim=1)))
    assert not np.allclose(swapped, h)


def test_silu_mul_f64_matches_bf16_version_on_exact_inputs():
    gu = inputs.rows_normal(33, 0, 4, 2 * 96, std=2.0)
    assert np.array_equal(oracle.silu_mul_f64(gu.double().numpy()), oracle.silu_mul(bits(gu)))


def test_matmul_silu_mul_composes_the_definitions():
    """Fused gate/up + glue: integer A, B make g and u exact, so h is the closed form of exact g, u."""
    M, K, F = 3, 32, 16
    a = inputs.rows_int(34, 0, M, K)
    w = inputs.weight_int(35, (2 * F, K))
    gu = py_matmul(ints(a).tolist(), ints(w).T.tolist())
    h = oracle.matmul_silu_mul(bits(a), bits(w), "nk")
    for i in range(M):
        for j in range(F):
            g, u = gu[i][j], gu[i][F + j]
            assert math.isclose(h[i, j], g / (1 + math.exp(-g)) * u, rel_tol=1e-15, abs_tol=1e-300)


def test_oracle_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.matmul(np.zeros((2, 3), np.uint16), np.zeros((4, 5), np.uint16), "kn")
    with pytest.raises(ValueError):
        oracle.rmsnorm(np.zeros((2, 3), np.uint16), np.zeros((4,), np.uint16), 1e-6)


def test_empty_batches():
    assert oracle.matmul(np.zeros((0, 8), np.uint16), np.zeros((8, 4), np.uint16), "kn").shape == (0, 4)
    assert oracle.mean(np.zeros((0, 8), np.float32)).shape == (0,)
    assert oracle.log_softmax(np.zeros((0, 8), np.float32)).shape == (0, 8)
