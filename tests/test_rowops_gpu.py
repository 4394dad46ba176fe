"""GPU parity and batch-invariance tests of the row kernels, through the C ABI.

Parity: kernel output vs the fp64 oracle on the same seeded inputs, at the tiny
sizes (full output) and at the workload sizes (sampled rows).  Invariance: each
row computed inside batches of many sizes, at several positions, equals bit for
bit the same row computed alone (M = 1); repeated runs are identical.
"""
import numpy as np
import pytest
import torch

from bi_testutil import (assert_bf16_close, assert_lsm_close, assert_mean_close, bf16_bits_np,
                         same_bits)
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


# ----------------------------------------------------------------------------- RMSNorm

@pytest.mark.parametrize("H", [256, 4096, 8, 24, 1000, 4104, 12288])
@pytest.mark.parametrize("M", [1, 3, 17])
def test_rmsnorm_parity_small(M, H):
    x = inputs.rows_normal_outliers(100 + H, 0, M, H, torch.bfloat16)
    w = inputs.gain(101, H)
    y = bi.bi_rmsnorm(x.to(DEV), w.to(DEV), EPS)
    ref = oracle.rmsnorm(bf16_bits_np(x), bf16_bits_np(w), EPS)
    assert_bf16_close(y, ref, f"rmsnorm M={M} H={H}")


def test_rmsnorm_integer_and_constant_rows():
    H = 4096
    x = inputs.rows_int(102, 0, 4, H)
    x[3] = 2.0
    w = inputs.gain(103, H)
    y = bi.bi_rmsnorm(x.to(DEV), w.to(DEV), EPS)
    assert_bf16_close(y, oracle.rmsnorm(bf16_bits_np(x), bf16_bits_np(w), EPS), "rmsnorm ints")


def test_rmsnorm_workload_sampled_rows():
    M, H = 16384, 4096
    x = inputs.rows_normal_outliers(104, 0, M, H, torch.bfloat16)
    w = inputs.gain(105, H)
    y = bi.bi_rmsnorm(x.to(DEV), w.to(DEV), EPS).cpu()
    rows = torch.tensor([0, 1, 127, 128, 4095, 9999, M - 1])
    ref = oracle.rmsnorm(bf16_bits_np(x[rows]), bf16_bits_np(w), EPS)
    assert_bf16_close(y[rows], ref, "rmsnorm 16384x4096 sampled")


# ----------------------------------------------------------------------------- mean

@pytest.mark.parametrize("H", [256, 4096, 7, 1000, 4100])
@pytest.mark.parametrize("M", [1, 3, 17])
def test_mean_parity_small(M, H):
    x = inputs.rows_normal_outliers(110 + H, 0, M, H, torch.float32)
    y = bi.bi_mean(x.to(DEV))
    xn = x.numpy()
    assert_mean_close(y, oracle.mean(xn), xn, f"mean M={M} H={H}")


@pytest.mark.parametrize("H", [16384, 151936, 16388, 16387])
def test_mean_parity_long_rows(H):
    """Long rows (the step's mean runs over 151936 log-probs), on the vector path and, for a
    row length that breaks the 16-byte rule (16387), the scalar path."""
    x = inputs.rows_normal_outliers(113 + H, 0, 5, H, torch.float32)
    y = bi.bi_mean(x.to(DEV))
    xn = x.numpy()
    assert_mean_close(y, oracle.mean(xn), xn, f"mean long rows H={H}")


def test_mean_long_rows_batch_invariance():
    H = 151936
    pool = inputs.rows_normal_outliers(115, 0, 512, H, torch.float32).to(DEV)
    _check_invariance(lambda x: bi.bi_mean(x), pool, [1, 2, 3, 8, 64, 77, 148, 256, 512], 116)
    first = bi.bi_mean(pool)
    for _ in range(100):
        assert same_bits(bi.bi_mean(pool), first)


@pytest.mark.parametrize("H", [256, 4096, 131072])
def test_mean_integer_exact(H):
    x = inputs.rows_int(111, 0, 9, H, dtype=torch.float32)
    y = bi.bi_mean(x.to(DEV)).cpu().double().numpy()
    ref = oracle.mean(x.numpy())
    assert np.array_equal(y, ref.astype(np.float32).astype(np.float64))


def test_mean_workload_sampled_rows():
    M, H = 16384, 4096
    x = inputs.rows_normal_outliers(112, 0, M, H, torch.float32)
    y = bi.bi_mean(x.to(DEV)).cpu()
    rows = torch.tensor([0, 5, 127, 128, 8191, M - 1])
    xs = x[rows].numpy()
    assert_mean_close(y[rows], oracle.mean(xs), xs, "mean 16384x4096 sampled")


# ----------------------------------------------------------------------------- log_softmax

@pytest.mark.parametrize("V", [1000, 8, 999, 4096, 16384, 98304, 98312, 151936])
@pytest.mark.parametrize("M", [1, 3, 17])
def test_log_softmax_parity_fp32(M, V):
    x = inputs.rows_normal(120 + V, 0, M, V, dtype=torch.float32)
    y = bi.bi_log_softmax(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(x.numpy()), f"log_softmax fp32 M={M} V={V}")


# 1001 takes the scalar path, the others the streamed path (a ring of 6 stages of 16 KB: rows of
# 1, 4, 14, 19, 24, 25 and 48 chunks).
@pytest.mark.parametrize("V", [151936, 1000, 1001, 110000, 155648, 155656, 4096, 32760, 32768, 196608,
                               196616, 393216])
def test_log_softmax_parity_bf16(V):
    M = 5
    x = inputs.rows_normal(121, 0, M, V, std=1.3)
    y = bi.bi_log_softmax(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), f"log_softmax bf16 V={V}")


def test_log_softmax_constant_and_extreme_rows():
    V = 151936
    x = torch.zeros(3, V, dtype=torch.bfloat16)
    x[1] = 3.5
    x[2, 17] = 60.0  # one dominant entry
    x[2, 18:] = -60.0
    y = bi.bi_log_softmax(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), "log_softmax constant/extreme")


def test_log_softmax_workload_sampled_rows():
    M, V = 1024, 151936
    x = inputs.rows_normal(122, 0, M, V, std=1.3)
    y = bi.bi_log_softmax(x.to(DEV)).cpu()
    rows = torch.tensor([0, 127, 128, 777, M - 1])
    assert_lsm_close(y[rows], oracle.log_softmax(bf16_bits_np(x[rows])), "log_softmax 1024x151936")


# ----------------------------------------------------------------------------- SiLU * up

@pytest.mark.parametrize("F", [12288, 8, 12, 1000])
@pytest.mark.parametrize("M", [1, 3, 17])
def test_silu_mul_parity(M, F):
    gu = inputs.rows_normal(130 + F, 0, M, 2 * F, std=2.0)
    h = bi.bi_silu_mul(gu.to(DEV))
    assert_bf16_close(h, oracle.silu_mul(bf16_bits_np(gu)), f"silu_mul M={M} F={F}")


# ----------------------------------------------------------------------------- invariance

ROW_SWEEP = [1, 2, 3, 4, 8, 16, 77, 128, 129, 1000, 1024, 2048]


def _pool_and_refs(fn, pool):
    refs = [fn(pool[i:i + 1]) for i in range(pool.shape[0])]
    return torch.cat(refs)


def _check_invariance(fn, pool, sweep, seed):
    ref = _pool_and_refs(fn, pool)
    perm = inputs.permutation(seed, pool.shape[0]).to(DEV)
    for M in sweep:
        for start in (0, pool.shape[0] - M):
            idx = perm[start:start + M]
            out = fn(pool[idx])
            assert same_bits(out, ref[idx]), f"M={M}: a row differs from its M=1 result"


def test_rmsnorm_batch_invariance():
    H = 4096
    pool = inputs.rows_normal_outliers(140, 0, 2048, H, torch.bfloat16).to(DEV)
    w = inputs.gain(141, H).to(DEV)
    _check_invariance(lambda x: bi.bi_rmsnorm(x, w, EPS), pool, ROW_SWEEP, 142)


def test_mean_batch_invariance():
    H = 4096
    pool = inputs.rows_normal_outliers(143, 0, 2048, H, torch.float32).to(DEV)
    _check_invariance(lambda x: bi.bi_mean(x), pool, ROW_SWEEP, 144)


def test_log_softmax_batch_invariance():
    V = 151936
    pool = inputs.rows_normal(145, 0, 256, V, std=1.3).to(DEV)
    _check_invariance(lambda x: bi.bi_log_softmax(x), pool, [1, 2, 3, 8, 64, 77, 128, 256], 146)


def test_log_softmax_streamed_rows_batch_invariance():
    V = 393216  # 48 ring chunks per row
    pool = inputs.rows_normal(149, 0, 64, V, std=1.3).to(DEV)
    _check_invariance(lambda x: bi.bi_log_softmax(x), pool, [1, 2, 3, 17, 64], 150)
    xf = pool[:8].float()
    _check_invariance(lambda x: bi.bi_log_softmax(x), xf, [1, 3, 8], 151)


def test_row_ops_repeatable_100_runs():
    H = 4096
    x = inputs.rows_normal_outliers(147, 0, 2048, H, torch.bfloat16).to(DEV)
    w = inputs.gain(148, H).to(DEV)
    xf = x.float()
    first_n = bi.bi_rmsnorm(x, w, EPS)
    first_m = bi.bi_mean(xf)
    for _ in range(100):
        assert same_bits(bi.bi_rmsnorm(x, w, EPS), first_n)
        assert same_bits(bi.bi_mean(xf), first_m)


def test_log_softmax_repeatable_100_runs():
    """The streamed kernel of the LM-head step: bulk copies complete on mbarriers, a stage is
    refilled right after the block has read it, and the second pass reads stages still
    resident.  A missing fence there would show up as a rare bit flip, so the step's own shape
    (bf16, M = 1024, V = 151936: 10 ring chunks, the last one partial) runs 100 times, and an
    fp32 row length whose last chunk holds 8 elements (98312 = 12 x 8192 + 8) as well."""
    x = inputs.rows_normal(152, 0, 1024, 151936, std=1.3).to(DEV)
    first = bi.bi_log_softmax(x)
    for _ in range(100):
        assert same_bits(bi.bi_log_softmax(x), first)
    xf = inputs.rows_normal(153, 0, 64, 98312, dtype=torch.float32).to(DEV)
    first = bi.bi_log_softmax(xf)
    for _ in range(100):
        assert same_bits(bi.bi_log_softmax(xf), first)


def test_silu_mul_repeatable_100_runs():
    gu = inputs.rows_normal(154, 0, 512, 2 * 12288, std=2.0).to(DEV)
    first = bi.bi_silu_mul(gu)
    for _ in range(100):
        assert same_bits(bi.bi_silu_mul(gu), first)


# ----------------------------------------------------------------------------- edge cases

def test_empty_batch_is_noop():
    x = torch.empty(0, 4096, dtype=torch.bfloat16, device=DEV)
    w = torch.ones(4096, dtype=torch.bfloat16, device=DEV)
    assert bi.bi_rmsnorm(x, w).shape == (0, 4096)
    assert bi.bi_mean(x.float()).shape == (0,)
    assert bi.bi_log_softmax(x).shape == (0, 4096)
    assert bi.bi_silu_mul(x).shape == (0, 2048)


def test_misaligned_vector_path_is_rejected():
    buf = torch.zeros(2 * 4096 + 8, dtype=torch.bfloat16, device=DEV)
    x = buf[1:1 + 2 * 4096].view(2, 4096)  # 2-byte offset: not 16-byte aligned
    w = torch.ones(4096, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_rmsnorm(x, w)
    assert e.value.status == bi.BI_ERR_ALIGNMENT
