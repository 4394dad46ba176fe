"""IEEE edge cases of the row kernels, through the C ABI, against the fp64 oracle.

Masked logits (-inf entries, routine in sampling: vocabulary padding, banned tokens,
grammar masks) must not poison a row's (max, sum of exp) fold, on every log_softmax path:
the one-block streamed kernel (bf16 and fp32 rows), its scalar path, the 4-CTA cluster
variant and the split variant.  Rows cover a fully masked leading ring chunk, alternating
masks, a masked tail and a row with one unmasked entry.  A row with every entry masked has
no defined log_softmax; the kernels return NaN there, as the oracle's plain definition does
(max = -inf, so x - max is NaN).  RMSNorm of an all-zero row is exactly zero; mean
propagates infinities and NaN as IEEE addition does.
"""
import math

import numpy as np
import pytest
import torch

from bi_testutil import assert_lsm_close_ieee, assert_mean_close, bf16_bits_np
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
NINF = float("-inf")


def masked_rows(V, dtype):
    """Six rows of N(0, 1.3) values with different -inf masks."""
    x = inputs.rows_normal(700, 0, 6, V, std=1.3, dtype=dtype)
    x[0, : min(V - 1, 40000)] = NINF      # leading chunks fully masked
    x[1, ::2] = NINF                       # every other entry masked
    x[2, V - min(V // 2, 267):] = NINF     # masked tail (vocabulary padding)
    x[3, :] = NINF
    x[3, V // 3] = 2.5                     # exactly one unmasked entry: y = 0 there, -inf elsewhere
    x[4, :] = NINF                         # fully masked: NaN
    return x                               # row 5 unmasked


def ref_of(x):
    return oracle.log_softmax(bf16_bits_np(x) if x.dtype == torch.bfloat16 else x.numpy())


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 151936), (torch.float32, 98312), (torch.bfloat16, 1001),
                                     (torch.float32, 1000), (torch.bfloat16, 4096)])
def test_log_softmax_masked_rows(dtype, V):
    x = masked_rows(V, dtype)
    y = bi.bi_log_softmax(x.to(DEV))
    ref = ref_of(x)
    assert np.isnan(ref[4]).all() and ref[3, V // 3] == 0.0
    assert_lsm_close_ieee(y, ref, f"log_softmax masked {dtype} V={V}")


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 151936), (torch.float32, 32768)])
def test_log_softmax_cluster_masked_rows(dtype, V):
    x = masked_rows(V, dtype)
    y = bi.bi_log_softmax_cluster(x.to(DEV))
    assert_lsm_close_ieee(y, ref_of(x), f"cluster masked {dtype} V={V}")


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 151936), (torch.float32, 8200)])
def test_log_softmax_split_masked_rows(dtype, V):
    x = masked_rows(V, dtype)
    y = bi.bi_log_softmax_split(x.to(DEV))
    assert_lsm_close_ieee(y, ref_of(x), f"split masked {dtype} V={V}")


@pytest.mark.parametrize("H", [4096, 1000])
def test_rmsnorm_zero_row_is_zero(H):
    x = inputs.rows_normal(701, 0, 3, H)
    x[1] = 0.0
    w = inputs.gain(702, H)
    y = bi.bi_rmsnorm(x.to(DEV), w.to(DEV), 1e-6).cpu()
    ref = oracle.rmsnorm(bf16_bits_np(x), bf16_bits_np(w), 1e-6)
    assert np.all(ref[1] == 0.0)
    assert torch.count_nonzero(y[1]) == 0


@pytest.mark.parametrize("H", [4096, 151936, 1001])
def test_mean_propagates_inf_and_nan(H):
    x = inputs.rows_normal(703, 0, 5, H, dtype=torch.float32)
    x[0, 17] = math.inf
    x[1, H - 1] = -math.inf
    x[2, 3] = math.inf
    x[2, H // 2] = -math.inf
    x[3, H // 3] = math.nan
    y = bi.bi_mean(x.to(DEV)).cpu().double().numpy()
    ref = oracle.mean(x.numpy())
    assert ref[0] == math.inf and ref[1] == -math.inf and math.isnan(ref[2]) and math.isnan(ref[3])
    assert y[0] == math.inf and y[1] == -math.inf and math.isnan(y[2]) and math.isnan(y[3])
    xs = x[4:5].numpy()
    assert_mean_close(torch.from_numpy(y[4:5]), ref[4:5], xs, f"mean finite row H={H}")
