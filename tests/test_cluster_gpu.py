"""bi_log_softmax_cluster: log_softmax of long rows by a cluster of 4 CTAs per row, through
the C ABI.

Parity against the fp64 oracle, agreement with the one-block-per-row bi_log_softmax to the
tolerance, bit-level batch invariance over M and row positions, repeatability, and the row
lengths it refuses.
"""
import numpy as np
import pytest
import torch

from bi_testutil import assert_lsm_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


# bf16 rows from 64 KB (V = 32768) to 4 slices of 96 KB (V = 196608): slices of 8192 to 49152
# elements, the last slice shorter when 32 does not divide V.
@pytest.mark.parametrize("V", [32768, 110000, 151936, 155648, 155656, 196608])
@pytest.mark.parametrize("M", [1, 5])
def test_cluster_parity_bf16(M, V):
    x = inputs.rows_normal(700, 0, M, V, std=1.3)
    y = bi.bi_log_softmax_cluster(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), f"cluster bf16 M={M} V={V}")
    assert bi.bi_get_device_status() == bi.BI_OK


@pytest.mark.parametrize("V", [16384, 65540, 98304])
def test_cluster_parity_fp32(V):
    x = inputs.rows_normal(701, 0, 3, V, dtype=torch.float32)
    y = bi.bi_log_softmax_cluster(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(x.numpy()), f"cluster fp32 V={V}")


def test_cluster_constant_and_extreme_rows():
    V = 151936
    x = torch.zeros(3, V, dtype=torch.bfloat16)
    x[1] = 3.5
    x[2, 17] = 60.0  # one dominant entry, in the first slice
    x[2, 18:] = -60.0
    y = bi.bi_log_softmax_cluster(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), "cluster constant/extreme")
    assert float((y[0] + np.log(V)).abs().max()) <= 1e-4


def test_cluster_workload_sampled_rows_and_one_block_agreement():
    M, V = 1024, 151936
    x = inputs.rows_normal(702, 0, M, V, std=1.3).to(DEV)
    y = bi.bi_log_softmax_cluster(x)
    rows = torch.tensor([0, 127, 128, 777, M - 1])
    assert_lsm_close(y.cpu()[rows], oracle.log_softmax(bf16_bits_np(x.cpu()[rows])), "cluster 1024x151936")
    assert float((y - bi.bi_log_softmax(x)).abs().max()) <= 1e-4


def test_cluster_batch_invariance_and_repeatability():
    V = 151936
    pool = inputs.rows_normal(703, 0, 256, V, std=1.3).to(DEV)
    ref = torch.cat([bi.bi_log_softmax_cluster(pool[i:i + 1]) for i in range(256)])
    perm = inputs.permutation(704, 256).to(DEV)
    for M in (1, 2, 3, 8, 64, 77, 128, 256):
        for start in (0, 256 - M):
            idx = perm[start:start + M]
            assert same_bits(bi.bi_log_softmax_cluster(pool[idx]), ref[idx]), f"M={M}"
    y = torch.empty(64, V, dtype=torch.float32, device=DEV)
    first = bi.bi_log_softmax_cluster(pool[:64]).clone()
    for _ in range(100):
        assert same_bits(bi.bi_log_softmax_cluster(pool[:64], out=y), first)


def test_cluster_refuses_other_row_lengths():
    for V, dt in ((32760, torch.bfloat16), (196616, torch.bfloat16), (1000, torch.bfloat16),
                  (98312, torch.float32), (16380, torch.float32), (32770, torch.float32)):
        x = torch.zeros(2, V, dtype=dt, device=DEV)
        y = torch.zeros(2, V, dtype=torch.float32, device=DEV)
        with pytest.raises(bi.BiError) as e:
            bi.bi_log_softmax_cluster(x, out=y)
        assert e.value.status == bi.BI_ERR_UNSUPPORTED, V
    assert bi.bi_log_softmax_cluster(torch.empty(0, 151936, dtype=torch.bfloat16, device=DEV)).shape == (0, 151936)
