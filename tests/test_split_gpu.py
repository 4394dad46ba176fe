"""bi_log_softmax_split: log_softmax by many blocks per row (short batches), through the C ABI.

Parity against the fp64 oracle, bit-level batch invariance over M and row positions,
repeatability, and the scratch-size / alignment / shape errors.
"""
import pytest
import torch

from bi_testutil import assert_lsm_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("V", [8, 1000, 4096, 4104, 151936])
@pytest.mark.parametrize("M", [1, 3, 17])
def test_split_parity_bf16(M, V):
    x = inputs.rows_normal(500 + V, 0, M, V, std=1.3)
    y = bi.bi_log_softmax_split(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), f"split bf16 M={M} V={V}")


@pytest.mark.parametrize("V", [8, 1000, 8200])
def test_split_parity_fp32(V):
    x = inputs.rows_normal(501, 0, 5, V, dtype=torch.float32)
    y = bi.bi_log_softmax_split(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(x.numpy()), f"split fp32 V={V}")


def test_split_constant_and_extreme_rows():
    V = 151936
    x = torch.zeros(3, V, dtype=torch.bfloat16)
    x[1] = 3.5
    x[2, 17] = 60.0
    x[2, 18:] = -60.0
    y = bi.bi_log_softmax_split(x.to(DEV))
    assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(x)), "split constant/extreme")


def test_split_batch_invariance_and_repeatability():
    V = 151936
    pool = inputs.rows_normal(502, 0, 256, V, std=1.3).to(DEV)
    ref = torch.cat([bi.bi_log_softmax_split(pool[i:i + 1]) for i in range(256)])
    perm = inputs.permutation(503, 256).to(DEV)
    for M in (1, 2, 3, 8, 64, 77, 128, 256):
        for start in (0, 256 - M):
            idx = perm[start:start + M]
            assert same_bits(bi.bi_log_softmax_split(pool[idx]), ref[idx]), f"M={M}"
    scratch = torch.empty(bi.bi_log_softmax_split_scratch_bytes(64, V), dtype=torch.uint8, device=DEV)
    first = bi.bi_log_softmax_split(pool[:64], scratch)
    for _ in range(100):
        assert same_bits(bi.bi_log_softmax_split(pool[:64], scratch), first)


def test_split_argument_errors():
    V = 1024
    x = torch.zeros(4, V, dtype=torch.bfloat16, device=DEV)
    need = bi.bi_log_softmax_split_scratch_bytes(4, V)
    assert need == 4 * 1 * 8
    with pytest.raises(bi.BiError) as e:
        bi.bi_log_softmax_split(x, torch.empty(need - 8, dtype=torch.uint8, device=DEV))
    assert e.value.status == bi.BI_ERR_INVALID_ARG
    buf = torch.empty(need + 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_log_softmax_split(x, buf[4:])
    assert e.value.status == bi.BI_ERR_ALIGNMENT
    with pytest.raises(bi.BiError) as e:
        bi.bi_log_softmax_split(torch.zeros(2, 1001, dtype=torch.bfloat16, device=DEV))
    assert e.value.status == bi.BI_ERR_UNSUPPORTED
    assert bi.bi_log_softmax_split(torch.zeros(0, V, dtype=torch.bfloat16, device=DEV)).shape == (0, V)
