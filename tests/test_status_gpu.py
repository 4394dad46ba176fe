"""The failure path of the bounded device-side waits, without a GPU fault.

A kernel waits on a barrier that nothing completes, through the same bounded wait
the GEMM's pipeline uses; the wait gives up after its limit, records BI_ERR_TIMEOUT
in the device status word and returns, and the context stays usable.
"""
import time

import pytest
import torch

from invariant_bi_matmul_02_b200 import binding as bi

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    assert bi.bi_get_device_status() == bi.BI_OK
    t0 = time.perf_counter()
    bi.bi_selftest_wait_timeout(2_000_000)  # 2 ms
    assert bi.bi_get_device_status() == bi.BI_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert bi.bi_get_device_status() == bi.BI_OK  # reading clears the word
    a = torch.ones(4, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, 64, dtype=torch.bfloat16, device="cuda")
    c = bi.bi_matmul(a, w, "nk")
    assert torch.all(c == 64)
    assert bi.bi_get_device_status() == bi.BI_OK


def test_selftest_limit_is_validated():
    with pytest.raises(bi.BiError):
        bi.bi_selftest_wait_timeout(10)
