"""bi_log_softmax_split_noalloc: the split log_softmax for callers that cannot allocate.

Some callers cannot hand the library a scratch buffer, because they cannot allocate device
memory when they call it (a fixed memory budget owned by someone else's pool, a host
framework that controls all allocation, a hot path that cannot take a cudaMalloc's
synchronisation).  This entry point keeps the split path's partials in a fixed array inside
the library instead.  The test calls it through the C ABI and checks it against the entry
point that takes caller scratch, on two calls in a row (the second one finds the first one's
partials still in the shared array), and checks that a call beyond the array's size is
refused.  The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from bi_testutil import LSM_ABS, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def call_noalloc(x, y):
    lib = bi.load()
    dt = bi.BI_BF16 if x.dtype == torch.bfloat16 else bi.BI_F32
    return lib.bi_log_softmax_split_noalloc(ctypes.c_void_p(x.data_ptr()), dt, ctypes.c_void_p(y.data_ptr()),
                                            x.shape[0], x.shape[1],
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def reference(x):
    scratch = torch.empty(bi.bi_log_softmax_split_scratch_bytes(*x.shape), dtype=torch.uint8, device=DEV)
    return bi.bi_log_softmax_split(x, scratch)


@pytest.mark.parametrize("first,second", [
    ((5, 151936, torch.bfloat16), (33, 4096, torch.float32)),
    ((1724, 151936, torch.bfloat16), (2, 1000, torch.bfloat16)),
    ((2, 1000, torch.bfloat16), (1724, 151936, torch.bfloat16)),  # the second call writes more partials
])
def test_noalloc_matches_scratch_entry_point_on_two_calls(first, second):
    for seed, (M, V, dt) in enumerate((first, second)):
        x = inputs.rows_normal(600 + seed, 0, M, V, std=1.3, dtype=dt).to(DEV)
        y = torch.full((M, V), float("nan"), dtype=torch.float32, device=DEV)
        assert call_noalloc(x, y) == bi.BI_OK
        ref = reference(x)
        torch.cuda.synchronize()
        assert float((y - ref).abs().max()) <= LSM_ABS
        assert same_bits(y, ref)


def test_noalloc_python_wrapper():
    """The binding's wrapper passes its arguments in the C function's order and checks the
    output's shape before it calls anything."""
    x = inputs.rows_normal(610, 0, 9, 151936, std=1.3).to(DEV)
    y = torch.empty(9, 151936, dtype=torch.float32, device=DEV)
    for _ in range(2):
        assert bi.bi_log_softmax_split_noalloc(x, y) is y
        assert same_bits(y, reference(x))
    with pytest.raises(ValueError):
        bi.bi_log_softmax_split_noalloc(x, torch.empty(9, 151928, dtype=torch.float32, device=DEV))


def test_noalloc_refuses_sizes_beyond_its_array():
    V = 151936
    M = 1725  # 1725 rows x 38 chunks of 4096 = 65550 partials > 65536
    x = torch.zeros(M, V, dtype=torch.bfloat16, device=DEV)
    y = torch.zeros(M, V, dtype=torch.float32, device=DEV)
    assert call_noalloc(x, y) == bi.BI_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0  # nothing was launched
