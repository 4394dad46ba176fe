"""Greedy decoding of one prompt inside many random batch compositions (the pages'
1,000-completion experiment in miniature, with a random-weight decoder): with every
reduction on libbi.so the completion must be the same in every composition.  The count for
torch's default kernels is printed for comparison, not asserted.
"""
import pytest

import bench

pytestmark = pytest.mark.gpu


def test_one_completion_across_batch_compositions():
    res = bench.uniqueness(trials=24, new_tokens=16, max_batch=48, context=2048)
    print("unique completions:", res)
    assert res["bi"]["unique"] == 1, res
    assert res["bi"]["unique_logprob_bits"] == 1, res  # every step's log-probs, bit for bit
