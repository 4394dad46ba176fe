"""The seeded input recipe (inputs.py), on the CPU: row-keyed draws, the outlier rule, integer
mode, permutations and batch sizes."""
import numpy as np
import torch

from invariant_bi_matmul_02_b200 import inputs


def test_rows_are_keyed_by_seed_and_row():
    whole = inputs.rows_normal(5, 0, 40, 96)
    assert torch.equal(inputs.rows_normal(5, 13, 9, 96), whole[13:22])
    assert not torch.equal(inputs.rows_normal(6, 0, 40, 96), whole)
    assert whole.dtype == torch.bfloat16
    f = whole.float()
    assert abs(float(f.mean())) < 0.05 and abs(float(f.std()) - 1.0) < 0.05


def test_outliers_are_one_percent_scaled_by_fifty():
    base = inputs.rows_normal(7, 0, 200, 4096, dtype=torch.float32)
    x = inputs.with_outliers(base, 8)
    changed = x != base
    frac = float(changed.float().mean())
    assert 0.008 < frac < 0.012
    assert torch.allclose(x[changed], 50 * base[changed])
    # keyed by row as well: a slice of rows gets the same outliers
    assert torch.equal(inputs.with_outliers(base[50:60], 8, row0=50), x[50:60])


def test_integer_rows_are_small_exact_integers():
    x = inputs.rows_int(9, 0, 30, 500, dtype=torch.float32)
    v = x.numpy()
    assert np.array_equal(v, np.round(v)) and v.min() >= -4 and v.max() <= 4
    assert len(np.unique(v)) == 9
    assert torch.equal(inputs.rows_int(9, 10, 5, 500, dtype=torch.float32), x[10:15])


def test_weights_gain_and_bias_have_the_stated_spread():
    w = inputs.weight_normal(1, (512, 256)).float()
    assert abs(float(w.std()) - 0.02) < 0.002
    g = inputs.gain(2, 4096).float()
    assert abs(float(g.mean()) - 1.0) < 0.01 and abs(float(g.std()) - 0.1) < 0.01
    b = inputs.bias(3, 4096).float()
    assert abs(float(b.std()) - 0.01) < 0.001


def test_permutations_and_batch_sizes():
    p = inputs.permutation(4, 2048)
    assert torch.equal(torch.sort(p).values, torch.arange(2048))
    assert torch.equal(p, inputs.permutation(4, 2048))
    sizes = inputs.batch_sizes(5, 100, 1, 512)
    assert len(sizes) == 100 and min(sizes) >= 1 and max(sizes) <= 512
    assert sizes == inputs.batch_sizes(5, 100, 1, 512)
