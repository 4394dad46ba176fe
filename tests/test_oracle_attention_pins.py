"""Pins of the oracle's decode attention against closed forms and invariants.

Single-token sequences return their value row exactly; identical keys give the mean of the
values; a dominant score picks its value row; the output is linear in V and a convex
combination of the value rows; permuting the (key, value) pairs changes nothing; each query
head reads the kv head of its group.  A transposed or misindexed cache fails one of these.
"""
import math

import numpy as np
import torch

from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle


def bits(t):
    return inputs.bf16_bits(t)


def rand_cache(seed, B, L, Hkv, D):
    k = inputs.rows_normal(seed, 0, B * L * Hkv, D).view(B, L, Hkv, D)
    v = inputs.rows_normal(seed + 1, 0, B * L * Hkv, D).view(B, L, Hkv, D)
    return k, v


def test_single_token_returns_its_value_row():
    B, Hq, Hkv, D, L = 2, 8, 2, 16, 5
    q = inputs.rows_normal(700, 0, B * Hq, D).view(B, Hq, D)
    k, v = rand_cache(701, B, L, Hkv, D)
    o = oracle.decode_attention(bits(q), bits(k), bits(v), [1, 1], 1 / math.sqrt(D))
    for b in range(B):
        for h in range(Hq):
            assert np.array_equal(o[b, h], v[b, 0, h // (Hq // Hkv)].double().numpy())


def test_equal_keys_average_the_values_and_zero_scale_too():
    B, Hq, Hkv, D, L = 1, 4, 1, 8, 7
    q = inputs.rows_normal(702, 0, Hq, D).view(B, Hq, D)
    k = inputs.rows_normal(703, 0, 1, D).view(1, 1, 1, D).expand(B, L, Hkv, D).contiguous()
    _, v = rand_cache(704, B, L, Hkv, D)
    mean_v = v[0, :, 0].double().mean(0).numpy()
    o = oracle.decode_attention(bits(q), bits(k), bits(v), [L], 0.37)
    assert np.allclose(o[0], mean_v[None, :], rtol=0, atol=1e-14)
    k2, _ = rand_cache(705, B, L, Hkv, D)
    o0 = oracle.decode_attention(bits(q), bits(k2), bits(v), [L], 0.0)
    assert np.allclose(o0[0], mean_v[None, :], rtol=0, atol=1e-14)


def test_dominant_score_picks_its_row_and_outputs_are_convex():
    B, Hq, Hkv, D, L = 1, 2, 1, 8, 9
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16)
    q[:, :, 0] = 1.0
    k = torch.zeros(B, L, Hkv, D, dtype=torch.bfloat16)
    k[0, 6, 0, 0] = 64.0  # score 64 against 0: weight ratio e^-64
    _, v = rand_cache(706, B, L, Hkv, D)
    o = oracle.decode_attention(bits(q), bits(k), bits(v), [L], 1.0)
    assert np.allclose(o[0, 0], v[0, 6, 0].double().numpy(), rtol=0, atol=1e-25)
    q2 = inputs.rows_normal(707, 0, Hq, D).view(B, Hq, D)
    k2, v2 = rand_cache(708, B, L, Hkv, D)
    o2 = oracle.decode_attention(bits(q2), bits(k2), bits(v2), [L], 0.5)
    vv = v2[0, :, 0].double().numpy()
    assert np.all(o2[0] <= vv.max(0) + 1e-15) and np.all(o2[0] >= vv.min(0) - 1e-15)


def test_linear_in_values_and_permutation_invariant():
    B, Hq, Hkv, D, L = 1, 4, 2, 8, 11
    q = inputs.rows_normal(709, 0, Hq, D).view(B, Hq, D)
    k, _ = rand_cache(710, B, L, Hkv, D)
    v1 = inputs.rows_int(711, 0, B * L * Hkv, D).view(B, L, Hkv, D)
    v2 = inputs.rows_int(712, 0, B * L * Hkv, D).view(B, L, Hkv, D)
    vs = (v1.double() + v2.double()).to(torch.bfloat16)  # small integers: the sum is exact in bf16
    assert torch.equal(vs.double(), v1.double() + v2.double())
    s = 1 / math.sqrt(D)
    a = oracle.decode_attention(bits(q), bits(k), bits(v1), [L], s)
    b = oracle.decode_attention(bits(q), bits(k), bits(v2), [L], s)
    c = oracle.decode_attention(bits(q), bits(k), bits(vs), [L], s)
    assert np.allclose(c, a + b, rtol=1e-13, atol=1e-13)
    perm = torch.randperm(L, generator=torch.Generator().manual_seed(0))
    ap = oracle.decode_attention(bits(q), bits(k[:, perm].contiguous()), bits(v1[:, perm].contiguous()), [L], s)
    assert np.allclose(ap, a, rtol=1e-13, atol=1e-13)


def test_each_query_head_reads_its_group_kv_head():
    B, Hq, Hkv, D, L = 1, 8, 4, 8, 3
    q = inputs.rows_normal(713, 0, Hq, D).view(B, Hq, D)
    k, _ = rand_cache(714, B, L, Hkv, D)
    v = torch.zeros(B, L, Hkv, D, dtype=torch.bfloat16)
    for g in range(Hkv):
        v[0, :, g] = float(g + 1)  # kv head g's values are the constant g + 1
    o = oracle.decode_attention(bits(q), bits(k), bits(v), [L], 1.0)
    for h in range(Hq):
        assert np.allclose(o[0, h], h // (Hq // Hkv) + 1, rtol=0, atol=1e-14)


def test_lengths_are_respected():
    B, Hq, Hkv, D, Lmax = 2, 2, 1, 8, 6
    q = inputs.rows_normal(715, 0, B * Hq, D).view(B, Hq, D)
    k, v = rand_cache(716, B, Lmax, Hkv, D)
    full = oracle.decode_attention(bits(q), bits(k[:, :3].contiguous()), bits(v[:, :3].contiguous()), [3, 3],
                                   0.5)
    part = oracle.decode_attention(bits(q), bits(k), bits(v), [3, 3], 0.5)
    assert np.array_equal(full, part)
