"""bi_decode_attention through the C ABI: parity with the fp64 oracle, and batch invariance.

A sequence's output must be bit-identical whether it is decoded alone or inside batches of
other sequences of other lengths, at any position, whatever the cache's Lmax stride.
"""
import numpy as np
import pytest
import torch

from bi_testutil import assert_bf16_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


def make(seed, B, Hq, Hkv, Lmax, d=D):
    q = inputs.rows_normal(seed, 0, B * Hq, d).view(B, Hq, d)
    k = inputs.rows_normal(seed + 1, 0, B * Lmax * Hkv, d).view(B, Lmax, Hkv, d)
    v = inputs.rows_normal(seed + 2, 0, B * Lmax * Hkv, d).view(B, Lmax, Hkv, d)
    return q, k, v


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 8), (16, 2), (8, 1)])  # group sizes 4, 1, 2, 8, 8
@pytest.mark.parametrize("lens", [[1, 128, 300], [127, 129, 256, 257], [5], [511, 512, 513, 1100]])
def test_attention_parity(Hq, Hkv, lens):
    B, Lmax = len(lens), max(lens) + 3
    q, k, v = make(800, B, Hq, Hkv, Lmax)
    sl = torch.tensor(lens, dtype=torch.int32)
    o = bi.bi_decode_attention(q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV))
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), D ** -0.5)
    assert_bf16_close(o, ref, f"attention Hq={Hq} Hkv={Hkv} lens={lens}")
    assert bi.bi_get_device_status() == bi.BI_OK


def test_attention_batch_beyond_the_cached_lengths():
    """The kernel keeps the first 4096 sequence lengths in shared memory and reads the others from
    global memory: a batch of 5000 short sequences of mixed lengths checks both paths against the
    oracle, and a sequence past the cache gives the same bits as when it is decoded alone."""
    B, Hq, Hkv, Lmax = 5000, 1, 1, 3
    q, k, v = make(806, B, Hq, Hkv, Lmax)
    sl = torch.tensor([1 + (i * 7) % Lmax for i in range(B)], dtype=torch.int32)
    qd, kd, vd, ld = q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV)
    o = bi.bi_decode_attention(qd, kd, vd, ld)
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), D ** -0.5)
    assert_bf16_close(o, ref, "attention B=5000")
    for i in (0, 4095, 4096, 4999):
        alone = bi.bi_decode_attention(qd[i:i + 1], kd[i:i + 1], vd[i:i + 1], ld[i:i + 1])
        assert same_bits(alone, o[i:i + 1]), f"sequence {i}"
    assert bi.bi_get_device_status() == bi.BI_OK


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 2), (8, 8)])
@pytest.mark.parametrize("lens", [[1, 128, 300], [511, 512, 513, 1100]])
def test_attention_parity_head_size_64(Hq, Hkv, lens):
    """Head size 64 (one 64-wide TMA box per tile) against the oracle, at stage and split edges."""
    B, Lmax = len(lens), max(lens) + 3
    q, k, v = make(830, B, Hq, Hkv, Lmax, d=64)
    sl = torch.tensor(lens, dtype=torch.int32)
    o = bi.bi_decode_attention(q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV))
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), 64 ** -0.5)
    assert_bf16_close(o, ref, f"attention D=64 Hq={Hq} Hkv={Hkv} lens={lens}")
    assert bi.bi_get_device_status() == bi.BI_OK


def test_attention_head_size_64_invariance_and_repeats():
    P, Hq, Hkv, Lmax = 24, 16, 4, 1100
    q, k, v = make(831, P, Hq, Hkv, Lmax, d=64)
    lens = torch.tensor(inputs.batch_sizes(832, P, 1, Lmax), dtype=torch.int32)
    qd, kd, vd, ld = q.to(DEV), k.to(DEV), v.to(DEV), lens.to(DEV)
    ref = torch.cat([bi.bi_decode_attention(qd[i:i + 1], kd[i:i + 1], vd[i:i + 1], ld[i:i + 1]) for i in range(P)])
    for t, b in enumerate(inputs.batch_sizes(833, 10, 1, P)):
        idx = inputs.permutation(834 + t, P)[:b].to(DEV)
        assert same_bits(bi.bi_decode_attention(qd[idx], kd[idx], vd[idx], ld[idx]), ref[idx]), f"trial {t}"
    for _ in range(20):
        assert same_bits(bi.bi_decode_attention(qd, kd, vd, ld), ref)


def test_attention_long_sequences_sampled():
    B, Hq, Hkv, Lmax = 4, 32, 8, 4096
    q, k, v = make(801, B, Hq, Hkv, Lmax)
    sl = torch.tensor([4096, 1, 2049, 3000], dtype=torch.int32)
    o = bi.bi_decode_attention(q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV))
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), D ** -0.5)
    assert_bf16_close(o, ref, "attention Lmax=4096")


@pytest.mark.parametrize("d", [128, 64])
def test_attention_more_than_eight_splits(d):
    """Sequences of more than 8 splits of 512 tokens (the second launch folds them in chunks of
    weights staged in shared memory) and of exactly 8, against the oracle; each sequence alone,
    in a cache cut to its own length, gives the bits it has in the batch."""
    B, Hq, Hkv, Lmax = 3, 8, 2, 6000
    q, k, v = make(850, B, Hq, Hkv, Lmax, d=d)
    sl = torch.tensor([6000, 4097, 4096], dtype=torch.int32)
    qd, kd, vd, ld = q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV)
    o = bi.bi_decode_attention(qd, kd, vd, ld)
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), d ** -0.5)
    assert_bf16_close(o, ref, f"attention D={d} lens={sl.tolist()}")
    for i in range(B):
        alone = bi.bi_decode_attention(qd[i:i + 1], kd[i:i + 1, :int(sl[i])].contiguous(),
                                       vd[i:i + 1, :int(sl[i])].contiguous(), ld[i:i + 1])
        assert same_bits(alone, o[i:i + 1]), f"sequence {i}"
    assert bi.bi_get_device_status() == bi.BI_OK


@pytest.mark.parametrize("d", [128, 64])
def test_attention_one_split_caches_fold_in_launch_one(d):
    """With Lmax <= 512 every sequence is one split and launch 1 writes the output itself; the same
    sequences in a cache of Lmax = 600 take the combine launch.  The bits agree, and both match
    the oracle."""
    B, Hq, Hkv = 5, 16, 4
    lens = [500, 1, 129, 256, 417]
    q, k, v = make(860, B, Hq, Hkv, 600, d=d)
    sl = torch.tensor(lens, dtype=torch.int32)
    qd, ld = q.to(DEV), sl.to(DEV)
    two = bi.bi_decode_attention(qd, k.to(DEV), v.to(DEV), ld)
    one = bi.bi_decode_attention(qd, k[:, :500].contiguous().to(DEV), v[:, :500].contiguous().to(DEV), ld)
    assert same_bits(one, two)
    ref = oracle.decode_attention(bf16_bits_np(q), bf16_bits_np(k), bf16_bits_np(v), sl.numpy(), d ** -0.5)
    assert_bf16_close(one, ref, f"attention D={d} Lmax=500")
    assert bi.bi_get_device_status() == bi.BI_OK


def test_attention_batch_invariance_over_compositions():
    P, Hq, Hkv, Lmax = 48, 32, 8, 1024
    q, k, v = make(802, P, Hq, Hkv, Lmax)
    lens = torch.tensor(inputs.batch_sizes(803, P, 1, Lmax), dtype=torch.int32)
    qd, kd, vd, ld = q.to(DEV), k.to(DEV), v.to(DEV), lens.to(DEV)
    ref = torch.cat([bi.bi_decode_attention(qd[i:i + 1], kd[i:i + 1], vd[i:i + 1], ld[i:i + 1]) for i in range(P)])
    for t, b in enumerate(inputs.batch_sizes(804, 20, 1, P)):
        idx = inputs.permutation(805 + t, P)[:b].to(DEV)
        lmax = int(lens[idx.cpu()].max())
        # a batch's cache may be allocated with a smaller Lmax: the stride changes, the bits may not
        kk = kd[idx][:, :lmax].contiguous()
        vv = vd[idx][:, :lmax].contiguous()
        o = bi.bi_decode_attention(qd[idx], kk, vv, ld[idx])
        assert same_bits(o, ref[idx]), f"trial {t}: batch of {b} changed a sequence's output"


def test_attention_ignores_cache_contents_past_each_length():
    """Cache rows past a sequence's length may hold anything (a reused buffer, NaN or infinity
    bit patterns); the output must not change by a bit."""
    B, Hq, Hkv, Lmax = 4, 32, 8, 300
    q, k, v = make(809, B, Hq, Hkv, Lmax)
    lens = [1, 130, 255, 300]
    sl = torch.tensor(lens, dtype=torch.int32).to(DEV)
    clean = bi.bi_decode_attention(q.to(DEV), k.to(DEV), v.to(DEV), sl)
    k2, v2 = k.clone(), v.clone()
    for b, L in enumerate(lens):
        k2[b, L:] = float("nan")
        v2[b, L:] = float("inf") if b % 2 else float("nan")
    dirty = bi.bi_decode_attention(q.to(DEV), k2.to(DEV), v2.to(DEV), sl)
    assert same_bits(clean, dirty)


def test_attention_repeatable_100_runs():
    B, Hq, Hkv, Lmax = 16, 32, 8, 700
    q, k, v = make(806, B, Hq, Hkv, Lmax)
    sl = torch.tensor(inputs.batch_sizes(807, B, 1, Lmax), dtype=torch.int32).to(DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    scratch = torch.empty(bi.bi_decode_attention_scratch_bytes(B, Hq, D, Lmax), dtype=torch.uint8, device=DEV)
    first = bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch)
    for _ in range(100):
        assert same_bits(bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch), first)


def test_attention_scratch_contents_do_not_matter():
    """The splits' partial results live in caller scratch of any contents: random bytes, all
    ones, or 64-bit words with the top bit set give the bits of a zeroed scratch, also on a
    second call over what the first one left."""
    B, Hq, Hkv, Lmax = 6, 16, 4, 2600
    q, k, v = make(840, B, Hq, Hkv, Lmax)
    sl = torch.tensor([2600, 1, 512, 513, 2047, 1500], dtype=torch.int32).to(DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    n = bi.bi_decode_attention_scratch_bytes(B, Hq, D, Lmax)
    assert n % 8 == 0
    scratch = torch.zeros(n, dtype=torch.uint8, device=DEV)
    ref = bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch)
    rng = np.random.default_rng(841)
    stale = rng.integers(0, 1 << 62, n // 8, dtype=np.uint64) | np.uint64(1 << 63)
    fills = [rng.integers(0, 256, n, dtype=np.uint8), np.full(n, 255, dtype=np.uint8), stale.view(np.uint8)]
    for i, f in enumerate(fills):
        scratch.copy_(torch.from_numpy(f).to(DEV))
        assert same_bits(bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch), ref), f"fill {i}"
        assert same_bits(bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch), ref), f"fill {i}, again"
    assert bi.bi_get_device_status() == bi.BI_OK


def test_attention_replayed_from_a_cuda_graph():
    """Both launches of a call (the second dependent on the first through programmatic
    dependent launch) capture into a CUDA graph; new query rows before each replay give the
    bits of an eager call."""
    B, Hq, Hkv, Lmax = 8, 16, 4, 1500
    q, k, v = make(842, B, Hq, Hkv, Lmax)
    sl = torch.tensor(inputs.batch_sizes(843, B, 1, Lmax), dtype=torch.int32).to(DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    scratch = torch.empty(bi.bi_decode_attention_scratch_bytes(B, Hq, D, Lmax), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(qd)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch, out=out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        bi.bi_decode_attention(qd, kd, vd, sl, scratch=scratch, out=out)
    for t in range(6):
        qd.copy_(inputs.rows_normal(844 + t, 0, B * Hq, D).view(B, Hq, D).to(DEV))
        graph.replay()
        eager = bi.bi_decode_attention(qd, kd, vd, sl)
        assert same_bits(out, eager), f"replay {t}"
    del graph
    assert bi.bi_get_device_status() == bi.BI_OK


def test_attention_bad_lengths_are_reported():
    B, Hq, Hkv, Lmax = 2, 8, 2, 64
    q, k, v = make(808, B, Hq, Hkv, Lmax)
    sl = torch.tensor([0, 99], dtype=torch.int32, device=DEV)
    assert bi.bi_get_device_status() == bi.BI_OK
    bi.bi_decode_attention(q.to(DEV), k.to(DEV), v.to(DEV), sl)
    assert bi.bi_get_device_status() == bi.BI_ERR_INVALID_ARG


def test_attention_argument_errors():
    q = torch.zeros(2, 8, 96, dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros(2, 16, 2, 96, dtype=torch.bfloat16, device=DEV)
    sl = torch.ones(2, dtype=torch.int32, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_decode_attention(q, kv, kv, sl)  # D = 96: head sizes 64 and 128 are built
    assert e.value.status == bi.BI_ERR_UNSUPPORTED
    q = torch.zeros(2, 6, D, dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros(2, 16, 4, D, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_decode_attention(q, kv, kv, sl)  # 6 query heads over 4 kv heads
    assert e.value.status == bi.BI_ERR_INVALID_ARG
    q = torch.zeros(2, 8, D, dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros(2, 16, 2, D, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_decode_attention(q, kv, kv, sl, scratch=torch.empty(16, dtype=torch.uint8, device=DEV))
    assert e.value.status == bi.BI_ERR_INVALID_ARG
