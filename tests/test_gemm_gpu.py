"""GPU parity and batch-invariance tests of bi_matmul / bi_addmm, through the C ABI.

Parity: against the fp64 oracle (full outputs at tiny and ragged sizes, sampled
rows at the Qwen3-8B-shaped sizes), plus exact cases -- integer inputs whose fp32
sums are exact, and the identity -- that must match bit for bit.  Invariance: every
row of batches M = 1..2048, at any position, equals its M = 1 result bit for bit,
and 100 repeated runs agree.
"""
import numpy as np
import pytest
import torch

from bi_testutil import M_SWEEP, assert_bf16_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def weight(seed, N, K, layout, std=0.02):
    w = inputs.weight_normal(seed, (N, K), std=std)  # stored [N, K]
    return w if layout == "nk" else w.t().contiguous()


def wbits(w):
    return bf16_bits_np(w)


def abs_bits(bits):
    return bits & np.uint16(0x7FFF)  # |x| of a bf16 bit pattern: clear the sign bit


def assert_f32_close(gpu, ref, what, a_bits, b_bits, layout):
    """fp32-output bound: K/16 sequential fp32 additions of 16-product tensor-core steps
    (at most 16 roundings inside a step), each at most 2^-23 of the running |A||B| sum,
    plus the final rounding: |err| <= (K/16 + 16) 2^-23 (|A||B|)_ij + 2^-24 |ref_ij|."""
    g = gpu.detach().cpu().double().numpy()
    K = a_bits.shape[1]
    absprod = oracle.matmul(abs_bits(a_bits), abs_bits(b_bits), layout)
    bound = (K / 16 + 16) * 2.0 ** -23 * absprod + 2.0 ** -24 * np.abs(ref)
    err = np.abs(g - ref)
    assert np.all(err <= bound), f"{what}: worst excess {float((err - bound).max())}"


# ----------------------------------------------------------------------------- tiny config

@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("M", [1, 3, 8, 17])
def test_tiny_matmul_parity(M, layout):
    K, N = 256, 512
    a = inputs.rows_normal(200, 0, M, K)
    b = weight(201, N, K, layout)
    c = bi.bi_matmul(a.to(DEV), b.to(DEV), layout)
    ref = oracle.matmul(bf16_bits_np(a), wbits(b), layout)
    assert_bf16_close(c, ref, f"tiny matmul M={M} {layout}")
    c32 = bi.bi_matmul(a.to(DEV), b.to(DEV), layout, out_dtype=torch.float32)
    assert_f32_close(c32, ref, f"tiny matmul fp32 out M={M} {layout}", bf16_bits_np(a), wbits(b), layout)


@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("K", [256, 4096])
def test_integer_matmul_is_exact(K, layout):
    M, N = 37, 520
    a = inputs.rows_int(202, 0, M, K)
    w = inputs.weight_int(203, (N, K))
    b = w if layout == "nk" else w.t().contiguous()
    c = bi.bi_matmul(a.to(DEV), b.to(DEV), layout).cpu()
    exact = a.double().numpy().astype(np.int64) @ w.double().numpy().astype(np.int64).T
    assert np.array_equal(oracle.matmul(bf16_bits_np(a), wbits(b), layout), exact.astype(np.float64))
    expect = torch.from_numpy(exact.astype(np.float64)).to(torch.bfloat16)  # one RNE rounding
    assert same_bits(c, expect)
    c32 = bi.bi_matmul(a.to(DEV), b.to(DEV), layout, out_dtype=torch.float32).cpu()
    assert np.array_equal(c32.double().numpy(), exact.astype(np.float64))


@pytest.mark.parametrize("layout", ["kn", "nk"])
def test_identity_returns_a(layout):
    M, K = 300, 512
    a = inputs.rows_normal(204, 0, M, K).to(DEV)
    eye = torch.eye(K, dtype=torch.bfloat16, device=DEV)
    assert same_bits(bi.bi_matmul(a, eye, layout), a)


@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (129, 136, 40), (300, 520, 72), (5, 1000, 1000),
                                   (130, 264, 4104), (2, 8, 24), (257, 1032, 200)])
def test_ragged_shapes_parity(M, N, K, layout):
    a = inputs.rows_normal(205, 0, M, K)
    b = weight(206, N, K, layout, std=0.05)
    c = bi.bi_matmul(a.to(DEV), b.to(DEV), layout)
    assert_bf16_close(c, oracle.matmul(bf16_bits_np(a), wbits(b), layout), f"{M}x{N}x{K} {layout}")


@pytest.mark.parametrize("layout", ["kn", "nk"])
def test_leading_dimensions(layout):
    M, N, K = 70, 136, 96
    a_big = inputs.rows_normal(207, 0, M, K + 24).to(DEV)
    a = a_big[:, 8:8 + K]
    b_full = weight(208, N + 16, K + 16, "nk").to(DEV)  # [N+16, K+16]
    b = b_full[:N, :K] if layout == "nk" else b_full.t()[:K, :N]
    if layout == "kn":
        b = b.contiguous()
        b_big = torch.zeros(K, N + 40, dtype=torch.bfloat16, device=DEV)
        b_big[:, :N] = b
        b = b_big[:, :N]
    c_big = torch.full((M, N + 8), 7.0, dtype=torch.bfloat16, device=DEV)
    c = c_big[:, :N]
    bi.bi_matmul(a, b, layout, out=c)
    ref = oracle.matmul(bf16_bits_np(a.cpu().contiguous()), wbits(b.cpu().contiguous()), layout)
    assert_bf16_close(c, ref, "strided")
    assert torch.all(c_big[:, N:] == 7.0), "wrote outside C"


# ----------------------------------------------------------------------------- addmm

@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("M", [1, 17, 300])
def test_addmm_bias_and_residual(M, layout, out_dtype):
    K, N = 256, 520
    a = inputs.rows_normal(210, 0, M, K)
    b = weight(211, N, K, layout)
    bias = inputs.bias(212, N)
    resid = inputs.rows_normal(213, 0, M, N)
    for inp, name in ((bias, "bias"), (resid, "residual")):
        c = bi.bi_addmm(inp.to(DEV), a.to(DEV), b.to(DEV), layout, out_dtype=out_dtype)
        ref = oracle.addmm(bf16_bits_np(inp), bf16_bits_np(a), wbits(b), layout)
        if out_dtype == torch.bfloat16:
            assert_bf16_close(c, ref, f"addmm {name}")
        else:
            assert_f32_close(c, ref, f"addmm {name}", bf16_bits_np(a), wbits(b), layout)


def test_addmm_zero_lhs_and_k0():
    M, N, K = 33, 264, 64
    bias = inputs.bias(214, N).to(DEV)
    resid = inputs.rows_normal(215, 0, M, N).to(DEV)
    zero = torch.zeros(M, K, dtype=torch.bfloat16, device=DEV)
    b = weight(216, N, K, "nk").to(DEV)
    assert same_bits(bi.bi_addmm(resid, zero, b), resid)
    assert same_bits(bi.bi_addmm(bias, zero, b), bias.expand(M, N).contiguous())
    a0 = torch.empty(M, 0, dtype=torch.bfloat16, device=DEV)
    b0 = torch.empty(N, 0, dtype=torch.bfloat16, device=DEV)
    assert same_bits(bi.bi_addmm(resid, a0, b0), resid)
    assert torch.count_nonzero(bi.bi_matmul(a0, b0)) == 0


def test_integer_addmm_is_exact():
    M, N, K = 19, 264, 4096
    a = inputs.rows_int(217, 0, M, K)
    w = inputs.weight_int(218, (N, K))
    r = inputs.rows_int(219, 0, M, N)
    c = bi.bi_addmm(r.to(DEV), a.to(DEV), w.to(DEV), "nk", out_dtype=torch.float32).cpu()
    exact = (a.double().numpy() @ w.double().numpy().T) + r.double().numpy()
    assert np.array_equal(c.double().numpy(), exact)


# ----------------------------------------------------------------------------- workload sizes

QWEN_SHAPES = {"q/o": (4096, 4096), "k/v": (4096, 1024), "gate/up": (4096, 12288), "down": (12288, 4096)}


@pytest.mark.parametrize("name", list(QWEN_SHAPES))
def test_qwen_shapes_sampled_rows(name):
    K, N = QWEN_SHAPES[name]
    M = 2048
    a = inputs.rows_normal(220, 0, M, K)
    w = weight(221, N, K, "nk")
    bias = inputs.bias(222, N)
    ad, wd, bd = a.to(DEV), w.to(DEV), bias.to(DEV)
    c = bi.bi_matmul(ad, wd, "nk").cpu()
    cb = bi.bi_addmm(bd, ad, wd, "nk").cpu()
    rows = torch.tensor([0, 127, 128, 1000, M - 1])
    ref = oracle.matmul(bf16_bits_np(a[rows]), wbits(w), "nk")
    assert_bf16_close(c[rows], ref, f"{name} M=2048 sampled")
    assert_bf16_close(cb[rows], ref + bias.double().numpy()[None, :], f"{name} addmm sampled")


def test_lm_head_sampled_rows():
    K, N, M = 4096, 151936, 64
    a = inputs.rows_normal(223, 0, M, K)
    w = weight(224, N, K, "nk")
    c = bi.bi_matmul(a.to(DEV), w.to(DEV), "nk").cpu()
    rows = torch.tensor([0, 31, M - 1])
    assert_bf16_close(c[rows], oracle.matmul(bf16_bits_np(a[rows]), wbits(w), "nk"), "lm head")


# ----------------------------------------------------------------------------- invariance

@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("name", ["q/o", "k/v"])
def test_batch_invariance_sweep(name, layout):
    K, N = QWEN_SHAPES[name]
    pool = inputs.rows_normal(230, 0, 2048, K).to(DEV)
    w = weight(231, N, K, layout).to(DEV)
    ref = torch.cat([bi.bi_matmul(pool[i:i + 1], w, layout) for i in range(2048)])
    perm = inputs.permutation(232, 2048).to(DEV)
    for M in M_SWEEP:
        for start in (0, 2048 - M, (2048 - M) // 2):
            idx = perm[start:start + M]
            out = bi.bi_matmul(pool[idx], w, layout)
            assert same_bits(out, ref[idx]), f"{name} {layout} M={M}: a row differs from M=1"


@pytest.mark.parametrize("K,N", [(4096, 12288), (4096, 24576), (12288, 4096)])
def test_batch_invariance_sweep_wide_and_deep(K, N):
    """gate/up (N = 12288, and the fused [gate; up] N = 24576) and down (K = 12288) over the
    whole M sweep up to 2048: every row of every batch, at every position of three windows of
    a random permutation of the pool, equals the same row computed alone, bit for bit."""
    pool = inputs.rows_normal(238, 0, 2048, K).to(DEV)
    w = weight(239, N, K, "nk").to(DEV)
    ref = torch.empty(2048, N, dtype=torch.bfloat16, device=DEV)
    for i in range(2048):
        bi.bi_matmul(pool[i:i + 1], w, "nk", out=ref[i:i + 1])
    perm = inputs.permutation(240, 2048).to(DEV)
    for M in M_SWEEP:
        for start in (0, 2048 - M, (2048 - M) // 2):
            idx = perm[start:start + M]
            out = bi.bi_matmul(pool[idx], w, "nk")
            assert same_bits(out, ref[idx]), f"K={K} N={N} M={M}: a row differs from M=1"


@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("K", [4096, 4104])
def test_tile_width_does_not_change_bits(K, layout):
    """Weights of up to 1024 rows run the 128-column tile with 128-deep stages, wider ones the
    192-column tile with 128-deep stages ([N, K] storage, where it needs fewer cost-weighted
    waves) or the 256-column tile with 64-deep stages.  All take the same 16-wide K steps in
    ascending order, so the first 1024 columns of a 1280-column product equal, bit for bit, the
    product with only those 1024 weight rows (narrow tile) -- for plain, bias and fused SiLU * up
    outputs, at ragged M and K."""
    assert bi.bi_gemm_config(1024)["bn"] != bi.bi_gemm_config(1280)["bn"]
    w = weight(250, 1280, K, "nk").to(DEV)
    gate, up = w, weight(251, 1280, K, "nk").to(DEV)
    bias = inputs.bias(252, 1280).to(DEV)
    wk = w if layout == "nk" else w.t().contiguous()
    for M in (1, 77, 300):
        a = inputs.rows_normal(253, 0, M, K).to(DEV)
        wide = bi.bi_matmul(a, wk, layout)
        narrow = bi.bi_matmul(a, wk[:1024] if layout == "nk" else wk[:, :1024], layout)
        assert same_bits(wide[:, :1024], narrow), f"matmul M={M} K={K} {layout}"
        wide_b = bi.bi_addmm(bias, a, wk, layout)
        narrow_b = bi.bi_addmm(bias[:1024], a, wk[:1024] if layout == "nk" else wk[:, :1024], layout)
        assert same_bits(wide_b[:, :1024], narrow_b), f"addmm M={M} K={K} {layout}"
        gu_wide = torch.cat([gate, up])
        gu_narrow = torch.cat([gate[:1024], up[:1024]])
        if layout == "kn":
            gu_wide, gu_narrow = gu_wide.t().contiguous(), gu_narrow.t().contiguous()
        h_wide = bi.bi_matmul_silu_mul(a, gu_wide, layout)
        h_narrow = bi.bi_matmul_silu_mul(a, gu_narrow, layout)
        assert same_bits(h_wide[:, :1024], h_narrow), f"fused M={M} K={K} {layout}"


@pytest.mark.parametrize("K", [4096, 1000])
def test_mid_tile_matches_wide_tile_bits(K):
    """A 6144-row weight (the fused q/k/v projection) stored [N, K] runs the 192-column tile; the
    same weight stored [K, N] runs the 256-column tile.  Plain, bias and fused SiLU * up products
    agree bit for bit at ragged M, up to 1024 rows (where the tiles' wave counts differ)."""
    assert bi.bi_gemm_config(6144)["bn"] == 192 and bi.bi_gemm_config(0)["bn"] == 256
    w = weight(260, 6144, K, "nk").to(DEV)
    wt = w.t().contiguous()
    bias = inputs.bias(261, 6144).to(DEV)
    for M in (1, 77, 300, 1024):
        a = inputs.rows_normal(262, 0, M, K).to(DEV)
        assert same_bits(bi.bi_matmul(a, w, "nk"), bi.bi_matmul(a, wt, "kn")), f"matmul M={M} K={K}"
        assert same_bits(bi.bi_matmul(a, w, "nk", out_dtype=torch.float32),
                         bi.bi_matmul(a, wt, "kn", out_dtype=torch.float32)), f"matmul fp32 M={M} K={K}"
        assert same_bits(bi.bi_addmm(bias, a, w, "nk"), bi.bi_addmm(bias, a, wt, "kn")), f"addmm M={M} K={K}"
        assert same_bits(bi.bi_matmul_silu_mul(a, w, "nk"), bi.bi_matmul_silu_mul(a, wt, "kn")), \
            f"fused M={M} K={K}"
    assert bi.bi_get_device_status() == bi.BI_OK


def test_lm_head_logits_invariance():
    """LM-head logits [M, 151936] at M in {1, 8, 64, 256, 1024}: each row equals the row
    computed alone, bit for bit, at every position of two windows of a permutation."""
    K, N, P = 4096, 151936, 1024
    pool = inputs.rows_normal(241, 0, P, K).to(DEV)
    w = weight(242, N, K, "nk").to(DEV)
    ref = torch.empty(P, N, dtype=torch.bfloat16, device=DEV)
    for i in range(P):
        bi.bi_matmul(pool[i:i + 1], w, "nk", out=ref[i:i + 1])
    perm = inputs.permutation(243, P).to(DEV)
    for M in (1, 8, 64, 256, 1024):
        for start in (0, P - M):
            idx = perm[start:start + M]
            assert same_bits(bi.bi_matmul(pool[idx], w, "nk"), ref[idx]), f"LM head M={M}"


def test_addmm_repeatable_100_runs():
    K, N, M = 4096, 4096, 2048
    a = inputs.rows_normal(244, 0, M, K).to(DEV)
    w = weight(245, N, K, "nk").to(DEV)
    bias = inputs.bias(246, N).to(DEV)
    resid = inputs.rows_normal(247, 0, M, N).to(DEV)
    first_b = bi.bi_addmm(bias, a, w)
    first_r = bi.bi_addmm(resid, a, w)
    for _ in range(100):
        assert same_bits(bi.bi_addmm(bias, a, w), first_b)
        assert same_bits(bi.bi_addmm(resid, a, w), first_r)


def test_addmm_residual_invariance_positions():
    K, N = 12288, 4096
    pool = inputs.rows_normal(233, 0, 512, K).to(DEV)
    resid = inputs.rows_normal(234, 0, 512, N).to(DEV)
    w = weight(235, N, K, "nk").to(DEV)
    ref = torch.cat([bi.bi_addmm(resid[i:i + 1], pool[i:i + 1], w) for i in range(512)])
    for M in (2, 3, 77, 128, 129, 256, 512):
        for r in (0, 127, 128, 255, 256, M - 1):
            if r >= M:
                continue
            idx = torch.arange(M, device=DEV)
            # put pool row `M + 3 - r` (any fixed row) at position r
            target = (M + 3) % 512
            idx[r] = target
            out = bi.bi_addmm(resid[idx], pool[idx], w)
            assert same_bits(out[r], ref[target]), f"M={M} position {r}"


def test_matmul_repeatable_100_runs():
    K, N, M = 4096, 4096, 2048
    a = inputs.rows_normal(236, 0, M, K).to(DEV)
    w = weight(237, N, K, "nk").to(DEV)
    first = bi.bi_matmul(a, w)
    for _ in range(100):
        assert same_bits(bi.bi_matmul(a, w), first)


def test_tensor_map_cache_hits_on_repeated_calls():
    """A repeated call with the same buffers is served two tensor maps from the cache; a new
    activation buffer is one miss (its map) and one hit (the weights' map); results agree."""
    a = inputs.rows_normal(248, 0, 4, 256).to(DEV)
    w = weight(249, 512, 256, "nk").to(DEV)
    first = bi.bi_matmul(a, w)
    h0, m0 = bi.bi_tensor_map_cache_stats()
    again = bi.bi_matmul(a, w)
    h1, m1 = bi.bi_tensor_map_cache_stats()
    assert (h1 - h0, m1 - m0) == (2, 0)
    a2 = a.clone()
    other = bi.bi_matmul(a2, w)
    h2, m2 = bi.bi_tensor_map_cache_stats()
    assert (h2 - h1, m2 - m1) == (1, 1)
    assert same_bits(first, again) and same_bits(first, other)


# ----------------------------------------------------------------------------- errors

def test_invalid_arguments_are_rejected():
    a = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        bi.bi_matmul(a, torch.zeros(64, 32, dtype=torch.bfloat16, device=DEV), "nk")
    buf = torch.zeros(4 * 64 + 8, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bi.BiError) as e:
        bi.bi_matmul(buf[1:1 + 256].view(4, 64), w, "nk")
    assert e.value.status == bi.BI_ERR_ALIGNMENT
    assert bi.bi_matmul(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV), w).shape == (0, 64)
    assert bi.bi_get_device_status() == bi.BI_OK
