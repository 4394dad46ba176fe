"""bi_matmul_lse + bi_log_softmax_partials: the LM-head log_softmax split between the GEMM
epilogue (one (max, sum of exp) pair per row and 256-column tile) and one streaming pass.

Through the C ABI: the logits are bit-identical to bi_matmul's; every pair matches the fp64
oracle's per-tile statistics of those logits (max exactly, sum to fp32 rounding); y matches
the oracle's log_softmax of the same logits; and logits, pairs and y are bit-level
batch-invariant over M, row positions and repeated calls.
"""
import numpy as np
import pytest
import torch

from bi_testutil import M_SWEEP, assert_lsm_close, bf16_bits_np, same_bits, to_np64
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
TILE = 256
# fp32 sum of at most 256 terms in [0, 1], each exp with a few ulp of error: relative 2e-5.
SUM_REL = 2e-5


def weight(seed, N, K, layout):
    """On the device: [N, K] ('nk'), or [K, N] ('kn') in a buffer whose rows are padded to 16
    bytes (built there, because copying a strided view to the device would drop the padding)."""
    w = inputs.weight_normal(seed, (N, K)).to(DEV)
    if layout == "nk":
        return w
    kn = torch.zeros(K, -(-N // 8) * 8, dtype=w.dtype, device=DEV)
    kn[:, :N] = w.t()
    return kn[:, :N]


def c_buf(M, N, dtype=torch.bfloat16):
    """[M, N] view of a buffer whose rows are padded to a multiple of 8 columns (16-byte rows)."""
    return torch.empty(M, -(-N // 8) * 8, dtype=dtype, device=DEV)[:, :N]


def check_partials(logits: torch.Tensor, part: torch.Tensor, what: str):
    m_ref, s_ref = oracle.tile_max_sumexp(bf16_bits_np(logits.cpu()), TILE)
    p = to_np64(part)
    assert p.shape == (*m_ref.shape, 2), what
    assert np.array_equal(p[..., 0], m_ref), f"{what}: a tile max differs"
    err = np.abs(p[..., 1] - s_ref) / s_ref
    assert float(err.max()) <= SUM_REL, f"{what}: tile sum rel err {float(err.max())}"


@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("M,N,K", [(1, 1000, 256), (3, 151936, 512), (129, 1000, 1000), (300, 257, 72),
                                   (2, 8, 24), (257, 4104, 136), (17, 32000, 4096)])
def test_lse_parity(M, N, K, layout):
    a = inputs.rows_normal(900, 0, M, K)
    w = weight(901, N, K, layout)
    ad, wd = a.to(DEV), w
    lg, part = bi.bi_matmul_lse(ad, wd, layout, out=c_buf(M, N))
    assert same_bits(lg, bi.bi_matmul(ad, wd, layout, out=c_buf(M, N))), "logits differ from bi_matmul"
    check_partials(lg, part, f"M={M} N={N} K={K} {layout}")
    rs = torch.empty(M, 2, dtype=torch.float32, device=DEV)
    y = bi.bi_log_softmax_partials(lg, part, row_stats=rs)
    xb = bf16_bits_np(lg.cpu())
    assert_lsm_close(y, oracle.log_softmax(xb), f"y M={M} N={N} K={K}")
    # row_stats: the row max exactly, log of the row's sum of exp(x - max) to fp32 rounding
    x64 = lg.cpu().double().numpy()
    r = to_np64(rs)
    assert np.array_equal(r[:, 0], x64.max(axis=1))
    lse_ref = x64[:, :1] - oracle.log_softmax(xb)[:, :1] - x64.max(axis=1, keepdims=True)
    assert float(np.abs(r[:, 1:] - lse_ref).max()) <= 1e-5
    assert bi.bi_get_device_status() == bi.BI_OK


def test_lse_workload_sampled_rows():
    """The LM head of the benchmark step (M = 1024, K = 4096, V = 151936), sampled rows."""
    M, K, V = 1024, 4096, 151936
    a = inputs.rows_normal(902, 0, M, K).to(DEV)
    w = weight(903, V, K, "nk")
    lg, part = bi.bi_matmul_lse(a, w)
    y = bi.bi_log_softmax_partials(lg, part)
    rows = torch.tensor([0, 127, 128, 255, 256, 700, M - 1])
    lgr = lg.cpu()[rows]
    check_partials(lgr, part.cpu()[rows], "workload rows")
    assert_lsm_close(y.cpu()[rows], oracle.log_softmax(bf16_bits_np(lgr)), "workload y")
    # the single-pass log_softmax of the same logits agrees to the tolerance
    assert float((y - bi.bi_log_softmax(lg)).abs().max()) <= 1e-4


def test_lse_fp32_logits():
    M, N, K = 5, 1000, 512
    a = inputs.rows_normal(904, 0, M, K).to(DEV)
    w = weight(905, N, K, "nk")
    lg, part = bi.bi_matmul_lse(a, w, out_dtype=torch.float32)
    assert same_bits(lg, bi.bi_matmul(a, w, out_dtype=torch.float32))
    p = to_np64(part)
    x = to_np64(lg)
    for t in range(p.shape[1]):
        assert np.array_equal(p[:, t, 0], x[:, t * TILE:(t + 1) * TILE].max(axis=1))
    y = bi.bi_log_softmax_partials(lg, part)
    assert_lsm_close(y, oracle.log_softmax(lg.cpu().numpy()), "fp32 logits")


def test_lse_ragged_rows_and_strided_logits():
    M, K = 7, 256
    a = inputs.rows_normal(906, 0, M, K).to(DEV)
    for N in (1001, 255, 9):
        w = weight(907, N, K, "nk")
        lg, part = bi.bi_matmul_lse(a, w, out=c_buf(M, N))
        y = bi.bi_log_softmax_partials(lg, part)
        assert_lsm_close(y, oracle.log_softmax(bf16_bits_np(lg.cpu())), f"ragged N={N}")
    # logits in a wider buffer (row stride 1032 > V = 1000): same y as the contiguous case
    w = weight(908, 1000, K, "nk")
    wide = torch.zeros(M, 1032, dtype=torch.bfloat16, device=DEV)
    lg, part = bi.bi_matmul_lse(a, w, out=wide[:, :1000])
    lg2, part2 = bi.bi_matmul_lse(a, w)
    assert same_bits(part, part2)
    assert same_bits(bi.bi_log_softmax_partials(lg, part), bi.bi_log_softmax_partials(lg2, part2))


def test_lse_k0_and_constant_rows():
    """K = 0: every logit is 0, each pair is (0, column count) and y = -log V."""
    M, N = 4, 1000
    a = torch.empty(M, 0, dtype=torch.bfloat16, device=DEV)
    w = torch.empty(N, 0, dtype=torch.bfloat16, device=DEV)
    lg, part = bi.bi_matmul_lse(a, w)
    counts = [min(TILE, N - t * TILE) for t in range(bi.bi_lse_partials_per_row(N))]
    assert torch.equal(part[..., 0].cpu(), torch.zeros(M, len(counts)))
    assert torch.equal(part[..., 1].cpu(), torch.tensor([counts] * M, dtype=torch.float32))
    y = bi.bi_log_softmax_partials(lg, part)
    assert float((y + np.log(N)).abs().max()) <= 1e-4


@pytest.mark.parametrize("layout", ["nk", "kn"])
def test_lse_batch_invariance(layout):
    K, N, POOL = 1024, 32000, 2048
    pool = inputs.rows_normal(910, 0, POOL, K).to(DEV)
    w = weight(911, N, K, layout)
    lg_ref, part_ref = bi.bi_matmul_lse(pool, w, layout)
    y_ref = bi.bi_log_softmax_partials(lg_ref, part_ref)
    singles = [bi.bi_matmul_lse(pool[i:i + 1], w, layout) for i in range(0, POOL, 97)]
    for j, i in enumerate(range(0, POOL, 97)):
        assert same_bits(singles[j][1], part_ref[i:i + 1]), f"row {i} alone"
    perm = inputs.permutation(912, POOL).to(DEV)
    for M in M_SWEEP:
        for start in (0, POOL - M):
            idx = perm[start:start + M]
            lg, part = bi.bi_matmul_lse(pool[idx], w, layout)
            assert same_bits(lg, lg_ref[idx]), f"logits M={M}"
            assert same_bits(part, part_ref[idx]), f"pairs M={M}"
            assert same_bits(bi.bi_log_softmax_partials(lg, part), y_ref[idx]), f"y M={M}"


def test_lse_lm_head_invariance_and_repeatability():
    K, V = 4096, 151936
    pool = inputs.rows_normal(913, 0, 512, K).to(DEV)
    w = weight(914, V, K, "nk")
    lg_ref, part_ref = bi.bi_matmul_lse(pool, w)
    y_ref = bi.bi_log_softmax_partials(lg_ref, part_ref)
    perm = inputs.permutation(915, 512).to(DEV)
    for M in (1, 3, 77, 256, 300):
        idx = perm[:M]
        lg, part = bi.bi_matmul_lse(pool[idx], w)
        assert same_bits(bi.bi_log_softmax_partials(lg, part), y_ref[idx]), f"M={M}"
    y = torch.empty_like(y_ref)
    for _ in range(100):
        bi.bi_log_softmax_partials(lg_ref, part_ref, out=y)
        assert same_bits(y, y_ref)


def test_lse_argument_errors():
    lib = bi.load()
    N = 304
    a = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(N, 64, dtype=torch.bfloat16, device=DEV)
    c = torch.zeros(4, N, dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.bi_matmul_lse(a.data_ptr(), 64, w.data_ptr(), 64, bi.BI_B_NK, c.data_ptr(), N, bi.BI_BF16,
                             None, 4, N, 64, s) == bi.BI_ERR_INVALID_ARG
    part = torch.zeros(4 * 2 * 2 + 1, dtype=torch.float32, device=DEV)
    rs = torch.zeros(4 * 2 + 1, dtype=torch.float32, device=DEV)
    assert lib.bi_matmul_lse(a.data_ptr(), 64, w.data_ptr(), 64, bi.BI_B_NK, c.data_ptr(), N, bi.BI_BF16,
                             part.data_ptr() + 4, 4, N, 64, s) == bi.BI_ERR_ALIGNMENT
    y = torch.zeros(4, N, dtype=torch.float32, device=DEV)
    call = lambda ldx, p, r: lib.bi_log_softmax_partials(c.data_ptr(), ldx, bi.BI_BF16, p, r, y.data_ptr(), 4, N, s)
    assert call(N - 1, part.data_ptr(), rs.data_ptr()) == bi.BI_ERR_INVALID_ARG
    assert call(N, None, rs.data_ptr()) == bi.BI_ERR_INVALID_ARG
    assert call(N, part.data_ptr(), None) == bi.BI_ERR_INVALID_ARG
    assert call(N, part.data_ptr() + 4, rs.data_ptr()) == bi.BI_ERR_ALIGNMENT
    assert call(N, part.data_ptr(), rs.data_ptr() + 4) == bi.BI_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.count_nonzero(c) == 0 and torch.count_nonzero(y) == 0  # nothing was launched
