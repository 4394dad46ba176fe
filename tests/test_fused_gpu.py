"""bi_matmul_silu_mul: the gate/up GEMM with SiLU * up in its epilogue, through the C ABI.

Parity against the fp64 oracle (silu(A.gate) * (A.up) with no rounding in between),
bit-level batch invariance over M and positions, and the fused MLP chain over mixed
batches.
"""
import pytest
import torch

from bi_testutil import M_SWEEP, assert_bf16_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gate_up(seed, F, K, layout):
    w = inputs.weight_normal(seed, (2 * F, K))  # [gate; up], stored [2F, K]
    return w if layout == "nk" else w.t().contiguous()


@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("M,F,K", [(1, 512, 256), (3, 512, 256), (17, 512, 256), (300, 200, 72),
                                   (129, 1000, 1000), (2, 8, 24), (257, 136, 4104)])
def test_fused_parity(M, F, K, layout):
    a = inputs.rows_normal(400, 0, M, K)
    w = gate_up(401, F, K, layout)
    h = bi.bi_matmul_silu_mul(a.to(DEV), w.to(DEV), layout)
    ref = oracle.matmul_silu_mul(bf16_bits_np(a), bf16_bits_np(w), layout)
    assert_bf16_close(h, ref, f"fused M={M} F={F} K={K} {layout}")


def test_fused_workload_sampled_rows():
    M, F, K = 2048, 12288, 4096
    a = inputs.rows_normal(402, 0, M, K)
    w = gate_up(403, F, K, "nk")
    h = bi.bi_matmul_silu_mul(a.to(DEV), w.to(DEV)).cpu()
    rows = torch.tensor([0, 127, 128, 255, 256, 1500, M - 1])
    ref = oracle.matmul_silu_mul(bf16_bits_np(a[rows]), bf16_bits_np(w), "nk")
    assert_bf16_close(h[rows], ref, "fused 2048 x 12288 sampled")


def test_fused_and_unfused_paths_each_match_their_oracle():
    """The fused path feeds fp32 g, u to the glue; the unfused path rounds them to bf16
    first, so each is checked against the oracle of what it computes (stage by stage for
    the unfused chain), not against each other."""
    M, F, K = 300, 1024, 512
    a = inputs.rows_normal(404, 0, M, K).to(DEV)
    w = gate_up(405, F, K, "nk").to(DEV)
    fused = bi.bi_matmul_silu_mul(a, w)
    assert_bf16_close(fused, oracle.matmul_silu_mul(bf16_bits_np(a.cpu()), bf16_bits_np(w.cpu()), "nk"),
                      "fused")
    gu = bi.bi_matmul(a, w)
    unfused = bi.bi_silu_mul(gu)
    assert_bf16_close(unfused, oracle.silu_mul(bf16_bits_np(gu.cpu())), "unfused glue stage")


@pytest.mark.parametrize("layout", ["nk", "kn"])
def test_fused_batch_invariance(layout):
    F, K = 1536, 4096
    pool = inputs.rows_normal(406, 0, 2048, K).to(DEV)
    w = gate_up(407, F, K, layout).to(DEV)
    ref = torch.cat([bi.bi_matmul_silu_mul(pool[i:i + 1], w, layout) for i in range(2048)])
    perm = inputs.permutation(408, 2048).to(DEV)
    for M in M_SWEEP:
        for start in (0, 2048 - M):
            idx = perm[start:start + M]
            assert same_bits(bi.bi_matmul_silu_mul(pool[idx], w, layout), ref[idx]), f"M={M}"


def test_fused_repeatable_100_runs():
    M, F, K = 2048, 12288, 4096
    a = inputs.rows_normal(409, 0, M, K).to(DEV)
    w = gate_up(416, F, K, "nk").to(DEV)
    first = bi.bi_matmul_silu_mul(a, w)
    for _ in range(100):
        assert same_bits(bi.bi_matmul_silu_mul(a, w), first)


def test_fused_k0_and_empty():
    a0 = torch.empty(5, 0, dtype=torch.bfloat16, device=DEV)
    w0 = torch.empty(16, 0, dtype=torch.bfloat16, device=DEV)
    assert torch.count_nonzero(bi.bi_matmul_silu_mul(a0, w0)) == 0
    a = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(16, 64, dtype=torch.bfloat16, device=DEV)
    assert bi.bi_matmul_silu_mul(a, w).shape == (0, 8)


def test_fused_mlp_chain_over_mixed_batches():
    H, F, POOL = 4096, 12288, 2048
    pool = inputs.rows_normal(410, 0, POOL, H).to(DEV)
    g = inputs.gain(411, H).to(DEV)
    w_gu = inputs.weight_normal(412, (2 * F, H)).to(DEV)
    w_d = inputs.weight_normal(413, (H, F)).to(DEV)

    def run(x):
        return bi.bi_addmm(x, bi.bi_matmul_silu_mul(bi.bi_rmsnorm(x, g, 1e-6), w_gu), w_d)

    ref = run(pool)
    for t, b in enumerate(inputs.batch_sizes(414, 60, 1, 512)):
        idx = inputs.permutation(415 + t, POOL)[:b].to(DEV)
        assert same_bits(run(pool[idx]), ref[idx]), f"trial {t}, batch {b}"
