"""The MLP block chain over mixed batches, through the C ABI.

RMSNorm -> gate/up GEMM (4096 -> 2 x 12288) -> SiLU * up -> down GEMM (12288 -> 4096)
with the residual added in the down GEMM's epilogue.  Batches of 1..512 rows are
assembled from a seeded pool of 2048 rows in random order; every pool row's output
must be bit-identical in every batch it appears in, to its M = 1 result, and across
100 repeated runs.  Each stage is also checked against the oracle, stage by stage
(the oracle stage takes the device's bf16 input of that stage).
"""
import pytest
import torch

from bi_testutil import assert_bf16_close, bf16_bits_np, same_bits
from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs
from oracle import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
H, F, POOL, EPS = 4096, 12288, 2048, 1e-6


@pytest.fixture(scope="module")
def chain():
    pool = inputs.rows_normal(300, 0, POOL, H)
    g = inputs.gain(301, H)
    w_gu = inputs.weight_normal(302, (2 * F, H))
    w_d = inputs.weight_normal(303, (H, F))
    dev = {k: v.to(DEV) for k, v in dict(pool=pool, g=g, w_gu=w_gu, w_d=w_d).items()}

    def run(x):
        h = bi.bi_rmsnorm(x, dev["g"], EPS)
        gu = bi.bi_matmul(h, dev["w_gu"], "nk")
        a = bi.bi_silu_mul(gu)
        y = bi.bi_addmm(x, a, dev["w_d"], "nk")
        return h, gu, a, y

    return dict(host=dict(pool=pool, g=g, w_gu=w_gu, w_d=w_d), dev=dev, run=run)


def test_chain_stages_match_oracle(chain):
    rows = torch.tensor([0, 1, 129, 2047])
    x = chain["dev"]["pool"][rows.to(DEV)]
    h, gu, a, y = chain["run"](x)
    hst = chain["host"]
    assert_bf16_close(h, oracle.rmsnorm(bf16_bits_np(x.cpu()), bf16_bits_np(hst["g"]), EPS), "rmsnorm")
    assert_bf16_close(gu, oracle.matmul(bf16_bits_np(h.cpu()), bf16_bits_np(hst["w_gu"]), "nk"), "gate/up")
    assert_bf16_close(a, oracle.silu_mul(bf16_bits_np(gu.cpu())), "silu_mul")
    assert_bf16_close(y, oracle.addmm(bf16_bits_np(x.cpu()), bf16_bits_np(a.cpu()),
                                      bf16_bits_np(hst["w_d"]), "nk"), "down + residual")


def test_chain_rows_identical_across_batch_compositions(chain):
    pool = chain["dev"]["pool"]
    run = chain["run"]
    ref = run(pool)[3]  # the whole pool as one batch of 2048
    singles = torch.cat([run(pool[i:i + 1])[3] for i in range(0, POOL, 16)])
    assert same_bits(singles, ref[::16]), "M = 1 results differ from the M = 2048 batch"
    sizes = inputs.batch_sizes(304, 100, 1, 512)
    for t, b in enumerate(sizes):
        idx = inputs.permutation(305 + t, POOL)[:b].to(DEV)
        out = run(pool[idx])[3]
        assert same_bits(out, ref[idx]), f"trial {t}: batch of {b} changed a row's bits"


def test_chain_repeatable_100_runs(chain):
    x = chain["dev"]["pool"][:512]
    first = chain["run"](x)[3]
    for _ in range(100):
        assert same_bits(chain["run"](x)[3], first)
