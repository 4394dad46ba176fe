"""Guard canaries around every output buffer, through the C ABI.

Each kernel writes into the middle of a larger buffer whose bytes are first filled with a
sentinel pattern: a guard region before the output, one after it and, for outputs with a row
stride wider than the row, the padding between rows.  After the call every sentinel byte must
be unchanged.  Sizes are ragged (partial GEMM tiles in M and N, row tails), so a store past a
tile edge or a row end lands in a guard.
"""
import pytest
import torch

from invariant_bi_matmul_02_b200 import binding as bi
from invariant_bi_matmul_02_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096  # elements on each side (a multiple of 8, so the output stays 16-byte aligned)
SENTINEL = {torch.bfloat16: 0x7FA5, torch.float32: 0x7FC0DEAD}  # NaN payloads no kernel writes
INT_VIEW = {torch.bfloat16: torch.int16, torch.float32: torch.int32}


class Guarded:
    """A [rows, cols] output with row stride ld inside a sentinel-filled flat buffer."""

    def __init__(self, rows, cols, dtype, ld=None):
        self.rows, self.cols, self.ld = rows, cols, ld or cols
        self.buf = torch.empty(2 * GUARD + rows * self.ld, dtype=dtype, device=DEV)
        self.bits = self.buf.view(INT_VIEW[dtype])
        self.bits.fill_(SENTINEL[dtype])
        self.ref = self.bits.clone()
        inner = self.buf[GUARD:GUARD + rows * self.ld].view(rows, self.ld)
        self.view = inner[:, :cols]

    def flat(self):
        assert self.ld == self.cols
        return self.buf[GUARD:GUARD + self.rows * self.cols]

    def check(self, what):
        torch.cuda.synchronize()
        b, r = self.bits, self.ref
        assert torch.equal(b[:GUARD], r[:GUARD]), f"{what}: wrote before its output"
        end = GUARD + self.rows * self.ld
        assert torch.equal(b[end:], r[end:]), f"{what}: wrote past its output"
        if self.ld > self.cols:
            pad = b[GUARD:end].view(self.rows, self.ld)[:, self.cols:]
            assert torch.equal(pad, r[GUARD:end].view(self.rows, self.ld)[:, self.cols:]), \
                f"{what}: wrote into the row padding"


@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_outputs_stay_in_bounds(layout, out_dtype):
    M, N, K = 77, 1000, 200
    a = inputs.rows_normal(1100, 0, M, K).to(DEV)
    w = inputs.weight_normal(1101, (N, K)).to(DEV)
    if layout == "kn":
        w = w.t().contiguous()
    c = Guarded(M, N, out_dtype, ld=1008)
    bi.bi_matmul(a, w, layout, out=c.view)
    c.check(f"bi_matmul {layout} {out_dtype}")
    bias = inputs.bias(1102, N).to(DEV)
    c = Guarded(M, N, out_dtype, ld=1016)
    bi.bi_addmm(bias, a, w, layout, out=c.view)
    c.check(f"bi_addmm {layout} {out_dtype}")
    resid = inputs.rows_normal(1107, 0, M, N).to(DEV)
    c = Guarded(M, N, out_dtype, ld=1024)
    bi.bi_addmm(resid, a, w, layout, out=c.view)
    c.check(f"bi_addmm residual {layout} {out_dtype}")


@pytest.mark.parametrize("layout,F", [("nk", 500), ("kn", 504)])  # [K, 2F] needs F % 8 == 0
def test_fused_silu_output_stays_in_bounds(layout, F):
    M, K = 77, 200
    a = inputs.rows_normal(1103, 0, M, K).to(DEV)
    w = inputs.weight_normal(1104, (2 * F, K)).to(DEV)
    if layout == "kn":
        w = w.t().contiguous()
    h = Guarded(M, F, torch.bfloat16, ld=512)
    bi.bi_matmul_silu_mul(a, w, layout, out=h.view)
    h.check(f"bi_matmul_silu_mul {layout}")


@pytest.mark.parametrize("H", [4096, 1000, 1001])
def test_row_op_outputs_stay_in_bounds(H):
    M = 77
    x = inputs.rows_normal_outliers(1105, 0, M, H, torch.bfloat16).to(DEV)
    g = inputs.gain(1106, H).to(DEV)
    y = Guarded(M, H, torch.bfloat16)
    bi.bi_rmsnorm(x, g, 1e-6, out=y.flat().view(M, H))
    y.check(f"bi_rmsnorm H={H}")
    m = Guarded(M, 1, torch.float32)
    bi.bi_mean(x.float(), out=m.flat())
    m.check(f"bi_mean H={H}")
    ls = Guarded(M, H, torch.float32)
    bi.bi_log_softmax(x, out=ls.flat().view(M, H))
    ls.check(f"bi_log_softmax H={H}")
    if H % 2 == 0:
        s = Guarded(M, H // 2, torch.bfloat16)
        bi.bi_silu_mul(x, out=s.flat().view(M, H // 2))
        s.check(f"bi_silu_mul F={H // 2}")


@pytest.mark.parametrize("V", [151936, 110000, 4104])
def test_log_softmax_variants_stay_in_bounds(V):
    M = 5
    x = inputs.rows_normal(1107, 0, M, V, std=1.3).to(DEV)
    y = Guarded(M, V, torch.float32)
    bi.bi_log_softmax(x, out=y.flat().view(M, V))
    y.check(f"bi_log_softmax V={V}")
    y = Guarded(M, V, torch.float32)
    scr = Guarded(bi.bi_log_softmax_split_scratch_bytes(M, V) // 4, 1, torch.float32)
    bi.bi_log_softmax_split(x, scr.flat().view(torch.uint8), out=y.flat().view(M, V))
    y.check(f"bi_log_softmax_split V={V}")
    scr.check(f"bi_log_softmax_split scratch V={V}")
    if V >= 32768:
        y = Guarded(M, V, torch.float32)
        bi.bi_log_softmax_cluster(x, out=y.flat().view(M, V))
        y.check(f"bi_log_softmax_cluster V={V}")


@pytest.mark.parametrize("D", [64, 128])
def test_decode_attention_outputs_stay_in_bounds(D):
    B, Hq, Hkv, Lmax = 3, 16, 4, 300
    q = inputs.rows_normal(1108, 0, B * Hq, D).view(B, Hq, D).to(DEV)
    k = inputs.rows_normal(1109, 0, B * Lmax * Hkv, D).view(B, Lmax, Hkv, D).to(DEV)
    v = inputs.rows_normal(1110, 0, B * Lmax * Hkv, D).view(B, Lmax, Hkv, D).to(DEV)
    lens = torch.tensor([300, 1, 129], dtype=torch.int32, device=DEV)
    out = Guarded(B * Hq, D, torch.bfloat16)
    nscr = bi.bi_decode_attention_scratch_bytes(B, Hq, D, Lmax)
    scr = Guarded(nscr // 4, 1, torch.float32)
    bi.bi_decode_attention(q, k, v, lens, scratch=scr.flat().view(torch.uint8),
                           out=out.flat().view(B, Hq, D))
    out.check("bi_decode_attention output")
    scr.check("bi_decode_attention scratch")
