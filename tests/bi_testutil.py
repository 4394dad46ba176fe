"""Helpers shared by the GPU parity and invariance tests.

Tolerances (written here once, used by every parity test):
* bf16 outputs:        |gpu - ref| <= 2^-7 |ref| + 1e-3
* fp32 log_softmax:    |gpu - ref| <= 1e-4
* fp32 mean:           |gpu - ref| <= 1.01 d 2^-24 sum|x| / H + 2^-24 |ref|
  where d = mean_chain_depth(H) is the longest chain of fp32 additions an element passes
  through in bi_mean's fixed order (per-thread running sums, then the block tree): the
  first-order error bound of
  recursive summation in a fixed order (Higham, Accuracy and Stability of Numerical
  Algorithms, section 4.2), then one correctly rounded division
"""
import math

import numpy as np
import torch

from invariant_bi_matmul_02_b200 import inputs

BF16_REL = 2.0 ** -7
BF16_ABS = 1e-3
LSM_ABS = 1e-4
U32 = 2.0 ** -24


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_bf16_close(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = to_np64(gpu)
    err = np.abs(g - ref)
    bound = BF16_REL * np.abs(ref) + BF16_ABS
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} entries out of tolerance; first at {tuple(idx)}: "
            f"gpu={g[tuple(idx)]!r} ref={ref[tuple(idx)]!r}")


def assert_lsm_close(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = to_np64(gpu)
    err = np.abs(g - ref)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= LSM_ABS, f"{what}: max |err| {worst} > {LSM_ABS}"


def assert_lsm_close_ieee(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    """log_softmax parity on rows with masked (-inf) or non-finite entries: where the oracle's
    value is finite the kernel's must be within LSM_ABS of it; where it is +-inf the kernel's
    must be the same infinity; where it is NaN the kernel's must be NaN."""
    g = to_np64(gpu)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: finite entries differ from the oracle's"
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(g), nan), f"{what}: NaN entries differ from the oracle's"
    inf = ~fin & ~nan
    assert np.array_equal(g[inf], ref[inf]), f"{what}: infinite entries differ from the oracle's"
    if fin.any():
        worst = float(np.abs(g[fin] - ref[fin]).max())
        assert worst <= LSM_ABS, f"{what}: max |err| {worst} > {LSM_ABS}"


def mean_chain_depth(H: int) -> int:
    """Longest chain of fp32 additions in bi_mean's order for rows of H elements: one block of
    T threads per row (T = 32 ceil(((H / 4 + 3) / 4) / 32), clamped to [32, 1024]).
    H % 4 == 0: thread t keeps four running sums, one per lane of its float4 groups t, t + T,
    ...; each adds g = ceil(H / 4 / T) values, then the four meet in a 2-level tree.  Otherwise
    thread t adds its ceil(H / T) elements into one sum.  The block tree then adds 10 levels
    (warp butterfly, then a butterfly over the warp sums)."""
    v = (H // 4 + 3) // 4
    T = min(1024, max(32, -(-v // 32) * 32))
    if H % 4 == 0:
        return -(-(H // 4) // T) + 2 + 10
    return -(-H // T) + 10


def assert_mean_close(gpu: torch.Tensor, ref: np.ndarray, x: np.ndarray, what: str = ""):
    H = x.shape[1]
    g = to_np64(gpu)
    depth = 1.01 * mean_chain_depth(H)
    bound = depth * U32 * np.abs(x.astype(np.float64)).sum(axis=1) / H + U32 * np.abs(ref)
    err = np.abs(g - ref)
    assert np.all(err <= bound), f"{what}: worst excess {float((err - bound).max())}"


def bits16(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(torch.int16)


def bits32(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(torch.int32)


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    if a.dtype != b.dtype or a.shape != b.shape:
        return False
    view = bits16 if a.element_size() == 2 else bits32
    return bool(torch.equal(view(a), view(b)))


def bf16_bits_np(t: torch.Tensor) -> np.ndarray:
    return inputs.bf16_bits(t)


# The M values of the GEMM sweep: powers of two up to 2048, the odd sizes, and the sizes on
# either side of the GEMM's 128-token half-tile (a tile whose second half holds no token skips
# that half's MMAs): 129, 384, 385.
M_SWEEP = [1, 2, 3, 4, 8, 16, 32, 64, 77, 128, 129, 256, 384, 385, 512, 1000, 1024, 2048]
