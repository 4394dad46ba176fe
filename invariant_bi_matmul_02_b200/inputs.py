"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws numbers; it holds none of the arithmetic of the
operations.  Both the CUDA path and the CPU oracle read the tensors it
returns, bit for bit.

Recipe (all on the CPU with ``torch.Generator``, float32 draws rounded once to
bf16 by torch's round-to-nearest-even cast where a bf16 tensor is wanted):

* activations   N(0, 1)                      seed family 0
* weights       N(0, 0.02)                   seed family 1
* RMSNorm gain  1 + N(0, 0.1)                seed family 1
* bias          N(0, 0.01)                   seed family 2
* outliers      each entry independently with probability 0.01 is scaled x50,
                                             seed family 2
* integer mode  uniform integers in [-4, 4] (exact in bf16 and in fp32 sums)

Activations are drawn row by row from a generator keyed by (seed, row), so any
range of rows -- a batch slice, a shard of a multi-process run, a single row --
is reproduced exactly without drawing the rest.
"""
from __future__ import annotations

import numpy as np
import torch

ACT, WEIGHT, AUX = 0, 1, 2

# Qwen3-8B-shaped sizes used by the workloads.
HIDDEN = 4096
KV_OUT = 1024
FFN = 12288
VOCAB = 151936


def _gen(family: int, key: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((family << 48) ^ (key & ((1 << 48) - 1)))
    return g


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 tensor as a numpy uint16 array (CPU copy)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("bf16 tensor expected")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rows_normal(seed: int, row0: int, nrows: int, cols: int, std: float = 1.0,
                dtype=torch.bfloat16) -> torch.Tensor:
    """Rows row0 .. row0+nrows-1 of an N(0, std^2) activation matrix with `cols` columns."""
    out = torch.empty((nrows, cols), dtype=torch.float32)
    for r in range(nrows):
        g = _gen(ACT, (seed << 24) + row0 + r)
        out[r] = torch.randn(cols, generator=g)
    if std != 1.0:
        out.mul_(std)
    return out.to(dtype)


def rows_int(seed: int, row0: int, nrows: int, cols: int, lo: int = -4, hi: int = 4,
             dtype=torch.bfloat16) -> torch.Tensor:
    """Integer-valued rows, uniform on [lo, hi], keyed by row like rows_normal."""
    out = torch.empty((nrows, cols), dtype=torch.float32)
    for r in range(nrows):
        g = _gen(ACT, (seed << 24) + row0 + r + (1 << 40))
        out[r] = torch.randint(lo, hi + 1, (cols,), generator=g).to(torch.float32)
    return out.to(dtype)


def weight_normal(seed: int, shape, std: float = 0.02, dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(WEIGHT, seed)
    return (torch.randn(*shape, generator=g) * std).to(dtype)


def weight_int(seed: int, shape, lo: int = -4, hi: int = 4, dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(WEIGHT, seed + (1 << 40))
    return torch.randint(lo, hi + 1, tuple(shape), generator=g).to(torch.float32).to(dtype)


def gain(seed: int, n: int, std: float = 0.1, dtype=torch.bfloat16) -> torch.Tensor:
    """RMSNorm weight 1 + N(0, std^2)."""
    g = _gen(WEIGHT, seed + (1 << 41))
    return (1.0 + torch.randn(n, generator=g) * std).to(dtype)


def bias(seed: int, n: int, std: float = 0.01, dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(AUX, seed)
    return (torch.randn(n, generator=g) * std).to(dtype)


def with_outliers(x: torch.Tensor, seed: int, row0: int = 0, frac: float = 0.01,
                  scale: float = 50.0) -> torch.Tensor:
    """Scale an independent Bernoulli(frac) subset of entries by `scale` (row-keyed mask)."""
    xf = x.to(torch.float32).clone()
    for r in range(xf.shape[0]):
        g = _gen(AUX, (seed << 24) + row0 + r + (1 << 42))
        mask = torch.rand(xf.shape[1], generator=g) < frac
        xf[r, mask] *= scale
    return xf.to(x.dtype)


def rows_normal_outliers(seed: int, row0: int, nrows: int, cols: int, dtype) -> torch.Tensor:
    """Row-reduction workload rows: N(0, 1) with 1% of entries scaled x50."""
    x = rows_normal(seed, row0, nrows, cols, dtype=torch.float32)
    return with_outliers(x, seed, row0).to(dtype)


def permutation(seed: int, n: int) -> torch.Tensor:
    g = _gen(AUX, seed + (1 << 43))
    return torch.randperm(n, generator=g)


def batch_sizes(seed: int, count: int, lo: int, hi: int) -> list[int]:
    g = _gen(AUX, seed + (1 << 44))
    return [int(v) for v in torch.randint(lo, hi + 1, (count,), generator=g)]
