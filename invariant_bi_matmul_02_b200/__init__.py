"""Batch-invariant reduction kernels for B200 (sm_100a) behind a C ABI.

``binding`` exposes the entry points of include/bi.h (bi_matmul, bi_addmm,
bi_rmsnorm, bi_mean, bi_log_softmax, bi_silu_mul, ...) on torch tensors.
``inputs`` draws the seeded synthetic inputs of the workloads.
libbi.so is loaded on the first call into ``binding``.
"""
from .binding import (  # noqa: F401
    BiError,
    bi_addmm,
    bi_decode_attention,
    bi_decode_attention_scratch_bytes,
    bi_gemm_config,
    bi_get_device_status,
    bi_log_softmax,
    bi_log_softmax_split,
    bi_log_softmax_split_scratch_bytes,
    bi_matmul,
    bi_matmul_silu_mul,
    bi_mean,
    bi_rmsnorm,
    bi_selftest_wait_timeout,
    bi_silu_mul,
    bi_version,
    load,
)
