"""Python binding of libbi.so: the C ABI of include/bi.h, one function per entry point.

Argument marshalling only.  Each function checks device, dtype and layout of the
torch tensors it is given, allocates the output with torch when none is passed,
and calls the C entry point of the same name with raw device pointers, leading
dimensions and the current CUDA stream.  Every step of the computation runs in
libbi.so's kernels; there is no fallback.  If libbi.so is missing or a call fails
the function raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbi.so")

BI_OK, BI_ERR_INVALID_ARG, BI_ERR_UNSUPPORTED, BI_ERR_ALIGNMENT, BI_ERR_CUDA, BI_ERR_TIMEOUT = range(6)
BI_BF16, BI_F32 = 0, 1
BI_B_KN, BI_B_NK = 0, 1

# Every entry point declared in include/bi.h, with its ctypes signature.
_i64, _p, _i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32
SIGNATURES = {
    "bi_matmul": (ctypes.c_int, [_p, _i64, _p, _i64, ctypes.c_int, _p, _i64, ctypes.c_int,
                                 _i64, _i64, _i64, _p]),
    "bi_addmm": (ctypes.c_int, [_p, _i64, _p, _i64, _p, _i64, ctypes.c_int, _p, _i64, ctypes.c_int,
                                _i64, _i64, _i64, _p]),
    "bi_matmul_silu_mul": (ctypes.c_int, [_p, _i64, _p, _i64, ctypes.c_int, _p, _i64, _i64, _i64, _i64,
                                          _p]),
    "bi_rmsnorm": (ctypes.c_int, [_p, _p, _p, _i64, _i64, ctypes.c_float, _p]),
    "bi_mean": (ctypes.c_int, [_p, _p, _i64, _i64, _p]),
    "bi_log_softmax": (ctypes.c_int, [_p, ctypes.c_int, _p, _i64, _i64, _p]),
    "bi_log_softmax_cluster": (ctypes.c_int, [_p, ctypes.c_int, _p, _i64, _i64, _p]),
    "bi_log_softmax_split": (ctypes.c_int, [_p, ctypes.c_int, _p, _i64, _i64, _p, ctypes.c_size_t, _p]),
    "bi_log_softmax_split_scratch_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bi_log_softmax_split_noalloc": (ctypes.c_int, [_p, ctypes.c_int, _p, _i64, _i64, _p]),
    "bi_silu_mul": (ctypes.c_int, [_p, _p, _i64, _i64, _p]),
    "bi_decode_attention": (ctypes.c_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, ctypes.c_float,
                                           _p, ctypes.c_size_t, _p]),
    "bi_decode_attention_scratch_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _i64]),
    "bi_get_device_status": (ctypes.c_int, [_p, ctypes.POINTER(_i32)]),
    "bi_selftest_wait_timeout": (ctypes.c_int, [_i64, _p]),
    "bi_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bi_gemm_config": (None, [_i64] + [ctypes.POINTER(_i32)] * 5),
    "bi_tensor_map_cache_stats": (None, [ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "bi_version": (ctypes.c_int32, []),
}

_lib = None


class BiError(RuntimeError):
    def __init__(self, name: str, status: int):
        super().__init__(f"{name} failed: {status_string(status)} ({status})")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbi.so (once) and attach the ctypes signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"libbi.so not found at {path}: build it with __graft_entry__.build() or "
                "invariant_bi_matmul_02_b200/csrc/build.py")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().bi_status_string(int(status)).decode()


def _check(name: str, status: int):
    if status != BI_OK:
        raise BiError(name, status)


def _current_device() -> int:
    return torch.cuda.current_device()


def _same_device(index: int, name: str, cur: int | None = None):
    """The library launches on the current device and looks up its per-device state there, so
    every tensor and the stream of a call must live on that device.  `cur`: the current device,
    when the caller has already looked it up."""
    if cur is None:
        cur = _current_device()
    if index != cur:
        raise ValueError(f"{name} is on cuda:{index} but the current device is cuda:{cur}; "
                         "call under `with torch.cuda.device(...)`")


# The current stream's raw handle without building a torch.cuda.Stream object (3 us per call on
# the host otherwise); the public call where a torch build lacks it.
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, cur: int | None = None):
    if stream is None:
        if _raw_current_stream is not None:
            return _raw_current_stream(_current_device() if cur is None else cur)
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        _same_device(stream.device.index, "stream")
        return stream.cuda_stream
    return int(stream)


def _need_cuda(t: torch.Tensor, name: str, dtypes, cur: int | None = None) -> int:
    """Check that t is a CUDA tensor of one of `dtypes` on the current device; returns the
    current device, so that a call's other checks need not look it up again."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if cur is None:
        cur = _current_device()
    _same_device(t.get_device(), name, cur)
    return cur


def _ld(t: torch.Tensor, name: str) -> int:
    """Leading dimension of a 2-D tensor with unit-stride rows."""
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D")
    rows, cols = t.shape
    s0, s1 = t.stride()
    if cols > 1 and s1 != 1:
        raise ValueError(f"{name} rows must be contiguous")
    return s0 if rows > 1 else max(s0, cols)


def _contig(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_DT = {torch.bfloat16: BI_BF16, torch.float32: BI_F32}


def _gemm_shapes(a, b, b_layout):
    if b_layout not in ("kn", "nk"):
        raise ValueError("b_layout must be 'kn' ([K, N]) or 'nk' ([N, K])")
    M, K = a.shape
    if b_layout == "kn":
        Kb, N = b.shape
    else:
        N, Kb = b.shape
    if Kb != K:
        raise ValueError(f"inner dimensions differ: A has K={K}, B has K={Kb}")
    return M, N, K


def bi_matmul(a: torch.Tensor, b: torch.Tensor, b_layout: str = "nk", out: torch.Tensor | None = None,
              out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """C = A . B (b_layout 'kn': B [K, N]; 'nk': B [N, K], i.e. C = A . B^T)."""
    cur = _need_cuda(a, "A", (torch.bfloat16,))
    _need_cuda(b, "B", (torch.bfloat16,), cur)
    M, N, K = _gemm_shapes(a, b, b_layout)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _need_cuda(out, "C", (torch.bfloat16, torch.float32), cur)
    if tuple(out.shape) != (M, N):
        raise ValueError("C must be [M, N]")
    st = load().bi_matmul(a.data_ptr(), _ld(a, "A"), b.data_ptr(), _ld(b, "B"),
                          BI_B_KN if b_layout == "kn" else BI_B_NK, out.data_ptr(), _ld(out, "C"),
                          _DT[out.dtype], M, N, K, _stream(stream, cur))
    _check("bi_matmul", st)
    return out


def bi_addmm(input: torch.Tensor, a: torch.Tensor, b: torch.Tensor, b_layout: str = "nk",
             out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
             stream=None) -> torch.Tensor:
    """C = input + A . B; input is a bias [N] or a matrix [M, N] (bf16)."""
    cur = _need_cuda(a, "A", (torch.bfloat16,))
    _need_cuda(b, "B", (torch.bfloat16,), cur)
    _need_cuda(input, "input", (torch.bfloat16,), cur)
    M, N, K = _gemm_shapes(a, b, b_layout)
    if input.dim() == 1:
        if input.shape[0] != N:
            raise ValueError("bias must have N entries")
        if input.stride(0) != 1:
            raise ValueError("bias must be contiguous")
        ld_in = 0
    else:
        if tuple(input.shape) != (M, N):
            raise ValueError("input must be [N] or [M, N]")
        ld_in = _ld(input, "input")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _need_cuda(out, "C", (torch.bfloat16, torch.float32), cur)
    if tuple(out.shape) != (M, N):
        raise ValueError("C must be [M, N]")
    st = load().bi_addmm(input.data_ptr(), ld_in, a.data_ptr(), _ld(a, "A"), b.data_ptr(), _ld(b, "B"),
                         BI_B_KN if b_layout == "kn" else BI_B_NK, out.data_ptr(), _ld(out, "C"),
                         _DT[out.dtype], M, N, K, _stream(stream, cur))
    _check("bi_addmm", st)
    return out


def bi_matmul_silu_mul(a: torch.Tensor, b: torch.Tensor, b_layout: str = "nk",
                       out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H = silu(A . gate) * (A . up) with B the stacked [gate; up] weight ('nk': [2F, K];
    'kn': [K, 2F]); the glue runs in the GEMM's epilogue."""
    cur = _need_cuda(a, "A", (torch.bfloat16,))
    _need_cuda(b, "B", (torch.bfloat16,), cur)
    M, N2, K = _gemm_shapes(a, b, b_layout)
    if N2 % 2:
        raise ValueError("B must stack gate and up: an even number of output rows")
    F = N2 // 2
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=a.device)
    _need_cuda(out, "H", (torch.bfloat16,), cur)
    if tuple(out.shape) != (M, F):
        raise ValueError("H must be [M, F]")
    st = load().bi_matmul_silu_mul(a.data_ptr(), _ld(a, "A"), b.data_ptr(), _ld(b, "B"),
                                   BI_B_KN if b_layout == "kn" else BI_B_NK, out.data_ptr(),
                                   _ld(out, "H"), M, F, K, _stream(stream, cur))
    _check("bi_matmul_silu_mul", st)
    return out


def bi_rmsnorm(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """y = x / sqrt(mean(x^2) + eps) * w over the last dimension (bf16)."""
    _need_cuda(x, "x", (torch.bfloat16,))
    _need_cuda(w, "w", (torch.bfloat16,))
    _contig(x, "x")
    _contig(w, "w")
    M, H = x.shape
    if tuple(w.shape) != (H,):
        raise ValueError("w must be [H]")
    if out is None:
        out = torch.empty_like(x)
    _need_cuda(out, "y", (torch.bfloat16,))
    _contig(out, "y")
    _check("bi_rmsnorm", load().bi_rmsnorm(x.data_ptr(), w.data_ptr(), out.data_ptr(), M, H,
                                           float(eps), _stream(stream)))
    return out


def bi_mean(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y_i = mean_j x_ij (fp32)."""
    _need_cuda(x, "x", (torch.float32,))
    _contig(x, "x")
    M, H = x.shape
    if out is None:
        out = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need_cuda(out, "y", (torch.float32,))
    _contig(out, "y")
    _check("bi_mean", load().bi_mean(x.data_ptr(), out.data_ptr(), M, H, _stream(stream)))
    return out


def bi_log_softmax(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """log_softmax over the last dimension; x fp32 or bf16, y fp32."""
    _need_cuda(x, "x", (torch.float32, torch.bfloat16))
    _contig(x, "x")
    M, V = x.shape
    if out is None:
        out = torch.empty((M, V), dtype=torch.float32, device=x.device)
    _need_cuda(out, "y", (torch.float32,))
    _contig(out, "y")
    _check("bi_log_softmax", load().bi_log_softmax(x.data_ptr(), _DT[x.dtype], out.data_ptr(), M, V,
                                                   _stream(stream)))
    return out


def bi_log_softmax_cluster(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """log_softmax over the last dimension by a cluster of 4 CTAs per row (long rows only:
    32768 <= V <= 196608 for bf16, 16384 <= V <= 98304 for fp32)."""
    _need_cuda(x, "x", (torch.float32, torch.bfloat16))
    _contig(x, "x")
    M, V = x.shape
    if out is None:
        out = torch.empty((M, V), dtype=torch.float32, device=x.device)
    _need_cuda(out, "y", (torch.float32,))
    _contig(out, "y")
    _check("bi_log_softmax_cluster", load().bi_log_softmax_cluster(x.data_ptr(), _DT[x.dtype], out.data_ptr(), M,
                                                                   V, _stream(stream)))
    return out


def bi_log_softmax_split_scratch_bytes(M: int, V: int) -> int:
    return int(load().bi_log_softmax_split_scratch_bytes(int(M), int(V)))


def bi_log_softmax_split(x: torch.Tensor, scratch: torch.Tensor | None = None,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """log_softmax over the last dimension by many blocks per row (short batches).
    `scratch` is caller-owned device memory of at least bi_log_softmax_split_scratch_bytes."""
    _need_cuda(x, "x", (torch.float32, torch.bfloat16))
    _contig(x, "x")
    M, V = x.shape
    if out is None:
        out = torch.empty((M, V), dtype=torch.float32, device=x.device)
    _need_cuda(out, "y", (torch.float32,))
    _contig(out, "y")
    need = bi_log_softmax_split_scratch_bytes(M, V)
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    if not scratch.is_cuda:
        raise ValueError("scratch must be device memory")
    _same_device(scratch.get_device(), "scratch")
    nbytes = scratch.numel() * scratch.element_size()
    _check("bi_log_softmax_split", load().bi_log_softmax_split(
        x.data_ptr(), _DT[x.dtype], out.data_ptr(), M, V, scratch.data_ptr(), nbytes, _stream(stream)))
    return out


def bi_log_softmax_split_noalloc(x: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """bi_log_softmax_split with its partials in the library's fixed device array, for callers
    that cannot allocate device memory when they call it; `out` must be given."""
    _need_cuda(x, "x", (torch.float32, torch.bfloat16))
    _contig(x, "x")
    _need_cuda(out, "y", (torch.float32,))
    _contig(out, "y")
    M, V = x.shape
    if tuple(out.shape) != (M, V):
        raise ValueError("y must be [M, V]")
    _check("bi_log_softmax_split_noalloc", load().bi_log_softmax_split_noalloc(
        x.data_ptr(), _DT[x.dtype], out.data_ptr(), M, V, _stream(stream)))
    return out


def bi_silu_mul(gu: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h = silu(gu[:, :F]) * gu[:, F:] (bf16)."""
    _need_cuda(gu, "gu", (torch.bfloat16,))
    _contig(gu, "gu")
    M, F2 = gu.shape
    if F2 % 2:
        raise ValueError("gu must have 2F columns")
    F = F2 // 2
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=gu.device)
    _need_cuda(out, "h", (torch.bfloat16,))
    _contig(out, "h")
    _check("bi_silu_mul", load().bi_silu_mul(gu.data_ptr(), out.data_ptr(), M, F, _stream(stream)))
    return out


def bi_decode_attention_scratch_bytes(B: int, Hq: int, D: int, Lmax: int) -> int:
    return int(load().bi_decode_attention_scratch_bytes(int(B), int(Hq), int(D), int(Lmax)))


def bi_decode_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                        seq_lens: torch.Tensor, scale: float | None = None,
                        scratch: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """One decode step: q [B, Hq, D], caches [B, Lmax, Hkv, D] (bf16), seq_lens [B] int32."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cuda(t, n, (torch.bfloat16,))
        _contig(t, n)
    _need_cuda(seq_lens, "seq_lens", (torch.int32,))
    _contig(seq_lens, "seq_lens")
    B, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k_cache.shape
    if Bk != B or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(seq_lens.shape) != (B,):
        raise ValueError("shape mismatch between q, caches and seq_lens")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    _need_cuda(out, "out", (torch.bfloat16,))
    _contig(out, "out")
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be [B, Hq, D]")
    if scratch is None:
        scratch = torch.empty(max(bi_decode_attention_scratch_bytes(B, Hq, D, Lmax), 16), dtype=torch.uint8,
                              device=q.device)
    if not scratch.is_cuda:
        raise ValueError("scratch must be device memory")
    _same_device(scratch.get_device(), "scratch")
    nbytes = scratch.numel() * scratch.element_size()
    _check("bi_decode_attention", load().bi_decode_attention(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
        B, Hq, Hkv, D, Lmax, float(scale), scratch.data_ptr(), nbytes, _stream(stream)))
    return out


def bi_get_device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the device status word."""
    v = _i32(0)
    _check("bi_get_device_status", load().bi_get_device_status(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def bi_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("bi_selftest_wait_timeout", load().bi_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def bi_gemm_config(weight_rows: int = 0) -> dict:
    """Tile configuration of the GEMM entry points for an [N, K] weight of `weight_rows` rows
    (N of bi_matmul / bi_addmm, 2F of bi_matmul_silu_mul; <= 0: the 256-column tile)."""
    vals = [_i32(0) for _ in range(5)]
    load().bi_gemm_config(int(weight_rows), *[ctypes.byref(v) for v in vals])
    return dict(zip(("bm", "bn", "bk", "stages", "mma_k"), (int(v.value) for v in vals)))


def bi_tensor_map_cache_stats() -> tuple[int, int]:
    """(hits, misses) of the library's TMA tensor-map cache since it was loaded."""
    h, m = _i64(0), _i64(0)
    load().bi_tensor_map_cache_stats(ctypes.byref(h), ctypes.byref(m))
    return int(h.value), int(m.value)


def bi_version() -> int:
    return int(load().bi_version())
