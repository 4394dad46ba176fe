"""CPU-only checks of the C ABI: libbi.so loads, exports every entry point the header
declares, and rejects bad arguments on the host before touching a GPU.
"""
import ctypes
import os
import re

import pytest

from invariant_bi_matmul_02_b200 import binding
from invariant_bi_matmul_02_b200.csrc import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bi.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return binding.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("bi_matmul", "bi_addmm", "bi_rmsnorm", "bi_mean", "bi_log_softmax", "bi_silu_mul",
              "bi_get_device_status", "bi_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/bi.h but not exported"
    assert set(declared_functions()) == set(binding.SIGNATURES), "binding and header disagree"


def test_status_strings_and_config(lib):
    assert binding.status_string(binding.BI_OK) == "BI_OK"
    assert binding.status_string(binding.BI_ERR_TIMEOUT) == "BI_ERR_TIMEOUT"
    assert binding.status_string(99) == "BI_ERR_UNKNOWN"
    wide = binding.bi_gemm_config()
    # 256-column tiles where 192-column ones would not save a cost-weighted wave at 1024 rows
    # on 74 CTA pairs: q/o and down (4096 rows: 16 against 22 tiles per tile row, 1 wave against
    # 2), gate/up unfused (12288: 3 waves against 4 x 0.8), the LM head (151936: 33 against 43)
    for rows in (151936, 12288, 4096):
        assert binding.bi_gemm_config(rows) == wide, rows
    assert wide["bm"] == 256 and wide["bn"] == 256 and wide["bk"] == 64 and wide["mma_k"] == 16
    # 192-column tiles: fused q/k/v (6144: 2 waves against 2 x 0.8), fused gate/up (24576:
    # 6 against 7 x 0.8), and widths just above the narrow range (1025: 1 against 1 x 0.8)
    mid = binding.bi_gemm_config(6144)
    for rows in (24576, 2048, 1025):
        assert binding.bi_gemm_config(rows) == mid, rows
    assert mid["bm"] == 256 and mid["bn"] == 192 and mid["bk"] == 128 and mid["mma_k"] == 16
    narrow = binding.bi_gemm_config(1024)
    assert narrow == binding.bi_gemm_config(1)
    assert narrow["bm"] == 256 and narrow["bn"] == 128 and narrow["bk"] == 128 and narrow["mma_k"] == 16
    # every stage fits in the 227 KB a CTA may use, with room for the barriers
    for cfg in (wide, mid, narrow):
        assert cfg["stages"] >= 2
        assert cfg["stages"] * (128 + cfg["bn"] // 2) * cfg["bk"] * 2 <= 227 * 1024 - 1536
    assert binding.bi_version() >= 201


NULL = None


def test_host_validation_without_a_gpu(lib):
    I = binding.BI_ERR_INVALID_ARG
    U = binding.BI_ERR_UNSUPPORTED
    A = binding.BI_ERR_ALIGNMENT
    # negative sizes, bad enums, null pointers
    assert lib.bi_matmul(NULL, 8, NULL, 8, 1, NULL, 8, 0, -1, 8, 8, NULL) == I
    assert lib.bi_matmul(NULL, 8, NULL, 8, 7, NULL, 8, 0, 1, 8, 8, NULL) == I
    assert lib.bi_matmul(NULL, 8, NULL, 8, 1, NULL, 8, 5, 1, 8, 8, NULL) == I
    assert lib.bi_matmul(NULL, 8, NULL, 8, 1, NULL, 8, 0, 1, 8, 8, NULL) == I
    assert lib.bi_matmul(NULL, 8, NULL, 8, 1, NULL, 8, 0, 1 << 31, 8, 8, NULL) == U
    # leading dimension too small, misaligned pointers / leading dims
    fake = 0x10000
    assert lib.bi_matmul(fake, 4, fake, 8, 1, fake, 8, 0, 2, 8, 8, NULL) == I
    assert lib.bi_matmul(fake + 2, 8, fake, 8, 1, fake, 8, 0, 2, 8, 8, NULL) == A
    assert lib.bi_matmul(fake, 12, fake, 8, 1, fake, 8, 0, 2, 8, 8, NULL) == A
    assert lib.bi_matmul(fake, 8, fake, 8, 1, fake, 12, 0, 2, 8, 8, NULL) == A
    assert lib.bi_addmm(NULL, 0, fake, 8, fake, 8, 1, fake, 8, 0, 2, 8, 8, NULL) == I
    assert lib.bi_addmm(fake, 4, fake, 8, fake, 8, 1, fake, 8, 0, 2, 8, 8, NULL) == I
    # M = 0 is a no-op that succeeds without a device
    assert lib.bi_matmul(NULL, 8, NULL, 8, 1, NULL, 8, 0, 0, 8, 8, NULL) == binding.BI_OK
    assert lib.bi_rmsnorm(NULL, NULL, NULL, 0, 8, ctypes.c_float(1e-6), NULL) == binding.BI_OK
    # row ops
    assert lib.bi_rmsnorm(NULL, NULL, NULL, 2, 8, ctypes.c_float(1e-6), NULL) == I
    assert lib.bi_rmsnorm(fake, fake, fake, 2, 8, ctypes.c_float(-1.0), NULL) == I
    assert lib.bi_rmsnorm(fake + 2, fake, fake, 2, 8, ctypes.c_float(1e-6), NULL) == A
    assert lib.bi_mean(NULL, NULL, 2, 8, NULL) == I
    assert lib.bi_mean(fake + 4, fake, 2, 8, NULL) == A
    assert lib.bi_log_softmax(fake, 9, fake, 2, 8, NULL) == I
    assert lib.bi_log_softmax(fake + 4, 1, fake, 2, 8, NULL) == A
    assert lib.bi_silu_mul(NULL, NULL, 2, 8, NULL) == I
    # fused gate/up with [K, 2F] weights: the up half's first column F must be a multiple of 8
    assert lib.bi_matmul_silu_mul(fake, 200, fake, 1000, 0, fake, 504, 77, 500, 200, NULL) == A
    assert lib.bi_selftest_wait_timeout(10, NULL) == I
    # decode attention: shapes the kernel does not take are refused before any pointer is read
    da = lib.bi_decode_attention
    assert da(fake, fake, fake, fake, fake, 2, 32, 8, 96, 128, 1.0, fake, 1 << 20, NULL) == U  # D not 64 or 128
    assert da(fake, fake, fake, fake, fake, 2, 24, 8, 128, 128, 1.0, fake, 1 << 20, NULL) == U  # group 3
    assert da(fake, fake, fake, fake, fake, 2, 30, 8, 128, 128, 1.0, fake, 1 << 20, NULL) == I  # Hq % Hkv
    # B * Hkv * splits must stay below 2^31 (work items are 32-bit indices)
    assert da(fake, fake, fake, fake, fake, 60000, 40000, 40000, 128, 128, 1.0, fake, 1 << 20, NULL) == U
    v = ctypes.c_int32(0)
    assert lib.bi_get_device_status(NULL, None) == I


def test_binding_refuses_cpu_tensors():
    import torch
    a = torch.zeros(2, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.bi_matmul(a, a, "nk")
    with pytest.raises(ValueError):
        binding.bi_mean(a.float())


def test_binding_refuses_a_tensor_or_stream_off_the_current_device(monkeypatch):
    """The C ABI runs on the current device; a tensor or stream of another device is refused in
    the binding before anything is launched."""
    monkeypatch.setattr(binding, "_current_device", lambda: 1)
    binding._same_device(1, "x")
    with pytest.raises(ValueError, match="current device is cuda:1"):
        binding._same_device(0, "x")


def test_missing_library_fails_loudly(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(RuntimeError, match="libbi.so not found"):
            binding.load(str(tmp_path / "libbi.so"))
    finally:
        binding._lib = saved


def test_product_path_and_oracle_share_nothing():
    """The CUDA path (package, kernels, header) never names the oracle, and the oracle never
    names the package or its kernels: the two meet only in the tests, the smoke check and the
    benchmark's CPU baseline."""
    import glob
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    product = (glob.glob(os.path.join(root, "invariant_bi_matmul_02_b200", "*.py"))
               + glob.glob(os.path.join(root, "invariant_bi_matmul_02_b200", "csrc", "*"))
               + glob.glob(os.path.join(root, "include", "*.h")))
    for path in product:
        if os.path.isdir(path) or path.endswith((".so", ".pyc")):
            continue
        text = open(path, errors="replace").read()
        code = "\n".join(l for l in text.splitlines() if "import" in l or "#include" in l)
        assert not re.search(r"\boracle\b", code), f"{path} imports the oracle"
    for path in glob.glob(os.path.join(root, "oracle", "*.[pc]*")):
        text = open(path, errors="replace").read()
        assert "invariant_bi_matmul_02_b200" not in text and "csrc" not in text, f"{path} uses the CUDA path"
