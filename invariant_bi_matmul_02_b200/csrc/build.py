"""Build libbi.so (the CUDA kernels and the C ABI of include/bi.h) for sm_100a with nvcc.

The library is built in-tree next to the Python binding, with the CUDA runtime
linked statically, so it loads without a GPU and carries no JIT cache.
"""
import os
import subprocess
import sys

CSRC = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(CSRC)
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
SOURCES = [os.path.join(CSRC, "bi.cu")]
DEPS = SOURCES + [os.path.join(CSRC, n) for n in ("gemm.cuh", "gemm_pair.cuh", "rowops.cuh", "maxsum.cuh", "ptx.cuh", "attention.cuh")] + [
    os.path.join(INCLUDE, "bi.h")]
LIB = os.path.join(PKG, "libbi.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def nvcc():
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(home, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def build(force: bool = False, out: str = LIB, defines=(), verbose: bool = False) -> str:
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(p) for p in DEPS)
        if os.path.getmtime(out) >= newest:
            return out
    cmd = [nvcc(), *NVCC_FLAGS, "-I" + INCLUDE, *[f"-D{d}" for d in defines]]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", out, *SOURCES, "-ldl", "-lpthread", "-lrt"]
    subprocess.run(cmd, check=True)
    return out


PROBE_SRC = os.path.join(CSRC, "mma_probe.cu")
PROBE = os.path.join(PKG, "mma_probe")


def build_probe(force: bool = False) -> str:
    """The tcgen05 MMA cost probe (a stand-alone program, not part of libbi.so)."""
    deps = [PROBE_SRC, os.path.join(CSRC, "ptx.cuh")]
    if not force and os.path.exists(PROBE) and os.path.getmtime(PROBE) >= max(os.path.getmtime(p) for p in deps):
        return PROBE
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I" + CSRC, "-o", PROBE,
           PROBE_SRC]
    subprocess.run(cmd, check=True)
    return PROBE


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
