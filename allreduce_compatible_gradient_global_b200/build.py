"""Build libgq.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

    python -m allreduce_compatible_gradient_global_b200.build [--force] [--check]

Plain nvcc, one shared library, no JIT: the library lands next to this file so
it ships with the source tree.  --check also prints ptxas register and spill
counts (-Xptxas -v).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libgq.so")

SOURCES = ["gq_api.cu", "gq_kernels.cu", "gq_quant_tma.cu", "gq_bucket.cu", "gq_psgd.cu", "gq_logq.cu", "gq_noalloc.cu", "gq_nat.cu"]
HEADERS = ["gq_device.cuh", "gq_internal.h", "gq_pdl.cuh", "gq_psgd.h", "gq_nat.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "gq_api.h"))
    return files


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    newest = max(os.path.getmtime(f) for f in _inputs())
    if not force and not verbose_ptxas and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    cmd += ["-o", tmp, "-lcudart"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--check" in sys.argv))
