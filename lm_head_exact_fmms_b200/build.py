"""Build libfmms.so (the C-ABI library of include/fmms.h) for sm_100a with nvcc.

Usage: python -m lm_head_exact_fmms_b200.build [--force]

The library is built in-tree next to this file.  The fused kernel's modes
are instantiated in separate translation units (fmms_inst_*.cu), compiled in
parallel.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfmms.so")
OBJDIR = os.path.join(HERE, "_build")
SOURCES = ["fmms_inst_flat.cu", "fmms_inst_flat_pair.cu", "fmms_inst_grouped.cu",
           "fmms_inst_grouped_pair.cu", "fmms_inst_logits.cu", "fmms_kernel.cu", "aux_kernels.cu",
           "api.cu"]
HEADERS = ["fmms_kernel.cuh", "fmms_common.cuh", "sm100.cuh", "noise.cuh", "launch.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "fmms.h"))
    return files


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src, extra):
    obj = os.path.join(OBJDIR, os.path.splitext(src)[0] + ".o")
    cmd = [NVCC] + ARCH + FLAGS + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
    subprocess.run(cmd, check=True)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), SOURCES))
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart_static", "-ldl",
                                                                     "-lrt", "-lpthread"],
                   check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv))
