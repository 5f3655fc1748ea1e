"""Build libfmms.so (the C-ABI library of include/fmms.h) for sm_100a with nvcc.

Usage: python -m lm_head_exact_fmms_b200.build [--force] [--debug]

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
# The debug build: the same sources with -DFS_DEBUG (device-side bounds checks
# that report FS_ERR_DEVICE_BOUNDS through the status word instead of trapping).
DEBUG_LIB = os.path.join(HERE, "libfmms_debug.so")
DEBUG_OBJDIR = os.path.join(HERE, "_build", "debug")
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


def needs_build(lib=LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src, extra, objdir):
    obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
    cmd = [NVCC] + ARCH + FLAGS + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
    subprocess.run(cmd, check=True)
    return obj


def _link(lib, objs):
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart_static", "-ldl",
                                                                     "-lrt", "-lpthread"],
                   check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Builds libfmms.so (or, with debug=True, libfmms_debug.so) if a source
    is newer than it; returns its path."""
    lib, objdir = (DEBUG_LIB, DEBUG_OBJDIR) if debug else (LIB, OBJDIR)
    if not force and not needs_build(lib):
        return lib
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if debug:
        extra = extra + ["-DFS_DEBUG"]
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, objdir), SOURCES))
    _link(lib, objs)
    return lib


def build_all(force: bool = False) -> list:
    """Both libraries: the release build and the debug build."""
    return [build(force=force), build(force=force, debug=True)]


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv,
                debug="--debug" in sys.argv))
