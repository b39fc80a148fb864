"""Build libaaac.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m activation_aware_codebook_b200.csrc.build [--force] [--verbose] [--checks]

Each .cu file is compiled separately (-gencode arch=compute_100a,code=sm_100a,
-O3, -lineinfo) and linked with -shared into activation_aware_codebook_b200/
libaaac.so.  No PyTorch headers are involved.

--checks builds the debugging variant libaaac_checked.so instead (objects in
their own folder), compiled with -DAAAC_CHECKS: its kernels test the indices
they compute and record the first failure, read by aaac_device_checks.  The
binding loads it when AAAC_CHECKED=1 is set.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libaaac.so")
LIB_CHECKED = os.path.join(PKG, "libaaac_checked.so")
SOURCES = ["api.cu", "importance.cu", "init.cu", "fit.cu", "linear.cu", "gemm.cu", "awq.cu"]
BUILD_DIR = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "-I", INCLUDE, "-I", HERE]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    lib = LIB_CHECKED if checks else LIB
    bdir = os.path.join(BUILD_DIR, "checked") if checks else BUILD_DIR
    extra = ["-DAAAC_CHECKS"] if checks else []
    os.makedirs(bdir, exist_ok=True)
    headers = [os.path.join(HERE, h) for h in os.listdir(HERE) if h.endswith((".cuh", ".h"))]
    headers.append(os.path.join(INCLUDE, "aaac.h"))
    objs = []
    for src in SOURCES:
        s = os.path.join(HERE, src)
        o = os.path.join(bdir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers):
            cmd = ([NVCC] + ARCH + FLAGS + extra + (["-Xptxas", "-v"] if verbose else [])
                   + ["-c", s, "-o", o])
            subprocess.run(cmd, check=True)
    if force or _stale(lib, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", lib + ".tmp"] + objs + ["-lcudart"]
        subprocess.run(cmd, check=True)
        os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checks="--checks" in sys.argv))
