"""Build libgdr.so in-tree with nvcc for sm_100a (one object per .cu, then a
shared link with the static CUDA runtime).  build(checked=True) builds the
checked variant libgdr_check.so (-DGDR_CHECK: every kernel guards its
accesses; see include/gdr.h) from the same sources into its own objects."""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libgdr.so")
BUILD_CHECK = os.path.join(HERE, "_build_check")
LIB_CHECK = os.path.join(HERE, "libgdr_check.so")
SOURCES = ["gdr_api.cu", "decode.cu", "fwd_simt.cu", "fwd_tc.cu", "fwd_noalloc.cu", "product.cu",
           "frame.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, extra_flags=(), checked: bool = False) -> str:
    build_dir, lib_path = (BUILD_CHECK, LIB_CHECK) if checked else (BUILD, LIB)
    flags = FLAGS + (["-DGDR_CHECK"] if checked else [])
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(INCLUDE, "gdr.h"))

    def compile_one(src):
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        srcp = os.path.join(CSRC, src)
        if _newer(obj, [srcp, __file__] + headers) and not extra_flags:
            return obj
        cmd = [NVCC, *flags, *extra_flags, "-c", srcp, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        return obj

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    if not _newer(lib_path, objs) or extra_flags:
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               "-o", lib_path, *objs]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
    return lib_path


if __name__ == "__main__":
    print(build(verbose=True, checked="--checked" in sys.argv[1:]))
