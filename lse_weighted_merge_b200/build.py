"""Build the C-ABI shared library (liblse_merge.so) in-tree with nvcc for sm_100a,
and the small CPython extension (_fast) that forwards its per-call entry points.

    python -m lse_weighted_merge_b200.build [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblse_merge.so")
SOURCES = [os.path.join(CSRC, "plan.cpp"), os.path.join(CSRC, "lse_merge.cu"),
           os.path.join(CSRC, "decode_attention.cu"), os.path.join(CSRC, "cp_exchange.cu"),
           os.path.join(CSRC, "host_pipeline.cpp")]
HEADERS = [os.path.join(INCLUDE, "lse_merge.h"), os.path.join(CSRC, "plan.h"),
           os.path.join(CSRC, "device_common.cuh")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in SOURCES + HEADERS)


FAST_SRC = os.path.join(CSRC, "pyfast.c")


def fast_path() -> str:
    """In-tree path of the CPython extension that forwards the per-call entry points."""
    import sysconfig
    return os.path.join(PKG, "_fast" + sysconfig.get_config_var("EXT_SUFFIX"))


def build_fast(lib: str = LIB) -> str:
    """Compile pyfast.c (gcc, CPython headers) against liblse_merge.so, found at
    run time next to the extension ($ORIGIN)."""
    import sysconfig
    out = fast_path()
    cmd = ["gcc", "-O2", "-shared", "-fPIC", "-std=c11", "-I", INCLUDE,
           "-I", sysconfig.get_paths()["include"], FAST_SRC, "-L", os.path.dirname(lib),
           "-l:" + os.path.basename(lib), "-Wl,-rpath,$ORIGIN", "-o", out]
    subprocess.run(cmd, check=True)
    return out


def build(out: str = LIB, verbose: bool = False, extra: list[str] | None = None) -> str:
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", out]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    subprocess.run(cmd, check=True)
    if out == LIB:
        build_fast(out)
    return out


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv)
    print(LIB)
    print(fast_path())
