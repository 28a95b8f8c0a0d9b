"""Builds libecf8.so (host encoder + sm_100a decode kernels) in this directory."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libecf8.so")
# the same library with every kernel store and table read bounds-checked
# (-DECF8_CHECKED): a failed check sets ECF8_STATUS_BOUNDS instead of accessing
CHECKED_SO = os.path.join(HERE, "libecf8_checked.so")
SOURCES = [os.path.join(CSRC, f) for f in ("ecf8_host.cpp", "ecf8_decode.cu", "ecf8_pipeline.cpp", "ecf8_encode.cu",
                                                 "ecf8_bf16_host.cpp", "ecf8_bf16_decode.cu")]
HEADERS = [os.path.join(ROOT, "include", "ecf8.h"), os.path.join(CSRC, "ecf8_format.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC,-fopenmp,-O3",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale(so: str = SO) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    so = CHECKED_SO if checked else SO
    if force or stale(so):
        cmd = [nvcc(), *NVCC_FLAGS, *(["-DECF8_CHECKED"] if checked else []), "-I" + os.path.join(ROOT, "include"),
               "-I" + CSRC, "-o", so, *SOURCES, "-lgomp"]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
    return so


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
