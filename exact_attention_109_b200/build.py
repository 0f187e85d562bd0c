"""Build libfa_sm100.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", "fa_api.cu"),
           os.path.join(HERE, "csrc", "fa_noalloc.cu")]


def headers():
    """Every header the sources can include: all of csrc/*.cuh and include/*.h."""
    out = []
    for folder, ext in ((os.path.join(HERE, "csrc"), ".cuh"), (os.path.join(ROOT, "include"), ".h")):
        out += sorted(os.path.join(folder, f) for f in os.listdir(folder) if f.endswith(ext))
    return out

OUT = os.path.join(HERE, "libfa_sm100.so")


def nvcc_command(out: str = OUT, extra=()):
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
            "-I", os.path.join(ROOT, "include"), "-o", out, *SOURCES, *extra]


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(f) <= t for f in SOURCES + headers())


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        extra = ["-Xptxas", "-v"] if verbose else []
        subprocess.run(nvcc_command(extra=extra), check=True)
    return OUT


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(OUT)
