"""Builds the CUDA library libgptlayer.so in-tree for sm_100a.

    python -m transformer_layer_step_b200.build

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically,
so the library needs only the NVIDIA driver at run time; the TMA encoder is
taken from the driver through the runtime's entry-point query.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libgptlayer.so")
SOURCES = [os.path.join(PKG, "csrc", "libgptlayer.cu")]


def deps() -> list:
    """Every source and header the library is built from (rebuild if any is newer)."""
    out = []
    for d, exts in ((os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")),
                    (os.path.join(ROOT, "include"), (".h",))):
        out += [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith(exts)]
    return out + [os.path.abspath(__file__)]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=()) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++20", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2", "-shared",
            "-cudart", "static", "-I", os.path.join(ROOT, "include"), *extra,
            "-o", out, *SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = command()
    if verbose:
        print(" ".join(cmd), flush=True)
    tmp = LIB + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
