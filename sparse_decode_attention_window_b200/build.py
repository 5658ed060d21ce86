"""Build libkvc.so in-tree with nvcc for sm_100a (no GPU needed to compile).

    python -m sparse_decode_attention_window_b200.build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkvc.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

SOURCES = ["kvc.cu"]
# every header under csrc/ (the unity build includes them all)
HEADERS = sorted(f for f in os.listdir(CSRC) if f.endswith(".cuh"))


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "kvc.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "--extended-lambda",
           "-I", INCLUDE, "-o", LIB + ".tmp"] + [os.path.join(CSRC, f) for f in SOURCES]
    if extra:
        cmd[1:1] = extra
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = None
    if "--ptxas-v" in args:
        extra = ["-Xptxas", "-v"]
    print(build(force=True, verbose=True, extra=extra))
