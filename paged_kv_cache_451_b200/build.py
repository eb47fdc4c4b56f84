"""Build the native library libpagedkv.so in-tree with nvcc (sm_100a only)."""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpagedkv.so")
SOURCES = [os.path.join(CSRC, "pagedkv.cu"), os.path.join(CSRC, "prefill.cu"),
           os.path.join(CSRC, "alloc.cpp"), os.path.join(CSRC, "serve.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [
    os.path.join(ROOT, "include", "pagedkv.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared",
           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
           "-I", os.path.join(ROOT, "include"), "-o", out] + SOURCES
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS if os.path.exists(f))


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run(command(tmp, verbose_ptxas), check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="-v" in sys.argv)
    print(LIB)
