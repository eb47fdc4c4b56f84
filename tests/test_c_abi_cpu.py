"""The boundary from plain C: tests/c/host_abi.c includes include/pagedkv.h
under strict C99 (and C++17), links libpagedkv.so and drives the allocator,
the scheduling step and its packed form with no Python in between (host
entry points only, so no GPU is needed)."""

import os
import shutil
import subprocess

import pytest

import paged_kv_cache_451_b200 as pk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "host_abi.c")
LIBDIR = os.path.dirname(pk.LIB_PATH)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
@pytest.mark.parametrize("compiler,std", [("gcc", ["-x", "c", "-std=c99", "-pedantic"]),
                                          ("g++", ["-x", "c++", "-std=c++17"])])
def test_host_abi_from_c(tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"no {compiler}")
    exe = str(tmp_path / "host_abi")
    cmd = [compiler, *std, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), SRC,
           "-x", "none", "-L", LIBDIR, "-lpagedkv", f"-Wl,-rpath,{LIBDIR}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    lines = run.stdout.splitlines()
    assert len(lines) == 17 and all(ln.startswith("ok ") for ln in lines)
