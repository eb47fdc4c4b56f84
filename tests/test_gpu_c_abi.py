"""The GPU path driven from plain C, with no Python in between.
tests/c/decode_from_c.c allocates device memory with the CUDA runtime, binds
a pool and runs paged_kv_write and paged_attention_decode through
include/pagedkv.h; tests/c/serve_from_c.c runs the continuous-batching loop
(allocator, scheduler, kv_serve_* over three buffer sets with host staging).
Pools must equal the oracle's mirror bit for bit, outputs the fp64 oracle
within the fp16/bf16 bound."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import paged_kv_cache_451_b200 as pk
from oracle.sched import BlockManager, Scheduler
from gpu_util import TOL, max_abs
from workloads import BF16, normal_bits, scattered_tables

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "decode_from_c.c")
SERVE_SRC = os.path.join(ROOT, "tests", "c", "serve_from_c.c")
CUDA = "/usr/local/cuda"


def compile_c(src, exe):
    libdir = os.path.dirname(pk.LIB_PATH)
    subprocess.run(["gcc", "-std=gnu11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"), src, "-L", libdir, "-lpagedkv",
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{libdir}",
                    f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe], check=True, capture_output=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_write_and_decode_from_c(tmp_path):
    rng = np.random.default_rng(404)
    nb, bs, hkv, d, hq = 64, 16, 2, 128, 8
    lens = np.array([1, 17, 300, 33, 250], np.int32)
    b = len(lens)
    tables = scattered_tables(rng, lens, bs, nb)
    shape = (nb, hkv, bs, d)
    kh, vh = normal_bits(rng, shape, BF16), normal_bits(rng, shape, BF16)
    q = normal_bits(rng, (b, hq, d), BF16)
    kn, vn = normal_bits(rng, (b, hkv, d), BF16), normal_bits(rng, (b, hkv, d), BF16)
    pos = lens - 1  # each sequence's newest token
    slots = (tables[np.arange(b), pos // bs].astype(np.int64) * bs + pos % bs).astype(np.int64)
    scale = np.float32(1.0 / np.sqrt(d))
    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        f.write(np.array([nb, bs, hkv, d, hq, b, tables.shape[1], b], np.int32).tobytes())
        f.write(np.array([scale], np.float32).tobytes())
        for a in (kh, vh, q, kn, vn):
            f.write(np.ascontiguousarray(a).tobytes())
        f.write(np.ascontiguousarray(tables, np.int32).tobytes())
        f.write(lens.tobytes())
        f.write(slots.tobytes())
    exe = str(tmp_path / "decode_from_c")
    compile_c(SRC, exe)
    out_path = tmp_path / "out.bin"
    run = subprocess.run([exe, str(inp), str(out_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
    res = np.fromfile(out_path, np.uint8)
    pool_n = kh.nbytes
    k_after = res[:pool_n].view(np.uint16).reshape(shape)
    out = res[pool_n:].view(np.float32).reshape(b, hq, d)
    kref, vref = kh.copy(), vh.copy()
    oracle.kv_write(kref, vref, BF16, kn, vn, BF16, slots, bs)
    assert np.array_equal(k_after, kref)
    ref = oracle.paged_decode(kref, vref, BF16, q, BF16, tables, lens, float(scale), bs)
    assert max_abs(out, ref) <= TOL[BF16]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_serving_loop_from_c(tmp_path):
    rng = np.random.default_rng(505)
    nb, bs, hkv, d, hq, steps = 64, 16, 2, 128, 8, 4
    scale = np.float32(1.0 / np.sqrt(d))
    order = rng.permutation(nb).astype(np.int32)
    reqs = [(7, 20), (8, 33), (9, 5)]
    bm = BlockManager(nb, bs, order)
    sch = Scheduler(bm, 4)
    for sid, plen in reqs:
        sch.add_request(sid, plen)
    shape = (nb, hkv, bs, d)
    kh, vh = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    inp = tmp_path / "in.bin"
    refs = []
    with open(inp, "wb") as f:
        f.write(np.array([nb, bs, hkv, d, hq, steps, len(reqs)], np.int32).tobytes())
        f.write(np.array([scale], np.float32).tobytes())
        f.write(order.tobytes())
        for sid, plen in reqs:
            f.write(np.array([sid], np.int64).tobytes() + np.array([plen], np.int32).tobytes())
        for _ in range(steps):
            want = sch.step([])
            T, B = len(want["slot_mapping"]), len(want["running"])
            q = normal_bits(rng, (B, hq, d), BF16)
            kn, vn = normal_bits(rng, (T, hkv, d), BF16), normal_bits(rng, (T, hkv, d), BF16)
            f.write(np.array([T, B], np.int32).tobytes())
            for a in (q, kn, vn):
                f.write(np.ascontiguousarray(a).tobytes())
            oracle.block_copy([kh, vh], want["cow_pairs"])
            oracle.kv_write(kh, vh, BF16, kn, vn, BF16, want["slot_mapping"], bs)
            width = max(len(t) for t in want["block_tables"])
            tables = np.full((B, width), -1, np.int32)
            for i, t in enumerate(want["block_tables"]):
                tables[i, :len(t)] = t
            lens = np.array(want["context_lens"], np.int32)
            refs.append(oracle.paged_decode(kh, vh, BF16, q, BF16, tables, lens, float(scale), bs))
    exe = str(tmp_path / "serve_from_c")
    compile_c(SERVE_SRC, exe)
    out_path = tmp_path / "out.bin"
    run = subprocess.run([exe, str(inp), str(out_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
    res = np.fromfile(out_path, np.uint8)
    off = 0
    for step, ref in enumerate(refs):
        n = ref.size * 4
        got = res[off:off + n].view(np.float32).reshape(ref.shape)
        off += n
        assert max_abs(got, ref) <= TOL[BF16], f"step {step}"
    assert np.array_equal(res[off:off + kh.nbytes].view(np.uint16).reshape(shape), kh)
    assert np.array_equal(res[off + kh.nbytes:].view(np.uint16).reshape(shape), vh)
