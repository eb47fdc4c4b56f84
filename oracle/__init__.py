"""CPU oracle for paged-attention decode — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
the two share no code: this package has its own format codecs, its own
layout arithmetic and its own allocator, all written from the pages:

* "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍" (fudengji.cn):
  - section "真正吃显存的是 KV Cache，不是模型权重": KV bytes per request;
  - section "PagedAttention：把操作系统的虚拟内存搬进 GPU": fixed-size physical
    blocks, a per-sequence block table, on-demand allocation, shared blocks;
  - section "连续批处理：别再等最慢的那个请求了": the scheduling loop
    (free finished requests, admit waiting ones FIFO, decode the running set);
  - section "vLLM 也不是银弹：真实部署中的坑": FP8 KV cache for long contexts.

Numerics live in ``oracle.c`` (plain C, fp64), compiled by :func:`build`
into ``liboracle.so``; the host-side mirrors of the cache write and block copy
are plain numpy here; the allocator and scheduler are in :mod:`oracle.sched`.

Every function here is pinned by ``tests/test_oracle_*.py`` against
something other than itself (library routines, closed forms, invariants,
brute force, the pages' worked example).
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC_PATH = os.path.join(HERE, "oracle.c")

# Element formats (this package's own numbering).
F16, BF16, E4M3, F32 = 0, 1, 2, 3
ELEM_BYTES = {F16: 2, BF16: 2, E4M3: 1, F32: 4}
STORAGE = {F16: np.uint16, BF16: np.uint16, E4M3: np.uint8, F32: np.float32}


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (fp64, OpenMP over (sequence, head) pairs)."""
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC_PATH)):
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", SRC_PATH, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        c_p, c_i, c_d, c_i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int64
        L.oracle_f16_to_double.restype = c_d
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = c_d
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_e4m3_to_double.restype = c_d
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_from_float.restype = ctypes.c_uint8
        L.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        L.oracle_decode_array.restype = None
        L.oracle_decode_array.argtypes = [c_p, c_i, c_i64, c_p]
        L.oracle_e4m3_encode_array.restype = None
        L.oracle_e4m3_encode_array.argtypes = [c_p, c_i64, c_p]
        L.oracle_kv_cache_bytes.restype = c_i64
        L.oracle_kv_cache_bytes.argtypes = [c_i64] * 5
        dec = [c_p, c_p, c_i, c_p, c_p, c_i, c_i, c_i, c_i, c_p, c_i, c_i, c_p, c_i, c_p, c_i, c_d]
        L.oracle_paged_decode.restype = c_i
        L.oracle_paged_decode.argtypes = dec + [c_p]
        L.oracle_paged_decode_partials.restype = c_i
        L.oracle_paged_decode_partials.argtypes = dec + [c_i, c_i, c_p, c_p, c_p]
        L.oracle_paged_prefill.restype = c_i
        L.oracle_paged_prefill.argtypes = [c_p, c_p, c_i, c_p, c_p, c_i, c_i, c_i, c_i, c_p, c_i, c_i,
                                           c_p, c_p, c_i, c_p, c_i, c_d, c_i, c_p]
        L.oracle_lse_merge.restype = None
        L.oracle_lse_merge.argtypes = [c_i64, c_i, c_i, c_p, c_p, c_p, c_p]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ formats

def decode(raw: np.ndarray, fmt: int) -> np.ndarray:
    """Exact float64 values of raw storage (uint16 bits, uint8 codes or f32)."""
    raw = np.ascontiguousarray(raw, dtype=STORAGE[fmt])
    out = np.empty(raw.shape, dtype=np.float64)
    lib().oracle_decode_array(_ptr(raw), fmt, raw.size, _ptr(out))
    return out


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 codes, round-to-nearest-even, saturating at +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def kv_cache_bytes(seq_len: int, layers: int, heads: int, head_dim: int, elem_bytes: int) -> int:
    """KV bytes of one request, per the pages' worked formula."""
    return int(lib().oracle_kv_cache_bytes(seq_len, layers, heads, head_dim, elem_bytes))


# ---------------------------------------------------------------- attention

def paged_decode(k_pool, v_pool, kv_fmt, q, q_fmt, block_tables, context_lens,
                 scale, block_size, k_scale=None, v_scale=None):
    """fp64 decode attention over a paged pool.

    k_pool, v_pool: raw storage shaped [num_blocks][kv_heads][block_size][head_dim]
    q: raw storage [batch][num_q_heads][head_dim]
    block_tables: int32 [batch][max_blocks]; context_lens: int32 [batch]
    k_scale, v_scale: float32 [num_blocks][kv_heads] (FP8 pools only)
    Returns float64 [batch][num_q_heads][head_dim].
    """
    k_pool = _c(k_pool, STORAGE[kv_fmt])
    v_pool = _c(v_pool, STORAGE[kv_fmt])
    q = _c(q, STORAGE[q_fmt])
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    nb, hkv, bs, d = k_pool.shape
    assert bs == block_size
    b, hq, d2 = q.shape
    assert d2 == d and hq % hkv == 0
    out = np.zeros((b, hq, d), dtype=np.float64)
    rc = lib().oracle_paged_decode(_ptr(k_pool), _ptr(v_pool), kv_fmt, _ptr(ks), _ptr(vs),
                                   nb, hkv, bs, d, _ptr(q), q_fmt, hq, _ptr(bt), bt.shape[1],
                                   _ptr(cl), b, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode failed: {rc}")
    return out


def paged_prefill(k_pool, v_pool, kv_fmt, q, q_fmt, cu_q, block_tables, context_lens,
                  scale, block_size, k_scale=None, v_scale=None, window=0):
    """fp64 multi-token (causal) attention over a paged pool.

    Sequence s has its last ``cu_q[s+1] - cu_q[s]`` cached tokens as new
    query tokens; new token i sits at position p = n - q_len + i and attends
    to positions max(0, p - window + 1) .. p (0 .. p when ``window`` is 0).
    q: raw storage [cu_q[-1]][num_q_heads][head_dim]; returns float64 of the
    same shape.  Raises ValueError on a bad block id or q_len > context.
    """
    k_pool = _c(k_pool, STORAGE[kv_fmt])
    v_pool = _c(v_pool, STORAGE[kv_fmt])
    q = _c(q, STORAGE[q_fmt])
    cu = _c(cu_q, np.int32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    nb, hkv, bs, d = k_pool.shape
    assert bs == block_size
    rows, hq, d2 = q.shape
    b = cl.shape[0]
    assert d2 == d and hq % hkv == 0 and cu.shape[0] == b + 1 and int(cu[-1]) == rows
    out = np.zeros((rows, hq, d), dtype=np.float64)
    rc = lib().oracle_paged_prefill(_ptr(k_pool), _ptr(v_pool), kv_fmt, _ptr(ks), _ptr(vs), nb, hkv,
                                    bs, d, _ptr(q), q_fmt, hq, _ptr(cu), _ptr(bt), bt.shape[1],
                                    _ptr(cl), b, float(scale), int(window), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_prefill failed: {rc}")
    return out


def paged_decode_partials(k_pool, v_pool, kv_fmt, q, q_fmt, block_tables, context_lens,
                          scale, block_size, partition_tokens, num_parts,
                          k_scale=None, v_scale=None):
    """Per-partition (o, m, l) in fp64: o [B][Hq][P][D], m and l [B][Hq][P]."""
    k_pool = _c(k_pool, STORAGE[kv_fmt])
    v_pool = _c(v_pool, STORAGE[kv_fmt])
    q = _c(q, STORAGE[q_fmt])
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    nb, hkv, bs, d = k_pool.shape
    b, hq, _ = q.shape
    o = np.zeros((b, hq, num_parts, d), dtype=np.float64)
    m = np.zeros((b, hq, num_parts), dtype=np.float64)
    l = np.zeros((b, hq, num_parts), dtype=np.float64)
    rc = lib().oracle_paged_decode_partials(
        _ptr(k_pool), _ptr(v_pool), kv_fmt, _ptr(ks), _ptr(vs), nb, hkv, bs, d, _ptr(q), q_fmt,
        hq, _ptr(bt), bt.shape[1], _ptr(cl), b, float(scale), int(partition_tokens),
        int(num_parts), _ptr(o), _ptr(m), _ptr(l))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_partials failed: {rc}")
    return o, m, l


def lse_merge(o, m, l):
    """Merge partials [..][P][D], [..][P], [..][P] -> [..][D] (fp64)."""
    o = np.ascontiguousarray(o, dtype=np.float64)
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    lead = o.shape[:-2]
    p, d = o.shape[-2:]
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (d,), dtype=np.float64)
    lib().oracle_lse_merge(rows, p, d, _ptr(o), _ptr(m), _ptr(l), _ptr(out))
    return out


# ------------------------------------------------ cache write and block copy

def kv_write(k_pool, v_pool, kv_fmt, k_new, v_new, src_fmt, slot_mapping, block_size,
             k_inv_scale=None, v_inv_scale=None):
    """Host mirror of the slot-mapped cache write, in place on raw pools.

    Token t's rows new[t][h] (every kv head h) go to physical block
    slot // block_size at offset slot % block_size; a negative slot is
    skipped.  For a 16-bit pool the bits are copied unchanged (the source
    format must equal the pool's).  For an FP8 pool each source value is
    widened to fp32 and multiplied in fp32 by inv_scale[block][h], then
    rounded to E4M3 (nearest even, saturating).  Slots are assumed distinct.
    Raises IndexError for a block outside the pool.
    """
    nb, hkv, bs, d = k_pool.shape
    assert bs == block_size
    slots = np.asarray(slot_mapping, dtype=np.int64).reshape(-1)
    keep = np.nonzero(slots >= 0)[0]
    blk, off = slots[keep] // block_size, slots[keep] % block_size
    if blk.size and blk.max() >= nb:
        raise IndexError("a slot is outside the pool")
    for pool, new, inv in ((k_pool, k_new, k_inv_scale), (v_pool, v_new, v_inv_scale)):
        rows = np.asarray(new)[keep]  # [n][hkv][d] raw source storage
        if kv_fmt == E4M3:
            x = decode(rows, src_fmt).astype(np.float32)  # exact: 16-bit values fit fp32
            # the fp32 product may overflow to +-inf, which the encoder saturates
            with np.errstate(over="ignore"):
                y = (x * np.asarray(inv, np.float32)[blk][:, :, None]).astype(np.float32)
            pool[blk, :, off, :] = e4m3_encode(y)
        else:
            assert src_fmt == kv_fmt
            pool[blk, :, off, :] = rows


def block_copy(pools, pairs):
    """Host mirror of copy-on-write block copies: for each (src, dst) pair and
    every array in ``pools`` (each indexed by physical block first — K and V
    of every layer, and FP8 scale arrays), array[dst] = array[src], pairs
    applied in order."""
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        for arr in pools:
            arr[dst] = arr[src]
