"""The native library loads, exports every entry point the header declares,
and rejects bad arguments on the host before touching the GPU."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

import paged_kv_cache_451_b200 as pk

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-zA-Z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 30
    lib = ctypes.CDLL(pk.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(pk.EXPORTED)


def test_only_abi_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", pk.LIB_PATH], capture_output=True, text=True).stdout
    syms = [ln.split()[-1] for ln in out.splitlines() if " T " in ln]
    assert syms and all(s.startswith(("kv_", "paged_", "block_copy")) for s in syms), syms


def test_version_and_error_string():
    assert pk.kv_version() == 1
    with pytest.raises(pk.KVError) as e:
        pk.kv_pool_create(15, 10, 1, 128, pk.KV_F16)
    assert e.value.code == pk.KV_ERR_ARG
    assert "block_size" in pk.kv_last_error()


@pytest.mark.parametrize("args", [
    (16, 0, 1, 128, pk.KV_F16, 1),      # no blocks
    (16, 4, 1, 96, pk.KV_F16, 1),       # head_dim
    (24, 4, 1, 128, pk.KV_F16, 1),      # block size not a multiple of 16
    (48, 4, 1, 128, pk.KV_F16, 1),      # block size not a power of two
    (16, 4, 1, 128, pk.KV_F32, 1),      # pool dtype
    (16, 4, 0, 128, pk.KV_BF16, 1),     # kv heads
    (16, 4, 1, 128, pk.KV_BF16, 0),     # layers
])
def test_pool_create_rejects_bad_geometry(args):
    with pytest.raises(pk.KVError) as e:
        pk.kv_pool_create(*args)
    assert e.value.code == pk.KV_ERR_ARG


def test_pool_bytes_and_workspace_sizes():
    pool = pk.kv_pool_create(16, 100, 8, 128, pk.KV_BF16, 2)
    kvb, sb = pk.kv_pool_bytes(pool)
    assert kvb == 100 * 8 * 16 * 128 * 2 and sb == 0
    # split partials (head_dim + 4 floats per partition and query head) plus
    # one int merge counter per (sequence, kv head), padded to 16 bytes
    def ws(b, parts):
        return b * 64 * parts * 132 * 4 + (b * 8 * 4 + 15) // 16 * 16

    # automatic policy: partitions of at most 4096 tokens ...
    assert pk.paged_attention_workspace_bytes(pool, 512, 64, 4096) == 0
    assert pk.paged_attention_workspace_bytes(pool, 512, 64, 8192) == ws(512, 2)
    # ... and more, down to 512 tokens, when there are few (sequence, kv head) units
    assert pk.paged_attention_workspace_bytes(pool, 4, 64, 1024) == ws(4, 2)
    assert pk.paged_attention_workspace_bytes(pool, 4, 64, 512) == 0
    pk.kv_pool_set_decode_config(pool, 4096, 0, 0)
    assert pk.paged_attention_workspace_bytes(pool, 4, 64, 4096) == 0
    pk.kv_pool_set_decode_config(pool, 256, 2, 4)
    assert pk.paged_attention_workspace_bytes(pool, 4, 64, 513) == ws(4, 3)
    for bad in ((8, 0, 0), (16400, 0, 0), (100, 0, 0), (0, 5, 0), (0, 1, 0), (0, 7, 0), (0, 0, 6), (0, 4, 8)):
        with pytest.raises(pk.KVError):
            pk.kv_pool_set_decode_config(pool, *bad)
    pk.kv_pool_destroy(pool)
    fp8 = pk.kv_pool_create(32, 10, 4, 64, pk.KV_FP8_E4M3, 1)
    assert pk.kv_pool_bytes(fp8) == (10 * 4 * 32 * 64, 10 * 4 * 4)
    pk.kv_pool_destroy(fp8)


@pytest.mark.skipif(torch.cuda.is_available(), reason="on a GPU the policy sees the device's real occupancy")
def test_partition_count_fills_the_last_wave():
    """Without a device the policy counts one resident CTA per SM on 148
    SMs.  2 x 16K-token FP8 contexts with 32 kv heads are 64 units: four
    waves need 10 partitions (640 CTAs, 4.3 waves, the last one 32% full);
    the count is raised to 16 (1024 CTAs, 6.9 waves, the last 92% full) of
    1024 tokens each.  A forced partition length is kept as it is."""
    fp8 = pk.kv_pool_create(16, 4096, 32, 128, pk.KV_FP8_E4M3, 1)
    per = 132 * 4  # head_dim + 4 floats per (sequence, head, partition)
    counters = (2 * 32 * 4 + 15) // 16 * 16
    assert pk.paged_attention_workspace_bytes(fp8, 2, 32, 16384) == 2 * 32 * 16 * per + counters
    # 8 sequences: 256 units, 4 partitions already fill 92% of their last wave
    assert pk.paged_attention_workspace_bytes(fp8, 8, 32, 16384) == 8 * 32 * 4 * per + (8 * 32 * 4 + 15) // 16 * 16
    pk.kv_pool_set_decode_config(fp8, 512, 0, 0)
    assert pk.paged_attention_workspace_bytes(fp8, 2, 32, 16384) == 2 * 32 * 32 * per + counters
    pk.kv_pool_destroy(fp8)


def test_gpu_entries_reject_bad_arguments_before_launch():
    pool = pk.kv_pool_create(16, 8, 2, 64, pk.KV_F16, 1)
    # layer not bound
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_decode(pool, 0, 16, pk.KV_F16, 2, 16, 1, 16, 1, 16, 0.1, 16, pk.KV_F16, stream=0)
    assert e.value.code == pk.KV_ERR_STATE
    with pytest.raises(pk.KVError) as e:
        pk.paged_kv_write(pool, 0, 16, 16, pk.KV_F16, 16, 1, stream=0)
    assert e.value.code == pk.KV_ERR_STATE
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_decode(pool, 3, 16, pk.KV_F16, 2, 16, 1, 16, 1, 16, 0.1, 16, pk.KV_F16, stream=0)
    assert e.value.code == pk.KV_ERR_ARG
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_prefill(pool, 0, 16, pk.KV_F16, 2, 16, 4, 4, 16, 1, 16, 1, 0.1, 16,
                                   pk.KV_F16, stream=0)
    assert e.value.code == pk.KV_ERR_STATE
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_prefill(pool, -1, 16, pk.KV_F16, 2, 16, 4, 4, 16, 1, 16, 1, 0.1, 16,
                                   pk.KV_F16, stream=0)
    assert e.value.code == pk.KV_ERR_ARG
    with pytest.raises(pk.KVError) as e:
        pk.block_copy(pool, 16, -1, stream=0)
    assert e.value.code == pk.KV_ERR_ARG
    with pytest.raises(pk.KVError):
        pk.kv_selftest_wait_timeout(0, stream=0)
    with pytest.raises(pk.KVError):
        pk.kv_pool_bind(pool, 0, 0, 0)
    with pytest.raises(pk.KVError):
        pk.kv_pool_bind(pool, 0, 24, 32)  # misaligned
    pk.kv_pool_destroy(pool)
