"""Decode for callers that cannot allocate device memory.

Some callers have no way to call cudaMalloc: a plain C host program or a
plugin that only receives the cache pool and its input tensors, a process
whose device memory is entirely handed to the KV pool, or a hot path that
must not call cudaMalloc because it can synchronise the device.
paged_attention_decode_noalloc serves them from a fixed scratch array that
the library keeps in device memory.  These tests call it through the C ABI
and check that it returns what paged_attention_decode returns with a caller
workspace, on two calls in a row that both split their contexts (so the
shared scratch is really used, and reused): bit for bit, since both run the
same kernels with the same partitioning, and against the fp64 oracle within
the tolerance of the other decode tests."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, DevicePool, decode, dev, max_abs
from workloads import BF16, E4M3, e4m3_codes, fp8_scales, normal_bits, scattered_tables

pytestmark = pytest.mark.gpu


def make(kv_fmt, q_fmt, hq, hkv, lens, seed, partition):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    bs, d = 16, 128
    nb = int(sum(-(-int(n) // bs) for n in lens)) + 3
    shape = (nb, hkv, bs, d)
    if kv_fmt == E4M3:
        k, v = e4m3_codes(rng, shape), e4m3_codes(rng, shape)
        ks, vs = fp8_scales(rng, (nb, hkv)), fp8_scales(rng, (nb, hkv))
    else:
        k, v = normal_bits(rng, shape, kv_fmt), normal_bits(rng, shape, kv_fmt)
        ks = vs = None
    pool = DevicePool(nb, hkv, d, bs, kv_fmt, k=[dev(k)], v=[dev(v)],
                      k_scale=None if ks is None else [dev(ks)], v_scale=None if vs is None else [dev(vs)],
                      partition=partition)
    tables = scattered_tables(rng, lens, bs, nb)
    q = normal_bits(rng, (len(lens), hq, d), q_fmt)
    ref = oracle.paged_decode(k, v, kv_fmt, q, q_fmt, tables, lens, 1.0 / math.sqrt(d), bs, ks, vs)
    return pool, dev(q), dev(tables), dev(lens), tables.shape[1], int(lens.max()), ref


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    cases = [
        (BF16, BF16, 8, 1, [1, 700, 1500, 33, 0, 2049], 1, 256),
        (E4M3, BF16, 4, 4, [4096, 17, 3001], 2, 512),
    ]
    for kv_fmt, q_fmt, hq, hkv, lens, seed, part in cases:
        pool, q, tables, lens_d, width, max_ctx, ref = make(kv_fmt, q_fmt, hq, hkv, lens, seed, part)
        b = len(lens)
        assert pk.paged_attention_workspace_bytes(pool.h, b, hq, max_ctx) > 0  # split in use
        scale = 1.0 / math.sqrt(128)
        want = decode(pool, q, q_fmt, hq, tables, lens_d, max_ctx, scale)
        for _ in range(2):  # two calls in a row on the shared scratch
            got = torch.full_like(want, float("nan"))
            pk.paged_attention_decode_noalloc(pool.h, 0, q, q_fmt, hq, tables, width, lens_d, b, max_ctx,
                                              scale, got, pk.KV_F32)
            torch.cuda.synchronize()
            assert pk.kv_get_device_error() == pk.KV_OK
            assert torch.equal(got, want)
            assert max_abs(got.cpu().numpy(), ref) <= TOL[kv_fmt]


def test_noalloc_rejects_sizes_beyond_its_scratch():
    pool = DevicePool(4, 8, 128, 16, BF16)
    b, hq, max_ctx = 256, 64, 8192
    need = pk.paged_attention_workspace_bytes(pool.h, b, hq, max_ctx)
    assert need > pk.KV_NOALLOC_WORKSPACE_BYTES
    # NULL inputs: if the size check ever stopped rejecting, the decode's own
    # argument check would still refuse before any launch
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_decode_noalloc(pool.h, 0, None, pk.KV_BF16, hq, None, 512, None, b, max_ctx,
                                          0.1, None, pk.KV_F32)
    assert e.value.code == pk.KV_ERR_ARG
    assert "static scratch" in pk.kv_last_error()
