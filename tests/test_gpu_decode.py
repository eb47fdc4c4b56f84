"""GPU parity of paged_attention_decode against the fp64 oracle.

Outputs are requested in fp32 and compared element by element with
max-abs 2e-3 (fp16 / bf16 caches) or 1e-2 (FP8 cache); outputs in the query
dtype must be within that plus one rounding of the format."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, DevicePool, assert_close_native, decode, dev, max_abs
from workloads import (BF16, E4M3, F16, F32, WORKLOADS, context_lens, e4m3_codes, fp8_scales,
                       normal_bits, random_pool, scattered_tables)

pytestmark = pytest.mark.gpu


def run_case(kv_fmt, q_fmt, d, bs, hq, hkv, lens, partition=0, stages=0, seed=0, spare=5,
             out_fmt=F32, scale=None, warps=0):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    nb = int(sum(-(-max(int(n), 1) // bs) for n in lens)) + spare
    shape = (nb, hkv, bs, d)
    if kv_fmt == E4M3:
        kh, vh = e4m3_codes(rng, shape), e4m3_codes(rng, shape)
        ks, vs = fp8_scales(rng, (nb, hkv)), fp8_scales(rng, (nb, hkv))
    else:
        kh, vh = normal_bits(rng, shape, kv_fmt), normal_bits(rng, shape, kv_fmt)
        ks = vs = None
    tables = scattered_tables(rng, np.maximum(lens, 1), bs, nb, pad_to=int(np.max(-(-np.maximum(lens, 1) // bs))) + 1)
    q = normal_bits(rng, (len(lens), hq, d), q_fmt)
    pool = DevicePool(nb, hkv, d, bs, kv_fmt, k=[dev(kh)], v=[dev(vh)],
                      k_scale=None if ks is None else [dev(ks)],
                      v_scale=None if vs is None else [dev(vs)], partition=partition, stages=stages,
                      warps=warps)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    max_ctx = int(lens.max()) if len(lens) else 0
    out = decode(pool, dev(q), q_fmt, hq, dev(tables), dev(lens), max_ctx, scale, out_fmt)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    ref = oracle.paged_decode(kh, vh, kv_fmt, q, q_fmt, tables, lens, scale, bs, ks, vs)
    return out, ref


EDGE_LENS = [1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257]


@pytest.mark.parametrize("kv_fmt,q_fmt", [(F16, F16), (BF16, BF16), (E4M3, BF16), (E4M3, F16)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2), (7, 1)])
def test_decode_matches_oracle_across_formats_and_groups(kv_fmt, q_fmt, d, hq, hkv):
    out, ref = run_case(kv_fmt, q_fmt, d, 16, hq, hkv, EDGE_LENS, seed=hq * 7 + d)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[kv_fmt]


@pytest.mark.parametrize("partition", [16, 48, 512, 4096])
@pytest.mark.parametrize("stages", [2, 3, 4, 6, 8])
@pytest.mark.parametrize("warps", [4, 8])
def test_split_and_pipeline_depths_match_oracle(partition, stages, warps):
    if stages * warps >= 32:  # 8 KB stages: more than 227 KB of shared memory per CTA
        pool = DevicePool(4, 1, 128, 16, BF16)
        with pytest.raises(pk.KVError) as e:
            pool.set_config(partition, stages, warps)
        assert e.value.code == pk.KV_ERR_ARG
        return
    lens = [1, 16, 47, 511, 512, 513, 1000, 1537, 0, 3]
    out, ref = run_case(BF16, BF16, 128, 16, 8, 1, lens, partition=partition, stages=stages,
                        warps=warps, seed=partition + stages + warps)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[BF16]
    assert np.all(out[8].cpu().numpy() == 0)  # empty context


@pytest.mark.parametrize("stages,warps", [(6, 4), (8, 4), (3, 8), (4, 8), (6, 8)])
@pytest.mark.parametrize("d", [64, 128])
def test_fp8_pipeline_shapes(stages, warps, d):
    out, ref = run_case(E4M3, BF16, d, 16, 8, 2, [1, 300, 2000, 17], partition=512, stages=stages,
                        warps=warps, seed=stages + warps + d)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[E4M3]


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_block_sizes(bs):
    out, ref = run_case(F16, F16, 128, bs, 4, 4, [1, bs - 1, bs, bs + 1, 3 * bs + 5, 700], seed=bs, partition=256)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[F16]


@pytest.mark.parametrize("kv_fmt,q_fmt", [(F16, F16), (BF16, BF16), (E4M3, BF16)])
def test_native_output_dtype(kv_fmt, q_fmt):
    out, ref = run_case(kv_fmt, q_fmt, 128, 16, 8, 2, [5, 77, 600], out_fmt=q_fmt, seed=11)
    assert_close_native(out, ref, q_fmt, TOL[kv_fmt])


def test_fp8_long_context_split():
    out, ref = run_case(E4M3, BF16, 128, 16, 4, 4, [4096, 3001], partition=512, seed=5)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[E4M3]


@pytest.mark.parametrize("partition", [0, 64, 256])
def test_fp8_extreme_scales_and_peaked_softmax(partition):
    """Per-block V scales spanning 2^-30 .. 2^20 with a large logit scale
    (peaked softmax) still match: the weights fed to the MMA are normalised
    by their own running maximum, not by the largest V scale."""
    rng = np.random.default_rng(9)
    nb, hkv, bs, d = 64, 2, 16, 128
    kh, vh = e4m3_codes(rng, (nb, hkv, bs, d)), e4m3_codes(rng, (nb, hkv, bs, d))
    ks = np.exp2(rng.uniform(-12, -2, (nb, hkv))).astype(np.float32)
    vs = np.exp2(rng.uniform(-30, 20, (nb, hkv))).astype(np.float32)
    lens = np.array([300, 17, 520], np.int32)
    tables = scattered_tables(rng, lens, bs, nb)
    q = normal_bits(rng, (3, 4, d), BF16)
    pool = DevicePool(nb, hkv, d, bs, E4M3, k=[dev(kh)], v=[dev(vh)], k_scale=[dev(ks)], v_scale=[dev(vs)],
                      partition=partition)
    out = decode(pool, dev(q), BF16, 4, dev(tables), dev(lens), 520, 3.0).cpu().numpy()
    ref = oracle.paged_decode(kh, vh, E4M3, q, BF16, tables, lens, 3.0, bs, ks, vs)
    rel = np.abs(out - ref) / (np.abs(ref).max(axis=-1, keepdims=True) + 1e-30)
    assert rel.max() <= 1e-2


def test_tiny_workload_write_then_decode():
    """The tiny workload end to end: one 1-token cache write per sequence,
    then one decode step over cached + 1 tokens."""
    w = WORKLOADS["tiny"]
    rng = np.random.default_rng(w.seed)
    lens = context_lens(w)  # cached + 1
    nb = w.extra["pool_blocks"]
    kh, vh, _, _ = random_pool(rng, w, nb)
    tables = scattered_tables(rng, lens, w.block_size, nb)
    q = normal_bits(rng, (w.batch, w.num_q_heads, w.head_dim), w.q_fmt)
    kn = normal_bits(rng, (w.batch, w.kv_heads, w.head_dim), w.kv_fmt)
    vn = normal_bits(rng, (w.batch, w.kv_heads, w.head_dim), w.kv_fmt)
    pos = lens - 1
    slots = np.array([tables[s, p // w.block_size] * w.block_size + p % w.block_size
                      for s, p in enumerate(pos)], np.int64)
    pool = DevicePool(nb, w.kv_heads, w.head_dim, w.block_size, w.kv_fmt, k=[dev(kh)], v=[dev(vh)])
    pk.paged_kv_write(pool.h, 0, dev(kn), dev(vn), w.kv_fmt, dev(slots), w.batch)
    out = decode(pool, dev(q), w.q_fmt, w.num_q_heads, dev(tables), dev(lens), int(lens.max()), w.scale)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    kref, vref = kh.copy(), vh.copy()
    oracle.kv_write(kref, vref, w.kv_fmt, kn, vn, w.kv_fmt, slots, w.block_size)
    assert np.array_equal(pool.k[0].cpu().numpy().view(np.uint16), kref)
    assert np.array_equal(pool.v[0].cpu().numpy().view(np.uint16), vref)
    ref = oracle.paged_decode(kref, vref, w.kv_fmt, q, w.q_fmt, tables, lens, w.scale, w.block_size)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[w.kv_fmt]


def test_bad_block_and_length_are_reported_not_read():
    rng = np.random.default_rng(3)
    nb, hkv, bs, d = 8, 1, 16, 64
    kh, vh = normal_bits(rng, (nb, hkv, bs, d), F16), normal_bits(rng, (nb, hkv, bs, d), F16)
    pool = DevicePool(nb, hkv, d, bs, F16, k=[dev(kh)], v=[dev(vh)])
    q = normal_bits(rng, (2, 1, d), F16)
    tables = np.array([[0, 1, 2, 3], [4, 99, 5, -7]], np.int32)
    lens = np.array([40, 60], np.int32)
    pk.kv_get_device_error()  # clear
    decode(pool, dev(q), F16, 1, dev(tables), dev(lens), 64, 0.125)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    # length above the launch bound
    decode(pool, dev(q), F16, 1, dev(tables[:1]), dev(np.array([64], np.int32)), 40, 0.125)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    assert pk.kv_get_device_error() == pk.KV_OK  # cleared by the read


def test_zero_batch_and_all_empty_contexts():
    out, ref = run_case(BF16, BF16, 128, 16, 8, 8, [0, 0, 0], seed=1)
    assert np.all(out.cpu().numpy() == 0) and np.all(ref == 0)
    pool = DevicePool(4, 1, 64, 16, F16)
    pk.paged_attention_decode(pool.h, 0, 0, F16, 1, 0, 1, 0, 0, 16, 0.1, 0, F16)  # batch 0: no-op


def test_bounded_wait_times_out_with_an_error_and_the_context_survives():
    """A pipeline wait that can never complete gives up after its limit and
    reports KV_ERR_TIMEOUT; the next decode on the same context is fine."""
    import time
    pk.kv_get_device_error()
    t0 = time.perf_counter()
    pk.kv_selftest_wait_timeout(50_000_000)  # 50 ms
    assert pk.kv_get_device_error() == pk.KV_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    out, ref = run_case(F16, F16, 64, 16, 2, 2, [5, 40], seed=3)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[F16]


def test_scheduling_order_does_not_change_outputs():
    """Any permutation in seq_order gives bit-identical outputs; an entry
    outside the batch is reported and skipped."""
    rng = np.random.default_rng(12)
    lens = np.array([700, 3, 129, 2049, 0, 16, 1500], np.int32)
    hq, hkv, d, bs = 8, 2, 128, 16
    nb = int(sum(-(-max(int(n), 1) // bs) for n in lens)) + 4
    kh, vh = normal_bits(rng, (nb, hkv, bs, d), BF16), normal_bits(rng, (nb, hkv, bs, d), BF16)
    tables = scattered_tables(rng, np.maximum(lens, 1), bs, nb)
    q = normal_bits(rng, (len(lens), hq, d), BF16)
    for part in (0, 256):
        pool = DevicePool(nb, hkv, d, bs, BF16, k=[dev(kh)], v=[dev(vh)], partition=part)
        b, width, max_ctx = len(lens), tables.shape[1], int(lens.max())
        wsb = pk.paged_attention_workspace_bytes(pool.h, b, hq, max_ctx)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
        outs = []
        for order in (None, np.argsort(-lens, kind="stable"), rng.permutation(b)):
            out = torch.full((b, hq, d), float("nan"), device="cuda")
            pk.paged_attention_decode(pool.h, 0, dev(q), BF16, hq, dev(tables), width, dev(lens), b, max_ctx,
                                      0.09, out, pk.KV_F32, ws, wsb,
                                      seq_order=None if order is None else dev(order.astype(np.int32)))
            outs.append(out.cpu().numpy())
        assert pk.kv_get_device_error() == pk.KV_OK
        assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
        ref = oracle.paged_decode(kh, vh, BF16, q, BF16, tables, lens, 0.09, bs)
        assert max_abs(outs[0], ref) <= TOL[BF16]
    bad = np.array([0, 1, 2, 3, 4, 5, 7], np.int32)
    out = torch.zeros((len(lens), hq, d), device="cuda")
    pk.paged_attention_decode(pool.h, 0, dev(q), BF16, hq, dev(tables), tables.shape[1], dev(lens), len(lens),
                              int(lens.max()), 0.09, out, pk.KV_F32, ws, wsb, seq_order=dev(bad))
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS


@pytest.mark.parametrize("kv_fmt,q_fmt", [(BF16, BF16), (E4M3, BF16)])
def test_every_layer_decodes_its_own_pool(kv_fmt, q_fmt):
    """A 5-layer pool whose layers hold different values: decoding layers 0,
    1 and 4 each matches the oracle on that layer's arrays (a wrong per-layer
    binding or tensor map would read another layer's values)."""
    rng = np.random.default_rng(77)
    L, nb, hkv, hq, bs, d = 5, 40, 2, 8, 16, 128
    lens = np.array([1, 100, 333, 17], np.int32)
    shape = (nb, hkv, bs, d)
    ks_h = vs_h = [None] * L
    if kv_fmt == E4M3:
        kh = [e4m3_codes(rng, shape) for _ in range(L)]
        vh = [e4m3_codes(rng, shape) for _ in range(L)]
        ks_h = [fp8_scales(rng, (nb, hkv)) for _ in range(L)]
        vs_h = [fp8_scales(rng, (nb, hkv)) for _ in range(L)]
    else:
        kh = [normal_bits(rng, shape, kv_fmt) for _ in range(L)]
        vh = [normal_bits(rng, shape, kv_fmt) for _ in range(L)]
    tables = scattered_tables(rng, lens, bs, nb)
    pool = DevicePool(nb, hkv, d, bs, kv_fmt, num_layers=L, k=[dev(a) for a in kh], v=[dev(a) for a in vh],
                      k_scale=None if ks_h[0] is None else [dev(a) for a in ks_h],
                      v_scale=None if vs_h[0] is None else [dev(a) for a in vs_h], partition=128)
    for layer in (0, 1, L - 1):
        q = normal_bits(rng, (len(lens), hq, d), q_fmt)
        out = decode(pool, dev(q), q_fmt, hq, dev(tables), dev(lens), int(lens.max()), 0.1, layer=layer)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        ref = oracle.paged_decode(kh[layer], vh[layer], kv_fmt, q, q_fmt, tables, lens, 0.1, bs,
                                  ks_h[layer], vs_h[layer])
        assert max_abs(out.cpu().numpy(), ref) <= TOL[kv_fmt], layer


@pytest.mark.parametrize("q_fmt", [BF16, F16])
def test_fp8_queries_spanning_many_binades(q_fmt):
    """FP8 caches take the query scaled by a power of two per head into f16
    (exact for bf16 queries, and for f16 ones up to components far below the
    head's largest, which leave the f16 range):
    queries whose components span 2^-24 .. 2^6 in magnitude, with a few huge
    and many tiny values per head, still match the oracle."""
    rng = np.random.default_rng(31)
    nb, hkv, hq, bs, d = 64, 2, 8, 16, 128
    kh, vh = e4m3_codes(rng, (nb, hkv, bs, d)), e4m3_codes(rng, (nb, hkv, bs, d))
    ks, vs = fp8_scales(rng, (nb, hkv)), fp8_scales(rng, (nb, hkv))
    lens = np.array([1, 40, 300, 513], np.int32)
    tables = scattered_tables(rng, lens, bs, nb)
    mag = np.exp2(rng.uniform(-24, 6, (len(lens), hq, d))) * rng.choice([-1.0, 1.0], (len(lens), hq, d))
    mag[:, 3, :] = 0.0  # an all-zero head
    x = torch.from_numpy(mag.astype(np.float32)).to(torch.float16 if q_fmt == F16 else torch.bfloat16)
    q = x.view(torch.int16).numpy().view(np.uint16)
    pool = DevicePool(nb, hkv, d, bs, E4M3, k=[dev(kh)], v=[dev(vh)], k_scale=[dev(ks)], v_scale=[dev(vs)],
                      partition=256)
    for scale in (1.0 / math.sqrt(d), 1e-3):
        out = decode(pool, dev(q), q_fmt, hq, dev(tables), dev(lens), int(lens.max()), scale).cpu().numpy()
        ref = oracle.paged_decode(kh, vh, E4M3, q, q_fmt, tables, lens, scale, bs, ks, vs)
        assert max_abs(out, ref) <= TOL[E4M3], scale
