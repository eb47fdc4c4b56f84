"""GPU paged_kv_write and block_copy against the oracle's host mirrors:
pool bytes must match bit for bit (including FP8 quantisation)."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import DevicePool, dev
from workloads import BF16, E4M3, F16, fp8_scales, normal_bits

pytestmark = pytest.mark.gpu


def raw(fmt):
    return np.uint8 if fmt == E4M3 else np.uint16


def pool_host(t, fmt):
    return t.cpu().numpy().view(raw(fmt))


@pytest.mark.parametrize("fmt,d,bs", [(F16, 64, 16), (BF16, 128, 16), (F16, 128, 32)])
def test_write_16bit_is_bit_exact(fmt, d, bs):
    rng = np.random.default_rng(40 + d + bs)
    nb, hkv, T = 37, 3, 300
    kh, vh = normal_bits(rng, (nb, hkv, bs, d), fmt), normal_bits(rng, (nb, hkv, bs, d), fmt)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[::17] = -1
    kn, vn = normal_bits(rng, (T, hkv, d), fmt), normal_bits(rng, (T, hkv, d), fmt)
    pool = DevicePool(nb, hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    pk.paged_kv_write(pool.h, 0, dev(kn), dev(vn), fmt, dev(slots), T)
    assert pk.kv_get_device_error() == pk.KV_OK
    oracle.kv_write(kh, vh, fmt, kn, vn, fmt, slots, bs)
    assert np.array_equal(pool_host(pool.k[0], fmt), kh)
    assert np.array_equal(pool_host(pool.v[0], fmt), vh)


@pytest.mark.parametrize("src", [BF16, F16])
@pytest.mark.parametrize("d", [64, 128])
def test_write_fp8_quantises_bit_exactly(src, d):
    rng = np.random.default_rng(50 + d + src)
    nb, hkv, bs, T = 29, 4, 16, 400
    kh = np.zeros((nb, hkv, bs, d), np.uint8)
    vh = np.zeros_like(kh)
    kinv = (1.0 / fp8_scales(rng, (nb, hkv))).astype(np.float32)
    vinv = (1.0 / fp8_scales(rng, (nb, hkv))).astype(np.float32)
    kinv[0, 0] = 1e6  # forces saturation for that (block, head)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    kn, vn = normal_bits(rng, (T, hkv, d), src), normal_bits(rng, (T, hkv, d), src)
    pool = DevicePool(nb, hkv, d, bs, E4M3)
    pk.paged_kv_write(pool.h, 0, dev(kn), dev(vn), src, dev(slots), T, dev(kinv), dev(vinv))
    assert pk.kv_get_device_error() == pk.KV_OK
    oracle.kv_write(kh, vh, E4M3, kn, vn, src, slots, bs, kinv, vinv)
    assert np.array_equal(pool_host(pool.k[0], E4M3), kh)
    assert np.array_equal(pool_host(pool.v[0], E4M3), vh)


@pytest.mark.parametrize("src", [BF16, F16])
def test_fp8_rounding_matches_oracle_for_every_finite_16bit_value(src):
    """Every finite bf16 / f16 bit pattern, times a few inverse scales, is
    quantised by the GPU exactly as the oracle's E4M3 encoder does."""
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.decode(codes, src)
    codes = codes[np.isfinite(vals)]
    d, hkv, bs = 128, 1, 16
    T = -(-codes.size // d)
    data = np.zeros(T * d, np.uint16)
    data[:codes.size] = codes
    data = data.reshape(T, hkv, d)
    nb = -(-T // bs)
    slots = np.arange(T, dtype=np.int64)
    for inv in (1.0, 0.013, 2.0 ** 7, 3.0e5):
        invs = np.full((nb, hkv), inv, np.float32)
        pool = DevicePool(nb, hkv, d, bs, E4M3)
        pk.paged_kv_write(pool.h, 0, dev(data), dev(data), src, dev(slots), T, dev(invs), dev(invs))
        kh = np.zeros((nb, hkv, bs, d), np.uint8)
        vh = np.zeros_like(kh)
        oracle.kv_write(kh, vh, E4M3, data, data, src, slots, bs, invs, invs)
        got = pool_host(pool.k[0], E4M3)
        assert np.array_equal(got, kh), (inv, int(np.sum(got != kh)))


def test_write_reports_slots_outside_the_pool():
    rng = np.random.default_rng(60)
    nb, hkv, bs, d = 4, 1, 16, 64
    kh = normal_bits(rng, (nb, hkv, bs, d), F16)
    pool = DevicePool(nb, hkv, d, bs, F16, k=[dev(kh)], v=[dev(kh.copy())])
    kn = normal_bits(rng, (2, hkv, d), F16)
    pk.kv_get_device_error()
    pk.paged_kv_write(pool.h, 0, dev(kn), dev(kn), F16, dev(np.array([nb * bs + 3, 5], np.int64)), 2)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    expect = kh.copy()
    expect[0, :, 5, :] = kn[1]
    assert np.array_equal(pool_host(pool.k[0], F16), expect)


@pytest.mark.parametrize("fmt", [BF16, E4M3])
def test_block_copy_all_layers_bit_exact(fmt):
    rng = np.random.default_rng(70 + fmt)
    nb, hkv, bs, d, L = 50, 8, 16, 128, 3
    if fmt == E4M3:
        from workloads import e4m3_codes
        ks = [e4m3_codes(rng, (nb, hkv, bs, d)) for _ in range(L)]
        vs = [e4m3_codes(rng, (nb, hkv, bs, d)) for _ in range(L)]
        ksc = [fp8_scales(rng, (nb, hkv)) for _ in range(L)]
        vsc = [fp8_scales(rng, (nb, hkv)) for _ in range(L)]
    else:
        ks = [normal_bits(rng, (nb, hkv, bs, d), fmt) for _ in range(L)]
        vs = [normal_bits(rng, (nb, hkv, bs, d), fmt) for _ in range(L)]
        ksc = vsc = None
    pool = DevicePool(nb, hkv, d, bs, fmt, num_layers=L, k=[dev(x) for x in ks], v=[dev(x) for x in vs],
                      k_scale=None if ksc is None else [dev(x) for x in ksc],
                      v_scale=None if vsc is None else [dev(x) for x in vsc])
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:12], perm[12:24]], axis=1).astype(np.int32)
    pk.block_copy(pool.h, dev(pairs), len(pairs))
    assert pk.kv_get_device_error() == pk.KV_OK
    arrays = ks + vs + ([] if ksc is None else ksc + vsc)
    oracle.block_copy(arrays, pairs)
    for layer in range(L):
        assert np.array_equal(pool_host(pool.k[layer], fmt), ks[layer])
        assert np.array_equal(pool_host(pool.v[layer], fmt), vs[layer])
        if fmt == E4M3:
            assert np.array_equal(pool.ks[layer].cpu().numpy(), ksc[layer])
            assert np.array_equal(pool.vs[layer].cpu().numpy(), vsc[layer])


def test_block_copy_reports_ids_outside_the_pool():
    pool = DevicePool(4, 1, 64, 16, F16)
    pk.kv_get_device_error()
    pk.block_copy(pool.h, dev(np.array([[0, 1], [2, 9]], np.int32)), 2)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
