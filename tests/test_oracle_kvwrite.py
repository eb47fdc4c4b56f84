"""Pins for the oracle's host mirrors of the cache write and the block copy.

The write is checked by reading the pool back through torch tensor indexing
(pool[block, :, offset, :]) rather than the mirror's own arithmetic, and the
FP8 path against torch's float8 cast of the fp32 product."""

import numpy as np
import pytest
import torch

import oracle
from workloads import BF16, E4M3, F16, fp8_scales, normal_bits


@pytest.mark.parametrize("fmt", [F16, BF16])
def test_write_places_each_row_at_its_slot(fmt):
    rng = np.random.default_rng(20)
    nb, hkv, bs, d, T = 9, 3, 16, 8, 25
    kp = normal_bits(rng, (nb, hkv, bs, d), fmt)
    vp = normal_bits(rng, (nb, hkv, bs, d), fmt)
    before_k, before_v = kp.copy(), vp.copy()
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1  # skipped tokens
    kn = normal_bits(rng, (T, hkv, d), fmt)
    vn = normal_bits(rng, (T, hkv, d), fmt)
    oracle.kv_write(kp, vp, fmt, kn, vn, fmt, slots, bs)
    tk, tv = torch.from_numpy(kp.view(np.int16)), torch.from_numpy(vp.view(np.int16))
    touched = np.zeros((nb, bs), dtype=bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        b, o = divmod(int(s), bs)
        touched[b, o] = True
        assert torch.equal(tk[b, :, o, :], torch.from_numpy(kn[t].view(np.int16)))
        assert torch.equal(tv[b, :, o, :], torch.from_numpy(vn[t].view(np.int16)))
    # every other slot is untouched
    assert np.array_equal(kp.transpose(0, 2, 1, 3)[~touched], before_k.transpose(0, 2, 1, 3)[~touched])
    assert np.array_equal(vp.transpose(0, 2, 1, 3)[~touched], before_v.transpose(0, 2, 1, 3)[~touched])


@pytest.mark.parametrize("src", [BF16, F16])
def test_fp8_write_quantises_like_torch(src):
    rng = np.random.default_rng(21)
    nb, hkv, bs, d, T = 6, 2, 16, 16, 30
    kp = np.zeros((nb, hkv, bs, d), np.uint8)
    vp = np.zeros_like(kp)
    kinv = (1.0 / fp8_scales(rng, (nb, hkv))).astype(np.float32)
    vinv = (1.0 / fp8_scales(rng, (nb, hkv))).astype(np.float32)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    kn = normal_bits(rng, (T, hkv, d), src)
    vn = normal_bits(rng, (T, hkv, d), src)
    oracle.kv_write(kp, vp, E4M3, kn, vn, src, slots, bs, kinv, vinv)
    tdt = torch.bfloat16 if src == BF16 else torch.float16
    for pool, new, inv in ((kp, kn, kinv), (vp, vn, vinv)):
        for t, s in enumerate(slots):
            b, o = divmod(int(s), bs)
            x = torch.from_numpy(new[t].view(np.int16)).view(tdt).float()
            y = x * torch.from_numpy(inv[b]).float()[:, None]
            finite = y.abs() < 464
            ref = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
            got = torch.from_numpy(pool[b, :, o, :])
            assert torch.equal(got[finite], ref[finite])
            assert torch.all(got[~finite] & 0x7F == 0x7E)  # saturated to +-448


def test_write_rejects_block_outside_pool():
    kp = np.zeros((2, 1, 16, 8), np.uint16)
    vp = np.zeros_like(kp)
    kn = np.zeros((1, 1, 8), np.uint16)
    with pytest.raises(IndexError):
        oracle.kv_write(kp, vp, F16, kn, kn, F16, np.array([2 * 16]), 16)


def test_block_copy_copies_blocks_of_every_array():
    rng = np.random.default_rng(22)
    arrs = [normal_bits(rng, (8, 2, 16, 4), F16) for _ in range(4)] + [fp8_scales(rng, (8, 2))]
    before = [a.copy() for a in arrs]
    pairs = np.array([[1, 5], [2, 6]], dtype=np.int32)
    oracle.block_copy(arrs, pairs)
    for a, b in zip(arrs, before):
        assert np.array_equal(a[5], b[1]) and np.array_equal(a[6], b[2])
        keep = [0, 1, 2, 3, 4, 7]
        assert np.array_equal(a[keep], b[keep])
