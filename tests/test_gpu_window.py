"""GPU parity of sliding-window decode against the fp64 oracle (multi-token
attention with q_len 1 and the same window).  Blocks wholly before each
window are released (table entry -1) and hold NaN bits, so a read before the
window shows up as an error or NaN."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, DevicePool, decode, dev, max_abs
from workloads import BF16, E4M3, F16, e4m3_codes, fp8_scales, normal_bits, scattered_tables

pytestmark = pytest.mark.gpu

NAN = {F16: 0x7E00, BF16: 0x7FC0, E4M3: 0x7F}


def run_case(fmt, d, bs, hq, hkv, lens, window, partition=0, seed=0, q_fmt=None):
    q_fmt = fmt if q_fmt is None else q_fmt
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    nb = int(sum(-(-int(n) // bs) for n in lens)) + 4
    shape = (nb, hkv, bs, d)
    if fmt == E4M3:
        kh, vh = e4m3_codes(rng, shape), e4m3_codes(rng, shape)
        ks, vs = fp8_scales(rng, (nb, hkv)), fp8_scales(rng, (nb, hkv))
    else:
        kh, vh = normal_bits(rng, shape, fmt), normal_bits(rng, shape, fmt)
        ks = vs = None
    tables = scattered_tables(rng, lens, bs, nb, pad_to=int(np.max(-(-lens // bs))) + 1)
    for s, n in enumerate(lens):  # release the blocks wholly before the window
        for i in range(max(0, int(n) - window) // bs):
            kh[tables[s, i]] = NAN[fmt]
            vh[tables[s, i]] = NAN[fmt]
            tables[s, i] = -1
    q = normal_bits(rng, (len(lens), hq, d), q_fmt)
    pool = DevicePool(nb, hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)],
                      k_scale=None if ks is None else [dev(ks)], v_scale=None if vs is None else [dev(vs)],
                      partition=partition)
    pk.kv_pool_set_sliding_window(pool.h, window)
    scale = 1 / math.sqrt(d)
    out = decode(pool, dev(q), q_fmt, hq, dev(tables), dev(lens), int(lens.max()), scale)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    cu = np.arange(len(lens) + 1, dtype=np.int32)
    ref = oracle.paged_prefill(kh, vh, fmt, q, q_fmt, cu, tables, lens, scale, bs, ks, vs, window=window)
    return out.cpu().numpy(), ref


LENS = [1, 15, 16, 17, 100, 255, 256, 257, 1000, 3000]


@pytest.mark.parametrize("window", [1, 15, 16, 17, 100, 1024, 5000])
@pytest.mark.parametrize("fmt,hq,hkv", [(F16, 8, 8), (BF16, 16, 2)])
def test_window_decode_matches_oracle(window, fmt, hq, hkv):
    out, ref = run_case(fmt, 128, 16, hq, hkv, LENS, window, seed=window + hq)
    assert not np.isnan(out).any()
    assert max_abs(out, ref) <= TOL[fmt]


@pytest.mark.parametrize("partition", [16, 64, 512])
def test_window_decode_split_partitions(partition):
    out, ref = run_case(BF16, 128, 16, 8, 8, [4000, 9000, 17, 600], 1000, partition=partition, seed=partition)
    assert max_abs(out, ref) <= TOL[BF16]


def test_window_decode_fp8_and_block_sizes():
    out, ref = run_case(E4M3, 128, 16, 8, 8, LENS, 200, seed=3, q_fmt=BF16)
    assert max_abs(out, ref) <= TOL[E4M3]
    for bs in (32, 64, 256):
        out, ref = run_case(F16, 64, bs, 4, 4, LENS, 300, seed=bs)
        assert max_abs(out, ref) <= TOL[F16]


def test_window_off_restores_full_attention():
    rng = np.random.default_rng(9)
    lens = np.array([300, 40], np.int32)
    nb = 30
    kh, vh = normal_bits(rng, (nb, 4, 16, 64), F16), normal_bits(rng, (nb, 4, 16, 64), F16)
    tables = scattered_tables(rng, lens, 16, nb)
    q = normal_bits(rng, (2, 4, 64), F16)
    pool = DevicePool(nb, 4, 64, 16, F16, k=[dev(kh)], v=[dev(vh)])
    pk.kv_pool_set_sliding_window(pool.h, 50)
    pk.kv_pool_set_sliding_window(pool.h, 0)
    out = decode(pool, dev(q), F16, 4, dev(tables), dev(lens), 300, 0.125)
    ref = oracle.paged_decode(kh, vh, F16, q, F16, tables, lens, 0.125, 16)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[F16]
    with pytest.raises(pk.KVError):
        pk.kv_pool_set_sliding_window(pool.h, -1)


def run_prefill_case(fmt, d, bs, hq, hkv, lens, q_lens, window, seed=0):
    """Multi-token attention over a windowed pool; blocks wholly before each
    sequence's first-row window are released (-1) and hold NaN bits."""
    rng = np.random.default_rng(seed)
    lens, q_lens = np.asarray(lens, np.int32), np.asarray(q_lens, np.int32)
    nb = int(sum(-(-int(n) // bs) for n in lens)) + 3
    shape = (nb, hkv, bs, d)
    kh, vh = normal_bits(rng, shape, fmt), normal_bits(rng, shape, fmt)
    tables = scattered_tables(rng, lens, bs, nb, pad_to=int(np.max(-(-lens // bs))) + 1)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        first = max(0, int(n) - int(ql) - window + 1)
        for i in range(first // bs):
            kh[tables[s, i]] = NAN[fmt]
            vh[tables[s, i]] = NAN[fmt]
            tables[s, i] = -1
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bits(rng, (int(cu[-1]), hq, d), fmt)
    pool = DevicePool(nb, hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    pk.kv_pool_set_sliding_window(pool.h, window)
    out = torch.full((int(cu[-1]), hq, d), float("nan"), dtype=torch.float32, device="cuda")
    pk.paged_attention_prefill(pool.h, 0, dev(q), fmt, hq, dev(cu), int(cu[-1]), int(q_lens.max()),
                               dev(tables), tables.shape[1], dev(lens), len(lens), 1 / math.sqrt(d), out,
                               pk.KV_F32)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    ref = oracle.paged_prefill(kh, vh, fmt, q, fmt, cu, tables, lens, 1 / math.sqrt(d), bs, window=window)
    return out.cpu().numpy(), ref


@pytest.mark.parametrize("window", [1, 16, 17, 100, 128, 129, 300, 2000])
@pytest.mark.parametrize("fmt,d,hq,hkv", [(BF16, 128, 16, 2), (F16, 64, 4, 4)])
def test_window_prefill_matches_oracle(window, fmt, d, hq, hkv):
    lens = [1, 129, 700, 1500, 300]
    q_lens = [1, 129, 300, 256, 1]  # whole prompts, chunks on cached prefixes, a decode row
    out, ref = run_prefill_case(fmt, d, 16, hq, hkv, lens, q_lens, window, seed=window + d)
    assert not np.isnan(out).any()
    assert max_abs(out, ref) <= TOL[fmt]
