"""GPU parity of paged_attention_prefill (multi-token causal attention on the
tensor cores) against the fp64 oracle.

Every pool slot that no sequence owns (the tail of each last block, spare
blocks) holds NaN bits, so a key read past a context or an unmasked stale
value shows up as NaN.  fp32 outputs must be within max-abs 2e-3 of the
oracle; outputs in the pool dtype within that plus one rounding."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import DEV, TOL, DevicePool, assert_close_native, dev, max_abs
from workloads import BF16, F16, F32, normal_bits, scattered_tables

pytestmark = pytest.mark.gpu

NAN_BITS = {F16: 0x7E00, BF16: 0x7FC0}


def make_pool(rng, fmt, d, bs, hkv, lens, spare=3):
    lens = np.asarray(lens, np.int32)
    nb = int(sum(-(-max(int(n), 1) // bs) for n in lens)) + spare
    shape = (nb, hkv, bs, d)
    kh = np.full(shape, NAN_BITS[fmt], np.uint16)
    vh = np.full(shape, NAN_BITS[fmt], np.uint16)
    tables = scattered_tables(rng, np.maximum(lens, 1), bs, nb,
                              pad_to=int(np.max(-(-np.maximum(lens, 1) // bs))) + 1)
    for s, n in enumerate(lens):
        t = np.arange(n)
        blk, off = tables[s][t // bs], t % bs
        kh[blk, :, off, :] = normal_bits(rng, (n, hkv, d), fmt)
        vh[blk, :, off, :] = normal_bits(rng, (n, hkv, d), fmt)
    return kh, vh, tables


def prefill(pool, q_dev, fmt, hq, cu_dev, total_q, max_q, tables_dev, lens_dev, scale, out_fmt=F32):
    out_dt = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[out_fmt]
    out = torch.full((total_q, hq, pool.head_dim), float("nan"), dtype=out_dt, device=DEV)
    pk.paged_attention_prefill(pool.h, 0, q_dev, fmt, hq, cu_dev, total_q, max_q, tables_dev,
                               tables_dev.shape[1], lens_dev, lens_dev.shape[0], scale, out, out_fmt)
    return out


def run_case(fmt, d, bs, hq, hkv, lens, q_lens, seed=0, out_fmt=F32, scale=None):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    q_lens = np.asarray(q_lens, np.int32)
    kh, vh, tables = make_pool(rng, fmt, d, bs, hkv, lens)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    total_q = int(cu[-1])
    q = normal_bits(rng, (total_q, hq, d), fmt)
    pool = DevicePool(kh.shape[0], hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = prefill(pool, dev(q), fmt, hq, dev(cu), total_q, int(q_lens.max()), dev(tables), dev(lens),
                  scale, out_fmt)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    ref = oracle.paged_prefill(kh, vh, fmt, q, fmt, cu, tables, lens, scale, bs)
    return out, ref


# full prompts of ragged lengths around the 128-key tile, a chunk on top of
# a cached prefix, a single decode-like token and an empty sequence
LENS = [1, 2, 127, 128, 129, 300, 700, 257, 40]
QLENS = [1, 2, 127, 128, 129, 300, 100, 1, 0]


@pytest.mark.parametrize("fmt", [F16, BF16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (6, 1)])
def test_prefill_matches_oracle_across_formats_and_groups(fmt, d, hq, hkv):
    out, ref = run_case(fmt, d, 16, hq, hkv, LENS, QLENS, seed=hq * 3 + d + fmt)
    got = out.cpu().numpy()
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[fmt]


@pytest.mark.parametrize("bs", [16, 32, 64, 128, 256])
def test_prefill_block_sizes(bs):
    out, ref = run_case(BF16, 128, bs, 8, 2, [33, 513, 250], [33, 200, 250], seed=bs)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[BF16]


@pytest.mark.parametrize("fmt", [F16, BF16])
def test_prefill_native_output(fmt):
    out, ref = run_case(fmt, 128, 16, 8, 8, [200, 129], [200, 64], seed=5, out_fmt=fmt)
    assert_close_native(out, ref, fmt, TOL[fmt])


@pytest.mark.parametrize("hq,hkv,n", [(8, 8, 2048), (32, 4, 1500), (64, 8, 1024)])
def test_prefill_long_prompts_many_tiles(hq, hkv, n):
    """Many query tiles and key tiles per sequence, the lazy rescale of O
    exercised across tiles."""
    out, ref = run_case(BF16, 128, 16, hq, hkv, [n, n // 2 + 37], [n, n // 3], seed=n)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[BF16]


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_many_items_per_persistent_cta(d):
    """Far more work items than SMs, so every persistent CTA takes over the
    items of CTAs whose launch it cancels and its barrier phases carry across
    items of different lengths; most sequences are much shorter than the
    longest, so runs of items without tokens are skipped in between."""
    rng = np.random.default_rng(77 + d)
    q_lens = rng.integers(1, 120, size=48).astype(np.int32)
    q_lens[[5, 30]] = [600, 400]
    prior = rng.integers(0, 300, size=48).astype(np.int32)
    out, ref = run_case(BF16, d, 16, 32, 4, prior + q_lens, q_lens, seed=11 + d)
    got = out.cpu().numpy()
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[BF16]


@pytest.mark.parametrize("fmt", [F16, BF16])
@pytest.mark.parametrize("d,scale", [(64, 0.9), (128, 0.6)])
def test_prefill_large_logits_move_the_reference_max(fmt, d, scale):
    """A scale that makes logits span many binades: a row's 16-key chunks
    often exceed its reference max by more than 2^8, in its first tile and in
    later ones, so the probabilities already stored for the tile (bf16: value
    and residual) and O are rescaled in TMEM."""
    out, ref = run_case(fmt, d, 16, 8, 2, [600, 300, 131], [600, 150, 131], seed=9 + d, scale=scale)
    got = out.cpu().numpy()
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[fmt]


def test_prefill_bf16_values_beyond_the_f16_range():
    """bf16 V values far beyond the f16 range (around 2^17, keys 130..140 of
    the first sequence: its second 128-key tile) and far below its normal
    range (around 2^-20, keys 300..319) in one prompt: P.V must keep bf16's
    range and precision.  Outputs are then large, so the bound is relative to
    the largest V; rows that never see the large values keep the plain
    bound."""
    rng = np.random.default_rng(41)
    lens, q_lens, d, hq, hkv, bs = [700, 300], [700, 120], 128, 16, 2, 16
    kh, vh, tables = make_pool(rng, BF16, d, bs, hkv, lens)
    vf = (vh.astype(np.uint32) << 16).view(np.float32)
    for t in range(130, 141):
        vf[tables[0][t // bs], :, t % bs, :] *= 2.0 ** 17
    for t in range(300, 320):
        vf[tables[0][t // bs], :, t % bs, :] *= 2.0 ** -20
    vh = (vf.view(np.uint32) >> 16).astype(np.uint16)  # the scalings are exact in bf16
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bits(rng, (int(cu[-1]), hq, d), BF16)
    pool = DevicePool(kh.shape[0], hkv, d, bs, BF16, k=[dev(kh)], v=[dev(vh)])
    scale = 1.0 / math.sqrt(d)
    lens_a = np.asarray(lens, np.int32)
    out = prefill(pool, dev(q), BF16, hq, dev(cu), int(cu[-1]), max(q_lens), dev(tables), dev(lens_a), scale)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    ref = oracle.paged_prefill(kh, vh, BF16, q, BF16, cu, tables, lens_a, scale, bs)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    vmax = float(np.abs(vf[np.isfinite(vf)]).max())
    assert max_abs(got, ref) <= TOL[BF16] + 1e-4 * vmax
    # rows whose keys never reach the large values stay within the plain bound
    assert max_abs(got[:130], ref[:130]) <= TOL[BF16]


@pytest.mark.parametrize("fmt,boost", [(BF16, 6), (F16, 3)])
def test_prefill_logit_jumps_inside_a_tile(fmt, boost):
    """Keys 300 and 301 of a 700-token prompt (the third 128-key tile, its
    third 16-key chunk) have K scaled by 2^boost, so the rows that see them
    find logits tens of binades above everything before, in the middle of a
    tile: the probabilities already computed for that tile, the sums and O
    must all move to the new reference."""
    rng = np.random.default_rng(43 + boost)
    lens, q_lens, d, hq, hkv, bs = [700, 260], [700, 260], 128, 8, 2, 16
    kh, vh, tables = make_pool(rng, fmt, d, bs, hkv, lens)
    if fmt == BF16:
        kf = (kh.astype(np.uint32) << 16).view(np.float32)
    else:
        kf = kh.view(np.float16).astype(np.float32)
    for t in (300, 301):
        kf[tables[0][t // bs], :, t % bs, :] *= 2.0 ** boost
    if fmt == BF16:
        kh = (kf.view(np.uint32) >> 16).astype(np.uint16)
    else:
        kh = kf.astype(np.float16).view(np.uint16)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bits(rng, (int(cu[-1]), hq, d), fmt)
    pool = DevicePool(kh.shape[0], hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    scale = 1.0 / math.sqrt(d)
    lens_a = np.asarray(lens, np.int32)
    out = prefill(pool, dev(q), fmt, hq, dev(cu), int(cu[-1]), max(q_lens), dev(tables), dev(lens_a), scale)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    ref = oracle.paged_prefill(kh, vh, fmt, q, fmt, cu, tables, lens_a, scale, bs)
    got = out.cpu().numpy()
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[fmt]


def test_write_then_prefill_end_to_end():
    """paged_kv_write the new tokens of a chunk, then prefill over the pool:
    the pool equals the oracle's write mirror bit for bit and the output the
    oracle's attention over it."""
    rng = np.random.default_rng(31)
    fmt, d, bs, hq, hkv = BF16, 128, 16, 16, 4
    prior = np.array([0, 300, 17], np.int32)
    q_lens = np.array([250, 130, 1], np.int32)
    lens = prior + q_lens
    nb = int(sum(-(-int(n) // bs) for n in lens)) + 2
    shape = (nb, hkv, bs, d)
    kh = np.full(shape, NAN_BITS[fmt], np.uint16)
    vh = np.full(shape, NAN_BITS[fmt], np.uint16)
    tables = scattered_tables(rng, lens, bs, nb)
    for s, n in enumerate(prior):
        t = np.arange(n)
        kh[tables[s][t // bs], :, t % bs, :] = normal_bits(rng, (n, hkv, d), fmt)
        vh[tables[s][t // bs], :, t % bs, :] = normal_bits(rng, (n, hkv, d), fmt)
    slots = np.concatenate([tables[s][(prior[s] + np.arange(q)) // bs].astype(np.int64) * bs
                            + (prior[s] + np.arange(q)) % bs for s, q in enumerate(q_lens)])
    total = int(q_lens.sum())
    k_new, v_new = normal_bits(rng, (total, hkv, d), fmt), normal_bits(rng, (total, hkv, d), fmt)
    q = normal_bits(rng, (total, hq, d), fmt)
    pool = DevicePool(nb, hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    pk.paged_kv_write(pool.h, 0, dev(k_new), dev(v_new), fmt, dev(slots), total, None, None)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    out = prefill(pool, dev(q), fmt, hq, dev(cu), total, int(q_lens.max()), dev(tables), dev(lens),
                  1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    oracle.kv_write(kh, vh, fmt, k_new, v_new, fmt, slots, bs)
    assert np.array_equal(pool.k[0].cpu().numpy().view(np.uint16), kh)
    assert np.array_equal(pool.v[0].cpu().numpy().view(np.uint16), vh)
    ref = oracle.paged_prefill(kh, vh, fmt, q, fmt, cu, tables, lens, 1 / math.sqrt(d), bs)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[fmt]


def test_single_token_rows_equal_decode():
    """q_len = 1 for every sequence is a decode step: both paths agree within
    their tolerances and with the oracle."""
    rng = np.random.default_rng(41)
    fmt, d, bs, hq, hkv = F16, 128, 16, 8, 2
    lens = np.array([1, 16, 17, 500, 1000], np.int32)
    kh, vh, tables = make_pool(rng, fmt, d, bs, hkv, lens)
    q = normal_bits(rng, (len(lens), hq, d), fmt)
    pool = DevicePool(kh.shape[0], hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    cu = np.arange(len(lens) + 1, dtype=np.int32)
    out = prefill(pool, dev(q), fmt, hq, dev(cu), len(lens), 1, dev(tables), dev(lens), 0.1)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(kh, vh, fmt, q, fmt, tables, lens, 0.1, bs)
    assert max_abs(out.cpu().numpy(), ref) <= TOL[fmt]


def test_bad_lengths_and_block_ids_are_reported():
    rng = np.random.default_rng(51)
    fmt, d, bs = BF16, 64, 16
    kh, vh, tables = make_pool(rng, fmt, d, bs, 2, [64, 64])
    pool = DevicePool(kh.shape[0], 2, d, bs, fmt, k=[dev(kh)], v=[dev(vh)])
    q = dev(normal_bits(rng, (80, 4, d), fmt))
    # q_len 48 > context 40 for sequence 1
    cu = np.array([0, 32, 80], np.int32)
    prefill(pool, q, fmt, 4, dev(cu), 80, 48, dev(tables), dev(np.array([64, 40], np.int32)), 0.1)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    bad = tables.copy()
    bad[0, 1] = kh.shape[0] + 7
    prefill(pool, q, fmt, 4, dev(cu), 80, 48, dev(bad), dev(np.array([64, 64], np.int32)), 0.1)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    # the context stays usable: a valid call afterwards is clean
    out = prefill(pool, q, fmt, 4, dev(cu), 80, 48, dev(tables), dev(np.array([64, 64], np.int32)), 0.1)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    assert not torch.isnan(out).any()


def test_unsupported_arguments_are_rejected_before_launch():
    rng = np.random.default_rng(61)
    kh, vh, tables = make_pool(rng, F16, 64, 16, 2, [32])
    pool = DevicePool(kh.shape[0], 2, 64, 16, F16, k=[dev(kh)], v=[dev(vh)])
    q = torch.zeros((32, 4, 64), dtype=torch.float16, device=DEV)
    out = torch.zeros((32, 4, 64), dtype=torch.float32, device=DEV)
    cu, tb, ln = dev(np.array([0, 32], np.int32)), dev(tables), dev(np.array([32], np.int32))

    def call(**kw):
        a = dict(q=q, q_dtype=F16, hq=4, scale=0.1, out=out, out_dtype=F32)
        a.update(kw)
        pk.paged_attention_prefill(pool.h, 0, a["q"], a["q_dtype"], a["hq"], cu, 32, 32, tb,
                                   tables.shape[1], ln, 1, a["scale"], a["out"], a["out_dtype"])

    call()
    for kw in (dict(q_dtype=BF16), dict(hq=3), dict(hq=18), dict(scale=0.0), dict(scale=-1.0),
               dict(scale=float("inf")), dict(out_dtype=BF16), dict(q=q[:, :, 1:])):
        with pytest.raises(pk.KVError) as e:
            call(**kw)
        assert e.value.code == pk.KV_ERR_ARG, kw
    fp8 = DevicePool(4, 2, 64, 16, pk.KV_FP8_E4M3)
    with pytest.raises(pk.KVError) as e:
        pk.paged_attention_prefill(fp8.h, 0, q, F16, 4, cu, 32, 32, tb, tables.shape[1], ln, 1, 0.1,
                                   out, F32)
    assert e.value.code == pk.KV_ERR_ARG
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
