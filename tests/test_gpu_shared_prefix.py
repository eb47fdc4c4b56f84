"""GPU parity of the shared-prefix decode against the fp64 oracle.

paged_attention_decode_shared_prefix must return what a plain decode of the
same batch returns: sequences that share their first blocks (forked from one
parent, or holding one common prompt, "vLLM 推理加速原理详解", section
"PagedAttention：把操作系统的虚拟内存搬进 GPU": blocks shared by reference
count) have the prefix attended once for all of them on the tensor cores,
their own tokens by the decode kernel, and both merged by the log-sum-exp
reduce.  Outputs are compared element by element with the oracle's (fp32
output, max-abs 2e-3) and with the plain decode on the GPU."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, DevicePool, decode, dev, max_abs
from workloads import BF16, E4M3, F16, F32, normal_bits

pytestmark = pytest.mark.gpu


def build(fmt, d, bs, hq, hkv, prefix_blocks, sharer_suffix, other_lens, seed, sharer_pos=None):
    """A pool whose sharers start with the same prefix_blocks blocks and then
    hold their own blocks; the other sequences hold only their own."""
    rng = np.random.default_rng(seed)
    P = prefix_blocks * bs
    lens, shared = [], []
    n_seq = len(sharer_suffix) + len(other_lens)
    pos = list(sharer_pos) if sharer_pos is not None else list(range(len(sharer_suffix)))
    it_s, it_o = iter(sharer_suffix), iter(other_lens)
    for s in range(n_seq):
        if s in pos:
            lens.append(P + next(it_s))
            shared.append(True)
        else:
            lens.append(next(it_o))
            shared.append(False)
    lens = np.array(lens, np.int32)
    own = [-(-int(n - (P if sh else 0)) // bs) for n, sh in zip(lens, shared)]
    nb = prefix_blocks + sum(own) + 3
    perm = rng.permutation(nb).astype(np.int32)
    pre = perm[:prefix_blocks]
    off = prefix_blocks
    width = max(-(-int(n) // bs) for n in lens) + 1
    tables = np.full((n_seq, width), -1, np.int32)
    for s in range(n_seq):
        k = 0
        if shared[s]:
            tables[s, :prefix_blocks] = pre
            k = prefix_blocks
        tables[s, k:k + own[s]] = perm[off:off + own[s]]
        off += own[s]
    shape = (nb, hkv, bs, d)
    kh, vh = normal_bits(rng, shape, fmt), normal_bits(rng, shape, fmt)
    q = normal_bits(rng, (n_seq, hq, d), fmt)
    sharers = np.array([s for s in range(n_seq) if shared[s]], np.int32)
    skip = np.array([P if sh else 0 for sh in shared], np.int32)
    return kh, vh, q, tables, lens, sharers, pre, P, skip


def run(fmt, d, bs, hq, hkv, prefix_blocks, sharer_suffix, other_lens, seed=0, sharer_pos=None,
        partition=0, order=None, scale=None):
    kh, vh, q, tables, lens, sharers, pre, P, skip = build(fmt, d, bs, hq, hkv, prefix_blocks, sharer_suffix,
                                                           other_lens, seed, sharer_pos)
    pool = DevicePool(kh.shape[0], hkv, d, bs, fmt, k=[dev(kh)], v=[dev(vh)], partition=partition)
    b, max_ctx = len(lens), int(lens.max())
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    wsb = pk.paged_attention_shared_prefix_workspace_bytes(pool.h, b, hq, max_ctx, len(sharers))
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    out = torch.full((b, hq, d), float("nan"), device="cuda")
    pk.paged_attention_decode_shared_prefix(pool.h, 0, dev(q), fmt, hq, dev(tables), tables.shape[1], dev(lens),
                                            b, max_ctx, dev(sharers), len(sharers), dev(pre), P, dev(skip),
                                            scale, out, F32, ws, wsb,
                                            seq_order=None if order is None else dev(order.astype(np.int32)))
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    plain = decode(pool, dev(q), fmt, hq, dev(tables), dev(lens), max_ctx, scale)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(kh, vh, fmt, q, fmt, tables, lens, scale, bs)
    got = out.cpu().numpy()
    return got, plain.cpu().numpy(), ref


@pytest.mark.parametrize("fmt", [F16, BF16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 1), (8, 2), (4, 4), (6, 1)])
def test_shared_prefix_matches_oracle(fmt, d, hq, hkv):
    suffix = [1, 15, 16, 17, 300, 2, 700, 33, 1]
    others = [5, 900, 129]
    got, plain, ref = run(fmt, d, 16, hq, hkv, 9, suffix, others, seed=hq + d + fmt,
                          sharer_pos=[0, 2, 3, 5, 6, 8, 9, 10, 11])
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[fmt]
    assert max_abs(got, plain) <= 2 * TOL[fmt]


@pytest.mark.parametrize("prefix_blocks,n_sharers", [(1, 1), (64, 40), (300, 5), (64, 130)])
def test_prefix_and_sharer_counts(prefix_blocks, n_sharers):
    """One block to 4800 tokens of prefix (many 128-key tiles); one sharer to
    130 (several query tiles and work items for groups of 8)."""
    rng = np.random.default_rng(prefix_blocks + n_sharers)
    suffix = [int(x) for x in rng.integers(0, 200, n_sharers)]
    others = [int(x) for x in rng.integers(1, 3000, 7)]
    got, plain, ref = run(BF16, 128, 16, 64, 8, prefix_blocks, suffix, others, seed=n_sharers)
    assert not np.isnan(got).any()
    assert max_abs(got, ref) <= TOL[BF16]


@pytest.mark.parametrize("bs", [32, 64])
def test_larger_blocks_and_split_suffixes(bs):
    """Block sizes above 16, and suffixes long enough that the decode splits
    them into several partitions after the prefix's."""
    suffix = [1, 4000, 2500, 63, 64, 65]
    others = [7000, 3]
    got, plain, ref = run(F16, 128, bs, 16, 2, 5, suffix, others, seed=bs, partition=1024)
    assert max_abs(got, ref) <= TOL[F16]


def test_scheduling_order_and_sharers_spread_through_the_batch():
    suffix = [3, 900, 40, 1, 2000]
    others = [10, 4000, 600, 1]
    order = np.array([8, 1, 7, 3, 0, 5, 2, 6, 4])
    got, plain, ref = run(BF16, 128, 16, 32, 4, 20, suffix, others, seed=5, sharer_pos=[1, 3, 4, 6, 8],
                          order=order)
    assert max_abs(got, ref) <= TOL[BF16]


def test_without_sharers_it_is_the_plain_decode():
    got, plain, ref = run(BF16, 128, 16, 8, 1, 0, [], [5, 300, 17], seed=2)
    assert np.array_equal(got, plain)
    assert max_abs(got, ref) <= TOL[BF16]


def test_bad_arguments_are_rejected():
    pool = DevicePool(8, 2, 128, 16, BF16)
    fp8 = DevicePool(8, 2, 128, 16, E4M3)
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    q = torch.zeros((2, 8, 128), dtype=torch.int16, device="cuda")
    out = torch.zeros((2, 8, 128), device="cuda")
    for p, prefix_len, n_sh in ((pool, 17, 1), (fp8, 16, 1), (pool, 16, 3)):
        with pytest.raises(pk.KVError) as e:
            pk.paged_attention_decode_shared_prefix(p.h, 0, q, BF16, 8, z, 4, z, 2, 48, z, n_sh, z, prefix_len, z,
                                                    0.1, out, F32, ws, 1 << 20)
        assert e.value.code == pk.KV_ERR_ARG
