"""Sliding window end to end: the scheduling step releases the blocks that
leave each sequence's window, the pool hands them to other sequences, and
the windowed decode never reads them.  Against a host mirror built only
from the oracle: scheduler outputs (released entries -1) equal the oracle's,
the GPU pool equals the mirror bit for bit, sampled decode rows match the
fp64 oracle with the same window."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, max_abs
from oracle.sched import BlockManager, Scheduler
from paged_kv_cache_451_b200.serving import DecodeLoop, NativeDecodeLoop
from workloads import BF16, device_normal_bits

pytestmark = pytest.mark.gpu


def host16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("native", [False, True])
def test_windowed_serving_loop_matches_oracle(native):
    """native: the same loop through the library's serving step (tables
    with released entries packed as they are)."""
    rng = np.random.default_rng(91)
    nb, bs, hkv, hq, d, W = 400, 16, 4, 16, 128, 200
    order = rng.permutation(nb).astype(np.int32)
    alloc = pk.kv_alloc_create(nb, bs, order)
    sched = pk.kv_sched_create(alloc, 48)
    pk.kv_sched_set_window(sched, W)
    bm = BlockManager(nb, bs, order)
    osch = Scheduler(bm, 48, window=W)
    k = torch.zeros((nb, hkv, bs, d), dtype=torch.int16, device="cuda")
    v = torch.zeros_like(k)
    pool = pk.kv_pool_create(bs, nb, hkv, d, BF16, 1)
    pk.kv_pool_bind(pool, 0, k, v)
    pk.kv_pool_set_sliding_window(pool, W)
    loop = (NativeDecodeLoop if native else DecodeLoop)(
        pool, sched, num_q_heads=hq, kv_heads=hkv, head_dim=d, block_size=bs, q_dtype=BF16,
        scale=1 / math.sqrt(d), max_batch=48, max_blocks=80, max_tokens=48 * 700, max_context=1200,
        order_policy="batch")
    if native:
        loop.full_plan = True
    kh = np.zeros((nb, hkv, bs, d), np.uint16)
    vh = np.zeros_like(kh)
    remaining, running, nxt, released = {}, [], 0, 0
    for it in range(70):
        for _ in range(int(rng.poisson(1.0 if it else 20.0))):
            plen = int(rng.integers(64, 600))
            pk.kv_sched_add_request(sched, nxt, plen)
            osch.add_request(nxt, plen)
            remaining[nxt] = int(rng.integers(20, 200))
            nxt += 1
        fin = [r for r in running if remaining[r] <= 0]
        plan = loop.schedule(fin)
        want = osch.step(fin)
        info = plan["info"]
        assert list(plan["running"]) == want["running"]
        for row, t in zip(plan["block_tables"], want["block_tables"]):
            assert list(row[:len(t)]) == t
        assert list(plan["slot_mapping"]) == want["slot_mapping"]
        released += sum(b == -1 for t in want["block_tables"] for b in t)
        T, B = info.num_tokens, info.batch
        kn = device_normal_bits((max(T, 1), hkv, d), BF16, "cuda", 1000 + 3 * it)
        vn = device_normal_bits((max(T, 1), hkv, d), BF16, "cuda", 1001 + 3 * it)
        q = device_normal_bits((max(B, 1), hq, d), BF16, "cuda", 1002 + 3 * it)
        out = torch.empty((max(B, 1), hq, d), dtype=torch.float32, device="cuda")
        loop.launch(plan, kn, vn, q, out)
        oracle.block_copy([kh, vh], want["cow_pairs"])
        oracle.kv_write(kh, vh, BF16, host16(kn)[:T], host16(vn)[:T], BF16, want["slot_mapping"], bs)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        if it % 10 == 9:
            assert np.array_equal(host16(k), kh) and np.array_equal(host16(v), vh), f"pool, iteration {it}"
        if B:
            picks = sorted({0, B // 2, B - 1})
            width = max(len(want["block_tables"][i]) for i in picks)
            tables = np.full((len(picks), width), -1, np.int32)
            for j, i in enumerate(picks):
                tables[j, :len(want["block_tables"][i])] = want["block_tables"][i]
            lens = np.array([want["context_lens"][i] for i in picks], np.int32)
            cu = np.arange(len(picks) + 1, dtype=np.int32)
            ref = oracle.paged_prefill(kh, vh, BF16, host16(q)[picks], BF16, cu, tables, lens, 1 / math.sqrt(d),
                                       bs, window=W)
            assert max_abs(out[picks].cpu().numpy(), ref) <= TOL[BF16], f"decode, iteration {it}"
        running = want["running"]
        for r in running:
            remaining[r] -= 1
    assert released > 0
    if native:
        loop.close()
    pk.kv_sched_destroy(sched)
    pk.kv_alloc_destroy(alloc)
    pk.kv_pool_destroy(pool)
