"""The packed scheduling step (kv_sched_step_packed), host side: every array
it lays into the upload buffer must equal the oracle scheduler's output for
the same step (running set, block tables padded with -1, context lengths,
slots, copy-on-write and swap pairs), the scheduling order must follow its
stated policy, and the admitted prompts' prefill arrays must follow from
the oracle's context lengths and cached-token counts.  The serving loop's
argument checks run before any CUDA call."""

import ctypes

import numpy as np
import pytest

import paged_kv_cache_451_b200 as pk
from oracle.sched import BlockManager, OracleOOM, PrefixCachingBlockManager, Scheduler


def aligned(nbytes):
    raw = np.zeros(nbytes + 64, np.uint8)
    off = (-raw.ctypes.data) % 16
    return raw[off:off + nbytes]


def section(buf, off, dtype, n):
    if n == 0:
        return np.zeros(0, dtype)
    assert off >= 0 and off % 16 == 0
    return buf[off:off + n * np.dtype(dtype).itemsize].view(dtype).copy()


def check_step(buf, lay, want, policy, cached):
    info = lay.info
    b, t, c, a, w = info.batch, info.num_tokens, info.num_cow, info.num_admitted, lay.table_width
    assert b == len(want["running"]) and t == len(want["slot_mapping"]) and a == len(want["admitted"])
    assert w == max([len(x) for x in want["block_tables"]] + [1])
    assert section(buf, lay.slot_mapping, np.int64, t).tolist() == want["slot_mapping"]
    lens = section(buf, lay.context_lens, np.int32, b)
    assert lens.tolist() == want["context_lens"]
    assert lay.max_context_len == (max(want["context_lens"]) if b else 0)
    tables = section(buf, lay.block_tables, np.int32, b * w).reshape(b, w)
    for row, tab in zip(tables, want["block_tables"]):
        assert row[:len(tab)].tolist() == list(tab) and np.all(row[len(tab):] == -1)
    assert section(buf, lay.cow_pairs, np.int32, 2 * c).reshape(c, 2).tolist() == [list(p) for p in want["cow_pairs"]]
    so, si = lay.num_swap_out, lay.num_swap_in
    assert section(buf, lay.swap_out_pairs, np.int32, 2 * so).reshape(so, 2).tolist() == \
        [list(p) for p in want.get("swap_out", [])]
    assert section(buf, lay.swap_in_pairs, np.int32, 2 * si).reshape(si, 2).tolist() == \
        [list(p) for p in want.get("swap_in", [])]
    if policy == pk.KV_ORDER_BATCH:
        assert lay.seq_order == -1
    else:
        order = section(buf, lay.seq_order, np.int32, b)
        assert sorted(order.tolist()) == list(range(b))
        if policy == pk.KV_ORDER_LONGEST:
            want_order = sorted(range(b), key=lambda i: (-lens[i], i))
        else:
            mean = lens.mean() if b else 0.0
            long = sorted((i for i in range(b) if lens[i] > mean), key=lambda i: (-lens[i], i))
            want_order = long + [i for i in range(b) if not lens[i] > mean]
        assert order.tolist() == want_order
    if a:
        # the admitted requests are the last rows; prompt = context - 1
        assert want["running"][b - a:] == want["admitted"]
        prompt = [want["context_lens"][b - a + i] - 1 for i in range(a)]
        fresh = [p - k for p, k in zip(prompt, cached)]
        assert section(buf, lay.cu_seqlens, np.int32, a + 1).tolist() == np.concatenate([[0], np.cumsum(fresh)]).tolist()
        assert section(buf, lay.prefill_context_lens, np.int32, a).tolist() == prompt
        assert lay.prefill_tokens == sum(fresh) and lay.max_prefill_len == max(fresh)
    else:
        assert lay.cu_seqlens == -1 and lay.prefill_context_lens == -1 and lay.prefill_tokens == 0
    offs = [o for o in (lay.slot_mapping, lay.block_tables, lay.context_lens, lay.seq_order, lay.cow_pairs,
                        lay.swap_out_pairs, lay.swap_in_pairs, lay.cu_seqlens, lay.prefill_context_lens) if o >= 0]
    assert all(o % 16 == 0 and o <= lay.bytes for o in offs)


@pytest.mark.parametrize("mode,policy,seed", [
    ("none", pk.KV_ORDER_BATCH, 0), ("none", pk.KV_ORDER_LONGEST, 1), ("none", pk.KV_ORDER_LONG_FIRST, 2),
    ("swap", pk.KV_ORDER_LONG_FIRST, 3), ("recompute", pk.KV_ORDER_BATCH, 4), ("swap", pk.KV_ORDER_LONGEST, 5),
    ("window", pk.KV_ORDER_LONG_FIRST, 6),
])
def test_packed_step_equals_the_oracle_scheduler(mode, policy, seed):
    rng = np.random.default_rng(700 + seed)
    nb, bs, max_seqs, slots = (48, 8, 16, 24) if mode in ("swap", "recompute") else (400, 16, 24, 0)
    order = rng.permutation(nb)
    bm = BlockManager(nb, bs, order)
    window = 40 if mode == "window" else 0  # blocks that left a sequence's last 40 positions are released
    sch = Scheduler(bm, max_seqs, window=window)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    s = pk.kv_sched_create(a, max_seqs)
    if window:
        pk.kv_sched_set_window(s, window)
    elif mode != "none":
        bm.set_swap_space(slots)
        sch.preemption = mode
        pk.kv_alloc_set_swap_space(a, slots)
        pk.kv_sched_set_preemption(s, pk.KV_PREEMPT_SWAP if mode == "swap" else pk.KV_PREEMPT_RECOMPUTE)
    width = nb
    cap = pk.kv_step_packed_bytes(max_seqs, 64 * max_seqs, width, slots)
    buf = aligned(cap)
    running_ids = np.zeros(max_seqs, np.int64)
    remaining, running, nxt, seen = {}, [], 0, set()
    for it in range(120):
        for _ in range(int(rng.poisson(0.7))):
            plen = int(rng.integers(1, 40))
            sch.add_request(nxt, plen)
            pk.kv_sched_add_request(s, nxt, plen)
            remaining[nxt] = int(rng.integers(3, 60))
            nxt += 1
        fin = [r for r in running if remaining[r] <= 0]
        want = sch.step(fin)
        lay = pk.kv_sched_step_packed(s, fin, policy, width, buf, cap, running_ids)
        assert running_ids[:lay.info.batch].tolist() == want["running"]
        check_step(buf, lay, want, policy, [0] * len(want["admitted"]))
        assert lay.bytes <= cap
        seen |= {k for k in ("cow_pairs", "swap_out", "swap_in", "admitted") if want.get(k)}
        if any(b == -1 for t in want["block_tables"] for b in t):
            seen.add("released")
        running = want["running"]
        for r in running:
            remaining[r] -= 1
    assert "admitted" in seen
    if mode == "swap":
        assert {"swap_out", "swap_in"} <= seen
    if mode == "window":
        assert "released" in seen
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_packed_step_with_prefix_caching_and_forks():
    """Cached prompt tokens shorten the prefill rows; forked sequences copy
    their shared last block on write."""
    rng = np.random.default_rng(77)
    nb, bs = 200, 16
    order = rng.permutation(nb)
    bm = PrefixCachingBlockManager(nb, bs, order)
    sch = Scheduler(bm, 32)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    pk.kv_alloc_enable_prefix_caching(a)
    s = pk.kv_sched_create(a, 32)
    bm.allocate(900, 37)
    pk.kv_alloc_allocate(a, 900, 37)
    for child in (901, 902, 903):
        bm.fork(900, child)
        pk.kv_alloc_fork(a, 900, child)
    for sid in (900, 901, 902, 903):
        sch.adopt(sid)
        pk.kv_sched_adopt(s, sid)
    system = list(rng.integers(0, 1000, size=120))
    cap = pk.kv_step_packed_bytes(32, 32 * 200, 64, 0)
    buf = aligned(cap)
    nxt, running, hit_steps, cow_steps = 0, [900, 901, 902, 903], 0, 0
    for it in range(40):
        for _ in range(int(rng.poisson(1.2))):
            toks = system[:int(rng.integers(0, 120))] + list(rng.integers(0, 1000, size=int(rng.integers(1, 50))))
            sch.add_request_tokens(nxt, toks)
            pk.kv_sched_add_request_tokens(s, nxt, toks)
            nxt += 1
        fin = [r for r in running if rng.random() < 0.1]
        want = sch.step(fin)
        lay = pk.kv_sched_step_packed(s, fin, pk.KV_ORDER_BATCH, 64, buf, cap)
        check_step(buf, lay, want, pk.KV_ORDER_BATCH, want["cached"])
        hit_steps += any(want["cached"])
        cow_steps += bool(want["cow_pairs"])
        running = want["running"]
    assert hit_steps > 0 and cow_steps > 0
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_packed_step_errors():
    a = pk.kv_alloc_create(64, 16)
    s = pk.kv_sched_create(a, 8)
    pk.kv_sched_add_request(s, 1, 100)  # 7 blocks
    cap = pk.kv_step_packed_bytes(8, 256, 16, 0)
    buf = aligned(cap + 16)
    # checked before the step: nothing changes
    for args in ((pk.KV_ORDER_BATCH, 16, buf[1:cap + 1], cap), (7, 16, buf, cap), (pk.KV_ORDER_BATCH, 0, buf, cap)):
        with pytest.raises(pk.KVError) as e:
            pk.kv_sched_step_packed(s, [], *args)
        assert e.value.code == pk.KV_ERR_ARG
    with pytest.raises(pk.KVError) as e:
        pk.kv_sched_step_packed(s, [5], pk.KV_ORDER_BATCH, 16, buf, cap)  # 5 is not running
    assert e.value.code == pk.KV_ERR_STATE
    assert pk.kv_sched_stats(s)[:2] == (0, 1)
    # a table wider than the buffer's rows: the step is taken, outputs stay readable
    with pytest.raises(pk.KVError) as e:
        pk.kv_sched_step_packed(s, [], pk.KV_ORDER_BATCH, 4, buf, cap)
    assert e.value.code == pk.KV_ERR_ARG and "step is taken" in pk.kv_last_error()
    out = pk.kv_sched_outputs(s, pk.kv_step_info(1, 101, 0, 1, 7))
    assert out["running"].tolist() == [1] and out["context_lens"].tolist() == [101]
    # a buffer too small for the step's arrays
    with pytest.raises(pk.KVError) as e:
        pk.kv_sched_step_packed(s, [], pk.KV_ORDER_BATCH, 16, buf, 32)
    assert e.value.code == pk.KV_ERR_ARG
    lay = pk.kv_sched_step_packed(s, [], pk.KV_ORDER_BATCH, 16, buf, cap)
    assert lay.info.batch == 1 and section(buf, lay.context_lens, np.int32, 1).tolist() == [103]
    assert lay.bytes == 16 + 32 + 16  # one slot, a 7-block row, one length
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_packed_bytes_bound_every_step_of_the_caps():
    assert pk.kv_step_packed_bytes(-1, 0, 1, 0) == 0
    n = pk.kv_step_packed_bytes(256, 4352, 521, 0)
    # slots + tables + lens + order + cow + cu + prefill lens, each rounded to 16
    assert n == 8 * 4352 + 4 * 256 * 521 + 4 * 256 + 4 * 256 + 8 * 256 + (4 * 257 + 12) + 4 * 256
    assert pk.kv_step_packed_bytes(256, 4352, 521, 10) == n + 2 * 80


def test_serve_create_checks_arguments_before_any_cuda_call():
    a = pk.kv_alloc_create(64, 16)
    s = pk.kv_sched_create(a, 8)
    pool = pk.kv_pool_create(16, 64, 1, 128, pk.KV_BF16, 1)
    need = pk.kv_step_packed_bytes(8, 64, 16, 0)
    h = [aligned(need), aligned(need)]
    d = [aligned(need), aligned(need)]  # stand-ins: never dereferenced on these paths
    ws = aligned(16)
    bad = [
        dict(meta_bytes=need - 16),                       # buffers too small
        dict(host=[h[0][1:], h[1]], meta_bytes=need - 16),  # misaligned host buffer
        dict(order=5),                                    # unknown policy
        dict(swap_slots=4),                               # swap slots without swap space
        dict(max_width=0),
        dict(host=[h[0]], dev=[d[0]]),                    # one buffer set
        dict(host=h * 3, dev=d * 3),                      # six sets, above KV_SERVE_MAX_SETS
    ]
    for b in bad:
        with pytest.raises(pk.KVError) as e:
            pk.kv_serve_create(pool, s, 8, pk.KV_BF16, 0.1, b.get("order", pk.KV_ORDER_BATCH), 8, 64,
                               b.get("max_width", 16), None, b.get("swap_slots", 0), b.get("host", h), b.get("dev", d),
                               b.get("meta_bytes", need), ws, 16)
        assert e.value.code == pk.KV_ERR_ARG
    for f in (lambda: pk.kv_serve_schedule(None, []), lambda: pk.kv_serve_launch(None, 0, 0, 0, 0, 0, pk.KV_F32),
              lambda: pk.kv_serve_upload(None, 0, 0, 0), lambda: pk.kv_serve_readback(None, 0, 0, 0, 0)):
        with pytest.raises(pk.KVError) as e:
            f()
        assert e.value.code == pk.KV_ERR_ARG
    assert pk._lib.kv_serve_destroy(None) == pk.KV_OK
    assert ctypes.sizeof(pk.kv_step_layout) == 128
    pk.kv_pool_destroy(pool)
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


@pytest.mark.parametrize("lens,policy,want", [
    ([9, 19, 29], pk.KV_ORDER_LONG_FIRST, [2, 0, 1]),           # 20 equals the mean: not long
    ([9, 19, 29], pk.KV_ORDER_LONGEST, [2, 1, 0]),
    ([4, 4, 4, 4], pk.KV_ORDER_LONG_FIRST, [0, 1, 2, 3]),       # nothing above the mean
    ([4, 4, 4, 4], pk.KV_ORDER_LONGEST, [0, 1, 2, 3]),          # ties keep batch order
    ([1, 50, 3, 50, 2], pk.KV_ORDER_LONG_FIRST, [1, 3, 0, 2, 4]),
    ([1, 50, 3, 50, 2], pk.KV_ORDER_LONGEST, [1, 3, 2, 4, 0]),
])
def test_packed_orders_on_chosen_lengths(lens, policy, want):
    """Contexts of chosen lengths (each step appends one token): the packed
    scheduling order against the policy worked by hand."""
    a = pk.kv_alloc_create(64, 16)
    s = pk.kv_sched_create(a, 8)
    for i, n in enumerate(lens):
        pk.kv_alloc_allocate(a, i, n)
        pk.kv_sched_adopt(s, i)
    cap = pk.kv_step_packed_bytes(8, 8, 8, 0)
    buf = aligned(cap)
    lay = pk.kv_sched_step_packed(s, [], policy, 8, buf, cap)
    assert section(buf, lay.context_lens, np.int32, len(lens)).tolist() == [n + 1 for n in lens]
    assert section(buf, lay.seq_order, np.int32, len(lens)).tolist() == want
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


from hypothesis import HealthCheck, example, given, settings
from hypothesis import strategies as st


@settings(max_examples=60, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
# a window's releases free blocks that later appends of the same step take:
# the step must not report running out of blocks when the appends, run in
# order, fit (found by this test)
@example(seed=23, window=24, policy=pk.KV_ORDER_BATCH, max_seqs=6, nb=23, reserve=0, mode="none")
@given(seed=st.integers(0, 2 ** 31 - 1), window=st.sampled_from([0, 0, 24, 64]),
       policy=st.sampled_from([pk.KV_ORDER_BATCH, pk.KV_ORDER_LONGEST, pk.KV_ORDER_LONG_FIRST]),
       max_seqs=st.integers(1, 6), nb=st.integers(8, 40), reserve=st.sampled_from([-1, -1, 0]),
       mode=st.sampled_from(["none", "swap", "recompute", "caching"]))
def test_packed_step_random_operations(seed, window, policy, max_seqs, nb, reserve, mode):
    """Random arrivals (1 to 70 tokens; with prefix caching, token prompts
    sharing a system prefix), a forked group sharing its blocks, random
    finishes (all at once included), empty steps, small pools that hold
    admissions back, swap or recompute preemption, and with no admission reserve the appends running out of
    blocks (the step where that happens must agree): every packed array, the
    swap outputs and the allocator's free list and refcounts equal the
    oracle scheduler's."""
    rng = np.random.default_rng(seed)
    bs = 8
    order = rng.permutation(nb)
    caching = mode == "caching"
    bm = (PrefixCachingBlockManager if caching else BlockManager)(nb, bs, order)
    sch = Scheduler(bm, max_seqs, min_blocks=None if reserve < 0 else reserve, window=window)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    slots = int(rng.integers(0, 30)) if mode == "swap" else 0
    if caching:
        pk.kv_alloc_enable_prefix_caching(a)
    if mode in ("swap", "recompute"):
        bm.set_swap_space(slots)
        sch.preemption = mode
        pk.kv_alloc_set_swap_space(a, slots)
    s = pk.kv_sched_create(a, max_seqs, reserve)
    if mode in ("swap", "recompute"):
        pk.kv_sched_set_preemption(s, pk.KV_PREEMPT_SWAP if mode == "swap" else pk.KV_PREEMPT_RECOMPUTE)
    if window:
        pk.kv_sched_set_window(s, window)
    width = nb + 32  # windowed tables keep their released entries (-1): rows may outgrow the pool
    cap = pk.kv_step_packed_bytes(max_seqs, 200 * max_seqs, width, slots)
    buf = aligned(cap)
    system = [int(x) for x in rng.integers(0, 50, size=60)]
    remaining, nxt = {}, 0
    # a forked group sharing its blocks (the partly filled last one included)
    plen, forks = int(rng.integers(1, 3 * bs)), int(rng.integers(0, 3))
    if not caching and bm.can_allocate(plen):
        bm.allocate(10_000, plen)
        pk.kv_alloc_allocate(a, 10_000, plen)
        for c in range(forks):
            bm.fork(10_000, 10_001 + c)
            pk.kv_alloc_fork(a, 10_000, 10_001 + c)
        for sid in ([10_000] + [10_001 + c for c in range(forks)])[:max_seqs]:
            sch.adopt(sid)
            pk.kv_sched_adopt(s, sid)
            remaining[sid] = int(rng.integers(2, 40))
    try:
        for _ in range(25):
            for _ in range(int(rng.integers(0, 3))):
                if caching:
                    toks = system[:int(rng.integers(0, 60))] + [int(x) for x in rng.integers(0, 50, size=int(rng.integers(1, 30)))]
                    sch.add_request_tokens(nxt, toks)
                    pk.kv_sched_add_request_tokens(s, nxt, toks)
                else:
                    plen = int(rng.integers(1, 71))
                    sch.add_request(nxt, plen)
                    pk.kv_sched_add_request(s, nxt, plen)
                remaining[nxt] = int(rng.integers(2, 40))
                nxt += 1
            run = list(sch.running)
            fin = run if rng.random() < 0.05 else [r for r in run if remaining[r] <= 0 or rng.random() < 0.1]
            try:
                want = sch.step(fin)
            except OracleOOM:  # the oracle ran out of blocks for the appends: the native step must too
                with pytest.raises(pk.KVError) as e:
                    pk.kv_sched_step_packed(s, fin, policy, width, buf, cap)
                assert e.value.code == pk.KV_ERR_OOM
                break
            lay = pk.kv_sched_step_packed(s, fin, policy, width, buf, cap)
            check_step(buf, lay, want, policy, want["cached"] if caching else [0] * len(want["admitted"]))
            sw = pk.kv_sched_swap_outputs(s)
            assert list(sw["preempted"]) == want["preempted"] and list(sw["recomputed"]) == want["recomputed"]
            assert list(sw["swapped_in"]) == want["swapped_in"]
            free, rc = pk.kv_alloc_snapshot(a, nb)
            assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
            for r in want["running"]:
                remaining[r] -= 1
    finally:
        pk.kv_sched_destroy(s)
        pk.kv_alloc_destroy(a)


@pytest.mark.parametrize("hkv,hq,fmt,max_b,max_ctx", [
    (8, 64, pk.KV_BF16, 256, 8324),      # the GQA serving trace
    (40, 40, pk.KV_F16, 64, 2048),       # the Llama layer
    (32, 32, pk.KV_FP8_E4M3, 8, 16384),  # long FP8 contexts
])
def test_serve_workspace_bounds_every_batch_and_shorter_context(hkv, hq, fmt, max_b, max_ctx):
    """kv_serve_workspace_bytes takes the largest need over the batch sizes
    at the longest context; no step with fewer sequences or shorter contexts
    may need more (the split policy divides short contexts too)."""
    pool = pk.kv_pool_create(16, 4096, hkv, 128, fmt, 1)
    try:
        cap = pk.kv_serve_workspace_bytes(pool, hq, max_b, max_ctx)
        for b in list(range(1, 41)) + list(range(41, max_b + 1, 9)) + [max_b]:
            if b > max_b:
                continue
            for c in list(range(1, 400, 13)) + list(range(400, max_ctx + 1, 97)) + [max_ctx]:
                assert pk.paged_attention_workspace_bytes(pool, b, hq, c) <= cap, (b, c)
    finally:
        pk.kv_pool_destroy(pool)
