"""Prefix caching: the oracle's block manager pinned to the FNV-1a test
vectors, to a closed form for its hits (the longest full-block common prefix
with any committed prompt, while nothing has been evicted) and to paging
invariants; then the native allocator and scheduler against the oracle,
operation by operation (bit-exact tables, cached counts, free lists,
refcounts)."""

import os

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import paged_kv_cache_451_b200 as pk
from oracle.sched import OracleOOM, OracleStateError, PrefixCachingBlockManager, Scheduler, block_key, fnv1a64

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fnv1a64_published_vectors():
    with open(os.path.join(HERE, "golden", "fnv1a64.txt")) as f:
        rows = [ln.rstrip("\n").split("\t") for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for text, want in rows:
        assert fnv1a64(text.strip('"').encode()) == int(want, 16)


def test_block_key_depends_on_parent_and_every_token():
    base = block_key(1, [5, 6, 7, 8])
    assert block_key(2, [5, 6, 7, 8]) != base
    for i in range(4):
        t = [5, 6, 7, 8]
        t[i] += 1
        assert block_key(1, t) != base


def lcp_blocks(a, b, bs):
    n = 0
    while (n + 1) * bs <= min(len(a), len(b)) and a[n * bs:(n + 1) * bs] == b[n * bs:(n + 1) * bs]:
        n += 1
    return n


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.lists(st.tuples(st.integers(0, 3), st.integers(1, 70)), min_size=1, max_size=12),
       st.sampled_from([4, 16]))
def test_hits_equal_longest_common_prefix_while_nothing_is_evicted(prompts, bs):
    """Prompts drawn from a few shared stems: with a pool that never evicts,
    a new prompt hits min((n - 1) // bs, max lcp over committed prompts)."""
    rng = np.random.default_rng(len(prompts) * 31 + bs)
    stems = [list(rng.integers(0, 50, size=80)) for _ in range(4)]
    bm = PrefixCachingBlockManager(4096, bs)
    committed = []
    for i, (stem, n) in enumerate(prompts):
        toks = stems[stem][:n]
        want = min((n - 1) // bs, max([lcp_blocks(toks, c, bs) for c in committed] or [0]))
        hit = bm.allocate_prompt(i, toks)
        assert hit == want * bs
        # the shared blocks are exactly those of a committed prompt with that prefix
        bm.commit(i)
        committed.append(toks)
        if i % 3 == 2:
            bm.free(i)
        assert bm.num_evictions == 0


def test_hits_stop_at_first_difference_and_need_the_same_position():
    bs = 4
    bm = PrefixCachingBlockManager(64, bs)
    a = list(range(100, 120))
    bm.allocate_prompt(0, a)
    bm.commit(0)
    b = a[:9] + [999] + a[10:]  # differs inside block 2
    assert bm.allocate_prompt(1, b) == 8
    assert bm.tables[1][:2] == bm.tables[0][:2] and bm.tables[1][2] != bm.tables[0][2]
    c = a[4:]  # same blocks shifted by one block: parents differ, no hit
    assert bm.allocate_prompt(2, c) == 0
    assert bm.allocate_prompt(3, a) == 16  # capped: the last token is always computed
    assert bm.allocate_prompt(4, a[:8]) == 4


def test_free_keeps_keys_until_eviction_deepest_first():
    bs = 4
    bm = PrefixCachingBlockManager(6, bs)
    a = list(range(12))
    bm.allocate_prompt(0, a + [50])  # 4 blocks, 3 full registered
    bm.commit(0)
    blocks = list(bm.tables[0])
    bm.free(0)
    assert list(bm.free_list)[-4:] == blocks[::-1]
    assert bm.allocate_prompt(1, a + [60]) == 12  # hits from the free list
    bm.free(1)
    # free list now [5, 3, 4, 2, 1, 0]: a foreign 4-block prompt takes 5, 3, 4
    # (never registered) and 2, the deepest cached block; the stem survives
    bm.allocate_prompt(2, list(range(500, 516)))
    assert bm.num_evictions == 1
    bm.free(2)
    assert bm.allocate_prompt(3, a + [70]) == 8


def test_paging_invariants_under_random_operations():
    rng = np.random.default_rng(5)
    bs = 8
    bm = PrefixCachingBlockManager(40, bs)
    stems = [list(rng.integers(0, 20, size=60)) for _ in range(3)]
    live = {}
    for step in range(400):
        op = rng.integers(0, 4)
        if op == 0 or not live:
            sid = step
            toks = stems[rng.integers(0, 3)][:int(rng.integers(1, 60))]
            try:
                hit = bm.allocate_prompt(sid, toks)
            except OracleOOM:
                continue
            live[sid] = toks
            tbl = bm.tables[sid]
            for i in range(hit // bs):  # every hit block holds the prompt's tokens
                assert bm.key_of[tbl[i]][2] == tuple(toks[i * bs:(i + 1) * bs])
            bm.commit(sid)
        elif op == 1:
            sid = list(live)[rng.integers(0, len(live))]
            bm.free(sid)
            del live[sid]
        elif op == 2:
            sid = list(live)[rng.integers(0, len(live))]
            try:
                bm.append_token(sid, int(rng.integers(0, 20)))
            except OracleOOM:
                pass
        else:
            sid = list(live)[rng.integers(0, len(live))]
            bm.commit(sid)
        held = {}
        for tbl in bm.tables.values():
            for b in tbl:
                held[b] = held.get(b, 0) + 1
        assert all(bm.refcount[b] == held.get(b, 0) for b in range(40))
        assert set(bm.free_list) == {b for b in range(40) if bm.refcount[b] == 0}
        assert len(set(bm.free_list)) == len(bm.free_list)
        for k, b in bm.cached.items():
            assert bm.key_of[b][0] == k


# ---------------------------------------------------------- native vs oracle

def native_state(a, n):
    free, rc = pk.kv_alloc_snapshot(a, n)
    return list(free), list(rc)


@pytest.mark.parametrize("seed", range(6))
def test_native_allocator_matches_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs = int(rng.integers(20, 60)), int(rng.choice([4, 16]))
    order = rng.permutation(nb)
    bm = PrefixCachingBlockManager(nb, bs, order)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    pk.kv_alloc_enable_prefix_caching(a)
    stems = [list(rng.integers(0, 30, size=120)) for _ in range(3)]
    live = []
    for step in range(300):
        op = int(rng.integers(0, 5))
        if op <= 1 or not live:
            toks = stems[int(rng.integers(0, 3))][:int(rng.integers(1, 120))]
            try:
                want = bm.allocate_prompt(step, toks)
            except OracleOOM:
                with pytest.raises(pk.KVError) as e:
                    pk.kv_alloc_allocate_prompt(a, step, toks)
                assert e.value.code == pk.KV_ERR_OOM
                continue
            assert pk.kv_alloc_allocate_prompt(a, step, toks) == want
            live.append(step)
        elif op == 2:
            sid = live.pop(int(rng.integers(0, len(live))))
            bm.free(sid)
            pk.kv_alloc_free(a, sid)
        elif op == 3:
            sid = live[int(rng.integers(0, len(live)))]
            tok = int(rng.integers(0, 30))
            try:
                want = bm.append_token(sid, tok)
            except OracleOOM:
                with pytest.raises(pk.KVError):
                    pk.kv_alloc_append_token(a, sid, tok)
                continue
            assert pk.kv_alloc_append_token(a, sid, tok) == want
        else:
            sid = live[int(rng.integers(0, len(live)))]
            assert pk.kv_alloc_commit(a, sid) == bm.commit(sid)
        for sid in live:
            assert list(pk.kv_alloc_block_table(a, sid)) == bm.tables[sid]
        assert native_state(a, nb) == (list(bm.free_list), bm.refcount)
        assert pk.kv_alloc_prefix_stats(a) == (bm.num_hits, bm.num_evictions, len(bm.cached))
    pk.kv_alloc_destroy(a)


def test_enable_after_allocation_is_rejected():
    a = pk.kv_alloc_create(8, 4)
    pk.kv_alloc_allocate(a, 1, 3)
    with pytest.raises(pk.KVError) as e:
        pk.kv_alloc_enable_prefix_caching(a)
    assert e.value.code == pk.KV_ERR_STATE
    pk.kv_alloc_destroy(a)


@pytest.mark.parametrize("seed", range(4))
def test_native_scheduler_with_prompt_tokens_matches_oracle(seed):
    rng = np.random.default_rng(200 + seed)
    nb, bs = 160, 16
    order = rng.permutation(nb)
    bm = PrefixCachingBlockManager(nb, bs, order)
    sch = Scheduler(bm, 24)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    pk.kv_alloc_enable_prefix_caching(a)
    s = pk.kv_sched_create(a, 24)
    system = list(rng.integers(0, 1000, size=200))  # a shared system prompt
    nxt = 0
    running = []
    for it in range(60):
        for _ in range(int(rng.poisson(1.5))):
            toks = system[:int(rng.integers(0, 200))] + list(rng.integers(0, 1000, size=int(rng.integers(1, 60))))
            sch.add_request_tokens(nxt, toks)
            pk.kv_sched_add_request_tokens(s, nxt, toks)
            nxt += 1
        fin = [r for r in running if rng.random() < 0.15]
        want = sch.step(fin)
        info = pk.kv_sched_step(s, fin)
        got = pk.kv_sched_outputs(s, info)
        assert list(got["running"]) == want["running"]
        assert [list(r[r >= 0]) for r in got["block_tables"]] == want["block_tables"]
        assert list(got["context_lens"]) == want["context_lens"]
        assert list(got["slot_mapping"]) == want["slot_mapping"]
        assert list(got["admitted"]) == want["admitted"]
        assert list(got["cached"]) == want["cached"]
        assert native_state(a, nb) == (list(bm.free_list), bm.refcount)
        running = want["running"]
    hits, _, _ = pk.kv_alloc_prefix_stats(a)
    assert hits > 0
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


@settings(max_examples=60, deadline=None, derandomize=True)
@given(seed=st.integers(0, 2 ** 31 - 1), nb=st.integers(3, 30), bs=st.sampled_from([4, 8]))
def test_native_prefix_caching_random_operations_match_oracle(seed, nb, bs):
    """Random prompts sharing a system prefix (cache hits, evictions),
    token appends and plain appends, commits, frees, forks and window
    releases: results, errors, the free list, refcounts and every live table
    equal the oracle's after each operation."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    bm = PrefixCachingBlockManager(nb, bs, order)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    pk.kv_alloc_enable_prefix_caching(a)
    system = [int(x) for x in rng.integers(0, 6, size=40)]
    live, nxt = [], 0
    try:
        for _ in range(60):
            kind = str(rng.choice(["prompt", "prompt", "append_tok", "append", "commit", "free", "fork", "release"]))
            if kind != "prompt" and not live:
                continue
            sid = int(rng.choice(live)) if kind != "prompt" else None
            toks = system[:int(rng.integers(0, 40))] + [int(x) for x in rng.integers(0, 6, size=int(rng.integers(1, 12)))]
            tk = int(rng.integers(0, 6))
            tok = int(rng.integers(-3, (bm.tokens[sid] if sid is not None else 0) + 5))
            ops = {
                "prompt": (lambda: bm.allocate_prompt(nxt, toks), lambda: pk.kv_alloc_allocate_prompt(a, nxt, toks)),
                "append_tok": (lambda: bm.append_token(sid, tk), lambda: pk.kv_alloc_append_token(a, sid, tk)),
                "append": (lambda: bm.append_slot(sid), lambda: pk.kv_alloc_append_slot(a, sid)),
                "commit": (lambda: bm.commit(sid), lambda: pk.kv_alloc_commit(a, sid)),
                "free": (lambda: bm.free(sid), lambda: pk.kv_alloc_free(a, sid)),
                "fork": (lambda: bm.fork(sid, nxt), lambda: pk.kv_alloc_fork(a, sid, nxt)),
                "release": (lambda: bm.release_before(sid, tok), lambda: pk.kv_alloc_release_before(a, sid, tok)),
            }[kind]
            try:
                want, oerr = ops[0](), None
            except (OracleOOM, OracleStateError) as e:
                want, oerr = None, e
            if oerr is not None:
                with pytest.raises(pk.KVError) as e:
                    ops[1]()
                assert e.value.code == (pk.KV_ERR_OOM if isinstance(oerr, OracleOOM) else pk.KV_ERR_STATE)
                continue
            got = ops[1]()
            if kind not in ("free", "fork"):
                assert tuple(np.atleast_1d(got)) == tuple(np.atleast_1d(want)), kind
            if kind in ("prompt", "fork"):
                live.append(nxt)
                nxt += 1
            elif kind == "free":
                live.remove(sid)
            assert native_state(a, nb) == (list(bm.free_list), bm.refcount)
            for x in live:
                assert list(pk.kv_alloc_block_table(a, x)) == bm.block_table(x)
    finally:
        pk.kv_alloc_destroy(a)
