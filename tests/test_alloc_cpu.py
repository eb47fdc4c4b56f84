"""The native allocator and scheduling step match the oracle's exactly:
the hand-traced scenarios, and random operation sequences / traces compared
state by state (tables, slots, copy-on-write pairs, free-list order,
refcounts)."""

import json
import os

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

import paged_kv_cache_451_b200 as pk
from oracle.sched import BlockManager, OracleOOM, OracleStateError, Scheduler

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sched_scenarios.json")


def native_state(a, nb):
    free, rc = pk.kv_alloc_snapshot(a, nb)
    return list(free), list(rc)


@pytest.mark.parametrize("name", ["admission", "head_of_line"])
def test_native_scheduler_matches_hand_traced_scenarios(name):
    sc = json.load(open(GOLDEN))[name]
    a = pk.kv_alloc_create(sc["num_blocks"], sc["block_size"], sc["initial_free_order"])
    s = pk.kv_sched_create(a, sc["max_num_seqs"])
    for sid, plen in sc["requests"]:
        pk.kv_sched_add_request(s, sid, plen)
    for want in sc["steps"]:
        info = pk.kv_sched_step(s, want["finished"])
        out = pk.kv_sched_outputs(s, info)
        assert list(out["admitted"]) == want["admitted"]
        assert list(out["running"]) == want["running"]
        tables = [list(r[r >= 0]) for r in out["block_tables"]]
        assert tables == want["block_tables"]
        assert list(out["context_lens"]) == want["context_lens"]
        assert list(out["slot_mapping"]) == want["slot_mapping"]
        assert out["cow_pairs"].tolist() == want["cow_pairs"]
        assert native_state(a, sc["num_blocks"])[0] == want["free_list"]
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_native_fork_and_copy_on_write_matches_hand_trace():
    sc = json.load(open(GOLDEN))["fork_cow"]
    a = pk.kv_alloc_create(sc["num_blocks"], sc["block_size"], sc["initial_free_order"])
    pk.kv_alloc_allocate(a, *sc["allocate"])
    pk.kv_alloc_fork(a, *sc["fork"])
    assert native_state(a, sc["num_blocks"])[1] == sc["refcounts_after_fork"]
    parent, child = sc["fork"]
    assert list(pk.kv_alloc_append_slot(a, child)) == sc["append_child"]
    assert list(pk.kv_alloc_block_table(a, child)) == sc["child_table_after"]
    assert list(pk.kv_alloc_append_slot(a, parent)) == sc["append_parent"]
    pk.kv_alloc_free(a, parent)
    pk.kv_alloc_free(a, child)
    assert native_state(a, sc["num_blocks"])[0] == sc["free_list_after_freeing_parent_then_child"]
    with pytest.raises(pk.KVError) as e:
        pk.kv_alloc_free(a, child)
    assert e.value.code == pk.KV_ERR_STATE
    pk.kv_alloc_destroy(a)


ops = st.lists(st.tuples(st.sampled_from(["alloc", "append", "fork", "free"]),
                         st.integers(0, 9), st.integers(0, 40)), max_size=100)


@settings(max_examples=200, deadline=None)
@given(ops, st.integers(0, 2 ** 31 - 1))
def test_native_allocator_matches_oracle_on_random_operations(seq, seed):
    rng = np.random.default_rng(seed)
    nb, bs = 20, 4
    order = rng.permutation(nb)
    ref = BlockManager(nb, bs, order)
    a = pk.kv_alloc_create(nb, bs, order)
    nid = 1
    for op, x, n in seq:
        ids = sorted(ref.tables)
        if op == "alloc":
            try:
                ref.allocate(nid, n)
                pk.kv_alloc_allocate(a, nid, n)
            except OracleOOM:
                with pytest.raises(pk.KVError) as e:
                    pk.kv_alloc_allocate(a, nid, n)
                assert e.value.code == pk.KV_ERR_OOM
            nid += 1
        elif op == "append" and ids:
            sid = ids[x % len(ids)]
            try:
                want = ref.append_slot(sid)
            except OracleOOM:
                with pytest.raises(pk.KVError) as e:
                    pk.kv_alloc_append_slot(a, sid)
                assert e.value.code == pk.KV_ERR_OOM
            else:
                assert pk.kv_alloc_append_slot(a, sid) == want
        elif op == "fork" and ids:
            ref.fork(ids[x % len(ids)], nid)
            pk.kv_alloc_fork(a, ids[x % len(ids)], nid)
            nid += 1
        elif op == "free" and ids:
            ref.free(ids[x % len(ids)])
            pk.kv_alloc_free(a, ids[x % len(ids)])
        assert native_state(a, nb) == tuple(map(list, ref.snapshot())) or \
            native_state(a, nb) == [list(v) for v in ref.snapshot()]
        for sid in ref.tables:
            assert list(pk.kv_alloc_block_table(a, sid)) == ref.tables[sid]
            assert pk.kv_alloc_num_tokens(a, sid) == ref.tokens[sid]
    assert pk.kv_alloc_num_free(a) == ref.get_num_free_blocks()
    assert pk.kv_alloc_counters(a) == (ref.num_alloc, ref.num_freed, ref.num_cow)
    pk.kv_alloc_destroy(a)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_native_scheduler_matches_oracle_on_random_traces(seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs = 96, 16
    order = rng.permutation(nb)
    ref_bm = BlockManager(nb, bs, order)
    ref = Scheduler(ref_bm, max_num_seqs=12)
    a = pk.kv_alloc_create(nb, bs, order)
    s = pk.kv_sched_create(a, 12)
    # a shared prefix: parent forked into sharers, all running
    ref_bm.allocate(0, 37)
    pk.kv_alloc_allocate(a, 0, 37)
    for c in (1, 2, 3):
        ref_bm.fork(0, c)
        pk.kv_alloc_fork(a, 0, c)
    for c in (0, 1, 2, 3):
        ref.adopt(c)
        pk.kv_sched_adopt(s, c)
    remaining = {c: int(rng.integers(1, 30)) for c in range(4)}
    sid = 10
    for it in range(200):
        for _ in range(int(rng.poisson(0.8))):
            plen = int(rng.integers(1, 100))
            ref.add_request(sid, plen)
            pk.kv_sched_add_request(s, sid, plen)
            remaining[sid] = int(rng.integers(1, 40))
            sid += 1
        done = [r for r in ref.running if remaining[r] <= 0]
        want = ref.step(done)
        info = pk.kv_sched_step(s, done)
        got = pk.kv_sched_outputs(s, info)
        assert list(got["running"]) == want["running"]
        assert [list(r[r >= 0]) for r in got["block_tables"]] == want["block_tables"]
        assert list(got["context_lens"]) == want["context_lens"]
        assert list(got["slot_mapping"]) == want["slot_mapping"]
        assert got["cow_pairs"].tolist() == [list(p) for p in want["cow_pairs"]]
        assert list(got["admitted"]) == want["admitted"]
        assert [list(x) for x in pk.kv_alloc_snapshot(a, nb)] == [list(x) for x in ref_bm.snapshot()]
        assert pk.kv_sched_stats(s) == ref.stats()
        for r in ref.running:
            remaining[r] -= 1
    assert ref_bm.num_cow >= 3  # the forked prefix was copied on write
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_native_scheduler_rejects_bad_finished_ids_without_changes():
    a = pk.kv_alloc_create(8, 4)
    s = pk.kv_sched_create(a, 4)
    pk.kv_sched_add_request(s, 1, 3)
    pk.kv_sched_step(s, [])
    before = pk.kv_alloc_snapshot(a, 8)
    for bad, msg in (([7], "7 is not running"), ([1, 1], "1 finished twice"), ([1, 7], "7 is not running"),
                     ([7, 1], "7 is not running")):
        with pytest.raises(pk.KVError) as e:
            pk.kv_sched_step(s, bad)
        assert e.value.code == pk.KV_ERR_STATE and msg in pk.kv_last_error()
    after = pk.kv_alloc_snapshot(a, 8)
    assert all(np.array_equal(x, y) for x, y in zip(before, after))
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_native_scheduler_reports_append_oom_with_explicit_small_reserve():
    a = pk.kv_alloc_create(2, 4)
    s = pk.kv_sched_create(a, 4, 0)  # MIN_BLOCKS = 0: no reserve
    pk.kv_sched_add_request(s, 1, 4)
    pk.kv_sched_add_request(s, 2, 4)
    with pytest.raises(pk.KVError) as e:
        pk.kv_sched_step(s, [])
    assert e.value.code == pk.KV_ERR_OOM
    assert pk.kv_sched_stats(s)[:2] == (2, 0)
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


@settings(max_examples=80, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(seed=st.integers(0, 2 ** 31 - 1), nb=st.integers(2, 30), bs=st.sampled_from([4, 8, 16]))
def test_native_allocator_random_operations_match_oracle(seed, nb, bs):
    """Random allocate / append / fork / free / window release sequences
    (release tokens below, at and past a sequence's length, exhaustion
    included): every result, error and the full allocator state (free list
    order, refcounts, every live table) equal the oracle's after each
    operation."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    bm = BlockManager(nb, bs, order)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    live, nxt = [], 0
    try:
        for _ in range(60):
            kind = str(rng.choice(["alloc", "append", "append", "fork", "free", "release"]))
            if kind != "alloc" and not live:
                continue
            sid = int(rng.choice(live)) if kind != "alloc" else None
            n = int(rng.integers(0, 40))
            tok = int(rng.integers(-5, bm.tokens[sid] + 6)) if kind == "release" else 0
            ops = {
                "alloc": (lambda: bm.allocate(nxt, n), lambda: pk.kv_alloc_allocate(a, nxt, n)),
                "append": (lambda: bm.append_slot(sid), lambda: pk.kv_alloc_append_slot(a, sid)),
                "fork": (lambda: bm.fork(sid, nxt), lambda: pk.kv_alloc_fork(a, sid, nxt)),
                "free": (lambda: bm.free(sid), lambda: pk.kv_alloc_free(a, sid)),
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
            if kind in ("append", "release"):
                assert tuple(np.atleast_1d(got)) == tuple(np.atleast_1d(want)), kind
            if kind in ("alloc", "fork"):
                live.append(nxt)
                nxt += 1
            elif kind == "free":
                live.remove(sid)
            free, rc = pk.kv_alloc_snapshot(a, nb)
            assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
            for x in live:
                assert list(pk.kv_alloc_block_table(a, x)) == bm.block_table(x)
    finally:
        pk.kv_alloc_destroy(a)
