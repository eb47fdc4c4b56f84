"""Sliding window, host side: the oracle's block release pinned to paging
invariants and a closed form (blocks kept = those holding the last `window`
positions), then the native allocator and scheduling step against it,
operation by operation."""

import numpy as np
import pytest

import paged_kv_cache_451_b200 as pk
from oracle.sched import BlockManager, Scheduler


def test_release_keeps_exactly_the_blocks_of_the_window():
    bs, W = 16, 40
    bm = BlockManager(64, bs)
    bm.allocate(1, 100)
    before = list(bm.tables[1])
    n = bm.release_before(1, 100 - W)  # positions 60..99 stay: blocks 3..6
    assert n == 3 and bm.tables[1][:3] == [-1, -1, -1] and bm.tables[1][3:] == before[3:]
    assert list(bm.free_list)[-3:] == before[:3]
    assert bm.release_before(1, 100 - W) == 0  # idempotent
    bm.free(1)
    assert sorted(bm.free_list) == list(range(64))


def test_release_of_a_shared_block_drops_one_reference():
    bm = BlockManager(16, 4)
    bm.allocate(1, 10)
    bm.fork(1, 2)
    b0 = bm.tables[1][0]
    bm.release_before(1, 8)
    assert bm.refcount[b0] == 1 and b0 not in bm.free_list
    bm.release_before(2, 8)
    assert bm.refcount[b0] == 0 and b0 in bm.free_list


@pytest.mark.parametrize("window", [1, 16, 50])
def test_native_scheduler_with_window_matches_oracle(window):
    rng = np.random.default_rng(window)
    nb, bs = 300, 16
    order = rng.permutation(nb)
    bm = BlockManager(nb, bs, order)
    sch = Scheduler(bm, 32, window=window)
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    s = pk.kv_sched_create(a, 32)
    pk.kv_sched_set_window(s, window)
    running, nxt = [], 0
    for it in range(80):
        for _ in range(int(rng.poisson(1.0))):
            plen = int(rng.integers(1, 120))
            sch.add_request(nxt, plen)
            pk.kv_sched_add_request(s, nxt, plen)
            nxt += 1
        fin = [r for r in running if rng.random() < 0.05]
        want = sch.step(fin)
        info = pk.kv_sched_step(s, fin)
        got = pk.kv_sched_outputs(s, info)
        assert list(got["running"]) == want["running"]
        for row, t in zip(got["block_tables"], want["block_tables"]):
            assert list(row[:len(t)]) == t  # released entries are -1 on both sides
        assert list(got["context_lens"]) == want["context_lens"]
        assert list(got["slot_mapping"]) == want["slot_mapping"]
        free, rc = pk.kv_alloc_snapshot(a, nb)
        assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
        # every running sequence holds only the blocks its window touches
        for sid, t, n in zip(want["running"], want["block_tables"], want["context_lens"]):
            if sid in want["admitted"]:
                continue
            held = [i for i, b in enumerate(t) if b >= 0]
            assert held == list(range(max(0, n - window) // bs, -(-n // bs)))
        running = want["running"]
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_native_release_before_matches_oracle():
    bm = BlockManager(20, 4)
    a = pk.kv_alloc_create(20, 4)
    for sid, n in ((1, 17), (2, 9)):
        bm.allocate(sid, n)
        pk.kv_alloc_allocate(a, sid, n)
    bm.fork(1, 3)
    pk.kv_alloc_fork(a, 1, 3)
    for sid, tok in ((1, 9), (3, 5), (2, 100), (1, 12)):
        assert pk.kv_alloc_release_before(a, sid, tok) == bm.release_before(sid, tok)
        assert list(pk.kv_alloc_block_table(a, sid)) == bm.tables[sid]
        free, rc = pk.kv_alloc_snapshot(a, 20)
        assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
    for sid in (1, 2, 3):
        bm.free(sid)
        pk.kv_alloc_free(a, sid)
    free, rc = pk.kv_alloc_snapshot(a, 20)
    assert list(free) == list(bm.free_list) and sorted(free) == list(range(20))
    pk.kv_alloc_destroy(a)


def test_release_covers_only_positions_the_sequence_holds():
    """Traced by hand: a window release past the sequence's length keeps the
    block that receives the next token.  9 tokens in blocks of 4: blocks 0
    and 1 (positions 0..7) go, block 2 (position 8, next token 9) stays and
    the append lands in it at offset 1.  16 tokens: all four full blocks go
    and the append takes a fresh block."""
    for native in (False, True):
        if native:
            a = pk.kv_alloc_create(8, 4)
            pk.kv_alloc_allocate(a, 1, 9)
            pk.kv_alloc_allocate(a, 2, 16)
            t1, t2 = list(pk.kv_alloc_block_table(a, 1)), list(pk.kv_alloc_block_table(a, 2))
            n1, n2 = pk.kv_alloc_release_before(a, 1, 100), pk.kv_alloc_release_before(a, 2, 100)
            slot1, _, _ = pk.kv_alloc_append_slot(a, 1)
            slot2, _, _ = pk.kv_alloc_append_slot(a, 2)
            tab1, tab2 = list(pk.kv_alloc_block_table(a, 1)), list(pk.kv_alloc_block_table(a, 2))
            pk.kv_alloc_destroy(a)
        else:
            bm = BlockManager(8, 4)
            bm.allocate(1, 9)
            bm.allocate(2, 16)
            t1, t2 = list(bm.tables[1]), list(bm.tables[2])
            n1, n2 = bm.release_before(1, 100), bm.release_before(2, 100)
            slot1, _, _ = bm.append_slot(1)
            slot2, _, _ = bm.append_slot(2)
            tab1, tab2 = list(bm.tables[1]), list(bm.tables[2])
        assert (n1, n2) == (2, 4)
        assert tab1 == [-1, -1, t1[2]] and slot1 == t1[2] * 4 + 1
        assert tab2[:4] == [-1, -1, -1, -1] and len(tab2) == 5 and tab2[4] >= 0 and slot2 == tab2[4] * 4
