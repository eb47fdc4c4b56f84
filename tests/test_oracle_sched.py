"""Pins for the oracle's block allocator and scheduling step.

Hand-traced scenarios (tests/golden/sched_scenarios.json) fix the step order
and the FIFO policies; property checks over random operation sequences fix
the paging invariants the pages state: blocks taken on demand
(ceil(tokens / block_size) per sequence), no external fragmentation (any
free block serves any request), and reference-counted sharing."""

import json
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle.sched import BlockManager, OracleOOM, OracleStateError, Scheduler, blocks_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sched_scenarios.json")


def load(name):
    with open(GOLDEN) as f:
        return json.load(f)[name]


@pytest.mark.parametrize("name", ["admission", "head_of_line"])
def test_hand_traced_scheduler_scenarios(name):
    sc = load(name)
    bm = BlockManager(sc["num_blocks"], sc["block_size"], sc["initial_free_order"])
    sched = Scheduler(bm, sc["max_num_seqs"])
    for sid, plen in sc["requests"]:
        sched.add_request(sid, plen)
    for want in sc["steps"]:
        got = sched.step(want["finished"])
        for key in ("admitted", "running", "block_tables", "context_lens", "slot_mapping"):
            assert got[key] == want[key], key
        assert [list(p) for p in got["cow_pairs"]] == want["cow_pairs"]
        assert bm.snapshot()[0] == want["free_list"]


def test_hand_traced_fork_and_copy_on_write():
    sc = load("fork_cow")
    bm = BlockManager(sc["num_blocks"], sc["block_size"], sc["initial_free_order"])
    bm.allocate(*sc["allocate"])
    bm.fork(*sc["fork"])
    assert bm.snapshot()[1] == sc["refcounts_after_fork"]
    child, parent = sc["fork"][1], sc["fork"][0]
    assert list(bm.append_slot(child)) == sc["append_child"]
    assert bm.block_table(child) == sc["child_table_after"]
    assert list(bm.append_slot(parent)) == sc["append_parent"]
    bm.free(parent)
    bm.free(child)
    assert bm.snapshot()[0] == sc["free_list_after_freeing_parent_then_child"]
    with pytest.raises(OracleStateError):
        bm.free(child)


def check_invariants(bm: BlockManager):
    free, rc = bm.snapshot()
    assert len(set(free)) == len(free)
    held = [0] * bm.num_blocks
    for sid, table in bm.tables.items():
        # on demand: exactly ceil(tokens / block_size) blocks
        assert len(table) == blocks_for(bm.tokens[sid], bm.block_size)
        for b in table:
            held[b] += 1
    assert held == rc  # a block's count is the number of tables holding it
    for b in free:
        assert rc[b] == 0  # never both free and referenced
    assert len(free) + sum(1 for c in rc if c > 0) == bm.num_blocks


ops = st.lists(st.tuples(st.sampled_from(["alloc", "append", "fork", "free"]),
                         st.integers(0, 9), st.integers(0, 40)), max_size=80)


@settings(max_examples=150, deadline=None)
@given(ops, st.integers(0, 2 ** 31 - 1))
def test_random_operations_keep_the_paging_invariants(seq, seed):
    rng = np.random.default_rng(seed)
    bm = BlockManager(24, 4, rng.permutation(24))
    next_id = 100
    for op, a, n in seq:
        ids = sorted(bm.tables)
        try:
            if op == "alloc":
                free_before = bm.get_num_free_blocks()
                ok = bm.can_allocate(n)
                try:
                    bm.allocate(next_id, n)
                    assert ok
                    # no external fragmentation: any free blocks will do
                    assert bm.get_num_free_blocks() == free_before - blocks_for(n, 4)
                except OracleOOM:
                    assert not ok
                next_id += 1
            elif op == "append" and ids:
                sid = ids[a % len(ids)]
                shared_before = bm.tables[sid][-1] if bm.tables[sid] else None
                pos = bm.tokens[sid]
                rc_last = bm.refcount[shared_before] if shared_before is not None else 0
                slot, cs, cd = bm.append_slot(sid)
                assert slot // 4 == bm.tables[sid][pos // 4] and slot % 4 == pos % 4
                if pos % 4 != 0 and rc_last > 1:
                    assert cs == shared_before and cd == bm.tables[sid][-1]
                else:
                    assert cs == cd == -1
            elif op == "fork" and ids:
                bm.fork(ids[a % len(ids)], next_id)
                next_id += 1
            elif op == "free" and ids:
                bm.free(ids[a % len(ids)])
        except OracleOOM:
            pass
        check_invariants(bm)


def test_free_and_can_allocate_edge_cases():
    bm = BlockManager(3, 16)
    assert bm.can_allocate(48) and not bm.can_allocate(49)
    bm.allocate(1, 0)
    assert bm.block_table(1) == [] and bm.get_num_free_blocks() == 3
    assert bm.append_slot(1) == (0, -1, -1)  # first token opens a block
    with pytest.raises(OracleStateError):
        bm.allocate(1, 5)
    with pytest.raises(OracleOOM):
        bm.allocate(2, 49)
    with pytest.raises(OracleStateError):
        bm.free(7)


def test_scheduler_never_fails_an_append_with_the_default_reserve():
    rng = np.random.default_rng(30)
    bm = BlockManager(64, 16, rng.permutation(64))
    sched = Scheduler(bm, max_num_seqs=16)
    sid = 0
    running_len = {}
    for it in range(300):
        for _ in range(rng.poisson(1.0)):
            sched.add_request(sid, int(rng.integers(1, 120)))
            running_len[sid] = int(rng.integers(1, 60))
            sid += 1
        done = [s for s in sched.running if running_len[s] <= 0]
        out = sched.step(done)
        for s in sched.running:
            running_len[s] -= 1
        assert len(out["slot_mapping"]) == len(out["running"]) + sum(
            bm.tokens[s] - 1 for s in out["admitted"])
        check_invariants(bm)
