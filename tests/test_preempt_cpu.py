"""Preemption with swap-out / swap-in and recompute, host side: a hand-traced
scenario of the oracle's policy (latest sequence preempted first, swapped
sequences back first in first out, nothing admitted while one is swapped
out), paging invariants, and the native scheduler against the oracle step by
step under a pool small enough to force preemption."""

import numpy as np
import pytest

import paged_kv_cache_451_b200 as pk
from oracle.sched import BlockManager, Scheduler


def test_hand_traced_swap_scenario():
    bs = 4
    bm = BlockManager(6, bs)
    bm.set_swap_space(8)
    sch = Scheduler(bm, 8, min_blocks=0)
    sch.preemption = "swap"
    sch.add_request(1, 4)  # 1 block; its first append opens block 2
    sch.add_request(2, 4)
    out = sch.step([])
    assert out["admitted"] == [1, 2] and out["running"] == [1, 2]
    # seq 1 and 2 each hold 2 blocks (4 prompt + 1 appended token) -> 2 free
    for _ in range(3):
        out = sch.step([])  # tokens 6, 7, 8: no new block needed
    assert bm.get_num_free_blocks() == 2
    out = sch.step([])  # token 9 of each opens a block: 2 needed, 2 free -> fits
    assert not out["preempted"] and bm.get_num_free_blocks() == 0
    for _ in range(3):
        sch.step([])
    held = list(bm.tables[2])
    out = sch.step([])  # token 13: both need a block, none free -> preempt seq 2 (the latest)
    assert out["preempted"] == [2] and out["running"] == [1]
    assert [b for b, _ in out["swap_out"]] == held and [s_ for _, s_ in out["swap_out"]] == [0, 1, 2]
    assert bm.tables[2] == [-2, -3, -4]
    sch.add_request(3, 2)
    out = sch.step([1])  # seq 1 finishes: seq 2 comes back (same slots) before seq 3 is admitted
    assert out["swapped_in"] == [2] and [s_ for s_, _ in out["swap_in"]] == [0, 1, 2]
    assert out["running"] == [2, 3] and out["admitted"] == [3]
    assert all(b >= 0 for b in bm.tables[2])


def test_recompute_requeues_the_whole_context_first():
    bm = BlockManager(4, 4)
    sch = Scheduler(bm, 8, min_blocks=0)
    sch.preemption = "recompute"
    sch.add_request(1, 7)
    sch.add_request(2, 4)
    sch.step([])
    sch.add_request(3, 1)
    out = sch.step([])  # seq 1 at 8 tokens + seq 2 at 6: appends need 1 block, 0 free -> seq 2 out
    assert out["recomputed"] == [2] and 2 not in bm.tables
    assert sch.waiting[0][:2] == (2, 5)  # its context (4 prompt + 1) is the new prompt, ahead of 3


@pytest.mark.parametrize("mode,seed", [("swap", 0), ("swap", 1), ("recompute", 2), ("swap", 3)])
def test_native_preemption_matches_oracle(mode, seed):
    rng = np.random.default_rng(300 + seed)
    nb, bs = 48, 8
    slots = 24 if seed != 3 else 4  # seed 3: swap space too small, falls back to recompute
    order = rng.permutation(nb)
    bm = BlockManager(nb, bs, order)
    bm.set_swap_space(slots)
    sch = Scheduler(bm, 16)
    sch.preemption = mode
    a = pk.kv_alloc_create(nb, bs, order.astype(np.int32))
    pk.kv_alloc_set_swap_space(a, slots)
    s = pk.kv_sched_create(a, 16)
    pk.kv_sched_set_preemption(s, pk.KV_PREEMPT_SWAP if mode == "swap" else pk.KV_PREEMPT_RECOMPUTE)
    remaining, running, nxt = {}, [], 0
    preempted = 0
    for it in range(150):
        for _ in range(int(rng.poisson(0.6))):
            plen = int(rng.integers(1, 40))
            sch.add_request(nxt, plen)
            pk.kv_sched_add_request(s, nxt, plen)
            remaining[nxt] = int(rng.integers(5, 80))
            nxt += 1
        fin = [r for r in running if remaining[r] <= 0]
        want = sch.step(fin)
        info = pk.kv_sched_step(s, fin)
        got = pk.kv_sched_outputs(s, info)
        sw = pk.kv_sched_swap_outputs(s)
        assert list(got["running"]) == want["running"]
        for row, t in zip(got["block_tables"], want["block_tables"]):
            assert list(row[:len(t)]) == t
        assert list(got["context_lens"]) == want["context_lens"]
        assert list(got["slot_mapping"]) == want["slot_mapping"]
        assert list(got["admitted"]) == want["admitted"]
        assert sw["swap_out"].tolist() == [list(p) for p in want["swap_out"]]
        assert sw["swap_in"].tolist() == [list(p) for p in want["swap_in"]]
        assert list(sw["preempted"]) == want["preempted"]
        assert list(sw["recomputed"]) == want["recomputed"]
        assert list(sw["swapped_in"]) == want["swapped_in"]
        assert sw["num_swapped"] == len(sch.swapped)
        free, rc = pk.kv_alloc_snapshot(a, nb)
        assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
        # paging invariants: every held block is referenced as often as tables name it
        held = {}
        for t in bm.tables.values():
            for b in t:
                if b >= 0:
                    held[b] = held.get(b, 0) + 1
        assert all(bm.refcount[b] == held.get(b, 0) for b in range(nb))
        host_held = sorted(-b - 2 for t in bm.tables.values() for b in t if b <= -2)
        assert sorted(host_held + list(bm.host_free)) == list(range(slots))
        preempted += len(want["preempted"]) + len(want["recomputed"])
        running = want["running"]
        for r in running:
            remaining[r] -= 1
    assert preempted > 0
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)
