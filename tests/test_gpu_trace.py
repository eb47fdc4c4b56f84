"""The GQA continuous-batching trace at full size (batch 256, 64/8 heads,
lognormal contexts up to 8192, half the batch sharing a 1024-token prefix,
100 iterations of Poisson arrivals) against a host mirror built only from
the oracle: every iteration the native scheduler's outputs must equal the
oracle scheduler's, the GPU pool must equal the mirror pool bit for bit at
checkpoints (copy-on-write included), and sampled decode outputs must match
the fp64 oracle."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, max_abs
from oracle.sched import BlockManager, Scheduler
from workloads import BF16, WORKLOADS, gqa_trace_plan
from workloads.gqa_trace import PARENT, GqaTrace

pytestmark = pytest.mark.gpu


def host16(t):
    return t.cpu().numpy().view(np.uint16)


def mirror_initial(tr, w, plan):
    """The same initial operations on the oracle allocator, and the initial
    cache content written by the oracle's cache-write mirror."""
    bs = w.block_size
    bm = BlockManager(tr.num_blocks, bs, tr.order)
    sched = Scheduler(bm, w.extra["max_num_seqs"])
    prefix = w.extra["prefix"] + plan["tail"]
    own = [s for s in range(w.batch) if s not in tr.sharers]
    bm.allocate(PARENT, prefix)
    for s in own:
        bm.allocate(s, int(plan["lens"][s]))

    def slots(sid, n):
        t = np.arange(n)
        return np.asarray(bm.tables[sid], np.int64)[t // bs] * bs + t % bs

    init_slots = np.concatenate([slots(PARENT, prefix)] + [slots(s, int(plan["lens"][s])) for s in own])
    for s in sorted(tr.sharers):
        bm.fork(PARENT, s)
    bm.free(PARENT)
    for s in range(w.batch):
        sched.adopt(s)
    shape = (tr.num_blocks, w.kv_heads, bs, w.head_dim)
    kh, vh = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    oracle.kv_write(kh, vh, BF16, host16(tr.init_k), host16(tr.init_v), BF16, init_slots, bs)
    return bm, sched, kh, vh, init_slots


class HostStaging:
    """Inputs drawn into pinned host memory and uploaded by the serving
    loop (kv_serve_upload) into the step's buffer set; outputs read back by
    it (kv_serve_readback) into pinned host memory."""

    def __init__(self, tr, w):
        e = w.extra
        self.loop, self.w = tr.loop, w
        hq, hkv, d = w.num_q_heads, w.kv_heads, w.head_dim
        n = (e["max_num_seqs"] * hq + 2 * tr.loop.max_tokens * hkv) * d
        self.host = torch.empty(n, dtype=torch.int16).pin_memory()
        sets = tr.loop.num_sets  # one input / output set per buffer set of the loop
        self.dev = [torch.empty(n, dtype=torch.int16, device="cuda") for _ in range(sets)]
        self.outs = [torch.empty((e["max_num_seqs"], hq, d), dtype=torch.float32, device="cuda") for _ in range(sets)]
        self.hout = [torch.empty((e["max_num_seqs"], hq, d), dtype=torch.float32).pin_memory() for _ in range(sets)]
        self.rb = torch.cuda.Stream()
        self.rng = np.random.default_rng(99)

    def inputs(self, T, B):
        w, k = self.w, self.loop.layout.buffer
        nq, nk = B * w.num_q_heads * w.head_dim, T * w.kv_heads * w.head_dim
        torch.cuda.current_stream().synchronize()  # the host buffer is rewritten: earlier uploads must be done
        self.loop.up.synchronize()
        bits = self.rng.standard_normal(nq + 2 * nk).astype(np.float32)
        self.host[:nq + 2 * nk].copy_(torch.from_numpy(bits).to(torch.bfloat16).view(torch.int16))
        self.loop.upload(self.dev[k], self.host, 2 * (nq + 2 * nk))
        buf = self.dev[k]
        return (buf[:nq].view(B, w.num_q_heads, w.head_dim), buf[nq:nq + nk].view(T, w.kv_heads, w.head_dim),
                buf[nq + nk:nq + 2 * nk].view(T, w.kv_heads, w.head_dim))


def run_trace(w, iters, check_pool_at, sample_every=1, shared_prefix=False, native=False, order_policy="batch",
              staging=False, serve_sets=3):
    plan = gqa_trace_plan(w)
    tr = GqaTrace(w, plan, shared_prefix=shared_prefix, native=native, order_policy=order_policy,
                  serve_sets=serve_sets)
    if native:
        tr.loop.full_plan = True  # the step's arrays, to compare with the oracle scheduler
    st = HostStaging(tr, w) if staging else None
    used_prefix = 0
    bm, sched, kh, vh, init_slots = mirror_initial(tr, w, plan)
    assert np.array_equal(init_slots, tr.init_slots)
    bs = w.block_size
    cow_total = 0
    for it in range(iters):
        if st is None:
            fin, arr, gplan, q, kn, vn, out = tr.iteration(it)
        else:
            k = it % tr.loop.num_sets
            fin, arr, gplan, q, kn, vn, out = tr.iteration(it, inputs=st.inputs, out=st.outs[k])
            assert gplan["layout"].buffer == k
            nout = gplan["info"].batch * w.num_q_heads * w.head_dim
            tr.loop.readback(st.hout[k], out, 4 * nout, st.rb)
            st.rb.synchronize()
            # the read-back waited for this step's decode
            assert torch.equal(st.hout[k].view(-1)[:nout], out.view(-1)[:nout].cpu())
        for sid, plen in arr:
            sched.add_request(sid, plen)
        want = sched.step(fin)
        info = gplan["info"]
        # allocator and scheduler: exact
        assert list(gplan["running"]) == want["running"]
        assert [list(r[r >= 0]) for r in gplan["block_tables"]] == want["block_tables"]
        assert list(gplan["context_lens"]) == want["context_lens"]
        assert list(gplan["slot_mapping"]) == want["slot_mapping"]
        assert gplan["cow_pairs"].tolist() == [list(p) for p in want["cow_pairs"]]
        assert list(gplan["admitted"]) == want["admitted"]
        free, rc = pk.kv_alloc_snapshot(tr.alloc, tr.num_blocks)
        assert list(free) == list(bm.free_list) and list(rc) == bm.refcount
        cow_total += len(want["cow_pairs"])
        # host mirror of copy-on-write and the cache write
        oracle.block_copy([kh, vh], want["cow_pairs"])
        T = info.num_tokens
        oracle.kv_write(kh, vh, BF16, host16(kn)[:T], host16(vn)[:T], BF16, want["slot_mapping"], bs)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        if it in check_pool_at:
            assert np.array_equal(host16(tr.k), kh), f"K pool differs after iteration {it}"
            assert np.array_equal(host16(tr.v), vh), f"V pool differs after iteration {it}"
        if it % sample_every == 0 and info.batch:
            B = info.batch
            picks = {0, B // 2, B - 1} | ({want["running"].index(want["admitted"][0])} if want["admitted"] else set())
            rows, _ = tr.loop.last_prefix
            if rows is not None:  # the shared-prefix decode ran: check sharers too
                used_prefix += 1
                picks |= {int(rows[0]), int(rows[len(rows) // 2]), int(rows[-1])}
            picks = sorted(picks)
            tables = np.full((len(picks), max(len(want["block_tables"][i]) for i in picks)), -1, np.int32)
            for j, i in enumerate(picks):
                tables[j, :len(want["block_tables"][i])] = want["block_tables"][i]
            lens = np.array([want["context_lens"][i] for i in picks], np.int32)
            ref = oracle.paged_decode(kh, vh, BF16, host16(q)[picks], BF16, tables, lens, w.scale, bs)
            assert max_abs(out[picks].cpu().numpy(), ref) <= TOL[BF16], f"iteration {it}"
    if shared_prefix:
        assert used_prefix > 0
    return tr, cow_total


def test_gqa_trace_full_size_matches_oracle():
    w = WORKLOADS["gqa_trace"]
    tr, cow_total = run_trace(w, w.extra["iters"], check_pool_at={0, 1, 50, w.extra["iters"] - 1})
    # every sharer but the last copied the shared partly filled block
    assert cow_total >= len(tr.sharers) - 1


@pytest.mark.parametrize("order_policy,iters", [("batch", 30), ("long_first", 12)])
def test_gqa_trace_through_the_native_serving_step(order_policy, iters):
    """The trace sequenced by the library (kv_serve_schedule packs the step
    into a pinned buffer and uploads it; kv_serve_launch enqueues copy,
    write and decode in the packed scheduling order): pool and sampled
    outputs still equal the oracle mirror's."""
    w = WORKLOADS["gqa_trace"]
    tr, cow_total = run_trace(w, iters, check_pool_at={0, iters - 1}, native=True, order_policy=order_policy)
    assert cow_total >= len(tr.sharers) - 1
    tr.loop.close()


@pytest.mark.parametrize("serve_sets", [2, 3])
def test_gqa_trace_with_host_staging_through_the_serving_loop(serve_sets):
    """Inputs uploaded from pinned host memory by kv_serve_upload into the
    loop's buffer sets in turn, outputs read back by kv_serve_readback: the
    pool, the sampled outputs and the read-back bytes all check."""
    w = WORKLOADS["gqa_trace"]
    tr, _ = run_trace(w, 10, check_pool_at={0, 9}, native=True, staging=True, serve_sets=serve_sets)
    tr.loop.close()


def test_gqa_trace_with_shared_prefix_decode_matches_oracle():
    """The same trace with the serving loop's shared-prefix decode: the
    sharers' common blocks are attended once per kv head on the tensor cores
    and merged with each sequence's own tokens; outputs (sharers sampled
    every iteration) still match the oracle."""
    w = WORKLOADS["gqa_trace"]
    run_trace(w, 40, check_pool_at={39}, shared_prefix=True)


def test_trace_with_block_aligned_prefix_needs_no_copy():
    """With no common tail the prefix ends on a block boundary: the first
    divergent token opens a fresh block and no copy-on-write happens."""
    base = WORKLOADS["gqa_trace"]
    w = dataclasses.replace(base, batch=32, extra=dict(base.extra, iters=3))
    plan = gqa_trace_plan(w)
    plan["tail"] = 0
    tr = GqaTrace(w, plan)
    _, _, gplan, *_ = tr.iteration(0)
    assert gplan["info"].num_cow == 0
    assert len(tr.sharers) == 16
