"""Retrieval-augmented serving trace with prefix caching, against a host
mirror built only from the oracle: every iteration the native scheduler's
outputs (cached token counts included) equal the oracle scheduler's, the GPU
pool equals the mirror pool bit for bit at checkpoints, and sampled prefill
rows (of prompts whose document came from the cache, too) and decode rows
match the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, max_abs
from oracle.sched import BlockManager, PrefixCachingBlockManager, Scheduler
from workloads import BF16, WORKLOADS
from workloads.rag_trace import RagTrace, rag_plan

pytestmark = pytest.mark.gpu


def host16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("caching,native", [(True, False), (False, False), (True, True)])
def test_rag_trace_matches_oracle(caching, native):
    """native: the same trace through the library's serving step, its
    prefill arrays packed by the library."""
    w = WORKLOADS["rag_trace"]
    plan = rag_plan(w)
    tr = RagTrace(w, plan, caching=caching, native=native)
    bs = w.block_size
    bm = (PrefixCachingBlockManager if caching else BlockManager)(tr.num_blocks, bs, tr.order)
    sched = Scheduler(bm, w.extra["max_num_seqs"])
    shape = (tr.num_blocks, w.kv_heads, bs, w.head_dim)
    kh, vh = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    iters = 24
    hits = 0
    for it in range(iters):
        fin, arr, gplan, q, kn, vn, out, pq, pout, P = tr.iteration(it)
        for sid, toks in arr:
            sched.add_request_tokens(sid, toks)
        want = sched.step(fin)
        info = gplan["info"]
        assert list(gplan["running"]) == want["running"]
        assert [list(r[r >= 0]) for r in gplan["block_tables"]] == want["block_tables"]
        assert list(gplan["context_lens"]) == want["context_lens"]
        assert list(gplan["slot_mapping"]) == want["slot_mapping"]
        assert list(gplan["admitted"]) == want["admitted"]
        assert list(gplan["cached"]) == want["cached"]
        hits += sum(want["cached"])
        T = info.num_tokens
        oracle.kv_write(kh, vh, BF16, host16(kn)[:T], host16(vn)[:T], BF16, want["slot_mapping"], bs)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        if it in (0, iters // 2, iters - 1):
            assert np.array_equal(host16(tr.k), kh) and np.array_equal(host16(tr.v), vh), f"pool, iteration {it}"
        B, A = info.batch, info.num_admitted
        if A:  # every admitted prompt's last new row, against the oracle
            lens = np.array(want["context_lens"][-A:], np.int32) - 1
            new = lens - np.array(want["cached"], np.int32)
            cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
            width = max(len(t) for t in want["block_tables"][-A:])
            tables = np.full((A, width), -1, np.int32)
            for i, t in enumerate(want["block_tables"][-A:]):
                tables[i, :len(t)] = t
            ref = oracle.paged_prefill(kh, vh, BF16, host16(pq)[:P], BF16, cu, tables, lens, w.scale, bs)
            rows = cu[1:] - 1
            assert max_abs(pout[rows].cpu().numpy(), ref[rows]) <= TOL[BF16], f"prefill, iteration {it}"
        if B:
            picks = sorted({0, B // 2, B - 1})
            width = max(len(want["block_tables"][i]) for i in picks)
            tables = np.full((len(picks), width), -1, np.int32)
            for j, i in enumerate(picks):
                tables[j, :len(want["block_tables"][i])] = want["block_tables"][i]
            lens = np.array([want["context_lens"][i] for i in picks], np.int32)
            ref = oracle.paged_decode(kh, vh, BF16, host16(q)[picks], BF16, tables, lens, w.scale, bs)
            assert max_abs(out[picks].cpu().numpy(), ref) <= TOL[BF16], f"decode, iteration {it}"
    assert (hits > 0) == caching
