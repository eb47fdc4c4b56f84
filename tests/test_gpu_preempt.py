"""Memory-pressure trace with preemption (swap and recompute) against a host
mirror built only from the oracle: the native scheduler's outputs and swap
pairs equal the oracle's every iteration; the GPU pool and the pinned host
swap space equal the mirror's bit for bit at checkpoints (after swap-outs and
swap-ins); sampled decode outputs match the fp64 oracle."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, max_abs
from oracle.sched import BlockManager, Scheduler
from workloads import BF16, WORKLOADS
from workloads.preempt_trace import PreemptTrace, preempt_plan

pytestmark = pytest.mark.gpu


def host16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("mode,native", [("swap", False), ("recompute", False), ("swap", True)])
def test_preempt_trace_matches_oracle(mode, native):
    """native: the same trace through the library's serving step
    (kv_serve_schedule / kv_serve_launch)."""
    w0 = WORKLOADS["preempt_trace"]
    w = dataclasses.replace(w0, extra=dict(w0.extra, out_lo=30, out_hi=80, num_blocks=2400, iters=45,
                                           arrival_rate=2.0))
    plan = preempt_plan(w)
    tr = PreemptTrace(w, plan, mode=mode, native=native)
    bs, nb = w.block_size, tr.num_blocks
    bm = BlockManager(nb, bs, tr.order)
    bm.set_swap_space(tr.swap_slots)
    sch = Scheduler(bm, w.extra["max_num_seqs"])
    sch.preemption = mode
    for sid, (plen, _) in enumerate(plan["initial"]):
        sch.add_request(sid, plen)
    shape = (nb, w.kv_heads, bs, w.head_dim)
    kh, vh = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    hs = np.zeros((max(tr.swap_slots, 1), 2) + shape[1:], np.uint16)
    seen = {"preempted": 0, "recomputed": 0, "swapped_in": 0}
    for it in range(w.extra["iters"]):
        fin, arr, gplan, q, kn, vn, out = tr.iteration(it)
        for sid, plen in arr:
            sch.add_request(sid, plen)
        want = sch.step(fin)
        info = gplan["info"]
        assert list(gplan["running"]) == want["running"]
        for row, t in zip(gplan["block_tables"], want["block_tables"]):
            assert list(row[:len(t)]) == t
        assert list(gplan["context_lens"]) == want["context_lens"]
        assert list(gplan["slot_mapping"]) == want["slot_mapping"]
        assert gplan["swap_out"].tolist() == [list(p) for p in want["swap_out"]]
        assert gplan["swap_in"].tolist() == [list(p) for p in want["swap_in"]]
        assert list(gplan["preempted"]) == want["preempted"]
        assert list(gplan["recomputed"]) == want["recomputed"]
        for k in seen:
            seen[k] += len(want[k])
        # host mirror, in the loop's order: swap out, swap in, copy-on-write, write
        for b, slot in want["swap_out"]:
            hs[slot, 0], hs[slot, 1] = kh[b], vh[b]
        for slot, b in want["swap_in"]:
            kh[b], vh[b] = hs[slot, 0], hs[slot, 1]
        oracle.block_copy([kh, vh], want["cow_pairs"])
        T = info.num_tokens
        oracle.kv_write(kh, vh, BF16, host16(kn)[:T], host16(vn)[:T], BF16, want["slot_mapping"], bs)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        if want["swap_out"] or want["swap_in"] or it in (0, w.extra["iters"] - 1):
            assert np.array_equal(host16(tr.k), kh) and np.array_equal(host16(tr.v), vh), f"pool, iteration {it}"
            if tr.swap_slots:
                got = tr.host.numpy().view(np.uint16).reshape(hs.shape)
                used = sorted({slot for _, slot in want["swap_out"]})
                assert np.array_equal(got[used], hs[used]), f"swap space, iteration {it}"
        B = info.batch
        if B:
            picks = sorted({0, B // 2, B - 1})
            width = max(len(want["block_tables"][i]) for i in picks)
            tables = np.full((len(picks), width), -1, np.int32)
            for j, i in enumerate(picks):
                tables[j, :len(want["block_tables"][i])] = want["block_tables"][i]
            lens = np.array([want["context_lens"][i] for i in picks], np.int32)
            ref = oracle.paged_decode(kh, vh, BF16, host16(q)[picks], BF16, tables, lens, w.scale, bs)
            assert max_abs(out[picks].cpu().numpy(), ref) <= TOL[BF16], f"decode, iteration {it}"
    if mode == "swap":
        assert seen["preempted"] > 0 and seen["swapped_in"] > 0
    else:
        assert seen["recomputed"] > 0


def test_swap_round_trip_fp8_with_scales():
    """kv_swap_out then kv_swap_in into other blocks moves data and FP8
    scales bit for bit, over every layer."""
    rng = np.random.default_rng(71)
    nb, hkv, bs, d, L = 24, 4, 16, 128, 3
    pool = pk.kv_pool_create(bs, nb, hkv, d, pk.KV_FP8_E4M3, L)
    ks_, vs_, kk, vv = [], [], [], []
    for layer in range(L):
        k = torch.from_numpy(rng.integers(0, 255, size=(nb, hkv, bs, d), dtype=np.uint8)).cuda()
        v = torch.from_numpy(rng.integers(0, 255, size=(nb, hkv, bs, d), dtype=np.uint8)).cuda()
        ks = torch.from_numpy(rng.random((nb, hkv), dtype=np.float32)).cuda()
        vs = torch.from_numpy(rng.random((nb, hkv), dtype=np.float32)).cuda()
        pk.kv_pool_bind(pool, layer, k, v, ks, vs)
        kk.append(k), vv.append(v), ks_.append(ks), vs_.append(vs)
    slots = 8
    host = torch.zeros(slots * pk.kv_swap_block_bytes(pool), dtype=torch.uint8).pin_memory()
    before = [(k.clone(), v.clone(), a.clone(), b.clone()) for k, v, a, b in zip(kk, vv, ks_, vs_)]
    out_pairs = torch.tensor([[3, 5], [10, 0], [17, 7]], dtype=torch.int32, device="cuda")
    pk.kv_swap_out(pool, host, slots, out_pairs, 3)
    in_pairs = torch.tensor([[5, 20], [0, 21], [7, 22]], dtype=torch.int32, device="cuda")
    pk.kv_swap_in(pool, host, slots, in_pairs, 3)
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    for layer in range(L):
        k0, v0, a0, b0 = before[layer]
        for src, dst in ((3, 20), (10, 21), (17, 22)):
            assert torch.equal(kk[layer][dst], k0[src]) and torch.equal(vv[layer][dst], v0[src])
            assert torch.equal(ks_[layer][dst], a0[src]) and torch.equal(vs_[layer][dst], b0[src])
    bad = torch.tensor([[3, slots]], dtype=torch.int32, device="cuda")
    pk.kv_swap_out(pool, host, slots, bad, 1)
    assert pk.kv_get_device_error() == pk.KV_ERR_BOUNDS
    with pytest.raises(pk.KVError):  # device memory is not a host swap space
        pk.kv_swap_out(pool, kk[0], slots, out_pairs, 3)
    pk.kv_pool_destroy(pool)
