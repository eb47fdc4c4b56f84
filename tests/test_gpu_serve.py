"""The library's serving step on a multi-layer pool, against a host mirror
built only from the oracle: per step one kv_serve_schedule, then one
kv_serve_launch per layer (the first also runs the step's copy-on-write for
every layer), with forked sequences writing into their shared partly filled
block, arrivals and finishes.  The scheduler's outputs must equal the oracle
scheduler's, every layer's pool must equal the mirror bit for bit, and every
layer's decode must match the fp64 oracle on sampled sequences."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, DevicePool, dev, max_abs
from oracle.sched import BlockManager, Scheduler
from paged_kv_cache_451_b200.serving import NativeDecodeLoop
from workloads import BF16, normal_bits

pytestmark = pytest.mark.gpu


def host16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("order_policy,num_sets", [("batch", 3), ("longest", 2), ("batch", 4)])
def test_serving_step_on_a_multi_layer_pool(order_policy, num_sets):
    rng = np.random.default_rng(5 if order_policy == "batch" else 6)
    nb, bs, hkv, hq, d, L, max_seqs = 160, 16, 2, 8, 128, 3, 12
    scale = 1.0 / np.sqrt(d)
    order = rng.permutation(nb).astype(np.int32)
    pool = DevicePool(nb, hkv, d, bs, BF16, num_layers=L)
    shape = (nb, hkv, bs, d)
    kh = [np.zeros(shape, np.uint16) for _ in range(L)]
    vh = [np.zeros(shape, np.uint16) for _ in range(L)]

    a = pk.kv_alloc_create(nb, bs, order)
    s = pk.kv_sched_create(a, max_seqs)
    bm = BlockManager(nb, bs, order)
    sch = Scheduler(bm, max_seqs)
    # a parent with a 40-token prompt, forked twice: the 2.5 shared blocks
    # are written once; the forks' first appends copy the partly filled one
    pk.kv_alloc_allocate(a, 100, 40)
    bm.allocate(100, 40)
    t = np.arange(40)
    slots = np.asarray(bm.tables[100], np.int64)[t // bs] * bs + t % bs
    for layer in range(L):
        kn, vn = normal_bits(rng, (40, hkv, d), BF16), normal_bits(rng, (40, hkv, d), BF16)
        pk.paged_kv_write(pool.h, layer, dev(kn), dev(vn), BF16, dev(slots), 40)
        oracle.kv_write(kh[layer], vh[layer], BF16, kn, vn, BF16, slots, bs)
    for child in (101, 102):
        pk.kv_alloc_fork(a, 100, child)
        bm.fork(100, child)
    for sid in (100, 101, 102):
        pk.kv_sched_adopt(s, sid)
        sch.adopt(sid)

    loop = NativeDecodeLoop(pool.h, s, num_q_heads=hq, kv_heads=hkv, head_dim=d, block_size=bs, q_dtype=BF16,
                            scale=scale, max_batch=max_seqs, max_blocks=32, max_tokens=max_seqs * 200,
                            max_context=500, order_policy=order_policy, num_sets=num_sets)
    loop.full_plan = True
    remaining = {100: 30, 101: 12, 102: 45}
    nxt, cow_total, admitted = 200, 0, 0
    for it in range(24):
        for _ in range(int(rng.poisson(0.6))):
            plen = int(rng.integers(1, 120))
            pk.kv_sched_add_request(s, nxt, plen)
            sch.add_request(nxt, plen)
            remaining[nxt] = int(rng.integers(4, 30))
            nxt += 1
        fin = [r for r in sch.running if remaining[r] <= 0]
        want = sch.step(fin)
        plan = loop.schedule(fin)
        info = plan["info"]
        assert list(plan["running"]) == want["running"]
        assert [list(r[r >= 0]) for r in plan["block_tables"]] == want["block_tables"]
        assert list(plan["slot_mapping"]) == want["slot_mapping"]
        assert plan["cow_pairs"].tolist() == [list(p) for p in want["cow_pairs"]]
        cow_total += info.num_cow
        admitted += info.num_admitted
        oracle.block_copy(kh + vh, want["cow_pairs"])
        T, B = info.num_tokens, info.batch
        qs, outs = [], []
        for layer in range(L):
            kn, vn = normal_bits(rng, (max(T, 1), hkv, d), BF16), normal_bits(rng, (max(T, 1), hkv, d), BF16)
            q = normal_bits(rng, (max(B, 1), hq, d), BF16)
            out = torch.full((max(B, 1), hq, d), float("nan"), device="cuda")
            loop.launch(plan, dev(kn), dev(vn), dev(q), out, layer=layer)
            oracle.kv_write(kh[layer], vh[layer], BF16, kn[:T], vn[:T], BF16, want["slot_mapping"], bs)
            qs.append(q)
            outs.append(out)
        torch.cuda.synchronize()
        assert pk.kv_get_device_error() == pk.KV_OK
        for layer in range(L):
            assert np.array_equal(host16(pool.k[layer]), kh[layer]), f"K layer {layer}, step {it}"
            assert np.array_equal(host16(pool.v[layer]), vh[layer]), f"V layer {layer}, step {it}"
        if B:
            picks = sorted({0, B // 2, B - 1})
            width = max(len(want["block_tables"][i]) for i in picks)
            tables = np.full((len(picks), width), -1, np.int32)
            for j, i in enumerate(picks):
                tables[j, :len(want["block_tables"][i])] = want["block_tables"][i]
            lens = np.array([want["context_lens"][i] for i in picks], np.int32)
            for layer in range(L):
                ref = oracle.paged_decode(kh[layer], vh[layer], BF16, qs[layer][picks], BF16, tables, lens,
                                          scale, bs)
                assert max_abs(outs[layer][picks].cpu().numpy(), ref) <= TOL[BF16], f"layer {layer}, step {it}"
        for r in want["running"]:
            remaining[r] -= 1
    assert cow_total >= 2 and admitted > 0
    loop.close()
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)


def test_serving_step_call_order_is_enforced():
    pool = DevicePool(32, 1, 128, 16, BF16)
    a = pk.kv_alloc_create(32, 16)
    s = pk.kv_sched_create(a, 4)
    loop = NativeDecodeLoop(pool.h, s, num_q_heads=4, kv_heads=1, head_dim=128, block_size=16, q_dtype=BF16,
                            scale=0.1, max_batch=4, max_blocks=8, max_tokens=256, max_context=128)
    buf = torch.zeros(64, dtype=torch.int16, device="cuda")
    with pytest.raises(pk.KVError) as e:  # nothing scheduled yet
        loop.launch(None, buf, buf, buf, buf)
    assert e.value.code == pk.KV_ERR_STATE
    pk.kv_sched_add_request(s, 1, 20)
    loop.schedule([])
    with pytest.raises(pk.KVError) as e:  # read-back before the launch
        loop.readback(torch.zeros(4, dtype=torch.int16).pin_memory(), buf, 8, torch.cuda.current_stream())
    assert e.value.code == pk.KV_ERR_STATE
    with pytest.raises(pk.KVError) as e:  # a second schedule before the first step is launched
        loop.schedule([])
    assert e.value.code == pk.KV_ERR_STATE
    out = torch.empty((1, 4, 128), device="cuda")
    kv = torch.zeros((21, 1, 128), dtype=torch.int16, device="cuda")
    q = torch.zeros((1, 4, 128), dtype=torch.int16, device="cuda")
    loop.launch(None, kv, kv, q, out)
    with pytest.raises(pk.KVError) as e:  # uploads go before the step's launch
        loop.upload(buf, torch.zeros(4, dtype=torch.int16).pin_memory(), 8)
    assert e.value.code == pk.KV_ERR_STATE
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    loop.close()
    pk.kv_sched_destroy(s)
    pk.kv_alloc_destroy(a)
