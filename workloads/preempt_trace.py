"""GPU-side driver of the memory-pressure trace (harness code: it sequences
calls into the library and draws seeded inputs; it does none of the method's
arithmetic).

Sequences grow one token per iteration until they outgrow the pool; the
scheduling step then preempts the latest ones (swap: their exclusive blocks
go to a pinned host swap space; recompute: they are requeued with their
whole context as the prompt), and brings swapped ones back when blocks free
up.  Each iteration follows :class:`serving.DecodeLoop`: swap copies,
copy-on-write, cache write of the step's new tokens (re-admitted contexts
included), decode of every running sequence.
"""

from __future__ import annotations

import numpy as np

from paged_kv_cache_451_b200 import (KV_PREEMPT_RECOMPUTE, KV_PREEMPT_SWAP, kv_alloc_create,
                                     kv_alloc_set_swap_space, kv_pool_bind, kv_pool_create,
                                     kv_sched_add_request, kv_sched_create, kv_sched_set_preemption,
                                     kv_swap_block_bytes)
from paged_kv_cache_451_b200.serving import DecodeLoop, NativeDecodeLoop

from . import device_normal_bits, rng_for


def preempt_plan(w):
    e = w.extra
    r = rng_for(w, 5)
    initial = [(int(r.integers(e["prompt_lo"], e["prompt_hi"] + 1)), int(r.integers(e["out_lo"], e["out_hi"] + 1)))
               for _ in range(w.batch)]
    arrivals = [[(int(r.integers(e["prompt_lo"], e["prompt_hi"] + 1)), int(r.integers(e["out_lo"], e["out_hi"] + 1)))
                 for _ in range(int(r.poisson(e["arrival_rate"])))] for _ in range(e["iters"])]
    return {"initial": initial, "arrivals": arrivals}


class PreemptTrace:
    def __init__(self, w, plan, mode="swap", device="cuda", seed=0, native=False):
        import torch

        self.torch, self.w, self.plan, self.seed, self.device = torch, w, plan, seed, device
        e = w.extra
        bs = w.block_size
        self.num_blocks = e["num_blocks"]
        self.swap_slots = e["swap_slots"] if mode == "swap" else 0
        rng = np.random.default_rng([w.seed, 17, seed])
        self.order = rng.permutation(self.num_blocks).astype(np.int32)
        self.alloc = kv_alloc_create(self.num_blocks, bs, self.order)
        kv_alloc_set_swap_space(self.alloc, self.swap_slots)
        self.sched = kv_sched_create(self.alloc, e["max_num_seqs"])
        kv_sched_set_preemption(self.sched, KV_PREEMPT_SWAP if mode == "swap" else KV_PREEMPT_RECOMPUTE)
        shape = (self.num_blocks, w.kv_heads, bs, w.head_dim)
        self.k = torch.zeros(shape, dtype=torch.int16, device=device)
        self.v = torch.zeros(shape, dtype=torch.int16, device=device)
        self.pool = kv_pool_create(bs, self.num_blocks, w.kv_heads, w.head_dim, w.kv_fmt, 1)
        kv_pool_bind(self.pool, 0, self.k, self.v)
        self.slot_bytes = kv_swap_block_bytes(self.pool)
        self.host = (torch.zeros(max(self.swap_slots, 1) * self.slot_bytes, dtype=torch.uint8).pin_memory()
                     if self.swap_slots else None)
        self.remaining = {}
        self.next_id = 0
        self.running = []
        for plen, olen in plan["initial"]:
            self._add(plen, olen)
        max_ctx = e["prompt_hi"] + e["out_hi"] + 2 * bs
        self.max_blocks = -(-max_ctx // bs)
        # native: the iteration sequenced inside the library (kv_serve_*)
        self.loop = (NativeDecodeLoop if native else DecodeLoop)(
            self.pool, self.sched, num_q_heads=w.num_q_heads, kv_heads=w.kv_heads, head_dim=w.head_dim,
            block_size=bs, q_dtype=w.q_fmt, scale=w.scale, max_batch=e["max_num_seqs"], max_blocks=self.max_blocks,
            max_tokens=e["max_num_seqs"] * (max_ctx + 1), max_context=max_ctx, device=device, host_swap=self.host,
            swap_slots=self.swap_slots)
        if native:
            self.loop.full_plan = True  # callers mirror the swap pairs

    def _add(self, plen, olen):
        sid = self.next_id
        self.next_id += 1
        kv_sched_add_request(self.sched, sid, plen)
        self.remaining[sid] = olen
        return sid

    def _seed(self, it, kind):
        return (self.w.seed * 1_000_003 + (it + 2) * 7919 + kind * 104_729 + self.seed) % (2 ** 62)

    def iteration(self, it, before_launch=None, after_launch=None):
        """One iteration; returns (finished, arrivals, plan, q, k_new, v_new, out)."""
        torch, w = self.torch, self.w
        fin = [s for s in self.running if self.remaining[s] <= 0]
        arr = [(self._add(plen, olen), plen) for plen, olen in self.plan["arrivals"][it]]
        plan = self.loop.schedule(fin)
        info = plan["info"]
        self.running = [int(x) for x in plan["running"]]
        T, B = info.num_tokens, info.batch
        d = self.device
        k_new = device_normal_bits((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, d, self._seed(it, 0))
        v_new = device_normal_bits((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, d, self._seed(it, 1))
        q = device_normal_bits((max(B, 1), w.num_q_heads, w.head_dim), w.q_fmt, d, self._seed(it, 2))
        out = torch.empty((max(B, 1), w.num_q_heads, w.head_dim), dtype=torch.float32, device=d)
        if before_launch is not None:
            before_launch()
        self.loop.launch(plan, k_new, v_new, q, out)
        if after_launch is not None:
            after_launch()
        for s in self.running:
            self.remaining[s] -= 1
        return fin, arr, plan, q, k_new, v_new, out
