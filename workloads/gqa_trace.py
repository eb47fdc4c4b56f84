"""GPU-side driver of the GQA continuous-batching trace (harness code: it
sequences calls into the library and draws seeded inputs; it does none of
the method's arithmetic).

Initial state: half of the batch are sharers forked from one parent that
holds a 1024-token prefix plus ``tail`` common tokens (the parent is then
freed, so the prefix blocks and the partly filled last block are held by
every sharer); the other half hold their own lognormal-length contexts.  In
the first iteration every sharer appends its first own token into the
shared partly filled block, so all but the last of them copy it on write.
Each iteration then follows :class:`serving.DecodeLoop` (or, with ``native``,
the library's own serving step through :class:`serving.NativeDecodeLoop`):
finished sequences leave, Poisson arrivals are admitted while blocks allow,
every running sequence writes one token and is decoded.

Values (q, K, V of new tokens) are drawn on the device from seeded torch
generators; the caller may copy them back to mirror the run on the host.
"""

from __future__ import annotations

import math

import numpy as np

from paged_kv_cache_451_b200 import (kv_alloc_allocate, kv_alloc_block_table, kv_alloc_create,
                                     kv_alloc_fork, kv_alloc_free, kv_alloc_num_free, kv_pool_bind,
                                     kv_pool_create, kv_sched_adopt, kv_sched_add_request,
                                     kv_sched_create, kv_pool_set_decode_config, paged_kv_write)
from paged_kv_cache_451_b200.serving import DecodeLoop, NativeDecodeLoop

from . import blocks_needed, device_normal_bits

PARENT = 1_000_000
FIRST_ARRIVAL = 10_000


class GqaTrace:
    def __init__(self, w, plan, device="cuda", seed=0, decode_config=None, order_policy="batch",
                 shared_prefix=False, native=False, serve_sets=3):
        import torch

        self.torch, self.w, self.plan, self.seed = torch, w, plan, seed
        self.draw = device_normal_bits
        e = w.extra
        bs = w.block_size
        lens, sharers, tail = plan["lens"], plan["sharers"], plan["tail"]
        self.sharers = set(int(s) for s in sharers)
        prefix = e["prefix"] + tail
        own = [s for s in range(w.batch) if s not in self.sharers]
        need = int(blocks_needed([prefix], bs)[0] + blocks_needed(lens[own], bs).sum())
        self.num_blocks = int(math.ceil(e["pool_factor"] * need))
        rng = np.random.default_rng([w.seed, 11, seed])
        self.order = rng.permutation(self.num_blocks).astype(np.int32)
        self.alloc = kv_alloc_create(self.num_blocks, bs, self.order)
        self.sched = kv_sched_create(self.alloc, e["max_num_seqs"])
        shape = (self.num_blocks, w.kv_heads, bs, w.head_dim)
        self.k = torch.zeros(shape, dtype=torch.int16, device=device)
        self.v = torch.zeros(shape, dtype=torch.int16, device=device)
        self.pool = kv_pool_create(bs, self.num_blocks, w.kv_heads, w.head_dim, w.kv_fmt, 1)
        kv_pool_bind(self.pool, 0, self.k, self.v)
        if decode_config:
            kv_pool_set_decode_config(self.pool, *decode_config)
        self.device = device

        # initial contexts: parent prefix (shared by forks), own contexts
        kv_alloc_allocate(self.alloc, PARENT, prefix)
        for s in own:
            kv_alloc_allocate(self.alloc, s, int(lens[s]))
        slots = [self._slots(PARENT, 0, prefix)] + [self._slots(s, 0, int(lens[s])) for s in own]
        self.init_slots = np.concatenate(slots).astype(np.int64)
        for s in sorted(self.sharers):
            kv_alloc_fork(self.alloc, PARENT, s)
        kv_alloc_free(self.alloc, PARENT)
        for s in range(w.batch):
            kv_sched_adopt(self.sched, s)
        T = len(self.init_slots)
        self.init_k = self.draw((T, w.kv_heads, w.head_dim), w.kv_fmt, device, self._seed(-1, 0))
        self.init_v = self.draw((T, w.kv_heads, w.head_dim), w.kv_fmt, device, self._seed(-1, 1))
        d_slots = torch.from_numpy(self.init_slots).to(device)
        paged_kv_write(self.pool, 0, self.init_k, self.init_v, w.kv_fmt, d_slots, T)

        # output tokens still to generate, indexed by sequence id (arrivals
        # take ids from FIRST_ARRIVAL on), and the running set's ids
        n_arr = sum(len(a) for a in plan["arrivals"])
        self.remaining = np.zeros(FIRST_ARRIVAL + n_arr + 1, np.int64)
        self.remaining[:w.batch] = np.asarray(plan["remaining"][:w.batch], np.int64)
        self.next_id = FIRST_ARRIVAL
        self.running = np.arange(w.batch, dtype=np.int64)
        self.max_blocks = int(math.ceil((e["cap"] + e["iters"] + 2 * bs) / bs))
        max_tokens = 256 + 16 * e["prompt_hi"]
        # native: the iteration sequenced inside the library (kv_serve_*)
        if native and shared_prefix:
            raise ValueError("the native serving step has no shared-prefix decode")
        kw = dict(num_q_heads=w.num_q_heads, kv_heads=w.kv_heads, head_dim=w.head_dim, block_size=bs,
                  q_dtype=w.q_fmt, scale=w.scale, max_batch=e["max_num_seqs"], max_blocks=self.max_blocks,
                  max_tokens=max_tokens, max_context=e["cap"] + e["iters"] + bs, device=device,
                  order_policy=order_policy)
        self.loop = (NativeDecodeLoop(self.pool, self.sched, num_sets=serve_sets, **kw) if native else
                     DecodeLoop(self.pool, self.sched, shared_prefix=shared_prefix, **kw))

    def _seed(self, it, kind):
        return (self.w.seed * 1_000_003 + (it + 2) * 7919 + kind * 104_729 + self.seed) % (2 ** 62)

    def _slots(self, sid, t0, t1):
        bs = self.w.block_size
        table = kv_alloc_block_table(self.alloc, sid)
        t = np.arange(t0, t1)
        return table[t // bs].astype(np.int64) * bs + t % bs

    def finished(self):
        return self.running[self.remaining[self.running] <= 0].tolist()

    def arrivals(self, it):
        """Queue this iteration's arrivals; returns [(id, prompt_len)]."""
        out = []
        for plen, olen in self.plan["arrivals"][it]:
            sid = self.next_id
            self.next_id += 1
            kv_sched_add_request(self.sched, sid, plen)
            self.remaining[sid] = olen
            out.append((sid, plen))
        return out

    def iteration(self, it, out_dtype=None, out=None, before_launch=None, after_launch=None,
                  before_decode=None, inputs=None, stream=None):
        """One trace iteration: returns (finished, arrivals, plan, q, k_new,
        v_new, out) with device tensors of this step's inputs and output.
        before_launch / after_launch are called right around the library
        calls (after the inputs are drawn), e.g. to record timing events.
        ``inputs(T, B)``, if given, supplies (q, k_new, v_new) instead of the
        seeded draws (e.g. views of buffers it uploads from host memory); it
        is called after before_launch.  ``stream``: the stream the kernels run
        on (default: the current one)."""
        torch, w = self.torch, self.w
        import time
        fin = self.finished()
        arr = self.arrivals(it)
        t0 = time.perf_counter()
        plan = self.loop.schedule(fin)
        self.last_schedule_s = time.perf_counter() - t0
        info = plan["info"]
        self.running = np.array(plan["running"], np.int64)
        T, B = info.num_tokens, info.batch
        if inputs is None:
            k_new = self.draw((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, self.device, self._seed(it, 0))
            v_new = self.draw((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, self.device, self._seed(it, 1))
            q = self.draw((max(B, 1), w.num_q_heads, w.head_dim), w.q_fmt, self.device, self._seed(it, 2))
        if out is None:
            dt = torch.float32 if out_dtype is None else {0: torch.float16, 1: torch.bfloat16}[out_dtype]
            out = torch.empty((max(B, 1), w.num_q_heads, w.head_dim), dtype=dt, device=self.device)
        if before_launch is not None:
            before_launch()
        if inputs is not None:
            q, k_new, v_new = inputs(max(T, 1), max(B, 1))
        self.loop.launch(plan, k_new, v_new, q, out, out_dtype=out_dtype, before_decode=before_decode,
                         stream=stream)
        if after_launch is not None:
            after_launch()
        self.remaining[self.running] -= 1
        return fin, arr, plan, q, k_new, v_new, out

    def free_blocks(self):
        return kv_alloc_num_free(self.alloc)
