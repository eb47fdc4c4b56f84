"""GPU-side driver of the retrieval-augmented serving trace (harness code: it
sequences calls into the library and draws seeded inputs; it does none of
the method's arithmetic).

Every request's prompt is one of a few shared documents followed by its own
question (token ids drawn from a seeded generator).  Each iteration follows
:class:`serving.DecodeLoop`: finished requests leave, arrivals are admitted
(with prefix caching, a document already in the cache is shared instead of
recomputed), the admitted prompts' uncached tokens are written and prefilled,
and every running sequence writes one token and is decoded.
"""

from __future__ import annotations

import numpy as np

from paged_kv_cache_451_b200 import (kv_alloc_create, kv_alloc_enable_prefix_caching, kv_pool_bind,
                                     kv_pool_create, kv_sched_add_request_tokens, kv_sched_create)
from paged_kv_cache_451_b200.serving import DecodeLoop, NativeDecodeLoop

from . import device_normal_bits, rng_for


def rag_plan(w):
    """Seeded draws: document token ids, and per iteration the arrivals
    (document index, question token ids, output length)."""
    e = w.extra
    r = rng_for(w, 9)
    docs = [r.integers(0, e["vocab"], size=e["doc_len"]).astype(np.int32) for _ in range(e["docs"])]
    arrivals = []
    for _ in range(e["iters"]):
        k = int(r.poisson(e["arrival_rate"]))
        arrivals.append([(int(r.integers(0, e["docs"])),
                          r.integers(0, e["vocab"], size=int(r.integers(e["question_lo"], e["question_hi"] + 1))).astype(np.int32),
                          int(r.integers(e["out_lo"], e["out_hi"] + 1))) for _ in range(k)])
    return {"docs": docs, "arrivals": arrivals}


class RagTrace:
    def __init__(self, w, plan, caching=True, device="cuda", seed=0, shared_prefix=False, native=False):
        import torch

        self.torch, self.w, self.plan, self.seed, self.device = torch, w, plan, seed, device
        e = w.extra
        bs = w.block_size
        self.num_blocks = e["num_blocks"]
        rng = np.random.default_rng([w.seed, 13, seed])
        self.order = rng.permutation(self.num_blocks).astype(np.int32)
        self.alloc = kv_alloc_create(self.num_blocks, bs, self.order)
        if caching:
            kv_alloc_enable_prefix_caching(self.alloc)
        self.sched = kv_sched_create(self.alloc, e["max_num_seqs"])
        shape = (self.num_blocks, w.kv_heads, bs, w.head_dim)
        self.k = torch.zeros(shape, dtype=torch.int16, device=device)
        self.v = torch.zeros(shape, dtype=torch.int16, device=device)
        self.pool = kv_pool_create(bs, self.num_blocks, w.kv_heads, w.head_dim, w.kv_fmt, 1)
        kv_pool_bind(self.pool, 0, self.k, self.v)
        self.remaining = {}
        self.prompts = {}
        self.next_id = 0
        self.running = []
        max_ctx = e["doc_len"] + e["question_hi"] + e["out_hi"] + e["iters"] + 2 * bs
        self.max_blocks = -(-max_ctx // bs)
        max_prompt_tokens = 16 * (e["doc_len"] + e["question_hi"])
        # native: the iteration sequenced inside the library (kv_serve_*)
        if native and shared_prefix:
            raise ValueError("the native serving step has no shared-prefix decode")
        kw = dict(num_q_heads=w.num_q_heads, kv_heads=w.kv_heads, head_dim=w.head_dim, block_size=bs,
                  q_dtype=w.q_fmt, scale=w.scale, max_batch=e["max_num_seqs"], max_blocks=self.max_blocks,
                  max_tokens=max_prompt_tokens + e["max_num_seqs"], max_context=max_ctx, device=device)
        if native:
            self.loop = NativeDecodeLoop(self.pool, self.sched, **kw)
            self.loop.full_plan = True  # the prefill sizes come from the step's arrays
        else:
            self.loop = DecodeLoop(self.pool, self.sched, shared_prefix=shared_prefix, **kw)

    def _seed(self, it, kind):
        return (self.w.seed * 1_000_003 + (it + 2) * 7919 + kind * 104_729 + self.seed) % (2 ** 62)

    def arrivals(self, it):
        out = []
        for doc, question, olen in self.plan["arrivals"][it]:
            sid = self.next_id
            self.next_id += 1
            toks = np.concatenate([self.plan["docs"][doc], question]).astype(np.int32)
            kv_sched_add_request_tokens(self.sched, sid, toks)
            self.remaining[sid] = olen
            self.prompts[sid] = toks
            out.append((sid, toks))
        return out

    def iteration(self, it, before_launch=None, after_launch=None):
        """One iteration; returns (finished, arrivals, plan, q, k_new, v_new,
        out, prefill_q, prefill_out) with device tensors of the step."""
        torch, w = self.torch, self.w
        fin = [s for s in self.running if self.remaining[s] <= 0]
        arr = self.arrivals(it)
        plan = self.loop.schedule(fin)
        info = plan["info"]
        self.running = [int(x) for x in plan["running"]]
        T, B = info.num_tokens, info.batch
        a, new, _ = DecodeLoop.prefill_sizes(plan)
        P = int(new.sum())
        d = self.device
        k_new = device_normal_bits((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, d, self._seed(it, 0))
        v_new = device_normal_bits((max(T, 1), w.kv_heads, w.head_dim), w.kv_fmt, d, self._seed(it, 1))
        q = device_normal_bits((max(B, 1), w.num_q_heads, w.head_dim), w.q_fmt, d, self._seed(it, 2))
        pq = device_normal_bits((max(P, 1), w.num_q_heads, w.head_dim), w.q_fmt, d, self._seed(it, 3))
        out = torch.empty((max(B, 1), w.num_q_heads, w.head_dim), dtype=torch.float32, device=d)
        pout = torch.empty((max(P, 1), w.num_q_heads, w.head_dim), dtype=torch.float32, device=d)
        if before_launch is not None:
            before_launch()
        self.loop.launch(plan, k_new, v_new, q, out, prefill_q=pq, prefill_out=pout)
        if after_launch is not None:
            after_launch()
        for s in self.running:
            self.remaining[s] -= 1
        return fin, arr, plan, q, k_new, v_new, out, pq, pout, P
