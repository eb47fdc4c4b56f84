"""Continuous-batching decode iteration over the C ABI.

Sequencing only: every step runs in the native library.  One iteration, in
the order of the scheduling loop on "vLLM 推理加速原理详解：大模型服务吞吐量为何能
提升 10 倍" (section "连续批处理：别再等最慢的那个请求了"):

1. ``kv_sched_step`` (native, host): free the finished sequences, admit
   waiting requests first come first served, append one slot per running
   sequence (copy-on-write pairs where a shared block is written);
2. upload the step's metadata (block tables, context lengths, slots, copy
   pairs) from pinned host buffers with one async copy each;
3. ``block_copy`` for the copy-on-write pairs;
4. ``paged_kv_write`` of the step's new tokens (admitted prompts, then one
   token per running sequence);
5. ``paged_attention_decode`` over the running set, with the scheduling
   order of :func:`schedule_order` (it only affects how CTAs are placed on
   the GPU, not the outputs).
"""

from __future__ import annotations

import numpy as np

from . import (KV_F32, block_copy, kv_sched_outputs, kv_sched_step, paged_attention_decode,
               paged_attention_workspace_bytes, paged_kv_write)


def schedule_order(context_lens, policy="long_first"):
    """Order in which the decode schedules the batch's sequences.

    ``longest``: all sequences by decreasing length, so long contexts do not
    start last and leave a tail of idle SMs (best measured for one decode
    step over independent contexts).  ``long_first``: sequences longer than
    the batch mean, longest first, then the rest in batch order.  ``batch``:
    batch order, which keeps sequences that read shared blocks (from L2,
    issue bound) evenly mixed with sequences streaming from HBM (best
    measured for the continuous-batching trace with a shared prefix).
    """
    lens = np.asarray(context_lens)
    n = lens.shape[0]
    if policy == "batch" or n == 0:
        return np.arange(n, dtype=np.int32)
    if policy == "longest":
        return np.argsort(-lens, kind="stable").astype(np.int32)
    long = np.nonzero(lens > lens.mean())[0]
    long = long[np.argsort(-lens[long], kind="stable")]
    rest = np.nonzero(lens <= lens.mean())[0]
    return np.concatenate([long, rest]).astype(np.int32)


class DecodeLoop:
    def __init__(self, pool, sched, *, num_q_heads, kv_heads, head_dim, block_size, q_dtype,
                 scale, max_batch, max_blocks, max_tokens, max_context, device="cuda",
                 order_policy="batch"):
        import torch
        self.torch = torch
        self.pool, self.sched = pool, sched
        self.hq, self.hkv, self.d, self.bs = num_q_heads, kv_heads, head_dim, block_size
        self.q_dtype, self.scale = q_dtype, scale
        self.max_batch, self.max_blocks, self.max_tokens = max_batch, max_blocks, max_tokens
        pin = dict(pin_memory=True)
        self.h_tables = torch.empty(max_batch * max_blocks, dtype=torch.int32, **pin)
        self.h_lens = torch.empty(max_batch, dtype=torch.int32, **pin)
        self.h_slots = torch.empty(max_tokens, dtype=torch.int64, **pin)
        self.h_cow = torch.empty(2 * max_batch, dtype=torch.int32, **pin)
        self.h_order = torch.empty(max_batch, dtype=torch.int32, **pin)
        self.d_tables = torch.empty(max_batch * max_blocks, dtype=torch.int32, device=device)
        self.d_lens = torch.empty(max_batch, dtype=torch.int32, device=device)
        self.d_slots = torch.empty(max_tokens, dtype=torch.int64, device=device)
        self.d_cow = torch.empty(2 * max_batch, dtype=torch.int32, device=device)
        self.d_order = torch.empty(max_batch, dtype=torch.int32, device=device)
        ws = paged_attention_workspace_bytes(pool, max_batch, num_q_heads, max_context)
        self.ws_cap = max(ws, 16)
        self.d_ws = torch.empty(self.ws_cap, dtype=torch.uint8, device=device)
        self.copy_done = None
        self.order_policy = order_policy

    def schedule(self, finished_ids):
        """Native scheduler step; returns the step's host outputs."""
        info = kv_sched_step(self.sched, finished_ids)
        if info.batch > self.max_batch or info.num_tokens > self.max_tokens:
            raise RuntimeError("step exceeds the loop's buffers")
        out = kv_sched_outputs(self.sched, info, self.max_blocks)
        out["info"] = info
        return out

    def launch(self, plan, k_new, v_new, q, out, k_inv=None, v_inv=None, out_dtype=None,
               layer=0, stream=None):
        """Upload the plan's metadata and enqueue copy, write and decode."""
        torch = self.torch
        info = plan["info"]
        b, t, c = info.batch, info.num_tokens, info.num_cow
        if self.copy_done is not None:  # pinned buffers are reused: previous uploads must be done
            self.copy_done.synchronize()
        self.h_tables[: b * self.max_blocks].numpy()[:] = plan["block_tables"].reshape(-1)
        self.h_lens[:b].numpy()[:] = plan["context_lens"]
        self.h_order[:b].numpy()[:] = schedule_order(plan["context_lens"], self.order_policy)
        self.h_slots[:t].numpy()[:] = plan["slot_mapping"]
        if c:
            self.h_cow[: 2 * c].numpy()[:] = plan["cow_pairs"].reshape(-1)
        self.d_tables[: b * self.max_blocks].copy_(self.h_tables[: b * self.max_blocks], non_blocking=True)
        self.d_lens[:b].copy_(self.h_lens[:b], non_blocking=True)
        self.d_order[:b].copy_(self.h_order[:b], non_blocking=True)
        self.d_slots[:t].copy_(self.h_slots[:t], non_blocking=True)
        if c:
            self.d_cow[: 2 * c].copy_(self.h_cow[: 2 * c], non_blocking=True)
        self.copy_done = torch.cuda.Event()
        self.copy_done.record()
        max_ctx = int(plan["context_lens"].max()) if b else 0
        if c:
            block_copy(self.pool, self.d_cow, c, stream)
        if t:
            paged_kv_write(self.pool, layer, k_new, v_new, self.q_dtype, self.d_slots, t, k_inv, v_inv,
                           stream)
        if b:
            need = paged_attention_workspace_bytes(self.pool, b, self.hq, max_ctx)
            if need > self.ws_cap:
                raise RuntimeError("decode workspace too small")
            paged_attention_decode(self.pool, layer, q, self.q_dtype, self.hq, self.d_tables,
                                   self.max_blocks, self.d_lens, b, max_ctx, self.scale, out,
                                   KV_F32 if out_dtype is None else out_dtype, self.d_ws, need, stream,
                                   seq_order=self.d_order)
        return max_ctx
