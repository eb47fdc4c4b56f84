"""Continuous-batching decode iteration over the C ABI.

Sequencing only: every step runs in the native library.  One iteration, in
the order of the scheduling loop on "vLLM 推理加速原理详解：大模型服务吞吐量为何能
提升 10 倍" (section "连续批处理：别再等最慢的那个请求了"):

1. ``kv_sched_step`` (native, host): free the finished sequences, admit
   waiting requests first come first served, append one slot per running
   sequence (copy-on-write pairs where a shared block is written);
2. upload the step's metadata (block tables, context lengths, slots,
   scheduling order, copy and swap pairs) with one async copy from a pinned
   buffer;
3. ``kv_swap_out`` / ``kv_swap_in`` for preempted and resumed sequences,
   then ``block_copy`` for the copy-on-write pairs;
4. ``paged_kv_write`` of the step's new tokens (admitted prompts' uncached
   tokens, then one token per running sequence);
5. optionally ``paged_attention_prefill`` over the admitted prompts' uncached
   tokens (the prompt tokens a prefix-cache hit supplies are only read);
6. ``paged_attention_decode`` over the running set, with the scheduling
   order of :func:`schedule_order` (it only affects how CTAs are placed on
   the GPU, not the outputs).
"""

from __future__ import annotations

import numpy as np

from . import (KV_F32, KV_ORDER_BATCH, KV_ORDER_LONG_FIRST, KV_ORDER_LONGEST, block_copy, kv_sched_outputs,
               kv_sched_step, kv_sched_swap_outputs, kv_serve_create, kv_serve_destroy, kv_serve_launch,
               kv_serve_readback, kv_serve_schedule, kv_serve_upload, kv_serve_workspace_bytes, kv_step_layout,
               kv_step_packed_bytes, kv_swap_in, kv_swap_out, paged_attention_decode,
               paged_attention_decode_shared_prefix, paged_attention_prefill,
               paged_attention_shared_prefix_workspace_bytes, paged_attention_workspace_bytes, paged_kv_write)

ORDER_POLICIES = {"batch": KV_ORDER_BATCH, "longest": KV_ORDER_LONGEST, "long_first": KV_ORDER_LONG_FIRST}


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


def find_shared_prefix(block_tables, context_lens, block_size, min_sharers=2, min_tokens=1):
    """The largest group of running sequences whose block tables start with
    the same physical blocks (forked sequences, a common prompt cached once):
    (batch indices of the group, the common leading block ids), cut to whole
    blocks inside every member's context; (None, None) when no group of at
    least min_sharers shares at least min_tokens tokens.  Only the first
    column is grouped: one shared prefix per step."""
    lens = np.asarray(context_lens)
    b = lens.shape[0]
    if b < min_sharers:
        return None, None
    tables = np.asarray(block_tables)[:b]
    first = tables[:, 0]
    vals, counts = np.unique(first[first >= 0], return_counts=True)
    if counts.size == 0 or counts.max() < min_sharers:
        return None, None
    rows = np.nonzero(first == vals[np.argmax(counts)])[0]
    sub = tables[rows]
    same = np.all(sub == sub[0], axis=0) & (sub[0] >= 0)
    k = sub.shape[1] if same.all() else int(np.argmin(same))
    k = min(k, int(lens[rows].min()) // block_size)
    if k * block_size < max(min_tokens, 1):
        return None, None
    return rows.astype(np.int32), sub[0, :k].astype(np.int32)


class DecodeLoop:
    """Runs the iteration above on one device.  The step's metadata (slots,
    block tables, context lengths, scheduling order, copy pairs) is packed
    into one pinned buffer and uploaded with one copy on a side stream, into
    one of two device buffers, so the upload of the next step overlaps the
    kernels of the current one; events keep each buffer alive until the
    kernels that read it have run."""

    def __init__(self, pool, sched, *, num_q_heads, kv_heads, head_dim, block_size, q_dtype,
                 scale, max_batch, max_blocks, max_tokens, max_context, device="cuda",
                 order_policy="batch", host_swap=None, swap_slots=0, shared_prefix=False,
                 min_sharers=8, min_prefix_tokens=256):
        import torch
        self.torch = torch
        self.pool, self.sched = pool, sched
        self.hq, self.hkv, self.d, self.bs = num_q_heads, kv_heads, head_dim, block_size
        self.q_dtype, self.scale = q_dtype, scale
        self.max_batch, self.max_blocks, self.max_tokens = max_batch, max_blocks, max_tokens
        self.order_policy = order_policy
        self.host_swap, self.swap_slots = host_swap, swap_slots
        # shared-prefix decode (paged_attention_decode_shared_prefix) when a
        # group of at least min_sharers sequences shares min_prefix_tokens
        self.shared_prefix = shared_prefix
        self.min_sharers, self.min_prefix_tokens = min_sharers, min_prefix_tokens
        self.last_prefix = (None, None)
        cap = 8 * max_tokens + 4 * (max_batch * max_blocks + 6 * max_batch + 1) + 256
        if shared_prefix:
            cap += 4 * (2 * max_batch + max_blocks) + 64
        if swap_slots:
            cap += 16 * swap_slots + 64
        self.cap = (cap + 255) // 256 * 256
        self.h_buf = [torch.empty(self.cap, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self.d_buf = [torch.empty(self.cap, dtype=torch.uint8, device=device) for _ in range(2)]
        self.copy_ev = [None, None]  # upload into buffer k finished
        self.done_ev = [None, None]  # kernels reading buffer k finished
        self.side = torch.cuda.Stream(device=device)
        self.it = 0
        # the split policy partitions more finely when fewer sequences run, so
        # the scratch is sized for the largest need over every batch size
        ws = max(paged_attention_workspace_bytes(pool, b, num_q_heads, max_context)
                 for b in range(1, max_batch + 1))
        if shared_prefix:
            ws = max(ws, max(paged_attention_shared_prefix_workspace_bytes(pool, b, num_q_heads, max_context, b)
                             for b in range(1, max_batch + 1)))
        self.ws_cap = max(ws, 16)
        self.d_ws = torch.empty(self.ws_cap, dtype=torch.uint8, device=device)

    def schedule(self, finished_ids):
        """Native scheduler step; returns the step's host outputs."""
        info = kv_sched_step(self.sched, finished_ids)
        if info.batch > self.max_batch or info.num_tokens > self.max_tokens:
            raise RuntimeError("step exceeds the loop's buffers")
        out = kv_sched_outputs(self.sched, info, self.max_blocks)
        out.update(kv_sched_swap_outputs(self.sched))
        out["info"] = info
        return out

    @staticmethod
    def _layout(b, t, c, width, a=0, so=0, si=0, sh=0, shb=0):
        off, lay = 0, {}
        for name, n, size in (("slots", t, 8), ("tables", b * width, 4), ("lens", b, 4),
                              ("order", b, 4), ("cow", 2 * c, 4), ("cu", a + 1 if a else 0, 4),
                              ("pf_lens", a, 4), ("swo", 2 * so, 4), ("swi", 2 * si, 4),
                              ("sh_seqs", sh, 4), ("sh_blocks", shb, 4), ("skip", b if sh else 0, 4)):
            lay[name] = (off, n)
            off += (n * size + 15) // 16 * 16
        return lay, off

    @staticmethod
    def prefill_sizes(plan):
        """(admitted count, new tokens per admitted prompt, cached tokens per
        admitted prompt): admitted sequences are the last rows of the running
        set, their prompt is their context minus this step's appended token."""
        a = int(plan["info"].num_admitted)
        if a == 0:
            return 0, np.zeros(0, np.int64), np.zeros(0, np.int64)
        plen = np.asarray(plan["context_lens"][-a:], np.int64) - 1
        cached = np.asarray(plan.get("cached", np.zeros(a)), np.int64)
        return a, plen - cached, cached

    def launch(self, plan, k_new, v_new, q, out, k_inv=None, v_inv=None, out_dtype=None,
               layer=0, stream=None, prefill_q=None, prefill_out=None, before_decode=None):
        """Upload the plan's metadata and enqueue copy, write, prefill of the
        admitted prompts (when prefill_q is given) and decode.
        ``before_decode(stream)``, if given, is called right before the
        decode is enqueued (e.g. to record a timing event)."""
        torch = self.torch
        info = plan["info"]
        b, t, c, w = info.batch, info.num_tokens, info.num_cow, self.max_blocks
        a, new, _ = self.prefill_sizes(plan) if prefill_q is not None else (0, None, None)
        so = len(plan.get("swap_out", ()))
        si = len(plan.get("swap_in", ()))
        if (so or si) and self.host_swap is None:
            raise RuntimeError("the step swaps but the loop has no host swap space")
        k = self.it % 2
        self.it += 1
        sh_rows = sh_blocks = None
        if self.shared_prefix and b:
            sh_rows, sh_blocks = find_shared_prefix(plan["block_tables"], plan["context_lens"], self.bs,
                                                    self.min_sharers, self.min_prefix_tokens)
        self.last_prefix = (sh_rows, sh_blocks)
        nsh, nshb = (len(sh_rows), len(sh_blocks)) if sh_rows is not None else (0, 0)
        lay, nbytes = self._layout(b, t, c, w, a, so, si, nsh, nshb)
        if nbytes > self.cap:
            raise RuntimeError("step metadata exceeds the loop's buffers")
        if self.copy_ev[k] is not None:  # the pinned buffer is reused: its last upload must be done
            self.copy_ev[k].synchronize()
        hb = self.h_buf[k].numpy()

        def put(name, arr, dtype):
            off, n = lay[name]
            if n:
                hb[off:off + n * np.dtype(dtype).itemsize].view(dtype)[:] = np.asarray(arr, dtype).reshape(-1)

        put("slots", plan["slot_mapping"], np.int64)
        put("tables", plan["block_tables"], np.int32)
        put("lens", plan["context_lens"], np.int32)
        put("order", schedule_order(plan["context_lens"], self.order_policy), np.int32)
        put("cow", plan["cow_pairs"], np.int32)
        if so:
            put("swo", plan["swap_out"], np.int32)
        if si:
            put("swi", plan["swap_in"], np.int32)
        if nsh:
            put("sh_seqs", sh_rows, np.int32)
            put("sh_blocks", sh_blocks, np.int32)
            skip = np.zeros(b, np.int32)
            skip[sh_rows] = nshb * self.bs
            put("skip", skip, np.int32)
        if a:
            put("cu", np.concatenate([[0], np.cumsum(new)]), np.int32)
            put("pf_lens", np.asarray(plan["context_lens"][-a:], np.int64) - 1, np.int32)
        main = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(self.side):
            if self.done_ev[k] is not None:  # the device buffer is reused after its readers ran
                self.side.wait_event(self.done_ev[k])
            self.d_buf[k][:nbytes].copy_(self.h_buf[k][:nbytes], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.side)
            self.copy_ev[k] = ev
        main.wait_event(ev)

        def dview(name, dtype):
            off, n = lay[name]
            return self.d_buf[k][off:off + n * (8 if dtype == torch.int64 else 4)].view(dtype)

        max_ctx = int(plan["context_lens"].max()) if b else 0
        if so:  # before this step's writes can reuse the freed blocks
            kv_swap_out(self.pool, self.host_swap, self.swap_slots, dview("swo", torch.int32), so, main)
        if si:
            kv_swap_in(self.pool, self.host_swap, self.swap_slots, dview("swi", torch.int32), si, main)
        if c:
            block_copy(self.pool, dview("cow", torch.int32), c, main)
        if t:
            paged_kv_write(self.pool, layer, k_new, v_new, self.q_dtype, dview("slots", torch.int64), t,
                           k_inv, v_inv, main)
        if a and int(new.sum()) > 0:
            tables = dview("tables", torch.int32).view(b, w)[b - a:]
            paged_attention_prefill(self.pool, layer, prefill_q, self.q_dtype, self.hq, dview("cu", torch.int32),
                                    int(new.sum()), int(new.max()), tables, w, dview("pf_lens", torch.int32),
                                    a, self.scale, prefill_out, KV_F32 if out_dtype is None else out_dtype,
                                    main)
        if b and nsh:
            need = paged_attention_shared_prefix_workspace_bytes(self.pool, b, self.hq, max_ctx, nsh)
            if need > self.ws_cap:
                raise RuntimeError("decode workspace too small")
            if before_decode is not None:
                before_decode(main)
            paged_attention_decode_shared_prefix(
                self.pool, layer, q, self.q_dtype, self.hq, dview("tables", torch.int32), w,
                dview("lens", torch.int32), b, max_ctx, dview("sh_seqs", torch.int32), nsh,
                dview("sh_blocks", torch.int32), nshb * self.bs, dview("skip", torch.int32), self.scale, out,
                KV_F32 if out_dtype is None else out_dtype, self.d_ws, need, main,
                seq_order=dview("order", torch.int32))
        elif b:
            need = paged_attention_workspace_bytes(self.pool, b, self.hq, max_ctx)
            if need > self.ws_cap:
                raise RuntimeError("decode workspace too small")
            if before_decode is not None:
                before_decode(main)
            paged_attention_decode(self.pool, layer, q, self.q_dtype, self.hq, dview("tables", torch.int32),
                                   w, dview("lens", torch.int32), b, max_ctx, self.scale, out,
                                   KV_F32 if out_dtype is None else out_dtype, self.d_ws, need, main,
                                   seq_order=dview("order", torch.int32))
        done = torch.cuda.Event()
        done.record(main)
        self.done_ev[k] = done
        return max_ctx


class NativeDecodeLoop:
    """The iteration of :class:`DecodeLoop` sequenced inside the library
    (``kv_serve_schedule`` / ``kv_serve_launch``): the scheduler step packs
    the step's metadata straight into one of ``num_sets`` pinned buffers
    (used in turn) and queues its upload on the loop's upload stream; one
    launch call per layer then enqueues
    the swaps, copy-on-write, cache write, optional prefill and decode.  No
    shared-prefix decode (use :class:`DecodeLoop` for that).  This class only
    owns the buffers and passes pointers.  With ``full_plan`` set, schedule()
    also returns every array of the step (kv_sched_outputs and the swap
    outputs), for callers that check or mirror it."""

    def __init__(self, pool, sched, *, num_q_heads, kv_heads, head_dim, block_size, q_dtype,
                 scale, max_batch, max_blocks, max_tokens, max_context, device="cuda",
                 order_policy="batch", host_swap=None, swap_slots=0, num_sets=3):
        import torch
        self.torch = torch
        self.pool, self.sched = pool, sched
        self.hq, self.hkv, self.d, self.bs = num_q_heads, kv_heads, head_dim, block_size
        self.max_batch, self.max_blocks, self.max_tokens = max_batch, max_blocks, max_tokens
        # buffer sets used in turn: a step's uploads wait for the kernels of
        # the step num_sets before it (3 lets uploads and kernels overlap fully)
        self.num_sets = num_sets
        self.meta_bytes = kv_step_packed_bytes(max_batch, max_tokens, max_blocks, swap_slots)
        self.h_buf = [torch.empty(self.meta_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(num_sets)]
        self.d_buf = [torch.empty(self.meta_bytes, dtype=torch.uint8, device=device) for _ in range(num_sets)]
        self.ws_cap = max(kv_serve_workspace_bytes(pool, num_q_heads, max_batch, max_context), 16)
        self.d_ws = torch.empty(self.ws_cap, dtype=torch.uint8, device=device)
        self.up = torch.cuda.Stream(device=device)
        self.host_swap = host_swap
        self.handle = kv_serve_create(pool, sched, num_q_heads, q_dtype, scale, ORDER_POLICIES[order_policy],
                                      max_batch, max_tokens, max_blocks, host_swap, swap_slots, self.h_buf,
                                      self.d_buf, self.meta_bytes, self.d_ws, self.ws_cap)
        self.running_buf = np.empty(max_batch, np.int64)
        self.layout = kv_step_layout()
        self.last_prefix = (None, None)
        self.full_plan = False

    def schedule(self, finished_ids):
        """Native scheduler step + packed upload; returns {"info", "layout",
        "running"} (``running`` is a view valid until the next step)."""
        lay = kv_serve_schedule(self.handle, finished_ids, self.up, self.running_buf, self.layout)
        if not self.full_plan:
            return {"info": lay.info, "layout": lay, "running": self.running_buf[:lay.info.batch]}
        out = kv_sched_outputs(self.sched, lay.info, lay.table_width)
        out.update(kv_sched_swap_outputs(self.sched))
        out.update(info=lay.info, layout=lay)
        return out

    def launch(self, plan, k_new, v_new, q, out, k_inv=None, v_inv=None, out_dtype=None,
               layer=0, stream=None, prefill_q=None, prefill_out=None, before_decode=None):
        """Enqueue the step's kernels for one layer (``before_decode`` is
        called before the single launch call, which holds the decode)."""
        main = self.torch.cuda.current_stream() if stream is None else stream
        if before_decode is not None:
            before_decode(main)
        kv_serve_launch(self.handle, layer, q, k_new, v_new, out, KV_F32 if out_dtype is None else out_dtype,
                        k_inv, v_inv, prefill_q, prefill_out, main)
        return self.layout.max_context_len

    def upload(self, dev_dst, host_src, nbytes):
        """Copy the step's inputs from pinned host memory into the caller's
        buffer set ``plan["layout"].buffer`` (between schedule and launch)."""
        kv_serve_upload(self.handle, dev_dst, host_src, nbytes)

    def readback(self, host_dst, dev_src, nbytes, stream):
        """Copy the step's outputs to pinned host memory on ``stream``
        (after launch)."""
        kv_serve_readback(self.handle, host_dst, dev_src, nbytes, stream)

    def close(self):
        if self.handle is not None:
            kv_serve_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001  (interpreter shutdown)
            pass
