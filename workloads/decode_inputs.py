"""Device-resident inputs of one single-step decode workload, drawn with torch.

Everything here is random draws and layout: context lengths, the scattered
block placement, per-layer K/V pools (and FP8 scales), queries, the step's
new K/V rows and the slots they go to (each sequence's last position).  No
attention, quantisation or cache-write arithmetic happens here.  Both the
product path (through the C ABI) and the CPU oracle consume these inputs, and
the oracle side never needs the product library to obtain them.

A step of these workloads writes each sequence's last token (position
len - 1) with the cache write and then decodes every sequence over its whole
context (or its sliding window).
"""

from __future__ import annotations

import numpy as np

from . import (E4M3, F16, WORKLOADS, blocks_needed, context_lens, device_normal_bits, device_pool,
               pool_blocks, scattered_tables)


class DecodeInputs:
    """Inputs of workload ``name`` for replica ``rank`` on the current CUDA
    device.  ``layers`` limits the layer count (the workload's own count if
    None); layer l's pool, queries and new rows are drawn from seeds that
    depend on l, so every layer holds different values."""

    def __init__(self, name: str, rank: int = 0, layers: int | None = None):
        import torch
        w = WORKLOADS[name]
        self.w = w
        self.lens = context_lens(w)
        self.nb = pool_blocks(w, self.lens)
        rng = np.random.default_rng([w.seed, 1000 + rank])
        self.tables = scattered_tables(rng, self.lens, w.block_size, self.nb)
        dev = torch.device("cuda")
        seed = w.seed * 7919 + rank
        self.L = w.num_layers if layers is None else int(layers)
        self.window = int(w.extra.get("window", 0))
        self.k, self.v, self.ks, self.vs = [], [], [], []
        for layer in range(self.L):
            k, v, ks, vs = device_pool(w, self.nb, dev, seed=seed + 13 * layer)
            self.k.append(k)
            self.v.append(v)
            self.ks.append(ks)
            self.vs.append(vs)
        B, Hq, Hkv, D = w.batch, w.num_q_heads, w.kv_heads, w.head_dim
        self.q = [device_normal_bits((B, Hq, D), w.q_fmt, dev, seed + 1 + 17 * l) for l in range(self.L)]
        self.kn = [device_normal_bits((B, Hkv, D), w.q_fmt, dev, seed + 2 + 17 * l) for l in range(self.L)]
        self.vn = [device_normal_bits((B, Hkv, D), w.q_fmt, dev, seed + 3 + 17 * l) for l in range(self.L)]
        pos = self.lens.astype(np.int64) - 1
        self.slots_h = (self.tables[np.arange(B), pos // w.block_size].astype(np.int64) * w.block_size
                        + pos % w.block_size)
        self.slots = torch.from_numpy(self.slots_h).to(dev)
        self.tables_d = torch.from_numpy(self.tables).to(dev)
        self.lens_d = torch.from_numpy(self.lens).to(dev)
        # FP8 writes take the inverse of each (block, kv head) scale
        self.inv = None
        if w.kv_fmt == E4M3:
            self.inv = [(1.0 / self.ks[l], 1.0 / self.vs[l]) for l in range(self.L)]
        self.max_ctx = int(self.lens.max())
        self.blocks_touched = int(blocks_needed(self.lens, w.block_size).sum())
        # attended tokens per sequence: the whole context, or the window
        self.attended = np.minimum(self.lens, self.window) if self.window else self.lens
        self.out_torch_dtype = torch.float16 if w.q_fmt == F16 else torch.bfloat16

    def host_sample(self, seqs, layer: int = 0):
        """Host copies of what the sampled sequences read and write in one
        layer, as they were drawn: their blocks (and FP8 scales), remapped
        to a small pool numbered in table order, the remapped tables, their
        queries, new rows, slots in the small pool and lengths."""
        import torch
        w = self.w
        bs = w.block_size
        seqs = [int(s) for s in seqs]
        used, sub = [], np.full((len(seqs), self.tables.shape[1]), -1, np.int32)
        for i, s in enumerate(seqs):
            for j in range(-(-int(self.lens[s]) // bs)):
                sub[i, j] = len(used)
                used.append(int(self.tables[s, j]))
        idx = torch.tensor(used if used else [0], dtype=torch.long, device=self.k[layer].device)
        raw = np.uint8 if w.kv_fmt == E4M3 else np.uint16
        kh = self.k[layer].index_select(0, idx).cpu().numpy().view(raw)
        vh = self.v[layer].index_select(0, idx).cpu().numpy().view(raw)
        ks = vs = inv_k = inv_v = None
        if w.kv_fmt == E4M3:
            ks = self.ks[layer].index_select(0, idx).cpu().numpy()
            vs = self.vs[layer].index_select(0, idx).cpu().numpy()
            inv_k = self.inv[layer][0].index_select(0, idx).cpu().numpy()
            inv_v = self.inv[layer][1].index_select(0, idx).cpu().numpy()
        pos = self.lens[seqs].astype(np.int64) - 1
        slots = sub[np.arange(len(seqs)), pos // bs].astype(np.int64) * bs + pos % bs
        sel = torch.tensor(seqs, dtype=torch.long, device=self.q[layer].device)
        q = self.q[layer].index_select(0, sel).cpu().numpy().view(np.uint16)
        kn = self.kn[layer].index_select(0, sel).cpu().numpy().view(np.uint16)
        vn = self.vn[layer].index_select(0, sel).cpu().numpy().view(np.uint16)
        return {"k": kh, "v": vh, "k_scale": ks, "v_scale": vs, "k_inv": inv_k, "v_inv": inv_v,
                "tables": sub, "q": q, "k_new": kn, "v_new": vn, "slots": slots,
                "lens": self.lens[seqs].astype(np.int32), "blocks": used}
