"""Seeded synthetic inputs for the paged-decode workloads.

This module only draws random numbers and lays out inputs: context lengths,
block placements (which physical block holds which logical block), query and
cache contents, FP8 scales and the arrival trace.  It holds none of the
attention or quantisation arithmetic; both the CUDA path and the CPU oracle
consume what it produces.

Workloads (sizes from the configurations the library is measured on):

* ``tiny``      1 layer, 4 sequences with cached lengths {1, 17, 33, 100}, 4 MHA
                heads, head_dim 64, block 16, fp16, a 64-block pool; one
                1-token cache write per sequence, then one decode step.
* ``llama13b``  one Llama-2-13B-shaped layer: 40 MHA heads, head_dim 128,
                block 16, fp16, batch 64, context lengths uniform in
                [128, 2048], pool 1.25x the blocks needed, scattered placement.
* ``kv_example`` the KV-size example of the pages: 32 layers x 32 heads x
                head_dim 128, bf16, block 16, batch 32, every sequence 2048
                tokens, placement randomly interleaved over a 4096-block pool.
* ``gqa_trace`` 64 query / 8 KV heads, head_dim 128, bf16, block 16, batch 256,
                lognormal context lengths (median 1024, capped 8192), half the
                sequences sharing a 1024-token prefix, 100-iteration trace.
* ``fp8_long``  32 MHA heads, head_dim 128, batch 8, context 16384, E4M3 cache
                with one fp32 scale per (block, kv head), bf16 queries.
* ``window_long`` 32 MHA heads, head_dim 128, bf16, batch 8, context 16384,
                sliding window of 4096 tokens (decode reads only the window).
* ``prefill_llama13b`` / ``prefill_gqa``  multi-token attention over whole
                prompts: 16 prompts of lengths uniform in [64, 2048] (the
                trace's arrival range), Llama-2-13B layer shape (fp16) or the
                64/8 GQA shape (bf16).
* ``chunked_gqa`` 16 sequences, each a 512-token prompt chunk on top of a
                cached prefix of 512..4096 tokens, 64/8 GQA, bf16.
* ``preempt_trace`` decode under memory pressure: 64 initial sequences
                (prompts U[256,1024]) plus Poisson arrivals (0.5 per
                iteration), U[100,400] output tokens, a 3000-block pool that
                the running set outgrows; preempted sequences are swapped to
                a 6000-slot host space or recomputed; 64/8 GQA, bf16.
* ``rag_trace`` retrieval-augmented serving: Poisson arrivals (3 per
                iteration, 60 iterations) whose prompt is one of 2 shared
                1536-token documents plus a U[32,256]-token question, U[16,64]
                output tokens; 64/8 GQA, bf16, 8192-block pool; prompts are
                prefilled, then every running sequence decodes each iteration.

Values of q, K and V are ~N(0, 1).  Seeds are 451 + the workload's index.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# element formats, as numbered by the product ABI and by the oracle
F16, BF16, E4M3, F32 = 0, 1, 2, 3


@dataclass
class Workload:
    name: str
    index: int
    num_layers: int
    num_q_heads: int
    kv_heads: int
    head_dim: int
    block_size: int
    kv_fmt: int
    q_fmt: int
    batch: int
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return 451 + self.index

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 4, 4, 64, 16, F16, F16, 4,
                     extra={"cached_lens": [1, 17, 33, 100], "pool_blocks": 64}),
    "llama13b": Workload("llama13b", 1, 1, 40, 40, 128, 16, F16, F16, 64,
                         extra={"ctx_lo": 128, "ctx_hi": 2048, "pool_factor": 1.25}),
    "kv_example": Workload("kv_example", 2, 32, 32, 32, 128, 16, BF16, BF16, 32,
                           extra={"ctx": 2048, "pool_blocks": 4096}),
    "gqa_trace": Workload("gqa_trace", 3, 1, 64, 8, 128, 16, BF16, BF16, 256,
                          extra={"median": 1024, "sigma": 1.0, "cap": 8192, "prefix": 1024,
                                 "share_frac": 0.5, "iters": 100, "arrival_rate": 2.5,
                                 "prompt_lo": 64, "prompt_hi": 2048, "max_num_seqs": 256,
                                 "pool_factor": 1.25}),
    "fp8_long": Workload("fp8_long", 4, 1, 32, 32, 128, 16, E4M3, BF16, 8,
                         extra={"ctx": 16384, "pool_factor": 1.25}),
    # sliding-window decode over long contexts
    "window_long": Workload("window_long", 9, 1, 32, 32, 128, 16, BF16, BF16, 8,
                            extra={"ctx": 16384, "window": 4096, "pool_factor": 1.25}),
    # multi-token attention (prompts and prompt chunks)
    "prefill_llama13b": Workload("prefill_llama13b", 5, 1, 40, 40, 128, 16, F16, F16, 16,
                                 extra={"new_lo": 64, "new_hi": 2048, "prior_lo": 0, "prior_hi": 0,
                                        "pool_factor": 1.25}),
    "prefill_gqa": Workload("prefill_gqa", 6, 1, 64, 8, 128, 16, BF16, BF16, 16,
                            extra={"new_lo": 64, "new_hi": 2048, "prior_lo": 0, "prior_hi": 0,
                                   "pool_factor": 1.25}),
    "chunked_gqa": Workload("chunked_gqa", 7, 1, 64, 8, 128, 16, BF16, BF16, 16,
                            extra={"new_lo": 512, "new_hi": 512, "prior_lo": 512, "prior_hi": 4096,
                                   "pool_factor": 1.25}),
    # decode under memory pressure: sequences outgrow the pool and are preempted
    "preempt_trace": Workload("preempt_trace", 10, 1, 64, 8, 128, 16, BF16, BF16, 64,
                              extra={"prompt_lo": 256, "prompt_hi": 1024, "out_lo": 100, "out_hi": 400,
                                     "arrival_rate": 0.5, "iters": 150, "max_num_seqs": 96,
                                     "num_blocks": 3000, "swap_slots": 6000}),
    # retrieval-augmented requests: a shared document + a question each
    "rag_trace": Workload("rag_trace", 8, 1, 64, 8, 128, 16, BF16, BF16, 128,
                          extra={"docs": 2, "doc_len": 1536, "question_lo": 32, "question_hi": 256,
                                 "out_lo": 16, "out_hi": 64, "arrival_rate": 3.0, "iters": 60,
                                 "max_num_seqs": 128, "num_blocks": 8192, "vocab": 32000}),
}


def prefill_lens(w: Workload):
    """(cached-before lengths, new-token counts) of a multi-token workload:
    new tokens uniform in [new_lo, new_hi] (the trace's prompt range for whole
    prompts), on top of a cached prefix uniform in [prior_lo, prior_hi]."""
    e = w.extra
    r = rng_for(w, 3)
    new = r.integers(e["new_lo"], e["new_hi"] + 1, size=w.batch).astype(np.int32)
    prior = r.integers(e["prior_lo"], e["prior_hi"] + 1, size=w.batch).astype(np.int32)
    return prior, new


def rng_for(w: Workload, salt: int = 0) -> np.random.Generator:
    return np.random.default_rng([w.seed, salt])


def blocks_needed(lens, block_size: int) -> np.ndarray:
    return (np.asarray(lens, dtype=np.int64) + block_size - 1) // block_size


def context_lens(w: Workload) -> np.ndarray:
    """Attended context length per sequence for a single decode step."""
    r = rng_for(w, 1)
    if w.name == "tiny":
        return np.asarray(w.extra["cached_lens"], dtype=np.int32) + 1
    if w.name == "llama13b":
        return r.integers(w.extra["ctx_lo"], w.extra["ctx_hi"] + 1, size=w.batch).astype(np.int32)
    if w.name in ("kv_example", "fp8_long", "window_long"):
        return np.full(w.batch, w.extra["ctx"], dtype=np.int32)
    if w.name == "gqa_trace":
        x = r.lognormal(math.log(w.extra["median"]), w.extra["sigma"], size=w.batch)
        return np.clip(np.rint(x), 1, w.extra["cap"]).astype(np.int32)
    if "new_lo" in w.extra:  # multi-token workloads: cached prefix + new tokens
        prior, new = prefill_lens(w)
        return prior + new
    raise KeyError(w.name)


def pool_blocks(w: Workload, lens) -> int:
    if "pool_blocks" in w.extra:
        return int(w.extra["pool_blocks"])
    need = int(blocks_needed(lens, w.block_size).sum())
    return int(math.ceil(w.extra.get("pool_factor", 1.25) * need))


def scattered_tables(rng: np.random.Generator, lens, block_size: int, num_blocks: int,
                     pad_to: int | None = None) -> np.ndarray:
    """Block tables that hand each sequence consecutive entries of one seeded
    permutation of the pool, so logically adjacent blocks are physically
    scattered.  Unused entries are -1."""
    need = blocks_needed(lens, block_size)
    total = int(need.sum())
    if total > num_blocks:
        raise ValueError("pool too small")
    perm = rng.permutation(num_blocks).astype(np.int32)
    width = int(need.max()) if pad_to is None else int(pad_to)
    tables = np.full((len(lens), max(width, 1)), -1, dtype=np.int32)
    off = 0
    for i, n in enumerate(need):
        tables[i, :n] = perm[off:off + n]
        off += n
    return tables


# ------------------------------------------------------------- value draws

def normal_bits(rng: np.random.Generator, shape, fmt: int) -> np.ndarray:
    """~N(0, 1) values rounded to fp16 or bf16, returned as raw uint16 bits."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if fmt == F16:
        return x.astype(np.float16).view(np.uint16)
    if fmt == BF16:
        import torch
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(fmt)


def e4m3_codes(rng: np.random.Generator, shape, spread: float = 96.0) -> np.ndarray:
    """Random E4M3 codes: ~N(0, 1) * spread, clipped to +-448, converted by
    torch's float8_e4m3fn cast."""
    import torch
    x = np.clip(rng.standard_normal(size=shape, dtype=np.float32) * spread, -448.0, 448.0)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def fp8_scales(rng: np.random.Generator, shape) -> np.ndarray:
    """Positive fp32 per-(block, head) scales, log-uniform in [2^-9, 2^-4]."""
    return np.exp2(rng.uniform(-9.0, -4.0, size=shape)).astype(np.float32)


def random_pool(rng: np.random.Generator, w: Workload, num_blocks: int):
    """Host K and V pools [num_blocks][kv_heads][block_size][head_dim] of raw
    storage filled with random values (every slot, used or not), plus FP8
    scales (None for 16-bit pools)."""
    shape = (num_blocks, w.kv_heads, w.block_size, w.head_dim)
    if w.kv_fmt == E4M3:
        k = e4m3_codes(rng, shape)
        v = e4m3_codes(rng, shape)
        ks = fp8_scales(rng, (num_blocks, w.kv_heads))
        vs = fp8_scales(rng, (num_blocks, w.kv_heads))
        return k, v, ks, vs
    return normal_bits(rng, shape, w.kv_fmt), normal_bits(rng, shape, w.kv_fmt), None, None


def device_pool(w: Workload, num_blocks: int, device, seed: int | None = None):
    """Same as :func:`random_pool` but drawn on the GPU with a seeded torch
    generator (fast for multi-GB pools).  Returns torch tensors of raw
    storage (int16 / uint8 views) and scales."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (num_blocks, w.kv_heads, w.block_size, w.head_dim)

    def draw16(fmt):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return t.to(torch.float16 if fmt == F16 else torch.bfloat16).view(torch.int16)

    if w.kv_fmt == E4M3:
        def draw8():
            t = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * 96.0
            return t.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        k, v = draw8(), draw8()
        ks = torch.exp2(torch.rand((num_blocks, w.kv_heads), generator=g, device=device) * 5.0 - 9.0)
        vs = torch.exp2(torch.rand((num_blocks, w.kv_heads), generator=g, device=device) * 5.0 - 9.0)
        return k, v, ks, vs
    return draw16(w.kv_fmt), draw16(w.kv_fmt), None, None


def device_normal_bits(shape, fmt: int, device, seed: int):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return t.to(torch.float16 if fmt == F16 else torch.bfloat16).view(torch.int16)


# ------------------------------------------------------------ trace inputs

def gqa_trace_plan(w: Workload):
    """Draws for the continuous-batching trace: initial context lengths, which
    sequences share the prefix, the common tail length r after the prefix,
    remaining output lengths, and per-iteration arrivals (prompt length,
    output length)."""
    e = w.extra
    r = rng_for(w, 7)
    lens = context_lens(w)
    sharers = np.sort(r.choice(w.batch, size=int(w.batch * e["share_frac"]), replace=False))
    tail = int(r.integers(1, 16))
    remaining = r.integers(1, 201, size=w.batch)
    arrivals = []
    for _ in range(e["iters"]):
        k = int(r.poisson(e["arrival_rate"]))
        arrivals.append([(int(r.integers(e["prompt_lo"], e["prompt_hi"] + 1)),
                          int(r.integers(50, 2001))) for _ in range(k)])
    return {"lens": lens, "sharers": sharers, "tail": tail, "remaining": remaining,
            "arrivals": arrivals}
