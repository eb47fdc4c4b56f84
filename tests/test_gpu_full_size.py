"""GPU parity at the measured workloads' full sizes, in the launch
configuration bench.py times.

Each test draws the whole workload on the device (every layer's pool with
its own values, scattered block placement), runs the step the bench times
through the C ABI — the cache write of every sequence's last token, then the
decode of every sequence with the automatic launch policy, longest contexts
scheduled first — and checks sampled sequences against the oracle:

* the written blocks of the sampled sequences bit for bit against the
  oracle's cache-write mirror applied to the same blocks as drawn;
* their decode output element by element (fp32 output, max-abs 2e-3 for
  16-bit caches, 1e-2 for FP8) and in the query dtype the bench writes
  (the same bound plus one rounding of the format).

The oracle's inputs are the generator's values copied back before the GPU
step runs, never anything the library wrote.  The pages require the kernel
to read correctly from non-contiguous blocks ("vLLM 推理加速原理详解", section
"PagedAttention：把操作系统的虚拟内存搬进 GPU"); these sizes are where the
placement is most scattered and where the automatic split policy decides the
partitioning.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from gpu_util import TOL, max_abs
from paged_kv_cache_451_b200.serving import schedule_order
from workloads import BF16, E4M3, F32
from workloads.decode_inputs import DecodeInputs

pytestmark = pytest.mark.gpu


def bind(inp, partition=0):
    w = inp.w
    pool = pk.kv_pool_create(w.block_size, inp.nb, w.kv_heads, w.head_dim, w.kv_fmt, inp.L)
    for layer in range(inp.L):
        pk.kv_pool_bind(pool, layer, inp.k[layer], inp.v[layer], inp.ks[layer], inp.vs[layer])
    if partition:
        pk.kv_pool_set_decode_config(pool, partition, 0, 0)
    return pool


def step(inp, pool, out_fmt, layers=None):
    """The bench's step over the given layers: write, then decode."""
    w = inp.w
    order = torch.from_numpy(schedule_order(inp.lens, "longest")).cuda()
    B, Hq, D = w.batch, w.num_q_heads, w.head_dim
    wsb = pk.paged_attention_workspace_bytes(pool, B, Hq, inp.max_ctx)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    outs = {}
    for layer in (range(inp.L) if layers is None else layers):
        inv = inp.inv[layer] if inp.inv else (None, None)
        pk.paged_kv_write(pool, layer, inp.kn[layer], inp.vn[layer], w.q_fmt, inp.slots, B, inv[0], inv[1])
        dt = torch.float32 if out_fmt == F32 else inp.out_torch_dtype
        out = torch.full((B, Hq, D), float("nan"), dtype=dt, device="cuda")
        pk.paged_attention_decode(pool, layer, inp.q[layer], w.q_fmt, Hq, inp.tables_d, inp.tables.shape[1],
                                  inp.lens_d, B, inp.max_ctx, w.scale, out, out_fmt, ws, wsb, seq_order=order)
        outs[layer] = out
    torch.cuda.synchronize()
    assert pk.kv_get_device_error() == pk.KV_OK
    return outs, wsb


def oracle_check(inp, samples, outs, layer, seqs, out_fmt):
    """Oracle cache write + decode on the sampled sequences' blocks as drawn;
    compares the GPU's written blocks and its outputs."""
    w = inp.w
    s = samples[layer]
    kref, vref = s["k"].copy(), s["v"].copy()
    oracle.kv_write(kref, vref, w.kv_fmt, s["k_new"], s["v_new"], w.q_fmt, s["slots"], w.block_size,
                    s["k_inv"], s["v_inv"])
    idx = torch.tensor(s["blocks"], dtype=torch.long, device="cuda")
    raw = np.uint8 if w.kv_fmt == E4M3 else np.uint16
    assert np.array_equal(inp.k[layer].index_select(0, idx).cpu().numpy().view(raw), kref), f"K, layer {layer}"
    assert np.array_equal(inp.v[layer].index_select(0, idx).cpu().numpy().view(raw), vref), f"V, layer {layer}"
    ref = oracle.paged_decode(kref, vref, w.kv_fmt, s["q"], w.q_fmt, s["tables"], s["lens"], w.scale,
                              w.block_size, s["k_scale"], s["v_scale"])
    got = outs[layer][list(seqs)].float().cpu().numpy().astype(np.float64)
    tol = TOL[w.kv_fmt]
    if out_fmt == F32:
        err = max_abs(got, ref)
        assert err <= tol, (layer, err)
    else:
        u = 2.0 ** -8 if w.q_fmt == BF16 else 2.0 ** -11
        excess = np.abs(got - ref) - (tol + 2 * u * np.abs(ref))
        assert np.all(excess <= 0), (layer, float(excess.max()))


def sampled(inp):
    """The longest, the shortest and a middle-length sequence."""
    order = np.argsort(inp.lens, kind="stable")
    return sorted({int(order[-1]), int(order[0]), int(order[len(order) // 2])})


@pytest.mark.parametrize("out_fmt", [F32, "native"])
def test_llama13b_layer_full_size(out_fmt):
    """64 sequences x 40 MHA heads, head_dim 128, fp16, contexts U[128, 2048],
    pool 1.25x the blocks needed with a scattered placement."""
    inp = DecodeInputs("llama13b")
    fmt = F32 if out_fmt == F32 else inp.w.q_fmt
    seqs = sampled(inp)
    samples = {0: inp.host_sample(seqs, 0)}
    pool = bind(inp)
    try:
        outs, _ = step(inp, pool, fmt)
        oracle_check(inp, samples, outs, 0, seqs, fmt)
    finally:
        pk.kv_pool_destroy(pool)


def test_kv_example_every_layer_is_its_own_pool():
    """The pages' KV-size example: 32 layers x 32 heads x head_dim 128, bf16,
    32 sequences of 2048 tokens over 4096 blocks per layer, decoded layer by
    layer through each layer's own bound pool.  Layers 0, 1, 17 and 31 are
    checked; every layer holds different values, so a decode that read
    another layer's pool (a wrong per-layer descriptor) fails."""
    inp = DecodeInputs("kv_example")
    assert inp.L == 32
    seqs = [0, 13, 31]
    checked = (0, 1, 17, 31)
    samples = {layer: inp.host_sample(seqs, layer) for layer in checked}
    pool = bind(inp)
    try:
        outs, wsb = step(inp, pool, F32)
        assert wsb == 0  # 1024 (sequence, head) units: no split
        for layer in checked:
            oracle_check(inp, samples, outs, layer, seqs, F32)
        # the layers really differ: layer 1's output is not layer 0's
        assert max_abs(outs[0][seqs].cpu().numpy(), outs[1][seqs].cpu().numpy()) > 0.05
        # the native-dtype outputs the bench writes, on two layers
        outs_n, _ = step(inp, pool, inp.w.q_fmt, layers=(0, 31))
        for layer in (0, 31):
            oracle_check(inp, samples, outs_n, layer, seqs, inp.w.q_fmt)
    finally:
        pk.kv_pool_destroy(pool)


@pytest.mark.parametrize("partition", [0, 512])
def test_fp8_long_context_full_size(partition):
    """8 x 16384-token contexts, 32 MHA heads, E4M3 cache with one fp32
    scale per (block, kv head), bf16 queries: under the automatic split
    (partition 0) and under 512-token partitions with the LSE reduce."""
    inp = DecodeInputs("fp8_long")
    w = inp.w
    seqs = [0, w.batch - 1]
    samples = {0: inp.host_sample(seqs, 0)}
    pool = bind(inp, partition)
    try:
        B, Hq, D = w.batch, w.num_q_heads, w.head_dim
        wsb = pk.paged_attention_workspace_bytes(pool, B, Hq, inp.max_ctx)
        np_parts = wsb // (B * Hq * (D + 4) * 4)
        if partition:
            assert np_parts == 16384 // 512
        else:
            assert np_parts > 1  # 256 (sequence, head) units are split for balance
        outs, _ = step(inp, pool, F32)
        oracle_check(inp, samples, outs, 0, seqs, F32)
        outs_n, _ = step(inp, pool, w.q_fmt)
        oracle_check(inp, samples, outs_n, 0, seqs, w.q_fmt)
    finally:
        pk.kv_pool_destroy(pool)
