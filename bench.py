"""Benchmark of the paged-decode hot path on B200.

One step = the cache write of the step's new tokens (paged_kv_write) and one
PagedAttention decode over every sequence (paged_attention_decode, with its
split-K reduce when contexts are split), all through the C ABI, on inputs
resident in HBM.  Default workload: the pages' KV-size example — 32 layers x
32 heads x head_dim 128, bf16, block 16, 32 sequences of 2048 tokens (about
1.07 GB of K/V per request, 34 GB in all) — one step covering all 32 layers.

Prints one JSON line (rank 0).  ``value`` is achieved GB/s of algorithmic
bytes (K/V read + q read + output write + the step's cache-write bytes) over
the device-timed step, summed over ranks; ``seqs_per_s`` is decode sequences
per second (a step decodes every sequence through all its layers).  On one
GPU the line also carries ``per_config``: the other measured decode
workloads (the Llama-2-13B-shaped layer, the GQA continuous-batching trace,
long-context FP8 under the automatic split and under 512-token partitions),
each timed for at least a second with its own roofline, end-to-end figure and
clock record.  ``--impl reference`` times the CPU oracle on the same workload
instead.

The CPU-baseline leg runs the oracle on sampled sequences of each workload,
times it, and checks the GPU outputs of those sequences against it (outside
every timed region); a mismatch makes the run exit non-zero.

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``: every rank runs
an independent replica (decode shards by sequence with no exchange), time is
the max over ranks, ``value`` the bytes of all ranks over that time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: achieved KV-read GB/s (% of HBM peak); decode seqs/s"
METRIC_PREFILL = "paged multi-token attention: achieved TFLOP/s (% of tensor peak); new tokens/s"
PREFILL_WORKLOADS = ("prefill_llama13b", "prefill_gqa", "chunked_gqa")
DECODE_WORKLOADS = ("tiny", "llama13b", "kv_example", "fp8_long", "window_long")
METRIC_RAG = "retrieval-augmented serving with prefix caching: generated tokens/s (vs no caching)"
METRIC_PREEMPT = "decode under memory pressure with swap preemption: generated tokens/s (vs recompute)"
FALLBACK_BF16_TFLOPS = 1590.0
# dense bf16 under the power cap in a seconds-long loop (the recipe's figure)
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
SUSTAINED_MS = 500.0  # a timed region this long runs under the power cap
FALLBACK_HBM_GBS = 6650.0
DTYPE_NAME = {0: "f16", 1: "bf16", 2: "e4m3"}
ELEM = {0: 2, 1: 2, 2: 1}
MIN_TIMED_S = 1.0  # every per-config measurement times at least this much device work


# ------------------------------------------------------------------ helpers

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak(sustained=False):
    """Dense bf16 peak: the burst figure for a kernel timed alone, the
    sustained one (a seconds-long loop under the power cap) for one timed
    over a long region."""
    key, fb = ("bf16_tflops_sustained", FALLBACK_BF16_TFLOPS_SUSTAINED) if sustained else \
        ("bf16_tflops", FALLBACK_BF16_TFLOPS)
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)[key]), "measured"
    except Exception:  # noqa: BLE001
        return fb, "fallback"


def stream_rooflines(torch, stream):
    """Two plain streams timed on this GPU as extra, context-only
    denominators beside the official peak: a read-only stream over 4 GiB
    (the faster of a bf16 vector-matrix product, which reads the matrix once,
    and a float32 sum of the same bytes), as the decode only reads its K/V,
    and a copy (1 Gi bf16 elements, counting read + write bytes, the method
    of the measured-peak file).  Best of 10 CUDA-event-timed passes after 3
    warm-ups; the inputs are far larger than L2."""
    def best(fn, nbytes):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return nbytes / (min(ts) * 1e-3) / 1e9
    with torch.cuda.stream(stream):
        x = torch.ones(1 << 31, dtype=torch.bfloat16, device="cuda")
        w = torch.ones(1 << 15, dtype=torch.bfloat16, device="cuda")
        mat = x.view(1 << 15, 1 << 16)
        gemv = best(lambda: w @ mat, x.numel() * 2)
        x32 = x.view(torch.float32)
        fsum = best(lambda: x32.sum(), x.numel() * 2)
        del x, w, mat, x32
        src = torch.ones(1 << 30, dtype=torch.bfloat16, device="cuda")
        dst = torch.empty_like(src)
        copy = best(lambda: dst.copy_(src), 2 * src.numel() * 2)
        del src, dst
    torch.cuda.empty_cache()
    return {"read_gbs": round(max(gemv, fsum), 1), "read_gemv_gbs": round(gemv, 1), "read_sum_gbs": round(fsum, 1),
            "copy_gbs": round(copy, 1),
            "method": "read: bf16 vector x [32768 x 65536] matrix (torch / cuBLAS) and a float32 sum of the same "
                      "4 GiB, the faster; copy: 1 Gi bf16 elements, read + write bytes (torch copy_); best of 10 "
                      "CUDA-event-timed passes; context only, the official peak stays MEASURED_PEAKS.json or "
                      "the fallback"}


def source_hash(files):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_451_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def decode_source_hash():
    return source_hash(("decode.cuh", "ptx.cuh", "pagedkv.cu"))


def prefill_source_hash():
    return source_hash(("prefill.cuh", "tcgen05.cuh", "ptx.cuh", "prefill.cu"))


def committed_traffic(workload, source_hash_=None):
    """DRAM bytes per launch of the workload's dominant kernel from a
    committed ncu capture, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(workload)
    except Exception:  # noqa: BLE001
        return None
    if not rec or rec.get("source_hash") != (source_hash_ or decode_source_hash()):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """Polls NVML (the library nvidia-smi reads) for the SM clock and the
    throttle reasons every 2 ms from start() to stop(), keeping a host
    timestamp with each sample; summary(t0, t1) describes the samples taken
    while a timed region ran.  Read-only: it changes no setting."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples = []  # (t, sm_mhz, reasons)
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:  # noqa: BLE001
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception:  # noqa: BLE001
            pass
        self._stop = threading.Event()
        self.t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                self.samples.append((t, mhz, int(self.get_reasons(self.h))))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok and self.t is None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.t is not None:
            self._stop.set()
            self.t.join()
            self.t = None

    def summary(self, t0, t1):
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        if not self.ok or not sel:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        bits = 0
        for s in sel:
            bits |= s[2]
        names = [n for bit, n in self.REASONS.items() if bits & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": self.max_mhz,
                "sm_min_mhz": min(s[1] for s in sel), "reasons": names, "samples": len(sel),
                "region_s": round(t1 - t0, 3), "source": "nvml, 2 ms polling during the timed region"}


def max_over_ranks(value, dist, device):
    """Max of a per-rank scalar over all ranks (timing plumbing only)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(bytes_per_rank, world, max_ms):
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


class L2Flush:
    """Evicts L2 (126 MB on B200) between timed steps: zero_() writes a
    256 MiB buffer and then reads another 256 MiB, so the dirty lines the
    write leaves are written back before the next step starts (otherwise
    the step pays for ~126 MB of write-backs that are not its own work)."""

    def __init__(self, torch):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(64 << 20, dtype=torch.float32, device="cuda")

    def zero_(self):
        self.w.zero_()
        self.r.sum()


L2_NOTE = "flushed between steps (256 MiB write, then 256 MiB read: no dirty lines left)"


def init_dist(world):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return dist


# ------------------------------------------------------- single-step decode

class Case:
    """Device-resident inputs of one decode workload replica (drawn by
    workloads.decode_inputs) bound to a pool of the product library."""

    def __init__(self, name, rank, torch, pk, args=None, layers=None, partition=None):
        from paged_kv_cache_451_b200.serving import schedule_order
        from workloads.decode_inputs import DecodeInputs
        inp = DecodeInputs(name, rank, layers)
        self.inp = inp
        self.w, self.torch, self.pk = inp.w, torch, pk
        w = self.w
        self.lens, self.nb, self.tables, self.L, self.window = inp.lens, inp.nb, inp.tables, inp.L, inp.window
        self.k, self.v, self.ks, self.vs = inp.k, inp.v, inp.ks, inp.vs
        self.q, self.kn, self.vn, self.inv = inp.q, inp.kn, inp.vn, inp.inv
        self.slots, self.tables_d, self.lens_d, self.max_ctx = inp.slots, inp.tables_d, inp.lens_d, inp.max_ctx
        self.pool = pk.kv_pool_create(w.block_size, self.nb, w.kv_heads, w.head_dim, w.kv_fmt, self.L)
        if self.window:
            pk.kv_pool_set_sliding_window(self.pool, self.window)
        for layer in range(self.L):
            pk.kv_pool_bind(self.pool, layer, self.k[layer], self.v[layer], self.ks[layer], self.vs[layer])
        part = getattr(args, "partition", 0) if partition is None else partition
        stages, warps = getattr(args, "stages", 0), getattr(args, "warps", 0)
        if part or stages or warps:
            pk.kv_pool_set_decode_config(self.pool, part, stages, warps)
        self.partition = part
        B, Hq, Hkv, D = w.batch, w.num_q_heads, w.kv_heads, w.head_dim
        # the caller's scheduling order (placement only): long contexts first
        self.order_name = getattr(args, "order", None) or "longest"
        self.order_h = schedule_order(self.lens, self.order_name)
        self.order_d = torch.from_numpy(self.order_h).to("cuda")
        self.out = [torch.empty((B, Hq, D), dtype=inp.out_torch_dtype, device="cuda") for _ in range(self.L)]
        self.ws_bytes = pk.paged_attention_workspace_bytes(self.pool, B, Hq, self.max_ctx)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device="cuda")
        self.split = self.ws_bytes > 0
        self.num_parts = self.ws_bytes // (B * Hq * (D + 4) * 4) if self.split else 1
        e_kv, e_q = ELEM[w.kv_fmt], ELEM[w.q_fmt]
        self.attended = inp.attended
        self.decode_bytes = self.L * (int(self.attended.astype(np.int64).sum()) * Hkv * D * 2 * e_kv
                                      + B * Hq * D * (e_q + e_q)
                                      + (2 * 4 * inp.blocks_touched * Hkv if w.kv_fmt == 2 else 0))
        self.write_bytes = self.L * B * Hkv * D * 2 * (e_q + e_kv)
        self.step_bytes = self.decode_bytes + self.write_bytes
        # the cache write and the decode (split partials are merged by the decode's
        # last partition CTA; the merge counters are zeroed by a memset)
        self.launches_per_step = self.L * 2

    def write(self, layer, kn=None, vn=None, slots=None):
        w, pk = self.w, self.pk
        inv = self.inv[layer] if self.inv else (None, None)
        pk.paged_kv_write(self.pool, layer, self.kn[layer] if kn is None else kn,
                          self.vn[layer] if vn is None else vn, w.q_fmt,
                          self.slots if slots is None else slots, w.batch, inv[0], inv[1])

    def decode(self, layer, q=None, tables=None, lens=None, out=None, order=None):
        w, pk = self.w, self.pk
        pk.paged_attention_decode(self.pool, layer, self.q[layer] if q is None else q, w.q_fmt,
                                  w.num_q_heads, self.tables_d if tables is None else tables,
                                  self.tables.shape[1], self.lens_d if lens is None else lens, w.batch,
                                  self.max_ctx, w.scale, self.out[layer] if out is None else out,
                                  w.q_fmt, self.ws, self.ws_bytes,
                                  seq_order=self.order_d if order is None else order)

    def destroy(self):
        self.pk.kv_pool_destroy(self.pool)


def timed_steps(case, K, flush, stream, clk):
    """K device-timed steps (L2 flushed before each): returns (step ms list,
    decode-launch ms list, clock summary).  A step is, for every layer, the
    cache write then the decode (and its reduce)."""
    torch = case.torch
    L = case.L
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    evw = [[torch.cuda.Event(enable_timing=True) for _ in range(L)] for _ in range(K)]
    evd = [[torch.cuda.Event(enable_timing=True) for _ in range(L)] for _ in range(K)]
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        for layer in range(L):
            case.write(layer)
            evw[i][layer].record(stream)
            case.decode(layer)
            evd[i][layer].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    step_ms = [ev0[i].elapsed_time(evd[i][-1]) for i in range(K)]
    dec_ms = [evw[i][l].elapsed_time(evd[i][l]) for i in range(K) for l in range(L)]
    return step_ms, dec_ms, clk.summary(t0, t1)


def decode_roofline(case, dec_ms, workload_key):
    peak, peak_kind = hbm_peak()
    dec_avg = sum(dec_ms) / len(dec_ms)
    per_launch = case.decode_bytes / case.L
    achieved = per_launch / (dec_avg * 1e-3) / 1e9
    return {
        "bound": "hbm",
        "kernel": "paged_attention_decode (decode kernel" + (", split partials merged by its last partition CTA)"
                                                            if case.split else ")"),
        "achieved": round(achieved, 2),
        "peak": peak,
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": committed_traffic(workload_key),
        "algorithmic_bytes_per_launch": per_launch,
        "launch_ms": round(dec_avg, 5),
        "peak_note": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback copy bandwidth",
    }


def measure_decode(case, args, stream, flush, clk, dist, world, K=None, min_s=None, key=None):
    """Warm-up, then the device-timed steps (exactly K, or enough for min_s
    seconds of device time), the end-to-end loop with host buffers, and the
    roofline of the decode kernel.  Returns a dict of figures."""
    torch, pk = case.torch, case.pk
    W = args.warmup
    for _ in range(W):
        flush.zero_()
        for layer in range(case.L):
            case.write(layer)
            case.decode(layer)
    torch.cuda.synchronize()
    if pk.kv_get_device_error() != pk.KV_OK:
        raise RuntimeError("device error during warm-up")
    if K is None:  # calibrate: enough steps for min_s seconds of device time
        cal, _, _ = timed_steps(case, 5, flush, stream, clk)
        K = max(5, int(math.ceil(min_s * 1e3 / (sum(cal) / len(cal)))))
    if dist:
        dist.barrier()
    step_ms, dec_ms, clocks = timed_steps(case, K, flush, stream, clk)
    if dist:
        dist.barrier()
    total_ms = max_over_ranks(sum(step_ms), dist, "cuda")
    ms_per_step = total_ms / K
    # end to end through the C ABI with host buffers (pinned), copies timed; a
    # second replica with its own pool alternates with this one when the step
    # has a single layer (see run_e2e); with several layers consecutive
    # decodes already read different pools
    twin = case
    if case.L == 1:
        twin = Case(case.w.name, 0, torch, pk, args, partition=case.partition)
        twin.ws_bytes, twin.ws, twin.split = case.ws_bytes, case.ws, case.split
    K_e2e = K if min_s is None else max(K, 5)
    e2e = run_e2e(case, twin, torch, stream, K_e2e, W, clk)
    if twin is not case:
        twin.destroy()
    del twin
    e2e_ms = max_over_ranks(e2e["ms_per_step"] * K_e2e, dist, "cuda") / K_e2e
    e2e["ms_per_step"] = round(e2e_ms, 5)
    e2e["value"] = round(job_value(case.step_bytes, world, e2e_ms), 2)
    e2e["steps"] = K_e2e
    if pk.kv_get_device_error() != pk.KV_OK:
        raise RuntimeError("device error during timing")
    peak, _ = hbm_peak()
    value = job_value(case.step_bytes, world, ms_per_step)
    return {
        "value": round(value, 2),
        "unit": "GB/s",
        "steps": K,
        "ms_per_step": round(ms_per_step, 5),
        "timed_device_s": round(total_ms / 1e3, 4),
        "seqs_per_s": round(world * case.w.batch / (ms_per_step * 1e-3), 1),
        "pct_of_hbm_peak": round(100.0 * value / world / peak, 2),
        "roofline": decode_roofline(case, dec_ms, key or case.w.name),
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": case.launches_per_step * K,
        "split_k": {"partitions": case.num_parts, "partition_tokens": case.partition or "auto"},
    }


def run_ours(args, rank, world, local_rank):
    import torch
    import paged_kv_cache_451_b200 as pk

    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    clk = ClockSampler(local_rank).start()
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()
    case = Case(args.workload, rank, torch, pk, args, layers=args.layers)
    key = args.workload if args.layers is None else f"{args.workload}_layers{args.layers}"
    m = measure_decode(case, args, stream, flush, clk, dist, world, K=args.steps, key=key)
    w = case.w
    line = {
        "metric": METRIC,
        "value": m["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_NAME[w.kv_fmt],
        "data": "synthetic (seeded N(0,1) q/K/V drawn on device; seeded lengths and scattered block placement)",
        "config": {
            "workload": describe(w, case),
            "global_batch": w.batch * world,
            "layers_per_step": case.L,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": L2_NOTE,
            "split_k": bool(case.split),
            "order": case.order_name,
        },
        "seqs_per_s": m["seqs_per_s"],
        "pct_of_hbm_peak": m["pct_of_hbm_peak"],
        "hbm_peak_gbs": hbm_peak()[0],
        "hbm_peak_kind": hbm_peak()[1],
        "roofline": m["roofline"],
        "e2e": m["e2e"],
        "clocks": m["clocks"],
        "gpu_launches": m["gpu_launches"],
    }
    # the same step repeated for at least a second, for a sustained figure
    # and a clock record over a long region
    if not args.no_extras:
        K_s = max(args.steps, int(math.ceil(MIN_TIMED_S * 1e3 / m["ms_per_step"])))
        if dist:
            dist.barrier()
        step_ms, _, clocks = timed_steps(case, K_s, flush, stream, clk)
        if dist:
            dist.barrier()
        tot = max_over_ranks(sum(step_ms), dist, "cuda")
        line["sustained"] = {"steps": K_s, "ms_per_step": round(tot / K_s, 5),
                             "value": round(job_value(case.step_bytes, world, tot / K_s), 2),
                             "timed_device_s": round(tot / 1e3, 3), "clocks": clocks}
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, target_s=args.cpu_seconds, check=True)
    case.destroy()
    del case
    torch.cuda.empty_cache()
    if not args.no_extras:
        sr = stream_rooflines(torch, stream)
        sr["decode_frac_of_read"] = round(m["roofline"]["achieved"] / sr["read_gbs"], 4)
        sr["decode_frac_of_copy"] = round(m["roofline"]["achieved"] / sr["copy_gbs"], 4)
        line["stream_rooflines"] = sr
    if world == 1 and not args.no_extras and args.workload == "kv_example":
        line["per_config"] = per_config(args, torch, pk, stream, flush, clk)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    clk.stop()
    return line


def per_config(args, torch, pk, stream, flush, clk):
    """The other measured decode workloads, each timed for at least
    MIN_TIMED_S seconds of device time, with its own roofline, end-to-end
    figure, clock record and (CPU-baseline leg) sampled oracle check."""
    res = {}
    for name, label, part in (("llama13b", "llama13b", None), ("fp8_long", "fp8_long", None),
                              ("fp8_long", "fp8_long_partition512", 512), ("window_long", "window_long", None)):
        case = Case(name, 0, torch, pk, args, partition=part or 0)
        m = measure_decode(case, args, stream, flush, clk, None, 1, min_s=MIN_TIMED_S, key=label)
        m["workload"] = describe(case.w, case)
        if not args.no_cpu_baseline:
            m["oracle_check"] = cpu_baseline(case, target_s=0.0, check=True)["check"]
        case.destroy()
        del case
        torch.cuda.empty_cache()
        res[label] = m
    res["gqa_trace"] = trace_measure(args, 0, 1, 0, None, clk, flush, stream, min_s=MIN_TIMED_S)
    # the multi-token workloads (each timed for MIN_TIMED_S of device work;
    # their end-to-end legs move hundreds of MB over PCIe per step, so 50
    # steps) and the two serving traces (their own iteration counts)
    import argparse
    base = {**vars(args), "no_cpu_baseline": True, "shared_prefix": False}
    for wl in PREFILL_WORKLOADS:
        res[wl] = run_prefill(argparse.Namespace(**{**base, "workload": wl, "steps": 20, "min_s": MIN_TIMED_S,
                                                    "e2e_steps": 50}), 0, 1, 0)
        torch.cuda.empty_cache()
    res["rag_trace"] = run_rag(argparse.Namespace(**{**base, "workload": "rag_trace", "steps": 50}), 0, 1, 0)
    torch.cuda.empty_cache()
    res["preempt_trace"] = run_preempt(argparse.Namespace(**{**base, "workload": "preempt_trace", "steps": 50}),
                                       0, 1, 0)
    torch.cuda.empty_cache()
    return res


def unique_and_logical_tokens(tables, lens, block_size):
    """Token slots the decode reads: counted once per physical block (unique,
    what DRAM must deliver when shared blocks hit in L2) and once per
    sequence (logical)."""
    best = {}
    logical = 0
    for row, n in zip(tables, lens):
        n = int(n)
        logical += n
        for j in range(-(-n // block_size)):
            b = int(row[j])
            best[b] = max(best.get(b, 0), min(block_size, n - j * block_size))
    return sum(best.values()), logical


def trace_measure(args, rank, world, local_rank, dist, clk, flush, stream, min_s=None, shared_prefix=None):
    """The GQA continuous-batching trace: one step = one trace iteration
    (native scheduler step, metadata upload, copy-on-write block copies,
    cache write, decode).  The trace's iterations after the warm-up are
    timed; with min_s the trace is replayed (same seed, a fresh pool each
    pass) until the timed regions span at least min_s seconds."""
    import torch
    import paged_kv_cache_451_b200 as pk
    from workloads import WORKLOADS, gqa_trace_plan
    from workloads.gqa_trace import GqaTrace

    w = WORKLOADS["gqa_trace"]
    plan = gqa_trace_plan(w)
    if shared_prefix is None:
        shared_prefix = args.shared_prefix
    iters = w.extra["iters"]
    W = min(args.warmup, iters - 1)
    K = max(1, min(args.steps, iters - W)) if min_s is None else iters - W
    hq, hkv, d = w.num_q_heads, w.kv_heads, w.head_dim
    per_tok = hkv * d * 2 * 2
    tot_ms = dec_ms = 0.0
    uniq_b = logi_b = other_b = dec_b = 0
    launches = steps = 0
    host_s = sched_s = 0.0
    regions = []
    passes = 0
    while True:
        tr = GqaTrace(w, plan, seed=rank, decode_config=(args.partition, args.stages, args.warps),
                      order_policy=args.order or "batch", shared_prefix=shared_prefix)
        for it in range(W):
            flush.zero_()
            tr.iteration(it, out_dtype=w.q_fmt)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        mids = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

        def gate_and_start(i):
            # keep the GPU busy (~1 ms device sleep) while the host enqueues
            # the iteration, so the timed interval is the fed-GPU time of the step
            torch.cuda._sleep(2_000_000)
            starts[i].record(stream)

        t0 = time.perf_counter()
        for i in range(K):
            flush.zero_()
            h0 = time.perf_counter()
            fin, arr, pl, q, kn, vn, out = tr.iteration(W + i, out_dtype=w.q_fmt,
                                                        before_launch=lambda: gate_and_start(i),
                                                        after_launch=lambda: ends[i].record(stream),
                                                        before_decode=lambda s: mids[i].record(s))
            host_s += time.perf_counter() - h0
            sched_s += tr.last_schedule_s
            info = pl["info"]
            u, l = unique_and_logical_tokens(pl["block_tables"], pl["context_lens"], w.block_size)
            uniq_b += u * per_tok
            logi_b += l * per_tok
            qo = info.batch * hq * d * 4
            dec_b += u * per_tok + qo
            other_b += (qo + info.num_tokens * hkv * d * 2 * 4
                        + info.num_cow * hkv * w.block_size * d * 2 * 2 * 2)
            launches += 2 + (1 if info.num_cow else 0)
        torch.cuda.synchronize()
        t1 = time.perf_counter()
        regions.append((t0, t1))
        if pk.kv_get_device_error() != pk.KV_OK:
            raise RuntimeError("device error during the trace")
        tot_ms += sum(starts[i].elapsed_time(ends[i]) for i in range(K))
        dec_ms += sum(mids[i].elapsed_time(ends[i]) for i in range(K))
        steps += K
        passes += 1
        del tr
        if min_s is None or sum(b - a for a, b in regions) >= min_s or passes >= 8:
            break
    total_ms = max_over_ranks(tot_ms, dist, "cuda")
    ms = total_ms / steps
    e2e = trace_e2e(args, rank, w, plan, W, K, stream, clk, uniq_b, other_b, steps, dist, world, shared_prefix)
    peak, peak_kind = hbm_peak()
    value = world * (uniq_b + other_b) / (total_ms * 1e-3) / 1e9
    logical = world * (logi_b + other_b) / (total_ms * 1e-3) / 1e9
    achieved = dec_b / (dec_ms * 1e-3) / 1e9
    # clocks over every pass's timed region
    samples = [s for a, b in regions for s in clk.samples if a <= s[0] <= b]
    clocks = clk.summary(regions[0][0], regions[-1][1]) if samples else clk.summary(0, -1)
    if samples:
        clocks["samples"] = len(samples)
        clocks["sm_mhz"] = statistics.median(s[1] for s in samples)
        clocks["region_s"] = round(sum(b - a for a, b in regions), 3)
    return {
        "value": round(value, 2), "unit": "GB/s", "steps": steps, "passes": passes, "warmup": W,
        "ms_per_step": round(ms, 5), "timed_device_s": round(total_ms / 1e3, 4),
        "workload": describe(w),
        "logical_gbs": round(logical, 2),
        "unique_bytes_per_step": int((uniq_b + other_b) / steps),
        "logical_bytes_per_step": int((logi_b + other_b) / steps),
        "host_scheduler_ms_per_step": round(1e3 * sched_s / steps, 3),
        "host_iteration_ms_per_step": round(1e3 * host_s / steps, 3),
        "pct_of_hbm_peak": round(100.0 * value / world / peak, 2),
        "roofline": {
            "bound": "hbm", "kernel": "paged_attention_decode (decode kernel; split partials merged in it)",
            "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": committed_traffic("gqa_trace"),
            "algorithmic_bytes_per_launch": int(dec_b / steps),
            "launch_ms": round(dec_ms / steps, 5),
            "bytes_note": "unique physical K/V bytes (shared prefix blocks counted once) + q + out",
            "peak_note": f"{peak_kind} copy bandwidth"},
        "clocks": clocks, "gpu_launches": launches, "e2e": e2e,
        "step": "one trace iteration: native scheduler step, metadata upload, copy-on-write block copies, "
                "cache write, decode" + (" (shared-prefix decode: the sharers' common blocks once per kv head "
                                         "on the tensor cores, merged with each sequence's own tokens)"
                                         if shared_prefix else ""),
        "shared_prefix_decode": bool(shared_prefix),
    }


def trace_e2e(args, rank, w, plan, W, K, stream, clk, uniq_b, other_b, steps, dist, world, shared_prefix):
    """The trace end to end from host buffers, run back to back as a serving
    loop runs it (no device-side gate): each iteration takes the library's
    serving step (kv_serve_schedule: scheduler step, metadata packed into a
    pinned buffer and uploaded; kv_serve_launch: copy-on-write, cache write,
    decode), uploads its queries and new K/V rows from one pinned host
    staging buffer with one copy on an upload stream into one of the loop's
    three device buffer sets (so uploads overlap the earlier iterations' kernels),
    and its output is read back on a read-back stream (overlapping the next
    iteration); the K iterations are timed as one region, host scheduling
    included.  Bytes per step are the device-timed run's."""
    import torch
    from workloads.gqa_trace import GqaTrace
    e = w.extra
    hq, hkv, d = w.num_q_heads, w.kv_heads, w.head_dim
    native = not shared_prefix  # the library's serving step has no shared-prefix decode
    tr = GqaTrace(w, plan, seed=rank, decode_config=(args.partition, args.stages, args.warps),
                  order_policy=args.order or "batch", shared_prefix=shared_prefix, native=native)
    max_b, max_t = e["max_num_seqs"], tr.loop.max_tokens
    g = torch.Generator().manual_seed(w.seed * 31 + rank)
    # one staging buffer per step: q rows, then new K rows, then new V rows
    n_max = (max_b * hq + 2 * max_t * hkv) * d
    host = torch.randn(n_max, generator=g).to(torch.bfloat16).view(torch.int16).pin_memory()
    nsets = tr.loop.num_sets if native else 2  # the caller's input / output sets follow the loop's
    devb = [torch.empty_like(host, device="cuda") for _ in range(nsets)]
    outs = [torch.empty((max_b, hq, d), dtype=torch.bfloat16, device="cuda") for _ in range(nsets)]
    hout = torch.empty(max_b * hq * d, dtype=torch.bfloat16).pin_memory()
    up, rb = torch.cuda.Stream(), torch.cuda.Stream()
    up_done = [torch.cuda.Event(), torch.cuda.Event()]    # inputs of buffer set k uploaded
    kern_done = [torch.cuda.Event(), torch.cuda.Event()]  # kernels reading buffer set k finished
    rb_done = [torch.cuda.Event(), torch.cuda.Event()]    # read-back of output k finished
    used = [False, False]
    moved = {"h2d": 0, "d2h": 0}
    cur = {"k": 0}

    def inputs(T, B):
        k, main = cur["k"], stream  # the loop's stream: the current one
        nq, nk = B * hq * d, T * hkv * d
        if used[k]:  # the kernels that read this set two iterations ago
            up.wait_event(kern_done[k])
        with torch.cuda.stream(up):
            devb[k][:nq + 2 * nk].copy_(host[:nq + 2 * nk], non_blocking=True)
        up_done[k].record(up)
        moved["h2d"] += 2 * (nq + 2 * nk)
        main.wait_event(up_done[k])
        if used[k]:  # this set's output was read back
            main.wait_event(rb_done[k])
        buf = devb[k]
        return (buf[:nq].view(B, hq, d), buf[nq:nq + nk].view(T, hkv, d),
                buf[nq + nk:nq + 2 * nk].view(T, hkv, d))

    def one(it):
        k = cur["k"] = it % 2
        fin, arr, pl, *_r = tr.iteration(it, out_dtype=w.q_fmt, inputs=inputs, out=outs[k], stream=stream)
        kern_done[k].record(stream)
        n = max(pl["info"].batch, 1) * hq * d
        rb.wait_event(kern_done[k])
        with torch.cuda.stream(rb):
            hout[:n].copy_(outs[k].view(-1)[:n], non_blocking=True)
        rb_done[k].record(rb)
        used[k] = True
        moved["d2h"] += 2 * n

    if native:
        # the library orders the staging copies: kv_serve_upload on the
        # loop's upload stream into buffer set layout.buffer (the step's
        # parity), kv_serve_readback on the read-back stream
        loop = tr.loop
        hb, hob = host.data_ptr(), hout.data_ptr()
        dbase, obase = [t.data_ptr() for t in devb], [t.data_ptr() for t in outs]

        def inputs(T, B):  # noqa: F811
            k = loop.layout.buffer
            nq, nk = B * hq * d, T * hkv * d
            loop.upload(dbase[k], hb, 2 * (nq + 2 * nk))
            moved["h2d"] += 2 * (nq + 2 * nk) + loop.layout.bytes
            return dbase[k], dbase[k] + 2 * nq, dbase[k] + 2 * (nq + nk)

        def one(it):  # noqa: F811
            k = it % nsets
            fin, arr, pl, *_r = tr.iteration(it, out_dtype=w.q_fmt, inputs=inputs, out=obase[k], stream=stream)
            assert pl["layout"].buffer == k
            n = max(pl["info"].batch, 1) * hq * d
            loop.readback(hob, obase[k], 2 * n, rb)
            moved["d2h"] += 2 * n

    for it in range(W):
        one(it)
    torch.cuda.synchronize()
    moved["h2d"] = moved["d2h"] = 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record(stream)
    for i in range(K):
        one(W + i)
    last = torch.cuda.Event()
    last.record(rb)  # every read-back ran on rb: the last one is inside the region
    stream.wait_event(last)
    b.record(stream)
    torch.cuda.synchronize()
    span = (t0, time.perf_counter())
    ms = max_over_ranks(a.elapsed_time(b), dist, "cuda") / K
    timeline = serving_timeline(tr, one, W + K, 60) if native and getattr(args, "timeline", False) else None
    if native:
        tr.loop.close()
    del tr
    return {**({"timeline": timeline} if timeline else {}),
            "value": round(world * (uniq_b + other_b) / steps / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 5), "steps": K, "h2d_bytes_per_step": int(moved["h2d"] / K),
            "d2h_bytes_per_step": int(moved["d2h"] / K),
            "mode": ("serving loop from host memory, pipelined: per iteration the library's serving step "
                     f"(kv_serve_schedule: native scheduler step, metadata packed in a pinned buffer and uploaded; "
                     f"kv_serve_launch: copy-on-write, cache write, decode), one upload of the step's q and new "
                     f"K/V rows from a pinned staging buffer (kv_serve_upload) into one of {nsets} device buffer "
                     f"sets used in turn, and the output read back on a read-back stream (kv_serve_readback); K "
                     f"iterations timed as one region (host scheduling included); h2d counts the packed "
                     f"metadata too" if native else
                     "serving loop from host memory, pipelined: per iteration the Python serving loop with the "
                     "shared-prefix decode, one upload of the step's q and new K/V rows from a pinned staging "
                     "buffer on an upload stream into one of two device buffer sets, and the output read back "
                     "on a read-back stream; K iterations timed as one region (host scheduling included)"),
            "serving_step": "native" if native else "python",
            "clocks": clk.summary(*span)}


def serving_timeline(tr, one, it0, n):
    """After the timed region (never inside it): n more iterations of the
    end-to-end loop with timing events around each input upload on the
    loop's upload stream, and host clocks around the library's scheduling
    step, to show what bounds the loop (the PCIe upload or the host)."""
    import torch
    n = min(n, len(tr.plan["arrivals"]) - it0)  # the trace's iterations left after the timed region
    if n < 8:
        return {"skipped": f"only {max(n, 0)} trace iterations left after the timed region"}
    loop = tr.loop
    ev, host = [], {"schedule": 0.0, "total": 0.0, "bytes": 0}
    sched, upload = loop.schedule, loop.upload

    def timed_schedule(fin):
        t0 = time.perf_counter()
        r = sched(fin)
        host["schedule"] += time.perf_counter() - t0
        return r

    def timed_upload(dst, src, nbytes):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(loop.up)
        upload(dst, src, nbytes)
        b.record(loop.up)
        ev.append((a, b))
        host["bytes"] += nbytes

    loop.schedule, loop.upload = timed_schedule, timed_upload
    try:
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(n):
            one(it0 + i)
        torch.cuda.synchronize()
        host["total"] = time.perf_counter() - t0
    finally:
        del loop.schedule, loop.upload  # back to the class methods
    start = ev[0][0]
    u0 = [start.elapsed_time(a) for a, _ in ev]
    u1 = [start.elapsed_time(b) for _, b in ev]
    busy = sum(y - x for x, y in zip(u0, u1))
    period = (u1[-1] - u1[0]) / (len(ev) - 1)
    return {"iterations": n, "period_ms": round(period, 4),
            "input_upload_ms": round(busy / len(ev), 4),
            "input_upload_gbs": round(host["bytes"] / (busy * 1e-3) / 1e9, 1),
            "input_upload_busy_frac": round(busy / (u1[-1] - u0[0]), 3),
            "host_ms_per_iteration": round(host["total"] * 1e3 / n, 4),
            "host_in_schedule_ms": round(host["schedule"] * 1e3 / n, 4),
            "buffer_sets": loop.num_sets,
            "note": "a separate pass after the timed region; the schedule call includes its wait for the "
                    "uploads of the step that last used its buffer set"}


def run_trace(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    clk = ClockSampler(local_rank).start()
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()
    m = trace_measure(args, rank, world, local_rank, dist, clk, flush, stream)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    clk.stop()
    line = {
        "metric": METRIC, "value": m["value"], "unit": "GB/s", "n_gpus": world, "steps": m["steps"],
        "warmup": m["warmup"], "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded lognormal lengths, shared prefix, Poisson arrivals; q/K/V drawn on device)",
        "config": {"workload": m["workload"], "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": L2_NOTE.replace("steps", "iterations"), "step": m["step"]},
    }
    for k in ("logical_gbs", "unique_bytes_per_step", "logical_bytes_per_step", "host_scheduler_ms_per_step",
              "host_iteration_ms_per_step", "pct_of_hbm_peak", "roofline", "e2e", "clocks", "gpu_launches",
              "shared_prefix_decode"):
        line[k] = m[k]
    line["hbm_peak_gbs"], line["hbm_peak_kind"] = hbm_peak()
    return line


def run_rag(args, rank, world, local_rank):
    """The retrieval-augmented trace, with and without prefix caching: one
    step = one iteration (scheduler step, metadata upload, cache write,
    prefill of the admitted prompts' uncached tokens, decode)."""
    import torch
    import paged_kv_cache_451_b200 as pk
    from workloads import WORKLOADS
    from workloads.rag_trace import RagTrace, rag_plan

    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    clk = ClockSampler(local_rank).start()
    w = WORKLOADS["rag_trace"]
    plan = rag_plan(w)
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()
    iters = w.extra["iters"]
    W = min(args.warmup, iters - 1)
    K = max(1, min(args.steps, iters - W))
    res = {}
    for caching in (True, False):
        tr = RagTrace(w, plan, caching=caching, seed=rank, shared_prefix=args.shared_prefix and caching)
        for it in range(W):
            tr.iteration(it)
        torch.cuda.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        gen = prefilled = cached = admitted = 0
        host_s = 0.0

        def gate_and_start(i):
            torch.cuda._sleep(2_000_000)  # keep the GPU fed while the host enqueues
            starts[i].record(stream)

        r0 = time.perf_counter()
        for i in range(K):
            flush.zero_()
            t0 = time.perf_counter()
            fin, arr, pl, *_rest, P = tr.iteration(W + i, before_launch=lambda: gate_and_start(i),
                                                   after_launch=lambda: ends[i].record(stream))
            host_s += time.perf_counter() - t0
            gen += pl["info"].batch
            prefilled += P
            cached += int(np.sum(pl["cached"]))
            admitted += pl["info"].num_admitted
        torch.cuda.synchronize()
        clocks = clk.summary(r0, time.perf_counter())
        if pk.kv_get_device_error() != pk.KV_OK:
            raise RuntimeError("device error during the trace")
        total_ms = max_over_ranks(sum(starts[i].elapsed_time(ends[i]) for i in range(K)), dist, "cuda")
        hits, evictions, nblocks = pk.kv_alloc_prefix_stats(tr.alloc)
        res[caching] = {"tokens_per_s": world * gen / (total_ms * 1e-3), "ms_per_step": total_ms / K,
                        "generated": gen, "prefilled_tokens": prefilled, "cached_tokens": cached,
                        "admitted": admitted, "host_ms_per_step": 1e3 * host_s / K, "clocks": clocks,
                        "hit_blocks": hits, "evictions": evictions}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    clk.stop()
    on, off = res[True], res[False]
    return {
        "metric": METRIC_RAG, "value": round(on["tokens_per_s"], 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(on["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded documents, questions and Poisson arrivals; q/K/V drawn on device)",
        "config": {"workload": describe(w), "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": L2_NOTE.replace("steps", "iterations"),
                   "step": "one iteration: scheduler step (prefix lookup), metadata upload, cache write, "
                           "prefill of uncached prompt tokens, decode of every running sequence"},
        "no_caching": {"tokens_per_s": round(off["tokens_per_s"], 1), "ms_per_step": round(off["ms_per_step"], 5),
                       "prefilled_tokens": off["prefilled_tokens"], "admitted": off["admitted"]},
        "speedup_vs_no_caching": round(on["tokens_per_s"] / off["tokens_per_s"], 3),
        "prefilled_tokens": on["prefilled_tokens"], "cached_tokens": on["cached_tokens"],
        "admitted": on["admitted"], "hit_blocks": on["hit_blocks"], "evictions": on["evictions"],
        "host_iteration_ms_per_step": round(on["host_ms_per_step"], 3),
        "clocks": on["clocks"],
    }


def swap_copy_bandwidth(torch, pk, blocks=1024):
    """kv_swap_out / kv_swap_in of `blocks` blocks (GQA 8 heads, bf16, block
    16, head_dim 128) against a plain pinned-host cudaMemcpyAsync of the same
    bytes in each direction (the copy-engine reference), CUDA events."""
    nb, hkv, bs, d = blocks * 2, 8, 16, 128
    pool = pk.kv_pool_create(bs, nb, hkv, d, pk.KV_BF16, 1)
    k = torch.zeros((nb, hkv, bs, d), dtype=torch.int16, device="cuda")
    v = torch.zeros_like(k)
    pk.kv_pool_bind(pool, 0, k, v)
    slot = pk.kv_swap_block_bytes(pool)
    host = torch.zeros(blocks * slot, dtype=torch.uint8).pin_memory()
    dev_buf = torch.zeros(blocks * slot, dtype=torch.uint8, device="cuda")
    out_pairs = torch.stack([torch.arange(0, nb, 2), torch.arange(blocks)], 1).to(torch.int32).cuda()
    in_pairs = torch.stack([torch.arange(blocks), torch.arange(1, nb, 2)], 1).to(torch.int32).cuda()
    res = {}

    def timed(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    nbytes = blocks * slot
    res["swap_out_gbs"] = nbytes / (timed(lambda: pk.kv_swap_out(pool, host, blocks, out_pairs, blocks)) * 1e-3) / 1e9
    res["swap_in_gbs"] = nbytes / (timed(lambda: pk.kv_swap_in(pool, host, blocks, in_pairs, blocks)) * 1e-3) / 1e9
    res["memcpy_d2h_gbs"] = nbytes / (timed(lambda: host.copy_(dev_buf, non_blocking=True)) * 1e-3) / 1e9
    res["memcpy_h2d_gbs"] = nbytes / (timed(lambda: dev_buf.copy_(host, non_blocking=True)) * 1e-3) / 1e9
    res["bytes_per_call"] = nbytes
    if pk.kv_get_device_error() != pk.KV_OK:
        raise RuntimeError("device error in the swap copies")
    pk.kv_pool_destroy(pool)
    return {k2: (round(v2, 2) if isinstance(v2, float) else v2) for k2, v2 in res.items()}


def run_preempt(args, rank, world, local_rank):
    """The memory-pressure trace with swap and with recompute preemption: one
    step = one iteration (scheduler step, metadata upload, swap copies,
    copy-on-write, cache write, decode)."""
    import torch
    import paged_kv_cache_451_b200 as pk
    from workloads import WORKLOADS
    from workloads.preempt_trace import PreemptTrace, preempt_plan

    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    clk = ClockSampler(local_rank).start()
    w = WORKLOADS["preempt_trace"]
    plan = preempt_plan(w)
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()
    iters = w.extra["iters"]
    W = min(args.warmup, iters - 1)
    K = max(1, min(args.steps, iters - W))
    res = {}
    for mode in ("swap", "recompute"):
        tr = PreemptTrace(w, plan, mode=mode, seed=rank)
        for it in range(W):
            tr.iteration(it)
        torch.cuda.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        gen = pre = rec = swapped_blocks = rewritten = 0

        def gate_and_start(i):
            torch.cuda._sleep(2_000_000)  # keep the GPU fed while the host enqueues
            starts[i].record(stream)

        r0 = time.perf_counter()
        for i in range(K):
            flush.zero_()
            fin, arr, pl, *_ = tr.iteration(W + i, before_launch=lambda: gate_and_start(i),
                                           after_launch=lambda: ends[i].record(stream))
            gen += pl["info"].batch
            pre += len(pl["preempted"])
            rec += len(pl["recomputed"])
            swapped_blocks += len(pl["swap_out"]) + len(pl["swap_in"])
            rewritten += pl["info"].num_tokens
        torch.cuda.synchronize()
        clocks = clk.summary(r0, time.perf_counter())
        if pk.kv_get_device_error() != pk.KV_OK:
            raise RuntimeError("device error during the trace")
        total_ms = max_over_ranks(sum(starts[i].elapsed_time(ends[i]) for i in range(K)), dist, "cuda")
        res[mode] = {"tokens_per_s": world * gen / (total_ms * 1e-3), "ms_per_step": total_ms / K,
                     "preempted": pre, "recomputed": rec, "swapped_blocks": swapped_blocks,
                     "written_tokens": rewritten, "clocks": clocks}
    swap_bw = swap_copy_bandwidth(torch, pk) if rank == 0 else None
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    clk.stop()
    sw, rc = res["swap"], res["recompute"]
    return {
        "metric": METRIC_PREEMPT, "value": round(sw["tokens_per_s"], 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(sw["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded prompt / output lengths and Poisson arrivals; q/K/V drawn on device)",
        "config": {"workload": describe(w), "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": L2_NOTE.replace("steps", "iterations"),
                   "step": "one iteration: scheduler step (preemption, swap-in), metadata upload, swap copies, "
                           "copy-on-write, cache write, decode"},
        "swap": {k2: (round(v2, 3) if isinstance(v2, float) else v2) for k2, v2 in sw.items() if k2 != "clocks"},
        "recompute": {k2: (round(v2, 3) if isinstance(v2, float) else v2) for k2, v2 in rc.items() if k2 != "clocks"},
        "swap_copy": swap_bw,
        "roofline": None if swap_bw is None else {
            "bound": "host link", "kernel": "kv_swap_out (swap_kernel, device to pinned host)",
            "achieved": swap_bw["swap_out_gbs"], "peak": swap_bw["memcpy_d2h_gbs"], "unit": "GB/s",
            "frac": round(swap_bw["swap_out_gbs"] / swap_bw["memcpy_d2h_gbs"], 4), "traffic": None,
            "peak_note": "pinned cudaMemcpyAsync device-to-host of the same bytes, measured in this run"},
        "clocks": sw["clocks"],
    }


def describe(w, case=None):
    names = {
        "tiny": "tiny: 1 layer, 4 seqs ctx {2,18,34,101}, 4 MHA heads, head_dim 64, block 16, fp16",
        "llama13b": "Llama-2-13B-shaped layer: 40 MHA heads, head_dim 128, block 16, fp16, batch 64, ctx U[128,2048]",
        "kv_example": "KV-size example: 32 layers x 32 heads x head_dim 128, bf16, block 16, batch 32, ctx 2048",
        "gqa_trace": "GQA 64/8 heads, head_dim 128, bf16, block 16, batch 256, lognormal ctx (median 1024, cap 8192)",
        "fp8_long": "long-context FP8: 32 MHA heads, head_dim 128, E4M3 cache + per-(block,head) scales, bf16 q, batch 8, ctx 16384",
        "window_long": "sliding-window decode: 32 MHA heads, head_dim 128, bf16, batch 8, ctx 16384, window 4096 "
                       "(bytes counted over the window)",
        "preempt_trace": "decode under memory pressure: GQA 64/8 heads, head_dim 128, bf16, block 16, 3000-block pool, "
                         "64 initial sequences (prompts U[256,1024]) + Poisson arrivals (0.5/iteration), U[100,400] "
                         "output tokens, swap space 6000 host blocks",
        "rag_trace": "retrieval-augmented serving: GQA 64/8 heads, head_dim 128, bf16, block 16, 8192-block pool, "
                     "Poisson arrivals (3/iteration) of 2 shared 1536-token documents + U[32,256]-token questions, "
                     "U[16,64] output tokens, up to 128 running",
    }
    s = names[w.name]
    if case is not None:
        s += f"; pool {case.nb} blocks; sum ctx {int(case.lens.sum())}"
    return s


def pipelined_e2e(torch, stream, ins, outs, launch, K, W):
    """Time K steps of a serving-style loop from pinned host memory: each
    step's inputs (the device tensors `ins`, copied once to the host) are
    packed in one pinned buffer and uploaded with one copy on an upload
    stream into one of two device buffers; `launch(views, outs_k)` enqueues
    the step's kernels on `stream` over those views, writing per-buffer
    copies of `outs`; the outputs go back to pinned host memory on a
    read-back stream.  The upload of step i + 1 overlaps the kernels of step
    i, and the read-back of step i the kernels of step i + 1.  The K steps
    are timed as one region (CUDA events on `stream`, every copy inside).
    `launch(k, views, outs)` also gets the buffer index k (0 or 1).
    Returns (ms per step, H2D bytes per step, D2H bytes per step, host
    time span of the timed region)."""
    offs, off = [], 0
    for t in ins:
        offs.append(off)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    h2d = sum(t.numel() * t.element_size() for t in ins)
    hbuf = torch.empty(off, dtype=torch.uint8).pin_memory()
    for t, o in zip(ins, offs):
        n = t.numel() * t.element_size()
        hbuf[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8).cpu())
    dbuf = [torch.empty(off, dtype=torch.uint8, device="cuda") for _ in range(2)]
    views = [[dbuf[k][o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
              for t, o in zip(ins, offs)] for k in range(2)]
    dout = [[torch.empty_like(o) for o in outs] for _ in range(2)]
    hout = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs] for _ in range(2)]
    d2h = sum(o.numel() * o.element_size() for o in outs)
    cs_up, cs_dn = torch.cuda.Stream(), torch.cuda.Stream()
    up = [torch.cuda.Event() for _ in range(2)]
    comp = [None, None]   # kernels that read device buffer k (and wrote dout[k])
    down = [None, None]   # read-back of dout[k]

    def step(i):
        k = i % 2
        with torch.cuda.stream(cs_up):
            if comp[k] is not None:
                cs_up.wait_event(comp[k])  # buffer k's previous readers are done
            dbuf[k].copy_(hbuf, non_blocking=True)
            up[k].record(cs_up)
        stream.wait_event(up[k])
        if down[k] is not None:
            stream.wait_event(down[k])  # dout[k] was read back
        launch(k, views[k], dout[k])
        ev = torch.cuda.Event()
        ev.record(stream)
        comp[k] = ev
        with torch.cuda.stream(cs_dn):
            cs_dn.wait_event(ev)
            for h, d in zip(hout[k], dout[k]):
                h.copy_(d, non_blocking=True)
            dn = torch.cuda.Event()
            dn.record(cs_dn)
            down[k] = dn

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    cs_up.wait_event(a)  # the first upload starts inside the region
    for i in range(K):
        step(W + i)
    stream.wait_event(down[(W + K - 1) % 2])  # the last read-back is inside the region
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / K, h2d, d2h, (t0, time.perf_counter())


PIPELINE_MODE = ("pipelined: one packed upload per step on an upload stream (double-buffered), "
                 "read-back of every step's output on a read-back stream; K steps timed as one region")


def run_e2e(case, twin, torch, stream, K, W, clk):
    """The decode step through the C ABI from pinned host memory, pipelined
    the way a serving loop runs it (pipelined_e2e): inputs are q, the new
    K/V of every layer, slots, tables, lengths and order.  Consecutive steps
    alternate between `case` and `twin`, a replica with its own pool memory
    (the same inputs address it): in a model, consecutive decode calls read
    different layers' pools, and each step reads more than L2 holds, so
    nothing one step leaves in L2 serves the next and no flush is needed in
    between."""
    L = case.L
    ins = list(case.q) + list(case.kn) + list(case.vn) + [case.slots, case.tables_d, case.lens_d, case.order_d]
    cases = (case, twin)

    def launch(k, v, outs):
        c = cases[k]
        for layer in range(L):
            c.write(layer, v[L + layer], v[2 * L + layer], v[3 * L])
            c.decode(layer, v[layer], v[3 * L + 1], v[3 * L + 2], out=outs[layer], order=v[3 * L + 3])

    ms, h2d, d2h, span = pipelined_e2e(torch, stream, ins, list(case.out), launch, K, W)
    return {"value": round(case.step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "mode": PIPELINE_MODE, "clocks": clk.summary(*span)}


# ------------------------------------------------------ multi-token leg

class PrefillCase:
    """Device-resident inputs of a multi-token workload: a pool with every
    sequence's cached prefix, the new tokens' K/V and slots, their queries.
    With pk None (the reference arm) the inputs are drawn with torch alone
    and no pool of the product library is created."""

    def __init__(self, name, rank, torch, pk):
        from workloads import (WORKLOADS, device_normal_bits, device_pool, pool_blocks,
                               prefill_lens, scattered_tables)
        w = WORKLOADS[name]
        self.w, self.torch, self.pk = w, torch, pk
        self.prior, self.new = prefill_lens(w)
        self.lens = (self.prior + self.new).astype(np.int32)
        self.nb = pool_blocks(w, self.lens)
        rng = np.random.default_rng([w.seed, 1000 + rank])
        self.tables = scattered_tables(rng, self.lens, w.block_size, self.nb)
        dev = torch.device("cuda")
        seed = w.seed * 7919 + rank
        self.L = 1
        k, v, _, _ = device_pool(w, self.nb, dev, seed=seed)
        self.k, self.v = [k], [v]
        self.pool = None
        if pk is not None:
            self.pool = pk.kv_pool_create(w.block_size, self.nb, w.kv_heads, w.head_dim, w.kv_fmt, 1)
            pk.kv_pool_bind(self.pool, 0, k, v, None, None)
        T, Hq, Hkv, D = int(self.new.sum()), w.num_q_heads, w.kv_heads, w.head_dim
        self.T = T
        self.cu_h = np.concatenate([[0], np.cumsum(self.new)]).astype(np.int32)
        self.q = device_normal_bits((T, Hq, D), w.q_fmt, dev, seed + 1)
        self.kn = device_normal_bits((T, Hkv, D), w.q_fmt, dev, seed + 2)
        self.vn = device_normal_bits((T, Hkv, D), w.q_fmt, dev, seed + 3)
        pos = np.concatenate([np.arange(p, p + n) for p, n in zip(self.prior, self.new)]).astype(np.int64)
        seq = np.repeat(np.arange(w.batch), self.new)
        self.slots_h = self.tables[seq, pos // w.block_size].astype(np.int64) * w.block_size + pos % w.block_size
        self.slots = torch.from_numpy(self.slots_h).to(dev)
        self.cu = torch.from_numpy(self.cu_h).to(dev)
        self.tables_d = torch.from_numpy(self.tables).to(dev)
        self.lens_d = torch.from_numpy(self.lens).to(dev)
        self.max_q = int(self.new.max())
        out_dt = torch.float16 if w.q_fmt == 0 else torch.bfloat16
        self.out = torch.empty((T, Hq, D), dtype=out_dt, device=dev)
        # algorithmic work: new token i of s sees prior_s + i + 1 keys; q.K and P.V
        visible = sum(int(p) * int(n) + int(n) * (int(n) + 1) // 2 for p, n in zip(self.prior, self.new))
        self.flops = 4.0 * D * Hq * visible
        e = ELEM[w.q_fmt]
        self.write_bytes = T * Hkv * D * 2 * (e + ELEM[w.kv_fmt])

    def write(self, kn=None, vn=None, slots=None):
        self.pk.paged_kv_write(self.pool, 0, self.kn if kn is None else kn, self.vn if vn is None else vn,
                               self.w.q_fmt, self.slots if slots is None else slots, self.T, None, None)

    def prefill(self, q=None, cu=None, tables=None, lens=None, out=None):
        w = self.w
        self.pk.paged_attention_prefill(self.pool, 0, self.q if q is None else q, w.q_fmt, w.num_q_heads,
                                        self.cu if cu is None else cu, self.T, self.max_q,
                                        self.tables_d if tables is None else tables, self.tables.shape[1],
                                        self.lens_d if lens is None else lens, w.batch, w.scale,
                                        self.out if out is None else out, w.q_fmt)


def describe_prefill(w, case=None):
    names = {
        "prefill_llama13b": "whole prompts, Llama-2-13B-shaped layer: 40 MHA heads, head_dim 128, fp16, "
                            "block 16, 16 prompts of U[64,2048] tokens",
        "prefill_gqa": "whole prompts, GQA 64/8 heads, head_dim 128, bf16, block 16, 16 prompts of U[64,2048] tokens",
        "chunked_gqa": "prompt chunks, GQA 64/8 heads, head_dim 128, bf16, block 16, 16 sequences x 512 new "
                       "tokens on U[512,4096] cached",
    }
    s = names[w.name]
    if case is not None:
        s += f"; {case.T} new tokens; pool {case.nb} blocks"
    return s


def run_prefill(args, rank, world, local_rank):
    import torch
    import paged_kv_cache_451_b200 as pk

    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    clk = ClockSampler(local_rank).start()
    case = PrefillCase(args.workload, rank, torch, pk)
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()

    def step(ev_w=None, ev_p=None):
        case.write()
        if ev_w is not None:
            ev_w.record(stream)
        case.prefill()
        if ev_p is not None:
            ev_p.record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if pk.kv_get_device_error() != pk.KV_OK:
        raise RuntimeError("device error during warm-up")
    K = args.steps
    min_s = getattr(args, "min_s", None)
    if min_s:  # calibrate: enough steps for min_s seconds of device time
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(5):
            flush.zero_()
            step()
        b.record(stream)
        b.synchronize()
        K = max(K, int(math.ceil(min_s * 1e3 / (a.elapsed_time(b) / 5))))
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    evw = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    evp = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    r0 = time.perf_counter()
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        step(evw[i], evp[i])
    torch.cuda.synchronize()
    clocks = clk.summary(r0, time.perf_counter())
    if dist:
        dist.barrier()
    step_ms = [ev0[i].elapsed_time(evp[i]) for i in range(K)]
    pf_ms = [evw[i].elapsed_time(evp[i]) for i in range(K)]
    total_ms = max_over_ranks(sum(step_ms), dist, "cuda")
    ms_per_step = total_ms / K
    pf_avg = sum(pf_ms) / K
    Ke = getattr(args, "e2e_steps", None) or K
    e2e = run_e2e_prefill(case, torch, stream, Ke, args.warmup, clk)
    e2e_ms = max_over_ranks(e2e["ms_per_step"] * Ke, dist, "cuda") / Ke
    e2e["ms_per_step"] = round(e2e_ms, 5)
    e2e["value"] = round(world * case.flops / (e2e_ms * 1e-3) / 1e12, 2)
    if pk.kv_get_device_error() != pk.KV_OK:
        raise RuntimeError("device error during timing")
    sustained = total_ms >= SUSTAINED_MS
    peak, peak_kind = tensor_peak(sustained)
    value = world * case.flops / (ms_per_step * 1e-3) / 1e12
    achieved = case.flops / (pf_avg * 1e-3) / 1e12
    w = case.w
    line = {
        "metric": METRIC_PREFILL,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_NAME[w.kv_fmt],
        "data": "synthetic (seeded N(0,1) q/K/V drawn on device; seeded lengths and scattered block placement)",
        "config": {
            "workload": describe_prefill(w, case),
            "global_batch": w.batch * world,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": L2_NOTE,
        },
        "new_tokens_per_s": round(world * case.T / (ms_per_step * 1e-3), 1),
        "pct_of_tensor_peak": round(100.0 * value / world / peak, 2),
        "roofline": {
            "bound": "tensor",
            "kernel": "paged_attention_prefill",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": committed_traffic(args.workload, prefill_source_hash()),
            "algorithmic_flops_per_launch": case.flops,
            "launch_ms": round(pf_avg, 5),
            "peak_note": f"{peak_kind} dense bf16 GEMM ("
                         + ("sustained: the timed region is a long loop under the power cap"
                            if sustained else "cuBLAS, burst") + "); f16 runs at the same rate",
        },
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": 2 * K,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(case, target_s=args.cpu_seconds)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    clk.stop()
    return line


def run_e2e_prefill(case, torch, stream, K, W, clk):
    """The multi-token step from pinned host memory, pipelined like the
    decode leg (pipelined_e2e): inputs are q, the new K/V, slots,
    cu_seqlens, tables and lengths; the output comes back every step.  The
    step moves hundreds of MB over PCIe, more than L2 holds."""
    ins = [case.q, case.kn, case.vn, case.slots, case.cu, case.tables_d, case.lens_d]

    def launch(k, v, outs):
        q, kn, vn, slots, cu, tables, lens = v
        case.write(kn, vn, slots)
        case.prefill(q, cu, tables, lens, out=outs[0])

    ms, h2d, d2h, span = pipelined_e2e(torch, stream, ins, [case.out], launch, K, W)
    return {"value": round(case.flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "mode": PIPELINE_MODE,
            "clocks": clk.summary(*span)}


# ---------------------------------------------------------- CPU oracle legs

PARITY_FAILURES = []


def oracle_decode_sample(oracle, inp, seqs, layer):
    """The oracle on the sampled sequences of one layer: their blocks as
    the device holds them, with the step's cache write redone by the
    oracle's own mirror (so the slot the GPU wrote is replaced by the
    oracle's value and no input comes from the product path).  Returns
    (fp64 output [n][Hq][D], attended tokens, seconds spent in the oracle's
    attention)."""
    w = inp.w
    s = inp.host_sample(seqs, layer)
    oracle.kv_write(s["k"], s["v"], w.kv_fmt, s["k_new"], s["v_new"], w.q_fmt, s["slots"], w.block_size,
                    s["k_inv"], s["v_inv"])
    t0 = time.perf_counter()
    if inp.window:
        cu = np.arange(len(seqs) + 1, dtype=np.int32)
        ref = oracle.paged_prefill(s["k"], s["v"], w.kv_fmt, s["q"], w.q_fmt, cu, s["tables"], s["lens"],
                                   w.scale, w.block_size, s["k_scale"], s["v_scale"], window=inp.window)
        att = np.minimum(s["lens"], inp.window)
    else:
        ref = oracle.paged_decode(s["k"], s["v"], w.kv_fmt, s["q"], w.q_fmt, s["tables"], s["lens"], w.scale,
                                  w.block_size, s["k_scale"], s["v_scale"])
        att = s["lens"]
    return ref, att, time.perf_counter() - t0


def check_outputs(got, ref, q_fmt, kv_fmt):
    """GPU outputs in the query dtype against the fp64 oracle: max-abs 2e-3
    (16-bit caches) or 1e-2 (FP8 cache), plus one rounding of the output
    format (2u|ref|).  Returns (passed, worst excess over the bound, max
    abs error)."""
    tol = 1e-2 if kv_fmt == 2 else 2e-3
    u = 2.0 ** -8 if q_fmt == 1 else 2.0 ** -11
    err = np.abs(got - ref)
    excess = float(np.max(err - (tol + 2 * u * np.abs(ref)))) if err.size else -tol
    return excess <= 0, excess, float(err.max()) if err.size else 0.0


def cpu_baseline(case, target_s=15.0, check=False, steps=1):
    """The oracle, as it stands, on a bounded sample of the same workload:
    sequences in batch order until about target_s seconds of CPU work (all
    layers of each sampled sequence).  With ``check`` (``case`` is a Case
    whose step has run), the GPU outputs of the sampled sequences — and of
    the longest and shortest sequences, through every layer — are compared
    with the oracle's; a mismatch is recorded and makes bench.py exit
    non-zero after printing its line."""
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    inp = getattr(case, "inp", case)
    w = inp.w
    L = inp.L
    # calibrate on one sequence of one layer, then size the sample
    _, _, one = oracle_decode_sample(oracle, inp, [0], 0)
    n = int(min(w.batch, max(1, target_s / max(one, 1e-3) / max(1, L)))) if target_s > 0 else 0
    seqs = list(range(n))
    total_s, total_bytes, passes = 0.0, 0, 0
    worst, max_err, checked = -1.0, 0.0, 0
    extra = sorted({int(np.argmax(inp.lens)), int(np.argmin(inp.lens))} - set(seqs)) if check else []
    while n and (passes < steps or total_s < 0.5 * target_s):
        for layer in range(L):
            ref, att, dt = oracle_decode_sample(oracle, inp, seqs, layer)
            total_s += dt
            total_bytes += (int(att.astype(np.int64).sum()) * w.kv_heads * w.head_dim * 2 * ELEM[w.kv_fmt]
                            + n * w.num_q_heads * w.head_dim * 2 * ELEM[w.q_fmt])
            if check and passes == 0:
                got = case.out[layer][seqs].float().cpu().numpy().astype(np.float64)
                ok, exc, err = check_outputs(got, ref, w.q_fmt, w.kv_fmt)
                worst, max_err, checked = max(worst, exc), max(max_err, err), checked + 1
        passes += 1
        if n < w.batch:
            break
    if check and extra:
        for layer in range(L):
            ref, _, _ = oracle_decode_sample(oracle, inp, extra, layer)
            got = case.out[layer][extra].float().cpu().numpy().astype(np.float64)
            ok, exc, err = check_outputs(got, ref, w.q_fmt, w.kv_fmt)
            worst, max_err, checked = max(worst, exc), max(max_err, err), checked + 1
    res = {"cores": cores, "kind": "oracle"}
    if n:
        res.update({"value": round(total_bytes / total_s / 1e9, 4), "unit": "GB/s",
                    "seqs_per_s": round(passes * n / total_s, 3),
                    "sample": f"{n} of {w.batch} sequences x {L} layer(s), decode only, fp64 C oracle "
                              f"(OpenMP over (sequence, head)); {total_s:.1f} s"})
    if check:
        passed = worst <= 0
        res["check"] = {"passed": passed, "sequences": sorted(set(seqs) | set(extra)), "layers": L,
                        "max_abs_err": round(max_err, 6), "worst_excess_over_bound": round(worst, 6),
                        "bound": "max-abs 2e-3 (16-bit cache) / 1e-2 (FP8) + one output rounding, vs fp64 oracle"}
        if not passed:
            PARITY_FAILURES.append((w.name, res["check"]))
    return res


def cpu_baseline_prefill(case, target_s=15.0):
    """The oracle, as it stands, on a bounded sample: the shortest sequences
    first until about target_s of CPU work."""
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    w, bs = case.w, case.w.block_size
    kh_all = case.k[0]
    order = np.argsort(case.lens, kind="stable")
    total_s, flops, tokens, done = 0.0, 0.0, 0, 0
    qh = case.q.cpu().numpy().view(np.uint16)
    for s in order:
        s = int(s)
        nblk = -(-int(case.lens[s]) // bs)
        idx = case.torch.tensor(case.tables[s, :nblk].astype(np.int64), device=kh_all.device)
        kh = case.k[0].index_select(0, idx).cpu().numpy().view(np.uint16)
        vh = case.v[0].index_select(0, idx).cpu().numpy().view(np.uint16)
        table = np.arange(nblk, dtype=np.int32)[None, :]
        rows = slice(int(case.cu_h[s]), int(case.cu_h[s + 1]))
        cu = np.array([0, int(case.new[s])], np.int32)
        t0 = time.perf_counter()
        oracle.paged_prefill(kh, vh, w.kv_fmt, qh[rows], w.q_fmt, cu, table, case.lens[s:s + 1], w.scale, bs)
        total_s += time.perf_counter() - t0
        p, n = int(case.prior[s]), int(case.new[s])
        flops += 4.0 * w.head_dim * w.num_q_heads * (p * n + n * (n + 1) // 2)
        tokens += n
        done += 1
        if total_s >= target_s:
            break
    return {"value": round(flops / total_s / 1e12, 6), "unit": "TFLOP/s",
            "new_tokens_per_s": round(tokens / total_s, 2), "cores": cores, "kind": "oracle",
            "sample": f"{done} of {w.batch} sequences (shortest first), attention only, fp64 C oracle "
                      f"(OpenMP over (sequence, head)); {total_s:.1f} s"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle timed on the host cores, each step a
    bounded sample of the same workload.  The inputs are drawn with torch
    alone (the GPU arm's generators); the product library is not loaded."""
    import torch
    if rank != 0:
        return None
    torch.cuda.set_device(0)
    if args.workload in PREFILL_WORKLOADS:
        return run_reference_prefill(args, world, torch)
    if args.workload in ("rag_trace", "preempt_trace", "gqa_trace"):
        return {"impl": "reference", "metric": METRIC, "workload": args.workload,
                "unavailable": "the CPU oracle has no serving-trace leg (the GPU line reports the host "
                               "scheduling time per iteration); time the single-step decode workloads instead"}
    from workloads.decode_inputs import DecodeInputs
    inp = DecodeInputs(args.workload, 0, args.layers)
    # warm-ups of about a second of oracle work each; the timed sample about
    # one second per requested step, at most 20 s (with the host copies of
    # the sampled blocks, the whole run stays within a few minutes)
    for _ in range(args.warmup):
        cpu_baseline(inp, target_s=1.0)
    res = cpu_baseline(inp, target_s=max(2.0, min(20.0, 1.0 * args.steps)), steps=1)
    w = inp.w
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": res["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": None,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": describe(w, inp), "global_batch": w.batch, "layers_per_step": inp.L},
        "seqs_per_s": res["seqs_per_s"],
        "cpu_baseline": res,
        "e2e": {"value": res["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_prefill(args, world, torch):
    case = PrefillCase(args.workload, 0, torch, None)
    per_step = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline_prefill(case, target_s=per_step)
    res = cpu_baseline_prefill(case, target_s=per_step * args.steps)
    return {
        "impl": "reference",
        "metric": METRIC_PREFILL,
        "value": res["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": None,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": describe_prefill(case.w, case), "global_batch": case.w.batch},
        "new_tokens_per_s": res["new_tokens_per_s"],
        "cpu_baseline": res,
        "e2e": {"value": res["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="kv_example",
                    choices=[*DECODE_WORKLOADS, "gqa_trace", "rag_trace", "preempt_trace", *PREFILL_WORKLOADS])
    ap.add_argument("--layers", type=int, default=None,
                    help="decode workloads: time only the first N layers (a small case for profiling)")
    ap.add_argument("--partition", type=int, default=0, help="decode partition tokens (0: auto)")
    ap.add_argument("--stages", type=int, default=0, help="pipeline stages per warp (0: auto)")
    ap.add_argument("--warps", type=int, default=0, help="warps per decode CTA (0: auto)")
    ap.add_argument("--order", default=None, choices=["long_first", "longest", "batch"],
                    help="decode scheduling order (default: longest first for one decode step, "
                         "batch order for the continuous-batching trace)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--timeline", action="store_true",
                    help="gqa_trace: after the timed region, time the end-to-end loop's input uploads and host "
                         "scheduling per iteration (added under e2e.timeline)")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="serving traces: the shared-prefix decode for the largest group of sequences "
                         "sharing leading blocks (default: the plain decode)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sustained loop and the per-config measurements")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    elif args.workload == "gqa_trace":
        line = run_trace(args, rank, world, local_rank)
    elif args.workload in PREFILL_WORKLOADS:
        line = run_prefill(args, rank, world, local_rank)
    elif args.workload == "rag_trace":
        line = run_rag(args, rank, world, local_rank)
    elif args.workload == "preempt_trace":
        line = run_preempt(args, rank, world, local_rank)
    else:
        line = run_ours(args, rank, world, local_rank)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if PARITY_FAILURES:
        print(f"oracle check failed: {PARITY_FAILURES}", file=sys.stderr, flush=True)
        sys.exit(3)


if __name__ == "__main__":
    main()
