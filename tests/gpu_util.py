"""Helpers for the GPU parity tests: device pools, decode calls through the
C ABI, oracle comparison on sampled sequences."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import paged_kv_cache_451_b200 as pk
from workloads import BF16, E4M3, F16, F32

DEV = "cuda"
TORCH_RAW = {F16: torch.int16, BF16: torch.int16, E4M3: torch.uint8}
TOL = {F16: 2e-3, BF16: 2e-3, E4M3: 1e-2}  # max-abs tolerance of fp32 outputs vs fp64


def dev(a: np.ndarray) -> torch.Tensor:
    """Host numpy array -> device tensor with the same bytes."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(DEV)


def host(t: torch.Tensor, like: np.dtype) -> np.ndarray:
    a = t.cpu().numpy()
    return a.view(like)


class DevicePool:
    """A pool handle plus the device tensors bound to it."""

    def __init__(self, num_blocks, kv_heads, head_dim, block_size, fmt, num_layers=1,
                 k=None, v=None, k_scale=None, v_scale=None, partition=0, stages=0, warps=0):
        self.fmt, self.num_blocks, self.kv_heads = fmt, num_blocks, kv_heads
        self.head_dim, self.block_size, self.num_layers = head_dim, block_size, num_layers
        self.h = pk.kv_pool_create(block_size, num_blocks, kv_heads, head_dim, fmt, num_layers)
        pk.kv_pool_set_decode_config(self.h, partition, stages, warps)
        shape = (num_blocks, kv_heads, block_size, head_dim)
        self.k, self.v, self.ks, self.vs = [], [], [], []
        for layer in range(num_layers):
            kt = k[layer] if k is not None else torch.zeros(shape, dtype=TORCH_RAW[fmt], device=DEV)
            vt = v[layer] if v is not None else torch.zeros(shape, dtype=TORCH_RAW[fmt], device=DEV)
            kst = vst = None
            if fmt == E4M3:
                kst = k_scale[layer] if k_scale is not None else torch.ones((num_blocks, kv_heads), device=DEV)
                vst = v_scale[layer] if v_scale is not None else torch.ones((num_blocks, kv_heads), device=DEV)
            self.k.append(kt)
            self.v.append(vt)
            self.ks.append(kst)
            self.vs.append(vst)
            pk.kv_pool_bind(self.h, layer, kt, vt, kst, vst)

    def set_config(self, partition=0, stages=0, warps=0):
        pk.kv_pool_set_decode_config(self.h, partition, stages, warps)

    def __del__(self):
        try:
            pk.kv_pool_destroy(self.h)
        except Exception:  # noqa: BLE001
            pass


def decode(pool: DevicePool, q_dev, q_fmt, num_q_heads, tables_dev, lens_dev, max_ctx, scale,
           out_fmt=F32, layer=0, stream=None):
    b = q_dev.shape[0]
    width = tables_dev.shape[1]
    out_dt = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[out_fmt]
    out = torch.empty((b, num_q_heads, pool.head_dim), dtype=out_dt, device=DEV)
    wsb = pk.paged_attention_workspace_bytes(pool.h, b, num_q_heads, max_ctx)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
    pk.paged_attention_decode(pool.h, layer, q_dev, q_fmt, num_q_heads, tables_dev, width, lens_dev,
                              b, max_ctx, scale, out, out_fmt, ws, wsb, stream)
    return out


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def assert_close_native(out_native: torch.Tensor, ref: np.ndarray, fmt: int, tol: float):
    """|gpu - ref| <= tol + one rounding of the output format (2u|ref|)."""
    u = 2.0 ** -8 if fmt == BF16 else 2.0 ** -11
    got = out_native.float().cpu().numpy().astype(np.float64)
    bound = tol + 2 * u * np.abs(ref)
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))


def sampled_oracle(pool: DevicePool, tables: np.ndarray, lens: np.ndarray, q_host: np.ndarray,
                   q_fmt: int, scale: float, seqs, layer=0):
    """Oracle output for the sampled sequences only: their blocks are copied
    from the device pool (inputs, never written by the library) into a small
    host pool with remapped tables."""
    seqs = list(seqs)
    bs = pool.block_size
    used = []
    sub_tables = np.full((len(seqs), tables.shape[1]), -1, np.int32)
    for i, s in enumerate(seqs):
        nblk = -(-int(lens[s]) // bs)
        for j in range(nblk):
            sub_tables[i, j] = len(used)
            used.append(int(tables[s, j]))
    idx = torch.tensor(used if used else [0], dtype=torch.long, device=DEV)
    raw = np.uint8 if pool.fmt == E4M3 else np.uint16
    kh = host(pool.k[layer].index_select(0, idx), raw)
    vh = host(pool.v[layer].index_select(0, idx), raw)
    ks = vs = None
    if pool.fmt == E4M3:
        ks = pool.ks[layer].index_select(0, idx).cpu().numpy()
        vs = pool.vs[layer].index_select(0, idx).cpu().numpy()
    return oracle.paged_decode(kh, vh, pool.fmt, q_host[seqs], q_fmt, sub_tables,
                               lens[seqs].astype(np.int32), scale, bs, ks, vs)
