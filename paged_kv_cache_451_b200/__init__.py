"""Python binding of the pagedkv C ABI (include/pagedkv.h).

Argument marshalling only: every function forwards to the native library
``libpagedkv.so`` under the same name, turning torch tensors / numpy arrays
into raw pointers and raising :class:`KVError` on a non-zero status.  There
is no fallback: if the native library is missing and cannot be built, the
import fails.
"""

from __future__ import annotations

import ctypes
import os

from . import build as _build

KV_F16, KV_BF16, KV_FP8_E4M3, KV_F32 = 0, 1, 2, 3
KV_PREEMPT_NONE, KV_PREEMPT_SWAP, KV_PREEMPT_RECOMPUTE = 0, 1, 2
KV_ORDER_BATCH, KV_ORDER_LONGEST, KV_ORDER_LONG_FIRST = 0, 1, 2
KV_SERVE_MAX_SETS = 4
KV_OK, KV_ERR_ARG, KV_ERR_OOM, KV_ERR_STATE, KV_ERR_BOUNDS, KV_ERR_CUDA, KV_ERR_TIMEOUT = (
    0, -1, -2, -3, -4, -5, -6)
ERROR_NAMES = {0: "KV_OK", -1: "KV_ERR_ARG", -2: "KV_ERR_OOM", -3: "KV_ERR_STATE",
               -4: "KV_ERR_BOUNDS", -5: "KV_ERR_CUDA", -6: "KV_ERR_TIMEOUT"}

LIB_PATH = _build.LIB


class KVError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if _build.stale():
        try:
            _build.build()
        except Exception as e:  # noqa: BLE001
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"native library {LIB_PATH} is missing and could not be built: {e}")
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"native library {LIB_PATH} is missing")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()

c_int, c_int64, c_size_t, c_float, c_void_p = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                               ctypes.c_float, ctypes.c_void_p)
P = ctypes.POINTER


class kv_step_info(ctypes.Structure):
    _fields_ = [("batch", c_int), ("num_tokens", c_int), ("num_cow", c_int),
                ("num_admitted", c_int), ("max_blocks", c_int)]


class kv_step_layout(ctypes.Structure):
    _fields_ = [("info", kv_step_info), ("table_width", c_int), ("max_context_len", c_int),
                ("num_swap_out", c_int), ("num_swap_in", c_int), ("prefill_tokens", c_int),
                ("max_prefill_len", c_int), ("buffer", c_int), ("bytes", c_int64), ("slot_mapping", c_int64),
                ("block_tables", c_int64), ("context_lens", c_int64), ("seq_order", c_int64),
                ("cow_pairs", c_int64), ("swap_out_pairs", c_int64), ("swap_in_pairs", c_int64),
                ("cu_seqlens", c_int64), ("prefill_context_lens", c_int64)]


_SIGS = {
    "kv_last_error": (ctypes.c_char_p, []),
    "kv_version": (c_int, []),
    "kv_pool_create": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, P(c_void_p)]),
    "kv_pool_bytes": (c_int, [c_void_p, P(c_size_t), P(c_size_t)]),
    "kv_pool_bind": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "kv_pool_set_decode_config": (c_int, [c_void_p, c_int, c_int, c_int]),
    "kv_pool_set_sliding_window": (c_int, [c_void_p, c_int]),
    "kv_alloc_release_before": (c_int, [c_void_p, c_int64, c_int64, P(c_int)]),
    "kv_sched_set_window": (c_int, [c_void_p, c_int]),
    "kv_alloc_set_swap_space": (c_int, [c_void_p, c_int]),
    "kv_sched_set_preemption": (c_int, [c_void_p, c_int]),
    "kv_sched_swap_info": (c_int, [c_void_p, P(c_int), P(c_int), P(c_int), P(c_int), P(c_int), P(c_int)]),
    "kv_sched_swap_outputs": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "kv_swap_block_bytes": (c_size_t, [c_void_p]),
    "kv_swap_out": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p]),
    "kv_swap_in": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p]),
    "kv_pool_destroy": (c_int, [c_void_p]),
    "paged_kv_write": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_int,
                               c_void_p, c_void_p, c_void_p]),
    "block_copy": (c_int, [c_void_p, c_void_p, c_int, c_void_p]),
    "paged_attention_workspace_bytes": (c_size_t, [c_void_p, c_int, c_int, c_int]),
    "paged_attention_decode": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_int,
                                       c_void_p, c_int, c_int, c_float, c_void_p, c_int, c_void_p,
                                       c_size_t, c_void_p, c_void_p]),
    "paged_attention_shared_prefix_workspace_bytes": (c_size_t, [c_void_p, c_int, c_int, c_int, c_int]),
    "paged_attention_decode_shared_prefix": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_int,
                                                     c_void_p, c_int, c_int, c_void_p, c_int, c_void_p, c_int,
                                                     c_void_p, c_float, c_void_p, c_int, c_void_p, c_size_t,
                                                     c_void_p, c_void_p]),
    "paged_attention_decode_noalloc": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_void_p,
                                               c_int, c_void_p, c_int, c_int, c_float, c_void_p,
                                               c_int, c_void_p]),
    "paged_attention_prefill": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_int,
                                        c_int, c_void_p, c_int, c_void_p, c_int, c_float, c_void_p,
                                        c_int, c_void_p]),
    "kv_selftest_wait_timeout": (c_int, [ctypes.c_uint64, c_void_p]),
    "kv_get_device_error": (c_int, [c_void_p, P(c_int)]),
    "kv_alloc_create": (c_int, [c_int, c_int, c_void_p, P(c_void_p)]),
    "kv_alloc_num_free": (c_int, [c_void_p, P(c_int)]),
    "kv_alloc_can_allocate": (c_int, [c_void_p, c_int, P(c_int)]),
    "kv_alloc_allocate": (c_int, [c_void_p, c_int64, c_int]),
    "kv_alloc_append_slot": (c_int, [c_void_p, c_int64, P(c_int64), P(ctypes.c_int32),
                                     P(ctypes.c_int32)]),
    "kv_alloc_fork": (c_int, [c_void_p, c_int64, c_int64]),
    "kv_alloc_free": (c_int, [c_void_p, c_int64]),
    "kv_alloc_block_table": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "kv_alloc_num_tokens": (c_int, [c_void_p, c_int64, P(c_int)]),
    "kv_alloc_refcount": (c_int, [c_void_p, ctypes.c_int32, P(c_int)]),
    "kv_alloc_snapshot": (c_int, [c_void_p, c_void_p, P(c_int), c_void_p]),
    "kv_alloc_counters": (c_int, [c_void_p, P(c_int64), P(c_int64), P(c_int64)]),
    "kv_alloc_destroy": (c_int, [c_void_p]),
    "kv_alloc_enable_prefix_caching": (c_int, [c_void_p]),
    "kv_alloc_allocate_prompt": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "kv_alloc_append_token": (c_int, [c_void_p, c_int64, ctypes.c_int32, P(c_int64),
                                      P(ctypes.c_int32), P(ctypes.c_int32)]),
    "kv_alloc_commit": (c_int, [c_void_p, c_int64, P(c_int)]),
    "kv_alloc_prefix_stats": (c_int, [c_void_p, P(c_int64), P(c_int64), P(c_int)]),
    "kv_sched_create": (c_int, [c_void_p, c_int, c_int, P(c_void_p)]),
    "kv_sched_add_request": (c_int, [c_void_p, c_int64, c_int]),
    "kv_sched_add_request_tokens": (c_int, [c_void_p, c_int64, c_void_p, c_int]),
    "kv_sched_admitted_cached": (c_int, [c_void_p, c_void_p]),
    "kv_sched_adopt": (c_int, [c_void_p, c_int64]),
    "kv_sched_step": (c_int, [c_void_p, c_void_p, c_int, P(kv_step_info)]),
    "kv_sched_outputs": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                 c_void_p, c_void_p]),
    "kv_sched_stats": (c_int, [c_void_p, P(c_int), P(c_int), P(c_int), P(c_int)]),
    "kv_sched_destroy": (c_int, [c_void_p]),
    "kv_step_packed_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "kv_sched_step_packed": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p,
                                     P(kv_step_layout)]),
    "kv_serve_workspace_bytes": (c_size_t, [c_void_p, c_int, c_int, c_int]),
    "kv_serve_create": (c_int, [c_void_p, c_void_p, c_int, c_int, c_float, c_int, c_int, c_int, c_int, c_void_p,
                                c_int, c_int, P(c_void_p), P(c_void_p), c_size_t, c_void_p, c_size_t,
                                P(c_void_p)]),
    "kv_serve_schedule": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, P(kv_step_layout)]),
    "kv_serve_launch": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_int, c_void_p, c_void_p, c_void_p]),
    "kv_serve_upload": (c_int, [c_void_p, c_void_p, c_void_p, c_size_t]),
    "kv_serve_readback": (c_int, [c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kv_serve_destroy": (c_int, [c_void_p]),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def _check(rc: int) -> None:
    if rc != KV_OK:
        raise KVError(rc, _lib.kv_last_error().decode())


def _ptr(x):
    """Raw address of a torch tensor, numpy array, int or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)!r}")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ------------------------------------------------------------------- misc

def kv_last_error() -> str:
    return _lib.kv_last_error().decode()


def kv_version() -> int:
    return _lib.kv_version()


# ------------------------------------------------------------------- pool

def kv_pool_create(block_size, num_blocks, kv_heads, head_dim, dtype, num_layers=1):
    h = c_void_p()
    _check(_lib.kv_pool_create(block_size, num_blocks, kv_heads, head_dim, dtype, num_layers,
                               ctypes.byref(h)))
    return h


def kv_pool_bytes(pool):
    a, b = c_size_t(), c_size_t()
    _check(_lib.kv_pool_bytes(pool, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def kv_pool_bind(pool, layer, k_base, v_base, k_scale=None, v_scale=None):
    _check(_lib.kv_pool_bind(pool, layer, _ptr(k_base), _ptr(v_base), _ptr(k_scale), _ptr(v_scale)))


def kv_pool_set_decode_config(pool, partition_tokens=0, stages=0, warps=0):
    _check(_lib.kv_pool_set_decode_config(pool, partition_tokens, stages, warps))


def kv_pool_set_sliding_window(pool, window):
    _check(_lib.kv_pool_set_sliding_window(pool, int(window)))


def kv_alloc_release_before(a, seq_id, token) -> int:
    n = c_int()
    _check(_lib.kv_alloc_release_before(a, seq_id, int(token), ctypes.byref(n)))
    return n.value


def kv_sched_set_window(s, window):
    _check(_lib.kv_sched_set_window(s, int(window)))


def kv_alloc_set_swap_space(a, num_slots):
    _check(_lib.kv_alloc_set_swap_space(a, int(num_slots)))


def kv_sched_set_preemption(s, mode):
    _check(_lib.kv_sched_set_preemption(s, int(mode)))


def kv_sched_swap_outputs(s):
    """Last step's swap outputs as numpy arrays (dict) plus the count of
    sequences now swapped out."""
    import numpy as np
    n = [c_int() for _ in range(6)]
    _check(_lib.kv_sched_swap_info(s, *[ctypes.byref(x) for x in n]))
    out = {"swap_out": np.empty((n[0].value, 2), np.int32), "swap_in": np.empty((n[1].value, 2), np.int32),
           "preempted": np.empty(n[2].value, np.int64), "recomputed": np.empty(n[3].value, np.int64),
           "swapped_in": np.empty(n[4].value, np.int64), "num_swapped": n[5].value}
    if n[0].value or n[1].value or n[2].value or n[3].value or n[4].value:  # else nothing to copy
        _check(_lib.kv_sched_swap_outputs(s, _ptr(out["swap_out"]), _ptr(out["swap_in"]), _ptr(out["preempted"]),
                                          _ptr(out["recomputed"]), _ptr(out["swapped_in"])))
    return out


def kv_swap_block_bytes(pool) -> int:
    return int(_lib.kv_swap_block_bytes(pool))


def kv_swap_out(pool, host_swap, num_slots, pairs, num_pairs, stream=None):
    _check(_lib.kv_swap_out(pool, _ptr(host_swap), int(num_slots), _ptr(pairs), int(num_pairs), _stream(stream)))


def kv_swap_in(pool, host_swap, num_slots, pairs, num_pairs, stream=None):
    _check(_lib.kv_swap_in(pool, _ptr(host_swap), int(num_slots), _ptr(pairs), int(num_pairs), _stream(stream)))


def kv_pool_destroy(pool):
    _check(_lib.kv_pool_destroy(pool))


# ------------------------------------------------------------ GPU entries

def paged_kv_write(pool, layer, k_new, v_new, src_dtype, slot_mapping, num_tokens,
                   k_inv_scale=None, v_inv_scale=None, stream=None):
    _check(_lib.paged_kv_write(pool, layer, _ptr(k_new), _ptr(v_new), src_dtype,
                               _ptr(slot_mapping), num_tokens, _ptr(k_inv_scale),
                               _ptr(v_inv_scale), _stream(stream)))


def block_copy(pool, pairs, num_pairs, stream=None):
    _check(_lib.block_copy(pool, _ptr(pairs), num_pairs, _stream(stream)))


def paged_attention_workspace_bytes(pool, batch, num_q_heads, max_context_len) -> int:
    return int(_lib.paged_attention_workspace_bytes(pool, batch, num_q_heads, max_context_len))


def paged_attention_decode(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq,
                           context_lens, batch, max_context_len, scale, out, out_dtype,
                           workspace=None, workspace_bytes=0, stream=None, seq_order=None):
    _check(_lib.paged_attention_decode(pool, layer, _ptr(q), q_dtype, num_q_heads,
                                       _ptr(block_tables), max_blocks_per_seq, _ptr(context_lens),
                                       batch, max_context_len, float(scale), _ptr(out), out_dtype,
                                       _ptr(workspace), int(workspace_bytes), _ptr(seq_order),
                                       _stream(stream)))


def paged_attention_prefill(pool, layer, q, q_dtype, num_q_heads, cu_seqlens_q, total_q, max_q_len,
                            block_tables, max_blocks_per_seq, context_lens, batch, scale, out,
                            out_dtype, stream=None):
    _check(_lib.paged_attention_prefill(pool, layer, _ptr(q), q_dtype, num_q_heads,
                                        _ptr(cu_seqlens_q), int(total_q), int(max_q_len),
                                        _ptr(block_tables), max_blocks_per_seq, _ptr(context_lens),
                                        batch, float(scale), _ptr(out), out_dtype, _stream(stream)))


def paged_attention_shared_prefix_workspace_bytes(pool, batch, num_q_heads, max_context_len, num_sharers) -> int:
    return int(_lib.paged_attention_shared_prefix_workspace_bytes(pool, batch, num_q_heads, max_context_len,
                                                                  num_sharers))


def paged_attention_decode_shared_prefix(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq,
                                         context_lens, batch, max_context_len, prefix_seqs, num_sharers,
                                         prefix_blocks, prefix_len, skip_lens, scale, out, out_dtype,
                                         workspace, workspace_bytes, stream=None, seq_order=None):
    _check(_lib.paged_attention_decode_shared_prefix(
        pool, layer, _ptr(q), q_dtype, num_q_heads, _ptr(block_tables), max_blocks_per_seq,
        _ptr(context_lens), batch, max_context_len, _ptr(prefix_seqs), num_sharers, _ptr(prefix_blocks),
        prefix_len, _ptr(skip_lens), float(scale), _ptr(out), out_dtype, _ptr(workspace), workspace_bytes,
        _ptr(seq_order), _stream(stream)))


KV_NOALLOC_WORKSPACE_BYTES = 16 << 20


def paged_attention_decode_noalloc(pool, layer, q, q_dtype, num_q_heads, block_tables,
                                   max_blocks_per_seq, context_lens, batch, max_context_len, scale,
                                   out, out_dtype, stream=None):
    _check(_lib.paged_attention_decode_noalloc(pool, layer, _ptr(q), q_dtype, num_q_heads,
                                               _ptr(block_tables), max_blocks_per_seq,
                                               _ptr(context_lens), batch, max_context_len,
                                               float(scale), _ptr(out), out_dtype, _stream(stream)))


def kv_selftest_wait_timeout(limit_ns, stream=None):
    _check(_lib.kv_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def kv_get_device_error(stream=None) -> int:
    e = c_int()
    _check(_lib.kv_get_device_error(_stream(stream), ctypes.byref(e)))
    return e.value


# -------------------------------------------------------------- allocator

def kv_alloc_create(num_blocks, block_size, initial_free_order=None):
    import numpy as np
    h = c_void_p()
    order = None if initial_free_order is None else np.ascontiguousarray(initial_free_order, np.int32)
    _check(_lib.kv_alloc_create(num_blocks, block_size, _ptr(order), ctypes.byref(h)))
    return h


def kv_alloc_num_free(a) -> int:
    n = c_int()
    _check(_lib.kv_alloc_num_free(a, ctypes.byref(n)))
    return n.value


def kv_alloc_can_allocate(a, num_tokens) -> bool:
    y = c_int()
    _check(_lib.kv_alloc_can_allocate(a, num_tokens, ctypes.byref(y)))
    return bool(y.value)


def kv_alloc_allocate(a, seq_id, num_tokens):
    _check(_lib.kv_alloc_allocate(a, seq_id, num_tokens))


def kv_alloc_append_slot(a, seq_id):
    slot, cs, cd = c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.kv_alloc_append_slot(a, seq_id, ctypes.byref(slot), ctypes.byref(cs),
                                     ctypes.byref(cd)))
    return slot.value, cs.value, cd.value


def kv_alloc_fork(a, parent, child):
    _check(_lib.kv_alloc_fork(a, parent, child))


def kv_alloc_free(a, seq_id):
    _check(_lib.kv_alloc_free(a, seq_id))


def kv_alloc_block_table(a, seq_id):
    import numpy as np
    n = c_int()
    _check(_lib.kv_alloc_block_table(a, seq_id, None, 0, ctypes.byref(n)))
    out = np.empty(n.value, np.int32)
    _check(_lib.kv_alloc_block_table(a, seq_id, _ptr(out), n.value, ctypes.byref(n)))
    return out


def kv_alloc_num_tokens(a, seq_id) -> int:
    n = c_int()
    _check(_lib.kv_alloc_num_tokens(a, seq_id, ctypes.byref(n)))
    return n.value


def kv_alloc_refcount(a, block) -> int:
    r = c_int()
    _check(_lib.kv_alloc_refcount(a, block, ctypes.byref(r)))
    return r.value


def kv_alloc_snapshot(a, num_blocks):
    import numpy as np
    n = c_int()
    free = np.empty(num_blocks, np.int32)
    rc = np.empty(num_blocks, np.int32)
    _check(_lib.kv_alloc_snapshot(a, _ptr(free), ctypes.byref(n), _ptr(rc)))
    return free[:n.value].copy(), rc


def kv_alloc_counters(a):
    x, y, z = c_int64(), c_int64(), c_int64()
    _check(_lib.kv_alloc_counters(a, ctypes.byref(x), ctypes.byref(y), ctypes.byref(z)))
    return x.value, y.value, z.value


def kv_alloc_destroy(a):
    _check(_lib.kv_alloc_destroy(a))


def kv_alloc_enable_prefix_caching(a):
    _check(_lib.kv_alloc_enable_prefix_caching(a))


def kv_alloc_allocate_prompt(a, seq_id, tokens) -> int:
    import numpy as np
    t = np.ascontiguousarray(tokens, np.int32)
    n = c_int()
    _check(_lib.kv_alloc_allocate_prompt(a, seq_id, _ptr(t) if t.size else None, int(t.size),
                                         ctypes.byref(n)))
    return n.value


def kv_alloc_append_token(a, seq_id, token):
    slot, cs, cd = c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.kv_alloc_append_token(a, seq_id, int(token), ctypes.byref(slot), ctypes.byref(cs),
                                      ctypes.byref(cd)))
    return slot.value, cs.value, cd.value


def kv_alloc_commit(a, seq_id) -> int:
    n = c_int()
    _check(_lib.kv_alloc_commit(a, seq_id, ctypes.byref(n)))
    return n.value


def kv_alloc_prefix_stats(a):
    h, e, c = c_int64(), c_int64(), c_int()
    _check(_lib.kv_alloc_prefix_stats(a, ctypes.byref(h), ctypes.byref(e), ctypes.byref(c)))
    return h.value, e.value, c.value


# -------------------------------------------------------------- scheduler

def kv_sched_create(a, max_num_seqs, min_blocks=-1):
    h = c_void_p()
    _check(_lib.kv_sched_create(a, max_num_seqs, min_blocks, ctypes.byref(h)))
    return h


def kv_sched_add_request(s, seq_id, prompt_len):
    _check(_lib.kv_sched_add_request(s, seq_id, prompt_len))


def kv_sched_add_request_tokens(s, seq_id, tokens):
    import numpy as np
    t = np.ascontiguousarray(tokens, np.int32)
    _check(_lib.kv_sched_add_request_tokens(s, seq_id, _ptr(t) if t.size else None, int(t.size)))


def kv_sched_adopt(s, seq_id):
    _check(_lib.kv_sched_adopt(s, seq_id))


def kv_sched_step(s, finished_ids=()):
    import numpy as np
    fin = np.ascontiguousarray(finished_ids, np.int64)
    info = kv_step_info()
    _check(_lib.kv_sched_step(s, _ptr(fin) if fin.size else None, int(fin.size),
                              ctypes.byref(info)))
    return info


def kv_sched_outputs(s, info, table_width=None):
    """Last step's outputs as numpy arrays (dict)."""
    import numpy as np
    w = max(info.max_blocks, 1) if table_width is None else table_width
    out = {
        "running": np.empty(info.batch, np.int64),
        "block_tables": np.empty((info.batch, w), np.int32),
        "context_lens": np.empty(info.batch, np.int32),
        "slot_mapping": np.empty(info.num_tokens, np.int64),
        "cow_pairs": np.empty((info.num_cow, 2), np.int32),
        "admitted": np.empty(info.num_admitted, np.int64),
    }
    _check(_lib.kv_sched_outputs(s, _ptr(out["running"]), _ptr(out["block_tables"]), w,
                                 _ptr(out["context_lens"]), _ptr(out["slot_mapping"]),
                                 _ptr(out["cow_pairs"]), _ptr(out["admitted"])))
    out["cached"] = np.empty(info.num_admitted, np.int32)
    _check(_lib.kv_sched_admitted_cached(s, _ptr(out["cached"])))
    return out


def kv_sched_stats(s):
    r, w, u, t = c_int(), c_int(), c_int(), c_int()
    _check(_lib.kv_sched_stats(s, ctypes.byref(r), ctypes.byref(w), ctypes.byref(u),
                               ctypes.byref(t)))
    return r.value, w.value, u.value, t.value


def kv_sched_destroy(s):
    _check(_lib.kv_sched_destroy(s))


# ------------------------------------------------------------ serving step

def kv_step_packed_bytes(max_batch, max_tokens, max_table_width, max_swap_pairs=0) -> int:
    return int(_lib.kv_step_packed_bytes(max_batch, max_tokens, max_table_width, max_swap_pairs))


def kv_sched_step_packed(s, finished_ids, order_policy, max_table_width, buf, buf_bytes, running_ids=None):
    """Scheduler step packed into ``buf`` (host, 16-byte aligned); returns
    the kv_step_layout."""
    import numpy as np
    fin = np.ascontiguousarray(finished_ids, np.int64)
    lay = kv_step_layout()
    _check(_lib.kv_sched_step_packed(s, _ptr(fin) if fin.size else None, int(fin.size), order_policy,
                                     max_table_width, _ptr(buf), buf_bytes, _ptr(running_ids),
                                     ctypes.byref(lay)))
    return lay


def kv_serve_workspace_bytes(pool, num_q_heads, max_batch, max_context_len) -> int:
    return int(_lib.kv_serve_workspace_bytes(pool, num_q_heads, max_batch, max_context_len))


def kv_serve_create(pool, sched, num_q_heads, q_dtype, scale, order_policy, max_batch, max_tokens,
                    max_table_width, host_swap, swap_slots, host_meta, dev_meta, meta_bytes, workspace,
                    workspace_bytes):
    """host_meta / dev_meta: one buffer per set (their count is num_sets)."""
    h = c_void_p()
    n = len(host_meta)
    if len(dev_meta) != n:
        raise ValueError("host_meta and dev_meta need the same number of sets")
    hm = (c_void_p * max(n, 1))(*[_ptr(x) for x in host_meta])
    dm = (c_void_p * max(n, 1))(*[_ptr(x) for x in dev_meta])
    _check(_lib.kv_serve_create(pool, sched, num_q_heads, q_dtype, float(scale), order_policy, max_batch,
                                max_tokens, max_table_width, _ptr(host_swap), swap_slots, n, hm, dm, meta_bytes,
                                _ptr(workspace), workspace_bytes, ctypes.byref(h)))
    return h


def kv_serve_schedule(sv, finished_ids, upload_stream=None, running_ids=None, layout=None):
    """Returns the step's kv_step_layout (``layout``, if given, is filled and
    returned)."""
    import numpy as np
    fin = np.ascontiguousarray(finished_ids, np.int64)
    lay = kv_step_layout() if layout is None else layout
    _check(_lib.kv_serve_schedule(sv, _ptr(fin) if fin.size else None, int(fin.size), _stream(upload_stream),
                                  _ptr(running_ids), ctypes.byref(lay)))
    return lay


def kv_serve_launch(sv, layer, q, k_new, v_new, out, out_dtype, k_inv_scale=None, v_inv_scale=None,
                    prefill_q=None, prefill_out=None, stream=None):
    _check(_lib.kv_serve_launch(sv, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_inv_scale),
                                _ptr(v_inv_scale), _ptr(out), out_dtype, _ptr(prefill_q), _ptr(prefill_out),
                                _stream(stream)))


def kv_serve_upload(sv, dev_dst, host_src, nbytes):
    _check(_lib.kv_serve_upload(sv, _ptr(dev_dst), _ptr(host_src), int(nbytes)))


def kv_serve_readback(sv, host_dst, dev_src, nbytes, readback_stream=None):
    _check(_lib.kv_serve_readback(sv, _ptr(host_dst), _ptr(dev_src), int(nbytes), _stream(readback_stream)))


def kv_serve_destroy(sv):
    _check(_lib.kv_serve_destroy(sv))
