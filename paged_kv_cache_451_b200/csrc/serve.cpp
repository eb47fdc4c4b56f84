// Native serving step: one continuous-batching iteration sequenced by the
// library ("vLLM 推理加速原理详解", section "连续批处理：别再等最慢的那个请求了":
// free the finished, admit first come first served, append one slot per
// running sequence, then run the step on the GPU).
//
// kv_sched_step_packed runs the scheduler step and writes all of the step's
// device metadata into one caller buffer (pinned host memory), so a single
// copy uploads it.  kv_serve_* cycle through 2 to 4 sets of such buffers and
// device buffers: the upload of step i + 1 runs on an upload stream while the
// kernels of step i read another set, with events ordering reuse.  Only
// host code here; every kernel is enqueued through the library's own entry
// points (block_copy, kv_swap_out / kv_swap_in, paged_kv_write,
// paged_attention_prefill, paged_attention_decode).

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <numeric>
#include <vector>

#include "host_common.h"

using pagedkv::fail;
using pagedkv::ok;

namespace {

constexpr int64_t kAlign = 16;

int64_t up16(int64_t n) { return (n + kAlign - 1) / kAlign * kAlign; }

// Bytes of the packed arrays for these counts, in the order they are laid out.
int64_t packed_bytes(int64_t tokens, int64_t batch, int64_t width, int64_t cow, int64_t swo, int64_t swi,
                     int64_t admitted, bool order) {
  return up16(8 * tokens) + up16(4 * batch * width) + up16(4 * batch) + (order ? up16(4 * batch) : 0) +
         up16(8 * cow) + up16(8 * swo) + up16(8 * swi) + (admitted ? up16(4 * (admitted + 1)) : 0) +
         up16(4 * admitted);
}

// Scheduling order of the decode's sequences (the grid row -> sequence map):
// longest: all by decreasing context, ties in batch order; long_first: those
// longer than the batch mean, longest first, then the rest in batch order.
void order_of(const int32_t* lens, int n, int policy, int32_t* order) {
  std::iota(order, order + n, 0);
  if (policy == KV_ORDER_LONGEST) {
    std::stable_sort(order, order + n, [&](int32_t a, int32_t b) { return lens[a] > lens[b]; });
    return;
  }
  int64_t sum = 0;
  for (int i = 0; i < n; ++i) sum += lens[i];
  // lens[i] > sum / n, compared exactly in integers
  std::stable_partition(order, order + n, [&](int32_t i) { return (int64_t)lens[i] * n > sum; });
  const int n_long = (int)std::count_if(lens, lens + n, [&](int32_t l) { return (int64_t)l * n > sum; });
  std::stable_sort(order, order + n_long, [&](int32_t a, int32_t b) { return lens[a] > lens[b]; });
}

}  // namespace

struct kv_serve {
  kv_pool* pool = nullptr;
  kv_sched* sched = nullptr;
  int hq = 0;
  kv_dtype q_dtype = KV_BF16;
  float scale = 1.f;
  int order = KV_ORDER_BATCH;
  int max_batch = 0, max_tokens = 0, max_width = 0;
  void* host_swap = nullptr;
  int swap_slots = 0;
  int sets = 2;  // buffer sets, used in turn by consecutive steps
  uint8_t* h[KV_SERVE_MAX_SETS] = {};
  uint8_t* d[KV_SERVE_MAX_SETS] = {};
  size_t meta_bytes = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  cudaEvent_t copy_ev[KV_SERVE_MAX_SETS] = {};  // uploads into buffer set k done
  cudaEvent_t done_ev[KV_SERVE_MAX_SETS] = {};  // kernels reading buffer set k done
  cudaEvent_t rb_ev[KV_SERVE_MAX_SETS] = {};    // read-back of output set k done
  bool copy_rec[KV_SERVE_MAX_SETS] = {}, done_rec[KV_SERVE_MAX_SETS] = {}, rb_rec[KV_SERVE_MAX_SETS] = {};
  cudaStream_t up = nullptr;  // the current step's upload stream
  int k = -1;              // buffer set of the current step
  bool scheduled = false;  // a step is scheduled and not launched yet
  int launches = 0;        // launch calls for the current step
  kv_step_layout lay{};
};

extern "C" {

size_t kv_step_packed_bytes(int max_batch, int max_tokens, int max_table_width, int max_swap_pairs) {
  if (max_batch < 0 || max_tokens < 0 || max_table_width < 0 || max_swap_pairs < 0) return 0;
  return (size_t)packed_bytes(max_tokens, max_batch, std::max(max_table_width, 1), max_batch, max_swap_pairs,
                              max_swap_pairs, max_batch, true);
}

int kv_sched_step_packed(kv_sched* s, const int64_t* finished_ids, int n_finished, int order_policy,
                         int max_table_width, void* buf, size_t buf_bytes, int64_t* running_ids,
                         kv_step_layout* layout) {
  if (!s || !buf || !layout || (n_finished > 0 && !finished_ids) || n_finished < 0 || max_table_width < 1 ||
      (order_policy != KV_ORDER_BATCH && order_policy != KV_ORDER_LONGEST && order_policy != KV_ORDER_LONG_FIRST))
    return fail(KV_ERR_ARG, "bad argument");
  if (reinterpret_cast<uintptr_t>(buf) % kAlign) return fail(KV_ERR_ARG, "buffer not 16-byte aligned");
  kv_step_info info{};
  int rc = kv_sched_step(s, finished_ids, n_finished, &info);
  if (rc != KV_OK) return rc;
  int so = 0, si = 0;
  kv_sched_swap_info(s, &so, &si, nullptr, nullptr, nullptr, nullptr);
  const int b = info.batch, t = info.num_tokens, c = info.num_cow, a = info.num_admitted;
  const int w = std::max(info.max_blocks, 1);
  const bool ord = order_policy != KV_ORDER_BATCH;
  if (w > max_table_width)
    return fail(KV_ERR_ARG, "the step's longest block table (%d) exceeds the table width %d; the scheduler "
                "step is taken", w, max_table_width);
  const int64_t need = packed_bytes(t, b, w, c, so, si, a, ord);
  if (need > (int64_t)buf_bytes)
    return fail(KV_ERR_ARG, "the step's metadata (%lld bytes) exceeds the buffer (%zu); the scheduler step is "
                "taken", (long long)need, buf_bytes);

  kv_step_layout L{};
  L.info = info;
  L.table_width = w;
  L.num_swap_out = so;
  L.num_swap_in = si;
  int64_t off = 0;
  auto place = [&](int64_t n_bytes, bool present) -> int64_t {
    if (!present) return -1;
    const int64_t at = off;
    off += up16(n_bytes);
    return at;
  };
  L.slot_mapping = place(8 * (int64_t)t, true);
  L.block_tables = place(4 * (int64_t)b * w, true);
  L.context_lens = place(4 * (int64_t)b, true);
  L.seq_order = place(4 * (int64_t)b, ord);
  L.cow_pairs = place(8 * (int64_t)c, true);
  L.swap_out_pairs = place(8 * (int64_t)so, true);
  L.swap_in_pairs = place(8 * (int64_t)si, true);
  L.cu_seqlens = place(4 * ((int64_t)a + 1), a > 0);
  L.prefill_context_lens = place(4 * (int64_t)a, a > 0);
  L.bytes = off;

  uint8_t* p = static_cast<uint8_t*>(buf);
  auto at = [&](int64_t o) { return o < 0 ? nullptr : p + o; };
  int32_t* lens = reinterpret_cast<int32_t*>(at(L.context_lens));
  rc = kv_sched_outputs(s, running_ids, reinterpret_cast<int32_t*>(at(L.block_tables)), w, lens,
                        reinterpret_cast<int64_t*>(at(L.slot_mapping)), reinterpret_cast<int32_t*>(at(L.cow_pairs)),
                        nullptr);
  if (rc != KV_OK) return rc;
  if (so || si) {
    rc = kv_sched_swap_outputs(s, reinterpret_cast<int32_t*>(at(L.swap_out_pairs)),
                               reinterpret_cast<int32_t*>(at(L.swap_in_pairs)), nullptr, nullptr, nullptr);
    if (rc != KV_OK) return rc;
  }
  int max_ctx = 0;
  for (int i = 0; i < b; ++i) max_ctx = std::max(max_ctx, (int)lens[i]);
  L.max_context_len = max_ctx;
  if (ord) order_of(lens, b, order_policy, reinterpret_cast<int32_t*>(at(L.seq_order)));
  if (a > 0) {
    // the admitted requests are the last a rows of the running set; each
    // prompt is its context minus this step's appended token, of which the
    // prefix cache supplied `cached` tokens
    std::vector<int32_t> cached(a);
    rc = kv_sched_admitted_cached(s, cached.data());
    if (rc != KV_OK) return rc;
    int32_t* cu = reinterpret_cast<int32_t*>(at(L.cu_seqlens));
    int32_t* pl = reinterpret_cast<int32_t*>(at(L.prefill_context_lens));
    cu[0] = 0;
    int max_new = 0;
    for (int i = 0; i < a; ++i) {
      const int prompt = lens[b - a + i] - 1;
      const int fresh = prompt - cached[i];
      cu[i + 1] = cu[i] + fresh;
      pl[i] = prompt;
      max_new = std::max(max_new, fresh);
    }
    L.prefill_tokens = cu[a];
    L.max_prefill_len = max_new;
  }
  *layout = L;
  return ok();
}

size_t kv_serve_workspace_bytes(const kv_pool* pool, int num_q_heads, int max_batch, int max_context_len) {
  // the split policy partitions more finely when fewer sequences run, so the
  // need is the largest over every batch size
  size_t need = 0;
  for (int b = 1; b <= max_batch; ++b)
    need = std::max(need, paged_attention_workspace_bytes(pool, b, num_q_heads, max_context_len));
  return need;
}

int kv_serve_create(kv_pool* pool, kv_sched* sched, int num_q_heads, kv_dtype q_dtype, float scale,
                    int order_policy, int max_batch, int max_tokens, int max_table_width, void* host_swap,
                    int swap_slots, int num_sets, void* const* host_meta, void* const* dev_meta,
                    size_t meta_bytes, void* workspace, size_t workspace_bytes, kv_serve** out) {
  if (!pool || !sched || !out || !host_meta || !dev_meta || num_q_heads <= 0 || max_batch <= 0 ||
      num_sets < 2 || num_sets > KV_SERVE_MAX_SETS ||
      max_tokens < 0 || max_table_width < 1 || swap_slots < 0 || (swap_slots > 0 && !host_swap) ||
      (order_policy != KV_ORDER_BATCH && order_policy != KV_ORDER_LONGEST && order_policy != KV_ORDER_LONG_FIRST))
    return fail(KV_ERR_ARG, "bad argument");
  for (int i = 0; i < num_sets; ++i) {
    if (!host_meta[i] || !dev_meta[i]) return fail(KV_ERR_ARG, "NULL metadata buffer");
    if (reinterpret_cast<uintptr_t>(host_meta[i]) % kAlign || reinterpret_cast<uintptr_t>(dev_meta[i]) % kAlign)
      return fail(KV_ERR_ARG, "metadata buffers must be 16-byte aligned");
  }
  if (meta_bytes < kv_step_packed_bytes(max_batch, max_tokens, max_table_width, swap_slots))
    return fail(KV_ERR_ARG, "metadata buffers of %zu bytes, %zu needed", meta_bytes,
                kv_step_packed_bytes(max_batch, max_tokens, max_table_width, swap_slots));
  kv_serve* s = new (std::nothrow) kv_serve();
  if (!s) return fail(KV_ERR_OOM, "host allocation failed");
  s->pool = pool;
  s->sched = sched;
  s->hq = num_q_heads;
  s->q_dtype = q_dtype;
  s->scale = scale;
  s->order = order_policy;
  s->max_batch = max_batch;
  s->max_tokens = max_tokens;
  s->max_width = max_table_width;
  s->host_swap = host_swap;
  s->swap_slots = swap_slots;
  s->sets = num_sets;
  s->k = num_sets - 1;
  for (int i = 0; i < num_sets; ++i) {
    s->h[i] = static_cast<uint8_t*>(host_meta[i]);
    s->d[i] = static_cast<uint8_t*>(dev_meta[i]);
  }
  s->meta_bytes = meta_bytes;
  s->ws = workspace;
  s->ws_bytes = workspace ? workspace_bytes : 0;
  for (int i = 0; i < num_sets; ++i) {
    if (cudaEventCreateWithFlags(&s->copy_ev[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s->done_ev[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s->rb_ev[i], cudaEventDisableTiming) != cudaSuccess) {
      const cudaError_t e = cudaGetLastError();
      kv_serve_destroy(s);
      return fail(KV_ERR_CUDA, "cudaEventCreate: %s", cudaGetErrorString(e));
    }
  }
  *out = s;
  return ok();
}

int kv_serve_schedule(kv_serve* s, const int64_t* finished_ids, int n_finished, kv_stream_t upload_stream,
                      int64_t* running_ids, kv_step_layout* layout) {
  if (!s) return fail(KV_ERR_ARG, "NULL serving loop");
  if (s->scheduled && s->launches == 0)
    return fail(KV_ERR_STATE, "the previous step was scheduled but never launched");
  const int k = (s->k + 1) % s->sets;
  // the pinned buffer is rewritten: its last upload must have finished
  if (s->copy_rec[k] && cudaEventSynchronize(s->copy_ev[k]) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaEventSynchronize: %s", cudaGetErrorString(cudaGetLastError()));
  kv_step_layout L{};
  int rc = kv_sched_step_packed(s->sched, finished_ids, n_finished, s->order, s->max_width, s->h[k],
                                s->meta_bytes, nullptr, &L);
  if (rc != KV_OK) return rc;
  if (L.info.batch > s->max_batch || L.info.num_tokens > s->max_tokens)
    return fail(KV_ERR_ARG, "the step (batch %d, %d tokens) exceeds the loop's sizes; the scheduler step is taken",
                L.info.batch, L.info.num_tokens);
  // only now that the batch is known to fit the caller's max_batch rows
  if (running_ids) {
    rc = kv_sched_outputs(s->sched, running_ids, nullptr, 0, nullptr, nullptr, nullptr, nullptr);
    if (rc != KV_OK) return rc;
  }
  if ((L.num_swap_out || L.num_swap_in) && !s->host_swap)
    return fail(KV_ERR_STATE, "the step swaps but the loop has no host swap space; the scheduler step is taken");
  cudaStream_t up = reinterpret_cast<cudaStream_t>(upload_stream);
  // the device buffer is rewritten: the kernels that last read it (the step
  // num_sets before this one) must be done
  if (s->done_rec[k] && cudaStreamWaitEvent(up, s->done_ev[k], 0) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaStreamWaitEvent: %s", cudaGetErrorString(cudaGetLastError()));
  if (L.bytes > 0 && cudaMemcpyAsync(s->d[k], s->h[k], (size_t)L.bytes, cudaMemcpyHostToDevice, up) != cudaSuccess)
    return fail(KV_ERR_CUDA, "metadata upload: %s", cudaGetErrorString(cudaGetLastError()));
  if (cudaEventRecord(s->copy_ev[k], up) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(cudaGetLastError()));
  s->copy_rec[k] = true;
  s->k = k;
  s->up = up;
  L.buffer = k;
  s->lay = L;
  s->scheduled = true;
  s->launches = 0;
  if (layout) *layout = L;
  return ok();
}

int kv_serve_launch(kv_serve* s, int layer, const void* q, const void* k_new, const void* v_new,
                    const float* k_inv_scale, const float* v_inv_scale, void* out, kv_dtype out_dtype,
                    const void* prefill_q, void* prefill_out, kv_stream_t stream) {
  if (!s) return fail(KV_ERR_ARG, "NULL serving loop");
  if (!s->scheduled) return fail(KV_ERR_STATE, "no step scheduled");
  const kv_step_layout& L = s->lay;
  const int b = L.info.batch, t = L.info.num_tokens, c = L.info.num_cow, a = L.info.num_admitted;
  if ((b > 0 && (!q || !out)) || (t > 0 && (!k_new || !v_new)) || ((prefill_q != nullptr) != (prefill_out != nullptr)))
    return fail(KV_ERR_ARG, "bad argument");
  size_t need = 0;
  if (b > 0) {
    need = paged_attention_workspace_bytes(s->pool, b, s->hq, L.max_context_len);
    if (need > s->ws_bytes) return fail(KV_ERR_ARG, "decode workspace of %zu bytes, %zu needed", s->ws_bytes, need);
  }
  const int k = s->k;
  uint8_t* d = s->d[k];
  auto i32 = [&](int64_t o) { return o < 0 ? nullptr : reinterpret_cast<const int32_t*>(d + o); };
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamWaitEvent(st, s->copy_ev[k], 0) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaStreamWaitEvent: %s", cudaGetErrorString(cudaGetLastError()));
  // outputs of set k are overwritten only after their last read-back
  if (s->launches == 0 && s->rb_rec[k] && cudaStreamWaitEvent(st, s->rb_ev[k], 0) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaStreamWaitEvent: %s", cudaGetErrorString(cudaGetLastError()));
  int rc = KV_OK;
  if (s->launches == 0) {
    // once per step, all layers: swaps before this step's writes can reuse
    // the freed blocks, then the copy-on-write pairs
    if (L.num_swap_out)
      rc = kv_swap_out(s->pool, s->host_swap, s->swap_slots, i32(L.swap_out_pairs), L.num_swap_out, stream);
    if (rc == KV_OK && L.num_swap_in)
      rc = kv_swap_in(s->pool, s->host_swap, s->swap_slots, i32(L.swap_in_pairs), L.num_swap_in, stream);
    if (rc == KV_OK && c) rc = block_copy(s->pool, i32(L.cow_pairs), c, stream);
  }
  if (rc == KV_OK && t)
    rc = paged_kv_write(s->pool, layer, k_new, v_new, s->q_dtype,
                        reinterpret_cast<const int64_t*>(d + L.slot_mapping), t, k_inv_scale, v_inv_scale, stream);
  if (rc == KV_OK && a && prefill_q && L.prefill_tokens > 0)
    rc = paged_attention_prefill(s->pool, layer, prefill_q, s->q_dtype, s->hq, i32(L.cu_seqlens), L.prefill_tokens,
                                 L.max_prefill_len, i32(L.block_tables) + (size_t)(b - a) * L.table_width,
                                 L.table_width, i32(L.prefill_context_lens), a, s->scale, prefill_out, out_dtype,
                                 stream);
  if (rc == KV_OK && b)
    rc = paged_attention_decode(s->pool, layer, q, s->q_dtype, s->hq, i32(L.block_tables), L.table_width,
                                i32(L.context_lens), b, L.max_context_len, s->scale, out, out_dtype, s->ws, need,
                                i32(L.seq_order), stream);
  // recorded even after a failed enqueue, so the buffer's reuse still waits
  // for whatever was enqueued
  if (cudaEventRecord(s->done_ev[k], st) != cudaSuccess && rc == KV_OK)
    rc = fail(KV_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(cudaGetLastError()));
  s->done_rec[k] = true;
  s->launches++;
  return rc;
}

int kv_serve_upload(kv_serve* s, void* dev_dst, const void* host_src, size_t bytes) {
  if (!s || (bytes && (!dev_dst || !host_src))) return fail(KV_ERR_ARG, "bad argument");
  if (!s->scheduled || s->launches) return fail(KV_ERR_STATE, "uploads go between kv_serve_schedule and the step's launch");
  if (!bytes) return ok();
  const int k = s->k;
  if (cudaMemcpyAsync(dev_dst, host_src, bytes, cudaMemcpyHostToDevice, s->up) != cudaSuccess)
    return fail(KV_ERR_CUDA, "upload: %s", cudaGetErrorString(cudaGetLastError()));
  if (cudaEventRecord(s->copy_ev[k], s->up) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(cudaGetLastError()));
  return ok();
}

int kv_serve_readback(kv_serve* s, void* host_dst, const void* dev_src, size_t bytes, kv_stream_t readback_stream) {
  if (!s || (bytes && (!host_dst || !dev_src))) return fail(KV_ERR_ARG, "bad argument");
  if (!s->scheduled || !s->launches) return fail(KV_ERR_STATE, "read-back goes after the step's launch");
  const int k = s->k;
  cudaStream_t rb = reinterpret_cast<cudaStream_t>(readback_stream);
  if (cudaStreamWaitEvent(rb, s->done_ev[k], 0) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaStreamWaitEvent: %s", cudaGetErrorString(cudaGetLastError()));
  if (bytes && cudaMemcpyAsync(host_dst, dev_src, bytes, cudaMemcpyDeviceToHost, rb) != cudaSuccess)
    return fail(KV_ERR_CUDA, "read-back: %s", cudaGetErrorString(cudaGetLastError()));
  if (cudaEventRecord(s->rb_ev[k], rb) != cudaSuccess)
    return fail(KV_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(cudaGetLastError()));
  s->rb_rec[k] = true;
  return ok();
}

int kv_serve_destroy(kv_serve* s) {
  if (!s) return ok();
  for (int i = 0; i < KV_SERVE_MAX_SETS; ++i) {
    if (s->rb_ev[i]) {
      cudaEventSynchronize(s->rb_ev[i]);
      cudaEventDestroy(s->rb_ev[i]);
    }
    if (s->copy_ev[i]) {
      cudaEventSynchronize(s->copy_ev[i]);
      cudaEventDestroy(s->copy_ev[i]);
    }
    if (s->done_ev[i]) {
      cudaEventSynchronize(s->done_ev[i]);
      cudaEventDestroy(s->done_ev[i]);
    }
  }
  delete s;
  return ok();
}

}  // extern "C"
