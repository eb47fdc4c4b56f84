// C ABI of multi-token attention over the paged cache: argument checks, the
// query tensor map and the launch.  The kernel is in prefill.cuh.

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "host_common.h"
#include "pool.h"
#include "prefill.cuh"

using pagedkv::fail;
using pagedkv::ok;

namespace pagedkv {

int* device_error_word();  // pagedkv.cu: the library's device error word

namespace {

constexpr int kMaxDevices = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

int cuda_fail(cudaError_t e, const char* what) {
  (void)cudaGetLastError();
  return fail(KV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Query view [total_q][num_q_heads][head_dim] as x = head_dim, y = query
// head, z = row; one box = 64 columns x the g heads of a kv head x 128 / g
// rows, i.e. a 128-row x 128-byte tile in the 128-byte swizzled layout.
int make_q_map(const void* q, int total_q, int num_q_heads, int head_dim, int group, int tq,
               CUtensorMap* map) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)total_q};
  cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)head_dim * 2 * num_q_heads};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)tq};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)r);
  return KV_OK;
}

int* error_word_cached() {
  static std::atomic<int*> words[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::atomic<int*>& w = words[dev % kMaxDevices];
  int* p = w.load(std::memory_order_acquire);
  if (!p) {
    p = device_error_word();
    if (p) w.store(p, std::memory_order_release);
  }
  return p;
}

template <bool kBf16, int D, int STAGES>
int launch(const PrefillParams& p, const CUtensorMap& qmap, const LayerBinding& lb, dim3 grid,
           cudaStream_t stream) {
  using S = PrefillShape<D, STAGES>;
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const uint64_t bit = 1ull << (dev % kMaxDevices);
  if (!(done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(paged_prefill_kernel<kBf16, D, STAGES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (prefill)");
    done.fetch_or(bit, std::memory_order_acq_rel);
  }
  paged_prefill_kernel<kBf16, D, STAGES>
      <<<grid, kPfThreads, S::SMEM_BYTES, stream>>>(p, qmap, lb.k_map, lb.v_map);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "paged_prefill_kernel launch");
  return KV_OK;
}

// Stage counts: two K/V stages of 32 KB each at head_dim 128 (next to the two
// 32 KB query tiles), four of 16 KB at 64; both leave one CTA per SM, which
// the 512 TMEM columns need.
template <bool kBf16>
int launch_d(int head_dim, const PrefillParams& p, const CUtensorMap& qmap,
             const LayerBinding& lb, dim3 grid, cudaStream_t stream) {
  return head_dim == 64 ? launch<kBf16, 64, 4>(p, qmap, lb, grid, stream)
                        : launch<kBf16, 128, 2>(p, qmap, lb, grid, stream);
}

static_assert(PrefillShape<128, 2>::SMEM_BYTES <= 227 * 1024, "prefill shared memory");
static_assert(PrefillShape<64, 4>::SMEM_BYTES * 2 > 228 * 1024, "one prefill CTA per SM");
static_assert(PrefillShape<128, 2>::SMEM_BYTES * 2 > 228 * 1024, "one prefill CTA per SM");

}  // namespace

int prefix_partials(const kv_pool* pool, int layer, const void* q_rows, int num_rows, int num_q_heads,
                    const int32_t* prefix_blocks, int num_prefix_blocks, const int32_t* meta,
                    float scale, float* part_o, float* part_ml, const int32_t* prefix_rows,
                    int num_parts, kv_stream_t stream) {
  const LayerBinding& lb = pool->layers[layer];
  const int g = num_q_heads / pool->kv_heads;
  const int tq = kPfRows / g;
  const int64_t pairs = ((int64_t)num_rows + kPfTiles * tq - 1) / (kPfTiles * tq);
  int* err = error_word_cached();
  if (!err) return fail(KV_ERR_CUDA, "device error word unavailable");
  CUtensorMap qmap;
  int rc = make_q_map(q_rows, num_rows, num_q_heads, pool->head_dim, g, tq, &qmap);
  if (rc != KV_OK) return rc;
  PrefillParams p;
  p.cu_q = meta;              // {0, num_rows}: one sequence of num_rows new tokens
  p.block_tables = prefix_blocks;
  p.context_lens = meta + 2;  // {prefix_len}
  p.out = part_o;             // unused: the epilogue writes partials
  p.err = err;
  p.out_kind = PF_OUT_F32;
  p.num_q_heads = num_q_heads;
  p.group = g;
  p.tokens_per_tile = tq;
  p.num_q_pairs = (int)pairs;
  p.kv_heads = pool->kv_heads;
  p.block_size = pool->block_size;
  p.num_blocks = pool->num_blocks;
  p.max_blocks = num_prefix_blocks;
  p.total_q = num_rows;
  p.window = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.batch = 1;
  p.num_items = pairs * pool->kv_heads;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.prefix_rows = prefix_rows;
  p.num_parts = num_parts;
  const dim3 grid((unsigned)p.num_items);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return pool->dtype == KV_BF16 ? launch_d<true>(pool->head_dim, p, qmap, lb, grid, s)
                                : launch_d<false>(pool->head_dim, p, qmap, lb, grid, s);
}

}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

int paged_attention_prefill(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                            int num_q_heads, const int32_t* cu_seqlens_q, int total_q,
                            int max_q_len, const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int batch, float scale, void* out,
                            kv_dtype out_dtype, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (layer < 0 || layer >= pool->num_layers) return fail(KV_ERR_ARG, "layer %d out of range", layer);
  const LayerBinding& lb = pool->layers[layer];
  if (!lb.bound) return fail(KV_ERR_STATE, "layer %d is not bound", layer);
  if (pool->dtype != KV_F16 && pool->dtype != KV_BF16)
    return fail(KV_ERR_ARG, "multi-token attention needs an f16 or bf16 pool");
  if (pool->head_dim != 64 && pool->head_dim != 128)
    return fail(KV_ERR_ARG, "multi-token attention needs head_dim 64 or 128");
  if (q_dtype != pool->dtype) return fail(KV_ERR_ARG, "q dtype must equal the pool dtype");
  if (out_dtype != q_dtype && out_dtype != KV_F32)
    return fail(KV_ERR_ARG, "out dtype must be the q dtype or KV_F32");
  if (batch < 0 || total_q < 0 || max_q_len < 0 || max_blocks_per_seq < 0)
    return fail(KV_ERR_ARG, "negative size");
  if (batch > 65535) return fail(KV_ERR_ARG, "batch %d above 65535", batch);
  if (pool->kv_heads > 65535) return fail(KV_ERR_ARG, "kv_heads above 65535");
  if (num_q_heads <= 0 || num_q_heads % pool->kv_heads != 0 || num_q_heads / pool->kv_heads > 8)
    return fail(KV_ERR_ARG, "num_q_heads %d must be a multiple of kv_heads %d, at most 8x",
                num_q_heads, pool->kv_heads);
  if (!std::isfinite(scale) || !(scale > 0.f)) return fail(KV_ERR_ARG, "scale must be finite and > 0");
  if (batch == 0 || total_q == 0 || max_q_len == 0) return ok();
  if (!q || !cu_seqlens_q || !block_tables || !context_lens || !out)
    return fail(KV_ERR_ARG, "NULL input");
  if (((uintptr_t)q & 15) || ((uintptr_t)out & 15))
    return fail(KV_ERR_ARG, "q and out must be 16-byte aligned");
  if (max_blocks_per_seq == 0) return fail(KV_ERR_ARG, "max_blocks_per_seq must be positive");

  const int g = num_q_heads / pool->kv_heads;
  const int tq = kPfRows / g;
  const int64_t pairs = ((int64_t)max_q_len + kPfTiles * tq - 1) / (kPfTiles * tq);
  if (pairs > 0x7fffffff) return fail(KV_ERR_ARG, "max_q_len too large");
  int* err = error_word_cached();
  if (!err) return fail(KV_ERR_CUDA, "device error word unavailable");

  CUtensorMap qmap;
  int rc = make_q_map(q, total_q, num_q_heads, pool->head_dim, g, tq, &qmap);
  if (rc != KV_OK) return rc;

  PrefillParams p;
  p.cu_q = cu_seqlens_q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.out = out;
  p.err = err;
  p.out_kind = out_dtype == KV_F32 ? PF_OUT_F32 : (out_dtype == KV_BF16 ? PF_OUT_BF16 : PF_OUT_F16);
  p.num_q_heads = num_q_heads;
  p.group = g;
  p.tokens_per_tile = tq;
  p.num_q_pairs = (int)pairs;
  p.kv_heads = pool->kv_heads;
  p.block_size = pool->block_size;
  p.num_blocks = pool->num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.total_q = total_q;
  p.window = pool->window;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.batch = batch;
  p.num_items = pairs * pool->kv_heads * batch;
  if (p.num_items > 0x7fffffff) return fail(KV_ERR_ARG, "too many query tiles");
  p.part_o = nullptr;
  p.part_ml = nullptr;
  p.prefix_rows = nullptr;
  p.num_parts = 0;

  // one CTA per work item, heaviest first; a CTA that finishes an item
  // cancels the launch of a CTA not yet started and takes over its item
  const dim3 grid((unsigned)p.num_items);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = pool->dtype == KV_BF16 ? launch_d<true>(pool->head_dim, p, qmap, lb, grid, s)
                              : launch_d<false>(pool->head_dim, p, qmap, lb, grid, s);
  if (rc != KV_OK) return rc;
  return ok();
}

}  // extern "C"
