// C ABI of the GPU path: pool descriptors, TMA descriptors, launches.
// All device code lives in this one translation unit (kernels in the .cuh
// files) so every kernel shares one device error word.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "cache.cuh"
#include "decode.cuh"
#include "device_common.cuh"
#include "host_common.h"
#include "pool.h"

using pagedkv::fail;
using pagedkv::ok;

namespace pagedkv {
namespace {

constexpr int kMaxLayers = 4096;
constexpr int kMaxDevices = 64;
constexpr int kMaxSmemPerCta = 227 * 1024;

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

// 3-D view of one layer's K (or V) array: x = head_dim elements, y = kv_heads
// * block_size rows, z = num_blocks; box = (up to 128 bytes of a row) x 16
// rows x 1 block, with the swizzle matching the box row width.
int make_map(const kv_pool* pool, void* base, CUtensorMap* map) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
  const int eb = elem_bytes(pool->dtype);
  const int rowb = pool->head_dim * eb;
  const int boxb = std::min(rowb, 128);
  cuuint64_t dims[3] = {(cuuint64_t)pool->head_dim, (cuuint64_t)pool->kv_heads * pool->block_size,
                        (cuuint64_t)pool->num_blocks};
  cuuint64_t strides[2] = {(cuuint64_t)rowb, (cuuint64_t)rowb * pool->kv_heads * pool->block_size};
  cuuint32_t box[3] = {(cuuint32_t)(boxb / eb), (cuuint32_t)kChunk, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 3,
                   base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   boxb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KV_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  (void)cudaGetLastError();  // do not leave this error pending for the next check
  return fail(KV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// cudaFuncSetAttribute once per (kernel, device); `done` must be a flag word
// owned by that kernel alone.
template <class K>
int ensure_smem(K kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const uint64_t bit = 1ull << (dev % kMaxDevices);
  if (done.load(std::memory_order_acquire) & bit) return KV_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done.fetch_or(bit, std::memory_order_acq_rel);
  return KV_OK;
}

// Pipeline shape: warps per CTA and stages per warp.  4 warps of 3 stages of
// 8 KB (16-bit, D 128: two CTAs per SM) for single heads and small groups;
// 2 stages (three CTAs per SM) for GQA groups of 4 or more, whose shared
// prefixes are read from L2 with shorter latency and whose CTAs cover fewer
// chunks; 3 stages of 4 KB (FP8 D 128, 16-bit D 64: four and three CTAs per
// SM); 6 stages of 2 KB.  Measured on B200: more warps per CTA or deeper rings
// were slower for every format.
struct PipeShape {
  int warps;
  int stages;
};

PipeShape pipe_for(kv_dtype dtype, int head_dim, int group, int stages, int warps) {
  const int stage_bytes = 2 * kChunk * head_dim * elem_bytes(dtype);
  PipeShape ps;
  if (stage_bytes >= 8192) ps = {4, group >= 4 ? 2 : 3};
  else if (stage_bytes >= 4096) ps = {4, 3};
  else ps = {4, 6};
  if (warps > 0) ps.warps = warps;
  if (stages > 0) ps.stages = stages;
  return ps;
}

PipeShape pipe_for(const kv_pool* pool, int group) {
  return pipe_for(pool->dtype, pool->head_dim, group, pool->stages, pool->warps);
}

template <int KV, int D, int W>
int smem_bytes_w(int stages) {
  switch (stages) {
    case 2: return DecodeShape<KV, D, W, 2>::MAX_SMEM_BYTES;
    case 3: return DecodeShape<KV, D, W, 3>::MAX_SMEM_BYTES;
    case 4: return DecodeShape<KV, D, W, 4>::MAX_SMEM_BYTES;
    case 6: return DecodeShape<KV, D, W, 6>::MAX_SMEM_BYTES;
    default: return DecodeShape<KV, D, W, 8>::MAX_SMEM_BYTES;
  }
}

template <int KV, int D>
int smem_bytes_d(PipeShape ps) {
  return ps.warps == 8 ? smem_bytes_w<KV, D, 8>(ps.stages) : smem_bytes_w<KV, D, 4>(ps.stages);
}

int smem_bytes(kv_dtype dtype, int head_dim, PipeShape ps) {
  const bool d64 = head_dim == 64;
  switch (dtype) {
    case KV_FP8_E4M3: return d64 ? smem_bytes_d<KV_KIND_E4M3, 64>(ps) : smem_bytes_d<KV_KIND_E4M3, 128>(ps);
    default: return d64 ? smem_bytes_d<KV_KIND_F16, 64>(ps) : smem_bytes_d<KV_KIND_F16, 128>(ps);
  }
}

int decode_occupancy(const kv_pool* pool, int group);  // defined with the launchers below

// Resident decode CTAs the current device holds at once.
int decode_slots(const kv_pool* pool, int group) {
  static std::atomic<int> sm_count[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  int sms = sm_count[dev % kMaxDevices].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
      (void)cudaGetLastError();
      sms = 148;
    }
    sm_count[dev % kMaxDevices].store(sms, std::memory_order_relaxed);
  }
  return sms * decode_occupancy(pool, group);
}

// Partition length in tokens.  Automatic: contexts are cut into partitions
// of at most kAutoPartition tokens.  If the (sequence, kv head) units then
// give fewer than kWavesKeep waves of resident CTAs, contexts are split
// further, into enough partitions (of at least kMinPartition tokens) for
// kWavesSplit waves, and then possibly a few more so that the last wave is
// nearly full.  Measured on B200: unsplit 2K-token contexts with 1024 units
// (32-layer example, 3.5 waves), 4K-token partitions for a 256-sequence
// lognormal batch (few long contexts; the others skip the reduce), 1K-token
// partitions for 8 x 16K-token FP8 contexts (256 units); a 4K-token window
// over 8 x 16K-token bf16 contexts runs the same with 0.5K to 1.4K-token
// partitions.
// The decode merges its own split partials up to this many partitions per
// context (measured in-kernel against the separate reduce: GQA trace, 3
// partitions, +3%; FP8 16K contexts, 16 and 32, -3% and -9%; a 4K-token
// window, 8, -3%).
constexpr int kFusedMergeMaxParts = 4;
constexpr int kWavesKeep = 3;
constexpr int kWavesSplit = 4;
constexpr int kAutoPartition = 4096;
constexpr int kMinPartition = 512;
constexpr int kWaveFillPct = 85;

int partition_tokens(const kv_pool* pool, int batch, int max_context_len, int group) {
  if (pool->partition_tokens > 0) return pool->partition_tokens;
  const int ctx = std::max(max_context_len, 1);
  const int64_t units = std::max<int64_t>(1, (int64_t)batch * pool->kv_heads);
  const int64_t slots = decode_slots(pool, group);
  auto per_of = [&](int64_t n) {  // tokens per partition for n partitions
    const int64_t per = (ctx + n - 1) / n;
    return std::min<int64_t>(kChunk * kMaxPartChunks, (per + kChunk - 1) / kChunk * kChunk);
  };
  int64_t np = (ctx + kAutoPartition - 1) / kAutoPartition;
  if (units < (int64_t)kWavesKeep * slots) {
    const int64_t np_cap = std::max<int64_t>(1, (ctx + kMinPartition - 1) / kMinPartition);
    np = std::max<int64_t>(np, (kWavesSplit * slots + units - 1) / units);
    np = std::min<int64_t>(np, np_cap);
    // Equal partitions finish in waves of `slots` CTAs: take the smallest
    // count up to twice that whose last wave is at least kWaveFillPct % full
    // (measured: 8 x 16K-token FP8 contexts, 32 heads, as 16 partitions of
    // 1024 tokens, 6.9 waves, ran 2% faster than as 10 of 1648, 4.3 waves).
    for (int64_t n = np; n <= std::min<int64_t>(2 * np, np_cap); ++n) {
      const int64_t parts = (ctx + per_of(n) - 1) / per_of(n);
      const int64_t rem = units * parts % slots;
      if (rem == 0 || rem * 100 >= slots * kWaveFillPct) {
        np = n;
        break;
      }
    }
  }
  return (int)per_of(np);
}

int num_parts_for(const kv_pool* pool, int batch, int max_context_len, int group) {
  const int pt = partition_tokens(pool, batch, max_context_len, group);
  return std::max(1, (max_context_len + pt - 1) / pt);
}

// Upper bound on the tokens one decode visits per sequence: with a sliding
// window of W tokens, the chunks from the one holding the window's first
// token to the last, i.e. at most 16 * ceil(W / 16) + 16.
int visited_len(const kv_pool* pool, int max_context_len) {
  if (pool->window <= 0) return max_context_len;
  const int64_t w = ((int64_t)pool->window + kChunk - 1) / kChunk * kChunk + kChunk;
  return (int)std::min<int64_t>(max_context_len, w);
}

// Resident CTAs per SM of one decode instantiation on the current device
// (occupancy API; registers and shared memory both count), with the chunk
// tables of the automatic policy's longest partition.
template <int KV, int D, int W, int STAGES>
int decode_occupancy() {
  using Shape = DecodeShape<KV, D, W, STAGES>;
  auto kernel = paged_decode_kernel<KV, D, W, STAGES, false>;
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  int v = cached[dev % kMaxDevices].load(std::memory_order_relaxed);
  if (v > 0) return v;
  const int smem = Shape::smem_bytes(kAutoPartition / kChunk);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Shape::MAX_SMEM_BYTES) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, W * 32, smem) != cudaSuccess ||
      v <= 0) {
    (void)cudaGetLastError();
    v = std::max(1, kMaxSmemPerCta / smem);  // no device: shared-memory bound
  }
  cached[dev % kMaxDevices].store(v, std::memory_order_relaxed);
  return v;
}

template <int KV, int D, int W>
int occupancy_w(int stages) {
  switch (stages) {
    case 2: return decode_occupancy<KV, D, W, 2>();
    case 3: return decode_occupancy<KV, D, W, 3>();
    case 4: return decode_occupancy<KV, D, W, 4>();
    case 6: return decode_occupancy<KV, D, W, 6>();
    default: return decode_occupancy<KV, D, W, 8>();
  }
}

template <int KV, int D>
int occupancy_d(PipeShape ps) {
  return ps.warps == 8 ? occupancy_w<KV, D, 8>(ps.stages) : occupancy_w<KV, D, 4>(ps.stages);
}

int decode_occupancy(const kv_pool* pool, int group) {
  const PipeShape ps = pipe_for(pool, group);
  const bool d64 = pool->head_dim == 64;
  switch (pool->dtype) {
    case KV_FP8_E4M3: return d64 ? occupancy_d<KV_KIND_E4M3, 64>(ps) : occupancy_d<KV_KIND_E4M3, 128>(ps);
    case KV_BF16: return d64 ? occupancy_d<KV_KIND_BF16, 64>(ps) : occupancy_d<KV_KIND_BF16, 128>(ps);
    default: return d64 ? occupancy_d<KV_KIND_F16, 64>(ps) : occupancy_d<KV_KIND_F16, 128>(ps);
  }
}

template <int KV, int D, int W, int STAGES, bool EXT>
int launch_decode_x(const DecodeParams& p, const LayerBinding& lb, dim3 grid, cudaStream_t stream) {
  using Shape = DecodeShape<KV, D, W, STAGES>;
  auto kernel = paged_decode_kernel<KV, D, W, STAGES, EXT>;
  static std::atomic<uint64_t> done{0};  // one flag word per instantiation
  int rc = ensure_smem(kernel, Shape::MAX_SMEM_BYTES, done);
  if (rc != KV_OK) return rc;
  kernel<<<grid, W * 32, Shape::smem_bytes(p.part_chunks), stream>>>(p, lb.k_map, lb.v_map);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "paged_decode_kernel launch");
  return KV_OK;
}

// Decodes that skip prefixes or merge their own partials run the extended
// instantiation (16-bit caches; FP8 callers pass neither)
template <int KV, int D, int W, int STAGES>
int launch_decode_t(const DecodeParams& p, const LayerBinding& lb, dim3 grid, cudaStream_t stream) {
  if constexpr (KV != KV_KIND_E4M3) {
    if (p.skip != nullptr || p.counters != nullptr)
      return launch_decode_x<KV, D, W, STAGES, true>(p, lb, grid, stream);
  } else {
    if (p.skip != nullptr || p.counters != nullptr) return fail(KV_ERR_ARG, "FP8 decode takes no skip or counters");
  }
  return launch_decode_x<KV, D, W, STAGES, false>(p, lb, grid, stream);
}

template <int KV, int D, int W>
int launch_decode_w(int stages, const DecodeParams& p, const LayerBinding& lb, dim3 grid,
                    cudaStream_t stream) {
  switch (stages) {
    case 2: return launch_decode_t<KV, D, W, 2>(p, lb, grid, stream);
    case 3: return launch_decode_t<KV, D, W, 3>(p, lb, grid, stream);
    case 4: return launch_decode_t<KV, D, W, 4>(p, lb, grid, stream);
    case 6: return launch_decode_t<KV, D, W, 6>(p, lb, grid, stream);
    case 8: return launch_decode_t<KV, D, W, 8>(p, lb, grid, stream);
    default: return fail(KV_ERR_ARG, "unsupported stage count %d", stages);
  }
}

template <int KV>
int launch_decode_kv(int head_dim, PipeShape ps, const DecodeParams& p, const LayerBinding& lb,
                     dim3 grid, cudaStream_t stream) {
  if (head_dim == 64)
    return ps.warps == 8 ? launch_decode_w<KV, 64, 8>(ps.stages, p, lb, grid, stream)
                         : launch_decode_w<KV, 64, 4>(ps.stages, p, lb, grid, stream);
  return ps.warps == 8 ? launch_decode_w<KV, 128, 8>(ps.stages, p, lb, grid, stream)
                       : launch_decode_w<KV, 128, 4>(ps.stages, p, lb, grid, stream);
}

bool valid_q_dtype(kv_dtype pool, kv_dtype q) {
  if (pool == KV_FP8_E4M3) return q == KV_F16 || q == KV_BF16;
  return q == pool;
}

int out_kind(kv_dtype t) { return t == KV_F32 ? OUT_F32 : (t == KV_BF16 ? OUT_BF16 : OUT_F16); }

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

namespace pagedkv {

// Device address of the error word, for kernels built in the library's other
// translation units (they record into the same word).
int* device_error_word() {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return static_cast<int*>(p);
}

}  // namespace pagedkv

extern "C" {

int kv_pool_create(int block_size, int num_blocks, int kv_heads, int head_dim, kv_dtype dtype,
                   int num_layers, kv_pool** out) {
  if (!out) return fail(KV_ERR_ARG, "out is NULL");
  if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128 &&
      block_size != 256)
    return fail(KV_ERR_ARG, "block_size %d must be 16, 32, 64, 128 or 256", block_size);
  if (head_dim != 64 && head_dim != 128)
    return fail(KV_ERR_ARG, "head_dim %d unsupported (64 or 128)", head_dim);
  if (dtype != KV_F16 && dtype != KV_BF16 && dtype != KV_FP8_E4M3)
    return fail(KV_ERR_ARG, "pool dtype %d unsupported", (int)dtype);
  if (num_blocks <= 0 || kv_heads <= 0 || num_layers <= 0 || num_layers > kMaxLayers)
    return fail(KV_ERR_ARG, "bad geometry: num_blocks %d kv_heads %d num_layers %d", num_blocks,
                kv_heads, num_layers);
  if ((int64_t)kv_heads * block_size > (1ll << 31))
    return fail(KV_ERR_ARG, "kv_heads * block_size too large");
  kv_pool* p = new (std::nothrow) kv_pool();
  if (!p) return fail(KV_ERR_OOM, "host allocation failed");
  p->block_size = block_size;
  p->num_blocks = num_blocks;
  p->kv_heads = kv_heads;
  p->head_dim = head_dim;
  p->dtype = dtype;
  p->num_layers = num_layers;
  p->layers.resize(num_layers);
  *out = p;
  return ok();
}

int kv_pool_bytes(const kv_pool* pool, size_t* kv_bytes_per_layer, size_t* scale_bytes_per_layer) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (kv_bytes_per_layer) *kv_bytes_per_layer = pool->layer_bytes();
  if (scale_bytes_per_layer) *scale_bytes_per_layer = pool->scale_bytes();
  return ok();
}

int kv_pool_bind(kv_pool* pool, int layer, void* k_base, void* v_base, float* k_scale,
                 float* v_scale) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (layer < 0 || layer >= pool->num_layers)
    return fail(KV_ERR_ARG, "layer %d out of range [0, %d)", layer, pool->num_layers);
  if (!k_base || !v_base) return fail(KV_ERR_ARG, "K/V base is NULL");
  if (((uintptr_t)k_base | (uintptr_t)v_base) & 15)
    return fail(KV_ERR_ARG, "K/V base must be 16-byte aligned");
  const bool fp8 = pool->dtype == KV_FP8_E4M3;
  if (fp8 && (!k_scale || !v_scale)) return fail(KV_ERR_ARG, "FP8 pools need K and V scales");
  if (!fp8 && (k_scale || v_scale)) return fail(KV_ERR_ARG, "scales are only for FP8 pools");
  LayerBinding lb;
  int rc = make_map(pool, k_base, &lb.k_map);
  if (rc != KV_OK) return rc;
  rc = make_map(pool, v_base, &lb.v_map);
  if (rc != KV_OK) return rc;
  lb.k = k_base;
  lb.v = v_base;
  lb.k_scale = k_scale;
  lb.v_scale = v_scale;
  lb.bound = true;
  pool->layers[layer] = lb;
  return ok();
}

int kv_pool_set_decode_config(kv_pool* pool, int partition_tokens, int stages, int warps) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (partition_tokens != 0 &&
      (partition_tokens < kChunk || partition_tokens > kChunk * kMaxPartChunks ||
       partition_tokens % kChunk != 0))
    return fail(KV_ERR_ARG, "partition_tokens %d must be 0 or a multiple of 16 in [16, %d]",
                partition_tokens, kChunk * kMaxPartChunks);
  if (stages != 0 && stages != 2 && stages != 3 && stages != 4 && stages != 6 && stages != 8)
    return fail(KV_ERR_ARG, "stages %d must be 0, 2, 3, 4, 6 or 8", stages);
  if (warps != 0 && warps != 4 && warps != 8)
    return fail(KV_ERR_ARG, "warps %d must be 0, 4 or 8", warps);
  const PipeShape ps = pipe_for(pool->dtype, pool->head_dim, 1, stages, warps);
  const int need = smem_bytes(pool->dtype, pool->head_dim, ps);
  if (need > kMaxSmemPerCta)
    return fail(KV_ERR_ARG, "%d warps x %d stages need %d bytes of shared memory per CTA, above %d",
                ps.warps, ps.stages, need, kMaxSmemPerCta);
  pool->partition_tokens = partition_tokens;
  pool->stages = stages;
  pool->warps = warps;
  return ok();
}

int kv_pool_set_sliding_window(kv_pool* pool, int window) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (window < 0) return fail(KV_ERR_ARG, "window %d must be >= 0", window);
  pool->window = window;
  return ok();
}

int kv_pool_destroy(kv_pool* pool) {
  delete pool;
  return ok();
}

int paged_kv_write(const kv_pool* pool, int layer, const void* k_new, const void* v_new,
                   kv_dtype src_dtype, const int64_t* slot_mapping, int num_tokens,
                   const float* k_inv_scale, const float* v_inv_scale, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (layer < 0 || layer >= pool->num_layers) return fail(KV_ERR_ARG, "layer %d out of range", layer);
  if (num_tokens < 0) return fail(KV_ERR_ARG, "num_tokens < 0");
  const LayerBinding& lb = pool->layers[layer];
  if (!lb.bound) return fail(KV_ERR_STATE, "layer %d is not bound", layer);
  const bool fp8 = pool->dtype == KV_FP8_E4M3;
  if (!valid_q_dtype(pool->dtype, src_dtype))
    return fail(KV_ERR_ARG, "source dtype %d does not fit pool dtype %d", (int)src_dtype,
                (int)pool->dtype);
  if (fp8 && (!k_inv_scale || !v_inv_scale)) return fail(KV_ERR_ARG, "FP8 writes need inverse scales");
  if (num_tokens == 0) return ok();
  if (!k_new || !v_new || !slot_mapping) return fail(KV_ERR_ARG, "NULL input");
  if (((uintptr_t)k_new | (uintptr_t)v_new) & 15) return fail(KV_ERR_ARG, "k_new/v_new must be 16-byte aligned");
  WriteParams p;
  p.k_new = static_cast<const uint8_t*>(k_new);
  p.v_new = static_cast<const uint8_t*>(v_new);
  p.slots = slot_mapping;
  p.k = static_cast<uint8_t*>(lb.k);
  p.v = static_cast<uint8_t*>(lb.v);
  p.k_inv = k_inv_scale;
  p.v_inv = v_inv_scale;
  p.rows = (int64_t)num_tokens * pool->kv_heads;
  p.kv_heads = pool->kv_heads;
  p.head_dim = pool->head_dim;
  p.block_size = pool->block_size;
  p.num_blocks = pool->num_blocks;
  p.src_bf16 = src_dtype == KV_BF16;
  const int64_t threads = p.rows * (pool->head_dim / 8);
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffff) return fail(KV_ERR_ARG, "too many tokens");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (fp8)
    kv_write_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(p);
  else
    kv_write_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kv_write_kernel launch");
  return ok();
}

int block_copy(const kv_pool* pool, const int32_t* pairs, int num_pairs, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (num_pairs < 0 || num_pairs > 0x7fffffff / 2) return fail(KV_ERR_ARG, "bad num_pairs");
  if (num_pairs == 0) return ok();
  if (!pairs) return fail(KV_ERR_ARG, "pairs is NULL");
  for (int l = 0; l < pool->num_layers; ++l)
    if (!pool->layers[l].bound) return fail(KV_ERR_STATE, "layer %d is not bound", l);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int l0 = 0; l0 < pool->num_layers; l0 += kCopyLayers) {
    const int nl = std::min(kCopyLayers, pool->num_layers - l0);
    CopyParams p;
    std::memset(&p, 0, sizeof p);
    p.pairs = pairs;
    p.num_pairs = num_pairs;
    p.num_blocks = pool->num_blocks;
    p.kv_heads = pool->kv_heads;
    p.block_bytes = (int64_t)pool->block_bytes();
    for (int i = 0; i < nl; ++i) {
      const LayerBinding& lb = pool->layers[l0 + i];
      p.k[i] = lb.k;
      p.v[i] = lb.v;
      p.ks[i] = lb.k_scale;
      p.vs[i] = lb.v_scale;
    }
    block_copy_kernel<<<dim3(num_pairs, nl, 2), 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "block_copy_kernel launch");
  }
  return ok();
}

size_t kv_swap_block_bytes(const kv_pool* pool) {
  if (!pool) return 0;
  const size_t scales = pool->dtype == KV_FP8_E4M3 ? ((size_t)pool->kv_heads * 4 + 15) / 16 * 16 : 0;
  return (size_t)pool->num_layers * 2 * (pool->block_bytes() + scales);
}

static int swap_copy(const kv_pool* pool, const void* host_swap, int num_slots, const int32_t* pairs,
                     int num_pairs, bool out, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (num_pairs < 0 || num_slots < 0) return fail(KV_ERR_ARG, "negative size");
  if (num_pairs == 0) return ok();
  if (!pairs || !host_swap) return fail(KV_ERR_ARG, "NULL argument");
  if ((uintptr_t)host_swap & 15) return fail(KV_ERR_ARG, "host swap space must be 16-byte aligned");
  for (int l = 0; l < pool->num_layers; ++l)
    if (!pool->layers[l].bound) return fail(KV_ERR_STATE, "layer %d is not bound", l);
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, host_swap);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr)
    return fail(KV_ERR_ARG, "host swap space must be pinned host memory mapped into the device");
  const int64_t scales = pool->dtype == KV_FP8_E4M3 ? ((int64_t)pool->kv_heads * 4 + 15) / 16 * 16 : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int l0 = 0; l0 < pool->num_layers; l0 += kCopyLayers) {
    const int nl = std::min(kCopyLayers, pool->num_layers - l0);
    SwapParams p;
    std::memset(&p, 0, sizeof p);
    p.pairs = pairs;
    p.num_pairs = num_pairs;
    p.num_blocks = pool->num_blocks;
    p.num_slots = num_slots;
    p.kv_heads = pool->kv_heads;
    p.layer0 = l0;
    p.num_layers = pool->num_layers;
    p.block_bytes = (int64_t)pool->block_bytes();
    p.per_bytes = p.block_bytes + scales;
    p.host = static_cast<uint8_t*>(attr.devicePointer);
    for (int i = 0; i < nl; ++i) {
      const LayerBinding& lb = pool->layers[l0 + i];
      p.k[i] = lb.k;
      p.v[i] = lb.v;
      p.ks[i] = lb.k_scale;
      p.vs[i] = lb.v_scale;
    }
    if (out) swap_kernel<true><<<dim3(num_pairs, nl, 2), 256, 0, s>>>(p);
    else swap_kernel<false><<<dim3(num_pairs, nl, 2), 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swap_kernel launch");
  }
  return ok();
}

int kv_swap_out(const kv_pool* pool, void* host_swap, int num_slots, const int32_t* pairs,
                int num_pairs, kv_stream_t stream) {
  return swap_copy(pool, host_swap, num_slots, pairs, num_pairs, true, stream);
}

int kv_swap_in(const kv_pool* pool, const void* host_swap, int num_slots, const int32_t* pairs,
               int num_pairs, kv_stream_t stream) {
  return swap_copy(pool, host_swap, num_slots, pairs, num_pairs, false, stream);
}

size_t paged_attention_workspace_bytes(const kv_pool* pool, int batch, int num_q_heads,
                                       int max_context_len) {
  if (!pool || batch <= 0 || num_q_heads <= 0 || max_context_len <= 0) return 0;
  const int group = num_q_heads % pool->kv_heads == 0 ? num_q_heads / pool->kv_heads : 1;
  const int np = num_parts_for(pool, batch, visited_len(pool, max_context_len), group);
  if (np <= 1) return 0;
  // partials, then one merge counter per (sequence, kv head)
  return (size_t)batch * num_q_heads * np * (pool->head_dim + 4) * sizeof(float) +
         ((size_t)batch * pool->kv_heads * sizeof(int) + 15) / 16 * 16;
}

}  // extern "C"

namespace pagedkv {
namespace {

// Argument checks shared by the decode entry points.
int check_decode_args(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype, int num_q_heads,
                      const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                      int batch, int max_context_len, float scale, void* out, kv_dtype out_dtype) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  if (layer < 0 || layer >= pool->num_layers) return fail(KV_ERR_ARG, "layer %d out of range", layer);
  if (!pool->layers[layer].bound) return fail(KV_ERR_STATE, "layer %d is not bound", layer);
  if (batch < 0 || max_context_len < 0 || max_blocks_per_seq < 0)
    return fail(KV_ERR_ARG, "negative size");
  if (batch > 65535) return fail(KV_ERR_ARG, "batch %d above 65535", batch);
  if (num_q_heads <= 0 || num_q_heads % pool->kv_heads != 0 ||
      num_q_heads / pool->kv_heads > kMaxGroup)
    return fail(KV_ERR_ARG, "num_q_heads %d must be a multiple of kv_heads %d, at most %dx",
                num_q_heads, pool->kv_heads, kMaxGroup);
  if (pool->kv_heads > 65535) return fail(KV_ERR_ARG, "kv_heads above 65535");
  if (!valid_q_dtype(pool->dtype, q_dtype))
    return fail(KV_ERR_ARG, "q dtype %d does not fit pool dtype %d", (int)q_dtype, (int)pool->dtype);
  if (out_dtype != q_dtype && out_dtype != KV_F32)
    return fail(KV_ERR_ARG, "out dtype must be the q dtype or KV_F32");
  if (!std::isfinite(scale)) return fail(KV_ERR_ARG, "scale is not finite");
  if (batch == 0) return KV_OK;
  if (!q || !block_tables || !context_lens || !out) return fail(KV_ERR_ARG, "NULL input");
  if ((uintptr_t)q & 7) return fail(KV_ERR_ARG, "q must be 8-byte aligned");
  if ((int64_t)max_blocks_per_seq * pool->block_size < max_context_len)
    return fail(KV_ERR_ARG, "max_blocks_per_seq %d cannot hold max_context_len %d",
                max_blocks_per_seq, max_context_len);
  return KV_OK;
}

// The decode launch (and the reduce when more than one partition exists):
// `grid_parts` partitions per sequence in the grid, `stride_parts` partials
// per (sequence, head) in part_o / part_ml, `skip` as in DecodeParams.
int enqueue_decode(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype, int num_q_heads,
                   const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                   int batch, int max_context_len, float scale, void* out, kv_dtype out_dtype,
                   float* part_o, float* part_ml, int grid_parts, int stride_parts, int part_tokens,
                   const int32_t* skip, int* counters, const int32_t* seq_order, cudaStream_t s) {
  const LayerBinding& lb = pool->layers[layer];
  const int group = num_q_heads / pool->kv_heads;
  DecodeParams p;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.skip = skip;
  p.counters = counters;
  p.seq_order = seq_order;
  p.k_scale = lb.k_scale;
  p.v_scale = lb.v_scale;
  p.out = out;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.q_bf16 = q_dtype == KV_BF16;
  p.out_kind = out_kind(out_dtype);
  p.num_q_heads = num_q_heads;
  p.group = group;
  p.kv_heads = pool->kv_heads;
  p.block_size = pool->block_size;
  p.cpb_shift = 0;
  while ((kChunk << p.cpb_shift) < pool->block_size) ++p.cpb_shift;
  p.num_blocks = pool->num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.part_chunks = part_tokens / kChunk;
  p.num_parts = stride_parts;
  p.ctx_cap = (int)std::min<int64_t>((int64_t)max_blocks_per_seq * pool->block_size, max_context_len);
  p.window = pool->window;
  p.scale_log2 = scale * 1.4426950408889634f;

  const dim3 grid(grid_parts, pool->kv_heads, batch);
  const PipeShape ps = pipe_for(pool, group);
  if (counters != nullptr && stride_parts > 1) {
    // the merge counters start at zero in every call (the workspace is the caller's)
    cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)batch * pool->kv_heads * sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (merge counters)");
  }
  int rc;
  switch (pool->dtype) {
    case KV_F16: rc = launch_decode_kv<KV_KIND_F16>(pool->head_dim, ps, p, lb, grid, s); break;
    case KV_BF16: rc = launch_decode_kv<KV_KIND_BF16>(pool->head_dim, ps, p, lb, grid, s); break;
    default: rc = launch_decode_kv<KV_KIND_E4M3>(pool->head_dim, ps, p, lb, grid, s); break;
  }
  if (rc != KV_OK) return rc;
  if (stride_parts > 1 && counters == nullptr) {  // merged by a separate launch
    const int64_t rows = (int64_t)batch * num_q_heads;
    const int blocks = (int)((rows + 7) / 8);
    lse_reduce_kernel<<<blocks, 256, 0, s>>>(p.part_o, p.part_ml, context_lens, out, p.out_kind,
                                             num_q_heads, pool->head_dim, stride_parts, part_tokens,
                                             p.ctx_cap, p.window, batch, skip);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "lse_reduce_kernel launch");
  }
  return KV_OK;
}

}  // namespace
}  // namespace pagedkv

extern "C" {

int paged_attention_decode(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                           int num_q_heads, const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* context_lens, int batch, int max_context_len,
                           float scale, void* out, kv_dtype out_dtype, void* workspace,
                           size_t workspace_bytes, const int32_t* seq_order, kv_stream_t stream) {
  int rc = check_decode_args(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq,
                             context_lens, batch, max_context_len, scale, out, out_dtype);
  if (rc != KV_OK) return rc;
  if (batch == 0) return ok();
  const int visited = visited_len(pool, max_context_len);
  const int group = num_q_heads / pool->kv_heads;
  const int pt = partition_tokens(pool, batch, visited, group);
  const int np = num_parts_for(pool, batch, visited, group);
  if (np > 65535) return fail(KV_ERR_ARG, "too many partitions");
  const size_t need = paged_attention_workspace_bytes(pool, batch, num_q_heads, max_context_len);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(KV_ERR_ARG, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if (need > 0 && ((uintptr_t)workspace & 15)) return fail(KV_ERR_ARG, "workspace must be 16-byte aligned");
  float* ws = static_cast<float*>(workspace);
  float* part_o = need ? ws : nullptr;
  float* part_ml = need ? ws + (size_t)batch * num_q_heads * np * pool->head_dim : nullptr;
  // the decode merges its own partials when contexts are split into few
  // partitions (few split sequences: a separate reduce launch would mostly
  // find nothing to do); with many partitions per sequence the separate
  // reduce, spread over every SM, is faster than the last CTAs' merges (FP8
  // decodes always use the separate reduce)
  int* counters = need && np <= kFusedMergeMaxParts && pool->dtype != KV_FP8_E4M3
                      ? reinterpret_cast<int*>(part_ml + (size_t)batch * num_q_heads * np * 4)
                      : nullptr;
  rc = enqueue_decode(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                      batch, max_context_len, scale, out, out_dtype, part_o, part_ml, np, np, pt, nullptr,
                      counters, seq_order, reinterpret_cast<cudaStream_t>(stream));
  if (rc != KV_OK) return rc;
  return ok();
}

size_t paged_attention_shared_prefix_workspace_bytes(const kv_pool* pool, int batch, int num_q_heads,
                                                     int max_context_len, int num_sharers) {
  if (!pool || batch <= 0 || num_q_heads <= 0 || max_context_len <= 0 || num_sharers < 0) return 0;
  const int group = num_q_heads % pool->kv_heads == 0 ? num_q_heads / pool->kv_heads : 1;
  const int np = num_parts_for(pool, batch, max_context_len, group) + 1;
  const size_t parts = (size_t)batch * num_q_heads * np * (pool->head_dim + 4) * sizeof(float);
  const size_t rows = (size_t)num_sharers * num_q_heads * pool->head_dim * 2;
  return parts + (rows + 15) / 16 * 16 + 16;
}

int paged_attention_decode_shared_prefix(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                                         int num_q_heads, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens, int batch,
                                         int max_context_len, const int32_t* prefix_seqs, int num_sharers,
                                         const int32_t* prefix_blocks, int prefix_len,
                                         const int32_t* skip_lens, float scale, void* out,
                                         kv_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                         const int32_t* seq_order, kv_stream_t stream) {
  int rc = check_decode_args(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq,
                             context_lens, batch, max_context_len, scale, out, out_dtype);
  if (rc != KV_OK) return rc;
  if (pool->dtype != KV_F16 && pool->dtype != KV_BF16)
    return fail(KV_ERR_ARG, "shared-prefix decode needs an f16 or bf16 pool");
  if (pool->window > 0) return fail(KV_ERR_ARG, "shared-prefix decode does not take a sliding window");
  if (num_sharers < 0 || prefix_len < 0 || num_sharers > batch)
    return fail(KV_ERR_ARG, "bad shared prefix: %d sequences, %d tokens", num_sharers, prefix_len);
  if (prefix_len % pool->block_size != 0 || prefix_len > max_context_len)
    return fail(KV_ERR_ARG, "prefix_len %d must be whole blocks within max_context_len %d", prefix_len,
                max_context_len);
  if (!(scale > 0.f)) return fail(KV_ERR_ARG, "scale must be > 0");
  if (batch == 0) return ok();
  if (num_sharers == 0 || prefix_len == 0)  // nothing shared: the plain decode
    return paged_attention_decode(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq,
                                  context_lens, batch, max_context_len, scale, out, out_dtype, workspace,
                                  workspace_bytes, seq_order, stream);
  if (!prefix_seqs || !prefix_blocks || !skip_lens) return fail(KV_ERR_ARG, "NULL shared-prefix input");
  if ((uintptr_t)q & 15) return fail(KV_ERR_ARG, "q must be 16-byte aligned for shared-prefix decode");
  const size_t need = paged_attention_shared_prefix_workspace_bytes(pool, batch, num_q_heads, max_context_len,
                                                                    num_sharers);
  if (!workspace || workspace_bytes < need)
    return fail(KV_ERR_ARG, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if ((uintptr_t)workspace & 15) return fail(KV_ERR_ARG, "workspace must be 16-byte aligned");
  const int group = num_q_heads / pool->kv_heads;
  const int pt = partition_tokens(pool, batch, max_context_len, group);
  const int np = num_parts_for(pool, batch, max_context_len, group);
  if (np + 1 > 65535) return fail(KV_ERR_ARG, "too many partitions");
  const int npa = np + 1;
  float* part_o = static_cast<float*>(workspace);
  float* part_ml = part_o + (size_t)batch * num_q_heads * npa * pool->head_dim;
  uint8_t* rows = reinterpret_cast<uint8_t*>(part_ml + (size_t)batch * num_q_heads * npa * 4);
  const size_t row_bytes = (size_t)num_sharers * num_q_heads * pool->head_dim * 2;
  int32_t* meta = reinterpret_cast<int32_t*>(rows + (row_bytes + 15) / 16 * 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // 1. the sharers' query rows, consecutive
  const int chunks_per_row = num_q_heads * pool->head_dim * 2 / 16;
  const int64_t threads = (int64_t)num_sharers * chunks_per_row;
  gather_rows_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
      static_cast<const uint4*>(q), prefix_seqs, num_sharers, batch, chunks_per_row,
      reinterpret_cast<uint4*>(rows), meta, prefix_len);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gather_rows_kernel launch");
  // 2. the prefix once for every sharer, on the tensor cores: partition 0
  rc = prefix_partials(pool, layer, rows, num_sharers, num_q_heads, prefix_blocks,
                       prefix_len / pool->block_size, meta, scale, part_o, part_ml, prefix_seqs, npa, stream);
  if (rc != KV_OK) return rc;
  // 3. every sequence's own tokens (after the prefix for sharers), then the merge
  rc = enqueue_decode(pool, layer, q, q_dtype, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                      batch, max_context_len, scale, out, out_dtype, part_o, part_ml, np, npa, pt, skip_lens,
                      nullptr, seq_order, s);
  if (rc != KV_OK) return rc;
  return ok();
}

}  // extern "C"

// Scratch for paged_attention_decode_noalloc: split-K partials of the calls
// that cannot allocate.  Shared by every such call on a device.
static __device__ __align__(256) float g_noalloc_scratch[KV_NOALLOC_WORKSPACE_BYTES / sizeof(float)];

namespace pagedkv {
namespace {

std::atomic<void*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (host code cannot use the symbol itself as a device address).
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= kMaxDevices) return fail(KV_ERR_ARG, "device %d beyond %d devices", dev, kMaxDevices);
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return KV_OK;
}

}  // namespace
}  // namespace pagedkv

extern "C" {

int paged_attention_decode_noalloc(const kv_pool* pool, int layer, const void* q,
                                   kv_dtype q_dtype, int num_q_heads,
                                   const int32_t* block_tables, int max_blocks_per_seq,
                                   const int32_t* context_lens, int batch, int max_context_len,
                                   float scale, void* out, kv_dtype out_dtype, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_ARG, "NULL pool");
  const size_t need = paged_attention_workspace_bytes(pool, batch, num_q_heads, max_context_len);
  if (need > KV_NOALLOC_WORKSPACE_BYTES)
    return fail(KV_ERR_ARG,
                "these sizes need %zu bytes of split-K scratch, above the %u-byte static scratch; "
                "call paged_attention_decode with a workspace instead",
                need, (unsigned)KV_NOALLOC_WORKSPACE_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    int rc = noalloc_scratch(&scratch);
    if (rc != KV_OK) return rc;
  }
  return paged_attention_decode(pool, layer, q, q_dtype, num_q_heads, block_tables,
                                max_blocks_per_seq, context_lens, batch, max_context_len, scale, out,
                                out_dtype, scratch, need > 0 ? KV_NOALLOC_WORKSPACE_BYTES : 0, nullptr,
                                stream);
}

int kv_selftest_wait_timeout(uint64_t limit_ns, kv_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return fail(KV_ERR_ARG, "limit_ns must be in (0, 10 s]");
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait_timeout_selftest_kernel launch");
  return ok();
}

int kv_get_device_error(kv_stream_t stream, int* err) {
  if (!err) return fail(KV_ERR_ARG, "err is NULL");
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  *err = h;
  return ok();
}

}  // extern "C"
