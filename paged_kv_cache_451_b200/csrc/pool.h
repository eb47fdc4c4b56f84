// Host-side pool descriptor.
#pragma once

#include <cuda.h>

#include <cstdint>
#include <vector>

#include "host_common.h"

namespace pagedkv {

struct alignas(64) LayerBinding {
  CUtensorMap k_map;  // 3-D TMA descriptors over [num_blocks][kv_heads*block_size][head_dim]
  CUtensorMap v_map;
  void* k = nullptr;
  void* v = nullptr;
  float* k_scale = nullptr;
  float* v_scale = nullptr;
  bool bound = false;
};

inline int elem_bytes(kv_dtype t) { return t == KV_FP8_E4M3 ? 1 : (t == KV_F32 ? 4 : 2); }

}  // namespace pagedkv

struct kv_pool;

namespace pagedkv {

// Shared-prefix partials on the tensor cores (prefill.cu): rows of q_rows
// ([num_rows][num_q_heads][head_dim], the pool dtype) attend to the
// prefix_len tokens held by prefix_blocks; row r writes partition 0 of
// sequence prefix_rows[r] in part_o / part_ml (num_parts per (sequence,
// head)).  meta: device int32 {0, num_rows, prefix_len}.  Enqueues one
// launch on `stream`; returns a KV_* status.
int prefix_partials(const kv_pool* pool, int layer, const void* q_rows, int num_rows, int num_q_heads,
                    const int32_t* prefix_blocks, int num_prefix_blocks, const int32_t* meta,
                    float scale, float* part_o, float* part_ml, const int32_t* prefix_rows,
                    int num_parts, kv_stream_t stream);

}  // namespace pagedkv

struct kv_pool {
  int block_size = 0;
  int num_blocks = 0;
  int kv_heads = 0;
  int head_dim = 0;
  int num_layers = 0;
  kv_dtype dtype = KV_F16;
  int partition_tokens = 0;  // 0: automatic
  int stages = 0;            // 0: automatic
  int warps = 0;             // 0: automatic
  int window = 0;            // > 0: decode attends only the last `window` tokens
  std::vector<pagedkv::LayerBinding> layers;

  size_t tile_bytes() const { return (size_t)block_size * head_dim * pagedkv::elem_bytes(dtype); }
  size_t block_bytes() const { return tile_bytes() * kv_heads; }
  size_t layer_bytes() const { return block_bytes() * num_blocks; }
  size_t scale_bytes() const {
    return dtype == KV_FP8_E4M3 ? sizeof(float) * (size_t)num_blocks * kv_heads : 0;
  }
};
