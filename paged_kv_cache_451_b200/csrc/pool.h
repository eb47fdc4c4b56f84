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
