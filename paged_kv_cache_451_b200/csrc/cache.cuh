// Slot-mapped cache write and copy-on-write block copy.
//
// "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍", section
// "PagedAttention：把操作系统的虚拟内存搬进 GPU": a sequence's cache grows a
// block at a time as tokens arrive, and several logical blocks may map to
// one physical block.  The write puts each new token's K/V row in the slot
// its block table assigns; the copy gives a writer its own copy of a shared
// block.  FP8 (section "vLLM 也不是银弹：真实部署中的坑") quantises on write.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "device_common.cuh"
#include "ptx.cuh"

namespace pagedkv {

struct WriteParams {
  const uint8_t* k_new;  // [T][kv_heads][D] 16-bit elements
  const uint8_t* v_new;
  const int64_t* slots;  // [T]
  uint8_t* k;            // pool [num_blocks][kv_heads][block_size][D]
  uint8_t* v;
  const float* k_inv;    // FP8: [num_blocks][kv_heads]
  const float* v_inv;
  int64_t rows;          // T * kv_heads
  int kv_heads;
  int head_dim;
  int block_size;
  int num_blocks;
  int src_bf16;
};

// One thread per 8 elements of one (token, head) row.  16-bit pools copy
// 16 bytes; FP8 pools widen to fp32, multiply by the (block, head) inverse
// scale in fp32 and round to E4M3 (nearest even, saturating).
template <bool kFp8>
__global__ void __launch_bounds__(256) kv_write_kernel(const WriteParams p) {
  const int tpr = p.head_dim / 8;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gid / tpr;
  const int part = (int)(gid - row * tpr);
  if (row >= p.rows) return;
  const int64_t t = row / p.kv_heads;
  const int h = (int)(row - t * p.kv_heads);
  const int64_t slot = p.slots[t];
  if (slot < 0) return;
  const int64_t blk = slot / p.block_size;
  const int off = (int)(slot - blk * p.block_size);
  if (blk >= p.num_blocks) {
    record_error(KV_ERR_BOUNDS);
    return;
  }
  const int64_t src = (row * p.head_dim + part * 8) * 2;
  const int64_t dst_elem = ((blk * p.kv_heads + h) * p.block_size + off) * (int64_t)p.head_dim + part * 8;
  const uint4 kx = *reinterpret_cast<const uint4*>(p.k_new + src);
  const uint4 vx = *reinterpret_cast<const uint4*>(p.v_new + src);
  if constexpr (!kFp8) {
    *reinterpret_cast<uint4*>(p.k + dst_elem * 2) = kx;
    *reinterpret_cast<uint4*>(p.v + dst_elem * 2) = vx;
  } else {
    const float ki = p.k_inv[blk * p.kv_heads + h];
    const float vi = p.v_inv[blk * p.kv_heads + h];
    auto quant = [&](const uint4& x, float inv) {
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint32_t q[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float a = bits_to_float(w[2 * j] & 0xffff, p.src_bf16) * inv;
        const float b = bits_to_float(w[2 * j] >> 16, p.src_bf16) * inv;
        const float c = bits_to_float(w[2 * j + 1] & 0xffff, p.src_bf16) * inv;
        const float d = bits_to_float(w[2 * j + 1] >> 16, p.src_bf16) * inv;
        q[j] = (uint32_t)f32x2_to_e4m3x2(a, b) | ((uint32_t)f32x2_to_e4m3x2(c, d) << 16);
      }
      return make_uint2(q[0], q[1]);
    };
    *reinterpret_cast<uint2*>(p.k + dst_elem) = quant(kx, ki);
    *reinterpret_cast<uint2*>(p.v + dst_elem) = quant(vx, vi);
  }
}

constexpr int kCopyLayers = 64;  // layers per block_copy launch

struct CopyParams {
  const int32_t* pairs;  // [num_pairs][2] (src, dst)
  int num_pairs;
  int num_blocks;
  int kv_heads;
  int64_t block_bytes;   // kv_heads * block_size * D * elem bytes (a multiple of 16)
  void* k[kCopyLayers];
  void* v[kCopyLayers];
  float* ks[kCopyLayers];
  float* vs[kCopyLayers];
};

// grid = (num_pairs, layers in this launch, 2 for K and V)
__global__ void __launch_bounds__(256) block_copy_kernel(const CopyParams p) {
  const int pi = blockIdx.x;
  const int layer = blockIdx.y;
  const bool is_v = blockIdx.z == 1;
  const int32_t src = p.pairs[2 * pi];
  const int32_t dst = p.pairs[2 * pi + 1];
  if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
    if (threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
    return;
  }
  if (src == dst) return;
  uint8_t* base = static_cast<uint8_t*>(is_v ? p.v[layer] : p.k[layer]);
  const uint4* s = reinterpret_cast<const uint4*>(base + (int64_t)src * p.block_bytes);
  uint4* d = reinterpret_cast<uint4*>(base + (int64_t)dst * p.block_bytes);
  const int64_t n16 = p.block_bytes / 16;
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) d[i] = s[i];
  float* sc = is_v ? p.vs[layer] : p.ks[layer];
  if (sc != nullptr)
    for (int h = threadIdx.x; h < p.kv_heads; h += blockDim.x)
      sc[(int64_t)dst * p.kv_heads + h] = sc[(int64_t)src * p.kv_heads + h];
}

// Swap copies between device blocks and a host swap space (pinned host
// memory mapped into the device address space, written / read directly by
// the kernel over the host link).  A slot holds, per layer, K then V:
// block_bytes of data followed (FP8) by the block's kv_heads scales, padded
// to 16 bytes.  kOut: device block -> slot; else slot -> device block.
struct SwapParams {
  const int32_t* pairs;  // [num_pairs][2]: (device block, slot) out, (slot, device block) in
  int num_pairs;
  int num_blocks;
  int num_slots;
  int kv_heads;
  int layer0;            // first layer of this launch
  int num_layers;        // all layers of the pool
  int64_t block_bytes;
  int64_t per_bytes;     // block_bytes + padded scale bytes
  uint8_t* host;         // device-accessible base of the swap space
  void* k[kCopyLayers];
  void* v[kCopyLayers];
  float* ks[kCopyLayers];
  float* vs[kCopyLayers];
};

// grid = (num_pairs, layers in this launch, 2 for K and V)
template <bool kOut>
__global__ void __launch_bounds__(256) swap_kernel(const SwapParams p) {
  const int pi = blockIdx.x;
  const int li = blockIdx.y;
  const bool is_v = blockIdx.z == 1;
  const int32_t dev = kOut ? p.pairs[2 * pi] : p.pairs[2 * pi + 1];
  const int32_t slot = kOut ? p.pairs[2 * pi + 1] : p.pairs[2 * pi];
  if (dev < 0 || dev >= p.num_blocks || slot < 0 || slot >= p.num_slots) {
    if (threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
    return;
  }
  const int layer = p.layer0 + li;
  uint8_t* hb = p.host + ((int64_t)slot * p.num_layers * 2 + layer * 2 + (is_v ? 1 : 0)) * p.per_bytes;
  uint8_t* db = static_cast<uint8_t*>(is_v ? p.v[li] : p.k[li]) + (int64_t)dev * p.block_bytes;
  const int64_t n16 = p.block_bytes / 16;
  uint4* d = reinterpret_cast<uint4*>(kOut ? hb : db);
  const uint4* s = reinterpret_cast<const uint4*>(kOut ? db : hb);
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) d[i] = s[i];
  float* sc = is_v ? p.vs[li] : p.ks[li];
  if (sc != nullptr) {
    float* hs = reinterpret_cast<float*>(hb + p.block_bytes);
    for (int h = threadIdx.x; h < p.kv_heads; h += blockDim.x) {
      if (kOut) hs[h] = sc[(int64_t)dev * p.kv_heads + h];
      else sc[(int64_t)dev * p.kv_heads + h] = hs[h];
    }
  }
}

// Self-test of the bounded-wait error path used by the decode pipeline: one
// warp waits on an mbarrier whose phase can never complete (a transaction
// count that no copy will satisfy).  After limit_ns the wait gives up, the
// kernel records KV_ERR_TIMEOUT and returns; nothing is in flight.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_arrive_expect_tx(b, 16);  // 16 bytes that never arrive
  __syncwarp();
  const bool ok = mbar_wait_bounded(b, 0, limit_ns);
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) record_error(KV_ERR_TIMEOUT);
}

}  // namespace pagedkv
