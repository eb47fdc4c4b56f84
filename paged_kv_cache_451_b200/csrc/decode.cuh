// PagedAttention decode for sm_100a.
//
// Method: "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍", section
// "PagedAttention：把操作系统的虚拟内存搬进 GPU": K/V sit in fixed-size
// physical blocks scattered through one pool; a per-sequence block table
// maps logical to physical blocks; the kernel reads K/V from those
// non-contiguous blocks.  The page names block prefetch and re-arranging KV
// in shared memory as the kernel's tricks; here both are done by the TMA
// engine: every 16-token tile of K and V is fetched by a 3-D bulk tensor copy
// into a per-warp ring of shared-memory stages, landing in the 128-byte
// swizzled layout that ldmatrix reads without bank conflicts.
//
// Work split: one CTA per (context partition, kv head, sequence).  Each warp
// of the CTA walks every WARPS-th 16-token chunk of the partition with its
// own pipeline (lane 0 issues the copies for the chunk STAGES ahead) and keeps
// its own running max / sum / output; warps are merged once at the end.
//
// Math per chunk, in transposed form (m16n8k16 tensor-core MMA, fp32
// accumulate), so that K and V tiles from ldmatrix are A operands as they are
// and the query group is a plain B operand:
//   S^T[16 tokens x 8 heads]  = K_chunk[16 x D] . Q^T[D x 8]   (heads of this kv
//                               head's GQA group, zero-padded to 8)
//   online softmax over each head (column) in the log2 domain (fp32), with a
//   lazily moved reference max per head
//   P^T (16 tokens x 8 heads) is split into a 16-bit value and its 16-bit
//   rounding residual (~16 significant bits together) and transposed into B
//   fragments with movmatrix
//   O^T[D x 8] += V^T[D x 16 tokens] . P^T, once for the value and once for the
//   residual (FP8 pools: P as one f16 value, one pass).
// FP8 (E4M3) pools are decoded to f16 in registers (exact); the queries are
// scaled by a power of two per head so they fit f16 without losing bits; the
// K scale of each (block, head) multiplies its logits.  The V scale enters
// the weights of P.V: besides the running max m_z of the logits (which
// normalises the softmax sum l) a second running max m_w of logit +
// log2|V scale| normalises the weights fed to the MMA, so the dominant terms
// of the output always sit near 1 in f16, whatever the spread of V scales;
// the output is (O / l) * 2^(m_w - m_z).
//
// A context longer than one partition is split: each partition writes its
// unnormalised output and (m_z, l, m_w), and lse_reduce_kernel merges them;
// a context within one partition is written normalised by its only CTA.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "device_common.cuh"
#include "ptx.cuh"

namespace pagedkv {

constexpr int kChunk = 16;           // tokens per MMA tile
constexpr int kMaxPartChunks = 1024;  // at most 16384 tokens per partition
constexpr int kMaxGroup = 8;         // query heads per kv head in one CTA
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// A row's reference max is only moved (and its output rescaled) when the
// chunk max exceeds it by more than this many binades; in between the
// probabilities are exp2(z - m) <= 2^kLazyLog2, exact in the 16-bit hi/lo
// split and harmless to the fp32 sums.
constexpr float kLazyLog2 = 8.f;

enum KvKind { KV_KIND_F16 = 0, KV_KIND_BF16 = 1, KV_KIND_E4M3 = 2 };
enum OutKind { OUT_F16 = 0, OUT_BF16 = 1, OUT_F32 = 3 };

struct DecodeParams {
  const void* q;                // [batch][num_q_heads][D] f16 / bf16
  const int32_t* block_tables;  // [batch][max_blocks]
  const int32_t* context_lens;  // [batch]
  // NULL or [batch]: leading tokens of each sequence attended elsewhere (a
  // shared prefix, a multiple of 16).  Such a sequence's decode starts after
  // them and always writes split partials, at partition index + 1 (partition
  // 0 holds the prefix's).
  const int32_t* skip;
  // NULL, or [batch][kv_heads] zeroed counters: the last CTA of a split
  // (sequence, kv head) to finish merges its partials into the output
  int* counters;
  const int32_t* seq_order;     // NULL or [batch]: sequence of grid row z
  const float* k_scale;         // FP8: [num_blocks][kv_heads]
  const float* v_scale;
  void* out;                    // [batch][num_q_heads][D]
  float* part_o;                // split: [batch][num_q_heads][num_parts][D]
  float* part_ml;               // split: [batch][num_q_heads][num_parts][4] = m_z, l, m_w, 0
  int q_bf16;
  int out_kind;
  int num_q_heads;
  int group;                    // num_q_heads / kv_heads, <= 8
  int kv_heads;
  int block_size;
  int cpb_shift;                // log2(block_size / 16)
  int num_blocks;
  int max_blocks;
  int ctx_cap;                  // min(max_blocks * block_size, max_context_len)
  int part_chunks;              // chunks per partition
  int num_parts;
  int window;                   // > 0: attend only the last `window` tokens
  float scale_log2;             // softmax scale * log2(e)
};

__device__ __forceinline__ void store_out(void* out, int kind, int64_t idx, float v) {
  if (kind == OUT_F32) {
    static_cast<float*>(out)[idx] = v;
  } else if (kind == OUT_BF16) {
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  } else {
    static_cast<__half*>(out)[idx] = __float2half_rn(v);
  }
}

template <int KV, int D, int WARPS, int STAGES>
struct DecodeShape {
  static constexpr bool kFp8 = KV == KV_KIND_E4M3;
  static constexpr int EB = kFp8 ? 1 : 2;           // bytes per stored element
  static constexpr int ROWB = D * EB;               // bytes per token row
  static constexpr int BOXB = ROWB < 128 ? ROWB : 128;  // bytes per TMA box row
  static constexpr int NBOX = ROWB / BOXB;
  static constexpr int CPR = BOXB / 16;             // 16-byte chunks per box row
  static constexpr uint32_t SWZ = BOXB == 128 ? 7u : 3u;
  static constexpr int TILEB = kChunk * ROWB;       // one K (or V) chunk
  static constexpr int STAGEB = 2 * TILEB;
  static constexpr int STAGES_BYTES = WARPS * STAGES * STAGEB;
  static constexpr int MERGE_BYTES = WARPS * kMaxGroup * D * 4;
  static constexpr int BUF_BYTES = STAGES_BYTES > MERGE_BYTES ? STAGES_BYTES : MERGE_BYTES;
  static constexpr int BAR_OFF = BUF_BYTES;
  static constexpr int ML_OFF = BAR_OFF + WARPS * STAGES * 8;
  // per-chunk tables, sized at launch by the partition's chunk count: block
  // id, and for FP8 the K scale, log2 |V scale| and the V scale's sign
  // ML: per (warp, head) m_z, l, m_w and the warp's merge weight; then per
  // head the output factor, M_z, L and M_w of the merged CTA
  static constexpr int TAB_OFF = (ML_OFF + (WARPS + 1) * kMaxGroup * 16 + 15) / 16 * 16;
  static constexpr int TAB_ENTRY = kFp8 ? 16 : 4;
  __host__ __device__ static constexpr int tab_cap(int chunks) { return (chunks + 3) / 4 * 4; }
  // dynamic shared memory of a launch whose partitions hold `chunks` chunks
  // (+ 1024 bytes of alignment slack)
  __host__ __device__ static constexpr int smem_bytes(int chunks) {
    return TAB_OFF + tab_cap(chunks) * TAB_ENTRY + 1024;
  }
  static constexpr int MAX_SMEM_BYTES = smem_bytes(kMaxPartChunks);
  static_assert(BOXB == 128 || BOXB == 64, "row bytes must be 64 or a multiple of 128");
};

// Byte offset of (row, 16-byte chunk) inside one K or V chunk tile made of
// NBOX boxes of 16 rows x BOXB bytes, each with the TMA swizzle applied.
template <class S>
__device__ __forceinline__ uint32_t tile_off(int row, int chunk16) {
  const int box = chunk16 / S::CPR;
  const uint32_t lin = row * S::BOXB + (chunk16 % S::CPR) * 16;
  return box * (kChunk * S::BOXB) + (lin ^ (((lin >> 7) & S::SWZ) << 4));
}

// Merge of one (sequence, query head)'s split partials by one warp: with
// partition p holding (o_p, m_z,p, l_p, m_w,p) in the log2 domain,
//   Mz = max m_z,p,  L = sum l_p 2^(m_z,p - Mz),
//   Mw = max m_w,p,  O = sum o_p 2^(m_w,p - Mw),   out = (O / L) 2^(Mw - Mz).
// (For 16-bit caches m_w = m_z.)  idx = sequence * num_q_heads + head; np
// partials of the num_parts slots are used; head_dim 64 or 128.  kL2: read
// the partials through L2 only (other SMs of the same launch wrote them);
// otherwise through the read-only path (a separate launch: the (m, l)
// slots, read three times, may also hit in L1).
template <bool kL2>
__device__ __forceinline__ float4 ld_part(const float4* p) {
  if constexpr (kL2) return __ldcg(p);
  else return __ldg(p);
}
template <bool kL2>
__device__ __forceinline__ float2 ld_part(const float2* p) {
  if constexpr (kL2) return __ldcg(p);
  else return __ldg(p);
}

template <bool kL2, int PER>
__device__ __forceinline__ void merge_head_partials_t(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int64_t idx,
                                                      int num_parts, int np, void* out, int out_kind,
                                                      int lane) {
  constexpr int HD = PER * 32;  // each lane owns PER consecutive dims
  using Vec = typename std::conditional<PER == 4, float4, float2>::type;
  const float4* ml = reinterpret_cast<const float4*>(part_ml) + idx * num_parts;
  // the first 32 partitions' (m_z, l, m_w): one load per lane, kept
  const float4 m0 = lane < np ? ld_part<kL2>(ml + lane) : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
  float Mz = m0.x, Mw = m0.z;
  for (int q = lane + 32; q < np; q += 32) {
    const float4 v = ld_part<kL2>(ml + q);
    Mz = fmaxf(Mz, v.x);
    Mw = fmaxf(Mw, v.z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Mz = fmaxf(Mz, __shfl_xor_sync(0xffffffffu, Mz, o));
    Mw = fmaxf(Mw, __shfl_xor_sync(0xffffffffu, Mw, o));
  }
  float L = m0.x != -INFINITY ? m0.y * ex2(m0.x - Mz) : 0.f;
  for (int q = lane + 32; q < np; q += 32) {
    const float4 v = ld_part<kL2>(ml + q);
    if (v.x != -INFINITY) L += v.y * ex2(v.x - Mz);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const bool empty = !(L > 0.f) || Mw == -INFINITY;
  const float scale = empty ? 0.f : ex2(Mw - Mz) / L;
  // partition weights computed once per 32 partitions and broadcast; the
  // partial rows are loaded 8 at a time so their latencies overlap (the sum
  // still runs in partition order)
  const float* po = part_o + idx * num_parts * HD + lane * PER;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  if (!empty) {
    for (int q0 = 0; q0 < np; q0 += 32) {
      float mq = m0.z;
      if (q0 > 0) mq = q0 + lane < np ? ld_part<kL2>(ml + q0 + lane).z : -INFINITY;
      const float wq = mq == -INFINITY ? 0.f : ex2(mq - Mw);
      const int nq = min(32, np - q0);
      for (int j0 = 0; j0 < nq; j0 += 8) {
        Vec v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (j0 + u < nq) v[u] = ld_part<kL2>(reinterpret_cast<const Vec*>(po + (int64_t)(q0 + j0 + u) * HD));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u < nq) {  // uniform over the warp
            const float wj = __shfl_sync(0xffffffffu, wq, j0 + u);
            acc[0] += wj * v[u].x;
            acc[1] += wj * v[u].y;
            if constexpr (PER == 4) {
              acc[2] += wj * v[u].z;
              acc[3] += wj * v[u].w;
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) store_out(out, out_kind, idx * HD + lane * PER + k, acc[k] * scale);
}

// head_dim 64 or 128
template <bool kL2>
__device__ __forceinline__ void merge_head_partials(const float* part_o, const float* part_ml, int64_t idx,
                                                    int num_parts, int np, int head_dim, void* out,
                                                    int out_kind, int lane) {
  if (head_dim == 128)
    merge_head_partials_t<kL2, 4>(part_o, part_ml, idx, num_parts, np, out, out_kind, lane);
  else
    merge_head_partials_t<kL2, 2>(part_o, part_ml, idx, num_parts, np, out, out_kind, lane);
}

// Resident CTAs per SM the register allocation is sized for: FP8 tiles
// need half the shared memory of 16-bit ones, so four 4-warp CTAs fit.
template <int KV, int WARPS>
constexpr int decode_min_blocks() {
  return WARPS == 8 ? 2 : (KV == KV_KIND_E4M3 ? 4 : 1);
}

// EXT: the instantiation honours DecodeParams::skip and ::counters (16-bit
// caches only); without it both are ignored and compiled out.
template <int KV, int D, int WARPS, int STAGES, bool EXT>
__global__ void __launch_bounds__(WARPS * 32, decode_min_blocks<KV, WARPS>())
paged_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeShape<KV, D, WARPS, STAGES>;
  constexpr bool kFp8 = S::kFp8;
  constexpr bool kBf16Mma = KV == KV_KIND_BF16;
  constexpr int MT = D / 16;  // 16-row tiles of the transposed output O^T
  constexpr int KS = D / 16;  // 16-deep k-steps of q.K

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2;  // MMA group id: query-head row / token column
  const int cq = lane & 3;   // thread in group

  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  int seq = blockIdx.z;
  if (p.seq_order != nullptr) {
    seq = p.seq_order[blockIdx.z];
    if (seq < 0 || seq >= (int)gridDim.z) {
      if (part == 0 && kvh == 0 && threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
      return;  // uniform over the CTA
    }
  }
  const int bs = p.block_size;
  const int cpb_shift = p.cpb_shift;  // log2(block_size / 16)

  int n = p.context_lens[seq];
  if (n < 0 || n > p.ctx_cap) {
    if (part == 0 && threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
    n = n < 0 ? 0 : p.ctx_cap;
  }
  // Skipped prefixes and the in-kernel merge: 16-bit caches only (the
  // shared-prefix decode takes 16-bit pools, and FP8 contexts long enough to
  // split run faster with the separate reduce)
  constexpr bool kExt = EXT && !kFp8;
  int skip = 0;
  if (kExt && p.skip != nullptr) {
    skip = p.skip[seq];
    if (skip < 0 || skip > n || (skip & (kChunk - 1))) {
      if (part == 0 && threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
      skip = skip < 0 ? 0 : min(skip, n) & ~(kChunk - 1);
    }
  }
  // sliding window: tokens [t_lo, n) only; chunks are counted from cb, the
  // chunk holding t_lo (blocks wholly before it may already be released);
  // a skipped prefix starts the visited range the same way
  const int t_lo = p.window > 0 ? max(0, n - p.window) : skip;
  const int cb = t_lo / kChunk;
  const int total_chunks = (n + kChunk - 1) / kChunk - cb;
  const int c0 = part * p.part_chunks;
  const int c1 = min(c0 + p.part_chunks, total_chunks);
  if (c0 >= c1 && part > 0) return;  // nothing in this partition (uniform per CTA)
  const int nchunks = max(c1 - c0, 0);

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + S::BAR_OFF;
  const int tab = S::tab_cap(p.part_chunks);
  int32_t* blk_ids = reinterpret_cast<int32_t*>(smem + S::TAB_OFF);
  float* ksc = reinterpret_cast<float*>(smem + S::TAB_OFF) + tab;  // FP8: K scale
  float* vsc = ksc + tab;                                           // FP8: log2 |V scale|
  float* vsg = vsc + tab;                                           // FP8: sign of the V scale
  float* mls = reinterpret_cast<float*>(smem + S::ML_OFF);

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  for (int i = threadIdx.x; i < nchunks; i += WARPS * 32) {
    const int c = cb + c0 + i;
    int32_t b = p.block_tables[(int64_t)seq * p.max_blocks + (c >> cpb_shift)];
    if (b < 0 || b >= p.num_blocks) {
      record_error(KV_ERR_BOUNDS);
      b = -1;
    }
    blk_ids[i] = b;
    if constexpr (kFp8) {
      float sk = 0.f, sv = 0.f;
      if (b >= 0) {
        sk = p.k_scale[(int64_t)b * p.kv_heads + kvh];
        sv = p.v_scale[(int64_t)b * p.kv_heads + kvh];
      }
      ksc[i] = sk;
      vsc[i] = sv != 0.f ? lg2(fabsf(sv)) : -INFINITY;
      vsg[i] = sv < 0.f ? -1.f : 1.f;
    }
  }
  if (lane == 0) {
    for (int st = 0; st < STAGES; ++st) mbar_init(bars + (warp * STAGES + st) * 8, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ---- queries of this kv head's group as MMA B fragments: lane (gq, cq)
  // holds head gq's values at MMA k = 2cq, 2cq+1 (qb[ks][0]) and 2cq+8, 2cq+9
  // (qb[ks][1]); heads beyond the group are zero.
  uint32_t qb[KS][2];
  float zrow;  // logit scale of head gq (log2 units)
  {
    const bool valid = gq < p.group;
    const int64_t qrow = ((int64_t)seq * p.num_q_heads + kvh * p.group + (valid ? gq : 0)) * D;
    const uint16_t* qh = static_cast<const uint16_t*>(p.q) + qrow;
    if constexpr (!kFp8) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = valid ? *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 2 * cq) : 0u;
        qb[ks][1] = valid ? *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 8 + 2 * cq) : 0u;
      }
      zrow = p.scale_log2;
    } else {
      // k-order for FP8 tiles: MMA k = 2c+j  <-> d = 16ks + 4c + j,
      //                        MMA k = 2c+8+j <-> d = 16ks + 4c + 2 + j   (j = 0, 1)
      float v[KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint2 w = valid ? *reinterpret_cast<const uint2*>(qh + ks * 16 + 4 * cq) : make_uint2(0, 0);
        v[ks][0] = bits_to_float(w.x & 0xffff, p.q_bf16);
        v[ks][1] = bits_to_float(w.x >> 16, p.q_bf16);
        v[ks][2] = bits_to_float(w.y & 0xffff, p.q_bf16);
        v[ks][3] = bits_to_float(w.y >> 16, p.q_bf16);
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fabsf(v[ks][j]));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // power-of-two e with amax * 2^e in [2^14, 2^15): exact in f16 for bf16 inputs
      int e = 0;
      if (amax > 0.f) e = 14 - (int)((__float_as_uint(amax) >> 23) & 0xff) + 127;
      e = max(-126, min(100, e));
      const float mult = __uint_as_float((uint32_t)(e + 127) << 23);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = pack2<false>(v[ks][0] * mult, v[ks][1] * mult);
        qb[ks][1] = pack2<false>(v[ks][2] * mult, v[ks][3] * mult);
      }
      zrow = p.scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23);
    }
  }
  // this lane's S^T columns are heads 2cq and 2cq + 1
  const float zs_a = __shfl_sync(0xffffffffu, zrow, (2 * cq) * 4);
  const float zs_b = __shfl_sync(0xffffffffu, zrow, (2 * cq + 1) * 4);

  // ---- per-warp pipeline over chunks i = warp, warp + WARPS, ...
  const int my_n = nchunks > warp ? (nchunks - warp + WARPS - 1) / WARPS : 0;
  const uint32_t wstage = sbase + warp * STAGES * S::STAGEB;
  const uint32_t wbar = bars + warp * STAGES * 8;

  auto issue = [&](int li, int st) {
    const int i = warp + li * WARPS;
    const uint32_t bar = wbar + st * 8;
    const int32_t b = blk_ids[i];
    if (b < 0) {
      mbar_arrive(bar);  // complete the phase without data; the chunk is skipped
      return;
    }
    const int y = kvh * bs + ((cb + c0 + i) & ((1 << cpb_shift) - 1)) * kChunk;
    const uint32_t kd = wstage + st * S::STAGEB;
    mbar_arrive_expect_tx(bar, S::STAGEB);
#pragma unroll
    for (int bx = 0; bx < S::NBOX; ++bx) {
      tma_load_3d(kd + bx * kChunk * S::BOXB, &kmap, bar, bx * (S::BOXB / S::EB), y, b);
      tma_load_3d(kd + S::TILEB + bx * kChunk * S::BOXB, &vmap, bar, bx * (S::BOXB / S::EB), y, b);
    }
  };

  if (lane == 0) {
    for (int li = 0; li < STAGES && li < my_n; ++li) issue(li, li);
  }
  __syncwarp();

  // Per-lane running state for its two heads (a = 2cq, b = 2cq + 1).
  float m_a = -INFINITY, m_b = -INFINITY;    // reference max of the logits (log2)
  float l_a = 0.f, l_b = 0.f;                // this lane's share of the softmax sums
  float mw_a = -INFINITY, mw_b = -INFINITY;  // FP8: reference max of logit + log2|V scale|
  // O^T accumulators: tile t covers 16 output dims (rows) x 8 heads (columns)
  float o[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;

  // ldmatrix row (token) and 16-byte column chunk of this lane
  const int krow = (lane & 7) + (((lane >> 3) & 1) << 3);  // K: m0 tok 0-7, m1 tok 8-15, ...
  const int kcol = lane >> 4;
  const int vrow = kFp8 ? krow : (lane & 7) + ((lane >> 4) << 3);
  const int vcol = kFp8 ? (lane >> 4) : ((lane >> 3) & 1);
  // Swizzled byte offsets of this lane's ldmatrix rows.  Column chunk
  // 2j + col of a tile sits in box (2j + col) / CPR; within a box the swizzle
  // XOR depends only on the lane's row, so the offsets repeat every CPR / 2
  // steps up to a whole-box (compile-time) displacement.
  constexpr int NOFF = S::CPR / 2;
  uint32_t koff[NOFF], voff[NOFF];
#pragma unroll
  for (int j = 0; j < NOFF; ++j) {
    koff[j] = tile_off<S>(krow, 2 * j + kcol);
    voff[j] = tile_off<S>(vrow, 2 * j + vcol);
  }

  int li = 0;
  int st = 0;           // stage of chunk li
  uint32_t parity = 0;  // barrier phase parity of chunk li
  bool failed = false;
  for (; li < my_n; ++li) {
    const bool ready = mbar_wait_bounded(wbar + st * 8, parity, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ready)) {
      failed = true;
      break;
    }
    const int i = warp + li * WARPS;
    if (blk_ids[i] >= 0) {
      const int ct = (cb + c0 + i) * kChunk;    // first token of the chunk
      const int vt = min(kChunk, n - ct);        // tokens [lt, vt) of the chunk are attended
      const int lt = max(0, t_lo - ct);
      const uint32_t kb = wstage + st * S::STAGEB;
      const uint32_t vb = kb + S::TILEB;

      // S^T = K . Q^T (16 tokens x 8 heads); even / odd k-steps accumulate
      // separately: lane (gq, cq) gets tokens gq, gq+8 of heads 2cq, 2cq+1
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      if constexpr (!kFp8) {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb + koff[ks % NOFF] + (ks / NOFF) * (kChunk * S::BOXB), a0, a1, a2, a3);
          mma_16816<kBf16Mma>(sacc[ks & 1], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + koff[kp % NOFF] + (kp / NOFF) * (kChunk * S::BOXB), r0, r1, r2, r3);
          uint32_t f0l, f0h, f1l, f1h, f2l, f2h, f3l, f3h;
          e4m3x4_to_f16x4(r0, f0l, f0h);
          e4m3x4_to_f16x4(r1, f1l, f1h);
          e4m3x4_to_f16x4(r2, f2l, f2h);
          e4m3x4_to_f16x4(r3, f3l, f3h);
          mma_16816<false>(sacc[0], f0l, f1l, f0h, f1h, qb[2 * kp][0], qb[2 * kp][1]);
          mma_16816<false>(sacc[1], f2l, f3l, f2h, f3h, qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
        }
      }

      // online softmax (log2 domain) for heads a, b over this lane's tokens
      float zsa = zs_a, zsb = zs_b;
      if constexpr (kFp8) {
        zsa *= ksc[i];
        zsb *= ksc[i];
      }
      float z[4] = {(sacc[0][0] + sacc[1][0]) * zsa, (sacc[0][1] + sacc[1][1]) * zsb,
                    (sacc[0][2] + sacc[1][2]) * zsa, (sacc[0][3] + sacc[1][3]) * zsb};
      if (vt < kChunk || lt > 0) {
        if (gq >= vt || gq < lt) z[0] = z[1] = -INFINITY;
        if (gq + 8 >= vt || gq + 8 < lt) z[2] = z[3] = -INFINITY;
      }
      // A head's max over the chunk is only needed when some value exceeds its
      // reference max by more than 2^kLazyLog2 (the first chunk, rarely later);
      // if no lane's own max does, no head max does, so all lanes agree.
      float mxa = fmaxf(z[0], z[2]), mxb = fmaxf(z[1], z[3]);
      float lw = 0.f;  // FP8: log2 |V scale| of this chunk
      if constexpr (kFp8) lw = vsc[i];
      bool need = mxa > m_a + kLazyLog2 || mxb > m_b + kLazyLog2;
      if constexpr (kFp8)
        need = need || mxa + lw > mw_a + kLazyLog2 || mxb + lw > mw_b + kLazyLog2;
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, off));
          mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, off));
        }
      }
      const bool grow_a = mxa > m_a + kLazyLog2, grow_b = mxb > m_b + kLazyLog2;
      const float ma = grow_a ? mxa : m_a, mb = grow_b ? mxb : m_b;
      const float alpha_a = grow_a ? ex2(m_a - ma) : 1.f;
      const float alpha_b = grow_b ? ex2(m_b - mb) : 1.f;
      float pr[4] = {ex2(z[0] - ma), ex2(z[1] - mb), ex2(z[2] - ma), ex2(z[3] - mb)};
      l_a = l_a * alpha_a + (pr[0] + pr[2]);
      l_b = l_b * alpha_b + (pr[1] + pr[3]);
      m_a = ma;
      m_b = mb;
      float ao_a = alpha_a, ao_b = alpha_b;  // rescale of O's columns a, b
      bool grow_o = grow_a || grow_b;
      if constexpr (kFp8) {
        // weights pr * 2^(lw + m - mw) = 2^(z + lw - mw) <= 2^kLazyLog2
        const bool gwa = mxa + lw > mw_a + kLazyLog2, gwb = mxb + lw > mw_b + kLazyLog2;
        const float nwa = gwa ? mxa + lw : mw_a, nwb = gwb ? mxb + lw : mw_b;
        ao_a = (gwa && nwa != -INFINITY) ? ex2(mw_a - nwa) : 1.f;
        ao_b = (gwb && nwb != -INFINITY) ? ex2(mw_b - nwb) : 1.f;
        grow_o = gwa || gwb;
        const float ca = nwa == -INFINITY ? 0.f : ex2(lw + ma - nwa) * vsg[i];
        const float cb = nwb == -INFINITY ? 0.f : ex2(lw + mb - nwb) * vsg[i];
        mw_a = nwa;
        mw_b = nwb;
        pr[0] *= ca;
        pr[2] *= ca;
        pr[1] *= cb;
        pr[3] *= cb;
      }
      if (__any_sync(0xffffffffu, grow_o)) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          o[t][0] *= ao_a;
          o[t][1] *= ao_b;
          o[t][2] *= ao_a;
          o[t][3] *= ao_b;
        }
      }

      // P^T as B fragments, transposed so lane (g, c) holds tokens 2c, 2c+1
      // of head g.  16-bit caches: P as 16-bit value + rounding residual
      // (P.V runs once per half; 16 (bf16) to 22 (f16) significant bits
      // together), for the 2e-3 bound.  FP8 caches: P as one f16 value; its relative
      // rounding error 2^-11 moves the output by at most 2^-11 max |v|, far
      // inside the FP8 bound of 1e-2, and the second P.V pass is saved.
      uint32_t h0, l0 = 0u, h1, l1 = 0u;
      if constexpr (kFp8) {
        h0 = pack2<false>(pr[0], pr[1]);  // token gq, heads a, b
        h1 = pack2<false>(pr[2], pr[3]);  // token gq + 8
      } else {
        split2<kBf16Mma>(pr[0], pr[1], h0, l0);
        split2<kBf16Mma>(pr[2], pr[3], h1, l1);
      }
      const uint32_t bh0 = movmatrix_t(h0), bh1 = movmatrix_t(h1);
      const uint32_t bl0 = kFp8 ? 0u : movmatrix_t(l0), bl1 = kFp8 ? 0u : movmatrix_t(l1);

      // O^T += V^T . P^T.  The last chunk of a context zeroes the V values of
      // its tokens >= vt (stale slots may hold any bits, and 0 * NaN is NaN);
      // full chunks skip the masking.
      auto pv = [&](uint32_t mlo, uint32_t mhi, auto masked) {
        constexpr bool kMask = decltype(masked)::value;
        if constexpr (!kFp8) {
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vb + voff[t % NOFF] + (t / NOFF) * (kChunk * S::BOXB), a0, a1, a2, a3);
            if constexpr (kMask) {
              a0 &= mlo;
              a1 &= mlo;
              a2 &= mhi;
              a3 &= mhi;
            }
            mma_16816<kBf16Mma>(o[t], a0, a1, a2, a3, bh0, bh1);
            mma_16816<kBf16Mma>(o[t], a0, a1, a2, a3, bl0, bl1);
          }
        } else {
#pragma unroll
          for (int cp = 0; cp < MT / 2; ++cp) {
            uint32_t r0, r1, r2, r3;
            ldsm_x4_t(vb + voff[cp % NOFF] + (cp / NOFF) * (kChunk * S::BOXB), r0, r1, r2, r3);
            if constexpr (kMask) {
              r0 &= mlo;
              r1 &= mhi;
              r2 &= mlo;
              r3 &= mhi;
            }
            // bytes of r: [tok 2c][d0], [tok 2c][d0+1], [tok 2c+1][d0], [tok 2c+1][d0+1],
            // d0 = 16 * chunk + 2g; tile rows 0..7 take the even dims, 8..15 the odd
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t lo = h ? r2 : r0, hi = h ? r3 : r1;
              // the even bytes (dim d0 of tokens 2c, 2c+1) and the odd bytes (dim
              // d0 + 1) of both registers, one permute each; each 16-bit half
              // then converts to an f16 pair
              uint32_t a0, a1, a2, a3;
              e4m3x4_to_f16x4(__byte_perm(lo, hi, 0x6420), a0, a2);
              e4m3x4_to_f16x4(__byte_perm(lo, hi, 0x7531), a1, a3);
              mma_16816<false>(o[2 * cp + h], a0, a1, a2, a3, bh0, bh1);
            }
          }
        }
      };
      if (vt == kChunk && lt == 0) {
        pv(0u, 0u, std::false_type{});
      } else {
        auto in = [&](int t) { return t >= lt && t < vt; };
        const uint32_t mlo = (in(2 * cq) ? 0x0000ffffu : 0u) | (in(2 * cq + 1) ? 0xffff0000u : 0u);
        const uint32_t mhi = (in(8 + 2 * cq) ? 0x0000ffffu : 0u) | (in(9 + 2 * cq) ? 0xffff0000u : 0u);
        pv(mlo, mhi, std::true_type{});
      }
    }
    __syncwarp();
    if (lane == 0 && li + STAGES < my_n) issue(li + STAGES, st);
    if (++st == STAGES) {
      st = 0;
      parity ^= 1u;
    }
  }

  if (failed) {
    // give the copies already in flight a bounded chance to land before the
    // shared memory is reused
    if (lane == 0) record_error(KV_ERR_TIMEOUT);
    for (int k = li; k < my_n && k < li + STAGES; ++k)
      (void)mbar_wait_bounded(wbar + (k % STAGES) * 8, (k / STAGES) & 1, kWaitLimitNs);
  }

  // ---- merge the warps
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {  // sum over the 8 lanes of heads a, b
    l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
  }
  __syncthreads();  // every warp is done with its stages: reuse them for the merge
  float* obuf = reinterpret_cast<float*>(smem);  // [WARPS][kMaxGroup][D]
  const int ha = 2 * cq, hb = 2 * cq + 1;
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    int d0, d1;  // output dims of accumulator rows gq and gq + 8
    if constexpr (!kFp8) {
      d0 = 16 * t + gq;
      d1 = d0 + 8;
    } else {
      d0 = 16 * t + 2 * gq;
      d1 = d0 + 1;
    }
    if (ha < p.group) {
      obuf[(warp * kMaxGroup + ha) * D + d0] = o[t][0];
      obuf[(warp * kMaxGroup + ha) * D + d1] = o[t][2];
    }
    if (hb < p.group) {
      obuf[(warp * kMaxGroup + hb) * D + d0] = o[t][1];
      obuf[(warp * kMaxGroup + hb) * D + d1] = o[t][3];
    }
  }
  if (gq == 0) {
    if (ha < p.group) {
      float* ml = mls + (warp * kMaxGroup + ha) * 4;
      ml[0] = m_a;
      ml[1] = l_a;
      ml[2] = kFp8 ? mw_a : m_a;
    }
    if (hb < p.group) {
      float* ml = mls + (warp * kMaxGroup + hb) * 4;
      ml[0] = m_b;
      ml[1] = l_b;
      ml[2] = kFp8 ? mw_b : m_b;
    }
  }
  __syncthreads();

  // Merge weights, once per head: with Mz = max over warps of m_z, Mw = max
  // of m_w, warp w's output enters with weight 2^(m_w,w - Mw), its sum with
  // 2^(m_z,w - Mz); the head's result is O * 2^(Mw - Mz) / L.
  float* hd = mls + WARPS * kMaxGroup * 4;  // per head: factor, Mz, L, Mw
  if (threadIdx.x < p.group) {
    const int g = threadIdx.x;
    float Mz = -INFINITY, Mw = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      Mz = fmaxf(Mz, mls[(w * kMaxGroup + g) * 4 + 0]);
      Mw = fmaxf(Mw, mls[(w * kMaxGroup + g) * 4 + 2]);
    }
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      float* ml = mls + (w * kMaxGroup + g) * 4;
      if (ml[0] != -INFINITY) L += ml[1] * ex2(ml[0] - Mz);
      ml[3] = ml[2] != -INFINITY ? ex2(ml[2] - Mw) : 0.f;
    }
    float fin = 0.f;
    if (L > 0.f && Mw != -INFINITY) fin = (kFp8 ? ex2(Mw - Mz) : 1.f) / L;
    hd[g * 4 + 0] = fin;
    hd[g * 4 + 1] = Mz;
    hd[g * 4 + 2] = L;
    hd[g * 4 + 3] = Mw;
  }
  __syncthreads();

  // a context that fits one partition is finished here even in split mode;
  // the reduce kernel skips it
  const bool split = (p.num_parts > 1 && total_chunks > p.part_chunks) || skip > 0;
  const int pidx = part + (skip > 0 ? 1 : 0);  // partition 0 of a skipping sequence is its prefix's
  for (int idx = threadIdx.x; idx < p.group * D; idx += WARPS * 32) {
    const int g = idx / D;
    const int d = idx - g * D;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) O += obuf[(w * kMaxGroup + g) * D + d] * mls[(w * kMaxGroup + g) * 4 + 3];
    const int h = kvh * p.group + g;
    const int64_t sh = (int64_t)seq * p.num_q_heads + h;
    if (!split) {
      store_out(p.out, p.out_kind, sh * D + d, O * hd[g * 4]);
    } else {
      const int64_t pi = sh * p.num_parts + pidx;
      p.part_o[pi * D + d] = O;
      if (d == 0) {
        p.part_ml[pi * 4 + 0] = hd[g * 4 + 1];
        p.part_ml[pi * 4 + 1] = hd[g * 4 + 2];
        p.part_ml[pi * 4 + 2] = hd[g * 4 + 3];
        p.part_ml[pi * 4 + 3] = 0.f;
      }
    }
  }
  if (kExt && split && p.counters != nullptr && skip == 0) {
    // the last of this (sequence, kv head)'s partition CTAs merges them all
    __shared__ int s_last;
    const int np_seq = (total_chunks + p.part_chunks - 1) / p.part_chunks;
    __threadfence();  // this thread's partials are visible to every SM
    __syncthreads();
    if (threadIdx.x == 0)
      s_last = atomicAdd(p.counters + (int64_t)seq * p.kv_heads + kvh, 1) == np_seq - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int g = warp; g < p.group; g += WARPS)
        merge_head_partials<true>(p.part_o, p.part_ml, (int64_t)seq * p.num_q_heads + kvh * p.group + g,
                            p.num_parts, np_seq, D, p.out, p.out_kind, lane);
    }
  }
}

// Merge of split partials (merge_head_partials), one warp per (sequence,
// head), as a separate launch: used when the decode was not asked to merge
// in its last partition CTA (shared-prefix decode, whose prefix partials
// come from another kernel).
__global__ void __launch_bounds__(256)
lse_reduce_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                  const int32_t* __restrict__ context_lens, void* out, int out_kind,
                  int num_q_heads, int head_dim, int num_parts, int part_tokens, int ctx_cap,
                  int window, int batch, const int32_t* __restrict__ skip_lens) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t idx = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (idx >= (int64_t)batch * num_q_heads) return;
  const int seq = (int)(idx / num_q_heads);
  int n = context_lens[seq];
  n = n < 0 ? 0 : (n > ctx_cap ? ctx_cap : n);
  int skip = skip_lens != nullptr ? skip_lens[seq] : 0;
  skip = skip < 0 ? 0 : min(skip, n) & ~(kChunk - 1);
  // partitions of the chunks the decode visited (from the window's first
  // chunk, or after a skipped prefix, whose partials come first)
  const int cb = window > 0 ? max(0, n - window) / kChunk : skip / kChunk;
  const int chunks = (n + kChunk - 1) / kChunk - cb;
  const int part_chunks = part_tokens / kChunk;
  const int np = max(1, (chunks + part_chunks - 1) / part_chunks) + (skip > 0 ? 1 : 0);
  if (np == 1) return;  // written by the decode kernel directly
  merge_head_partials<false>(part_o, part_ml, idx, num_parts, np, head_dim, out, out_kind, lane);
}

// Rows of the sequences that share a prefix, gathered into consecutive
// rows for the multi-token kernel: dst[i] = q[rows[i]] (num_q_heads * D
// 16-bit values each, 16-byte chunks); also writes that kernel's one-sequence
// metadata: cu = {0, num_rows}, ctx = {prefix_len}.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ q, const int32_t* __restrict__ rows, int num_rows,
                   int batch, int chunks_per_row, uint4* __restrict__ dst, int32_t* meta, int prefix_len) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    meta[0] = 0;
    meta[1] = num_rows;
    meta[2] = prefix_len;
  }
  if (i >= (int64_t)num_rows * chunks_per_row) return;
  const int r = (int)(i / chunks_per_row), c = (int)(i - (int64_t)r * chunks_per_row);
  const int src = rows[r];
  if (src < 0 || src >= batch) {
    record_error(KV_ERR_BOUNDS);
    dst[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  dst[i] = q[(int64_t)src * chunks_per_row + c];
}

}  // namespace pagedkv
