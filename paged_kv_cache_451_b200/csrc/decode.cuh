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
// Math per chunk (m16n8k16 tensor-core MMA, fp32 accumulate):
//   S[16 x 16]  = Q[16 x D] . K_chunk^T      rows 0..7: the query heads of this
//                                            kv head (GQA group, zero-padded),
//                                            rows 8..15: a copy of rows 0..7
//   online softmax over S in the log2 domain (fp32), with a lazily moved
//                                            reference max per row
//   O[16 x D]  += P[16 x 16] . V_chunk       rows 0..7 carry the 16-bit value of
//                                            the probabilities, rows 8..15 the
//                                            16-bit rounding residual, so the
//                                            product keeps ~16 significant bits
//                                            of P; O = rows 0..7 + rows 8..15.
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
// unnormalised output and (m_z, l, m_w), and lse_reduce_kernel merges them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

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
  static constexpr int BLK_OFF = BAR_OFF + WARPS * STAGES * 8;
  static constexpr int SCALE_ENTRIES = kFp8 ? kMaxPartChunks : 0;  // FP8 scale tables only
  static constexpr int KSC_OFF = BLK_OFF + kMaxPartChunks * 4;
  static constexpr int VSC_OFF = KSC_OFF + SCALE_ENTRIES * 4;
  static constexpr int VSG_OFF = VSC_OFF + SCALE_ENTRIES * 4;
  static constexpr int ML_OFF = VSG_OFF + SCALE_ENTRIES * 4;
  static constexpr int SMEM_BYTES = ML_OFF + WARPS * kMaxGroup * 16 + 1024;  // + alignment slack
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

template <int KV, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, WARPS == 8 ? 2 : 1)
paged_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap) {
  using S = DecodeShape<KV, D, WARPS, STAGES>;
  constexpr bool kFp8 = S::kFp8;
  constexpr bool kBf16Mma = KV == KV_KIND_BF16;
  constexpr int NT = D / 8;   // 8-column tiles of the output
  constexpr int KS = D / 16;  // 16-deep k-steps of q.K

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2;  // MMA group id: query-head row / token column
  const int cq = lane & 3;   // thread in group

  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  const int seq = blockIdx.z;
  const int bs = p.block_size;
  const int cpb_shift = p.cpb_shift;  // log2(block_size / 16)

  int n = p.context_lens[seq];
  if (n < 0 || n > p.ctx_cap) {
    if (part == 0 && threadIdx.x == 0) record_error(KV_ERR_BOUNDS);
    n = n < 0 ? 0 : p.ctx_cap;
  }
  const int total_chunks = (n + kChunk - 1) / kChunk;
  const int c0 = part * p.part_chunks;
  const int c1 = min(c0 + p.part_chunks, total_chunks);
  if (c0 >= c1 && part > 0) return;  // nothing in this partition (uniform per CTA)
  const int nchunks = max(c1 - c0, 0);

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + S::BAR_OFF;
  int32_t* blk_ids = reinterpret_cast<int32_t*>(smem + S::BLK_OFF);
  float* ksc = reinterpret_cast<float*>(smem + S::KSC_OFF);
  float* vsc = reinterpret_cast<float*>(smem + S::VSC_OFF);  // log2 |V scale|
  float* vsg = reinterpret_cast<float*>(smem + S::VSG_OFF);  // sign of the V scale
  float* mls = reinterpret_cast<float*>(smem + S::ML_OFF);

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  for (int i = threadIdx.x; i < nchunks; i += WARPS * 32) {
    const int c = c0 + i;
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

  // ---- queries of this kv head's group as MMA A fragments (rows 8..15 = rows 0..7)
  uint32_t qa[KS][2];
  float zrow;
  {
    const bool valid = gq < p.group;
    const int64_t qrow = ((int64_t)seq * p.num_q_heads + kvh * p.group + (valid ? gq : 0)) * D;
    const uint16_t* qh = static_cast<const uint16_t*>(p.q) + qrow;
    if constexpr (!kFp8) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = valid ? *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 2 * cq) : 0u;
        qa[ks][1] = valid ? *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 8 + 2 * cq) : 0u;
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
        qa[ks][0] = pack2<false>(v[ks][0] * mult, v[ks][1] * mult);
        qa[ks][1] = pack2<false>(v[ks][2] * mult, v[ks][3] * mult);
      }
      zrow = p.scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23);
    }
  }

  // ---- per-warp pipeline over chunks i = warp, warp + WARPS, ...
  const int my_n = nchunks > warp ? (nchunks - warp + WARPS - 1) / WARPS : 0;
  const uint32_t wstage = sbase + warp * STAGES * S::STAGEB;
  const uint32_t wbar = bars + warp * STAGES * 8;

  auto issue = [&](int li) {
    const int i = warp + li * WARPS;
    const int st = li % STAGES;
    const uint32_t bar = wbar + st * 8;
    const int32_t b = blk_ids[i];
    if (b < 0) {
      mbar_arrive(bar);  // complete the phase without data; the chunk is skipped
      return;
    }
    const int y = kvh * bs + ((c0 + i) & ((1 << cpb_shift) - 1)) * kChunk;
    const uint32_t kd = wstage + st * S::STAGEB;
    mbar_arrive_expect_tx(bar, S::STAGEB);
#pragma unroll
    for (int bx = 0; bx < S::NBOX; ++bx) {
      tma_load_3d(kd + bx * kChunk * S::BOXB, &kmap, bar, bx * (S::BOXB / S::EB), y, b);
      tma_load_3d(kd + S::TILEB + bx * kChunk * S::BOXB, &vmap, bar, bx * (S::BOXB / S::EB), y, b);
    }
  };

  if (lane == 0) {
    for (int li = 0; li < STAGES && li < my_n; ++li) issue(li);
  }
  __syncwarp();

  float m_run = -INFINITY;   // running max of the logits (log2 domain)
  float l_run = 0.f;         // running softmax sum, relative to m_run
  float mw_run = -INFINITY;  // FP8: running max of logit + log2|V scale|
  float o[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;

  int li = 0;
  bool failed = false;
  for (; li < my_n; ++li) {
    const int st = li % STAGES;
    const uint32_t parity = (li / STAGES) & 1;
    const bool ready = mbar_wait_bounded(wbar + st * 8, parity, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ready)) {
      failed = true;
      break;
    }
    const int i = warp + li * WARPS;
    if (blk_ids[i] >= 0) {
      const int vt = min(kChunk, n - (c0 + i) * kChunk);  // valid tokens in the chunk
      const uint32_t kb = wstage + st * S::STAGEB;
      const uint32_t vb = kb + S::TILEB;

      // S = Q . K^T: tile 0 = tokens 0..7, tile 1 = tokens 8..15.  Even and odd
      // k-steps accumulate separately (four independent MMA chains) and are
      // summed afterwards, halving the dependent-MMA latency per chunk.
      float sa[2][2][4] = {};
      if constexpr (!kFp8) {
        const int row = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + tile_off<S>(row, ks * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
          mma_16816<kBf16Mma>(sa[ks & 1][0], qa[ks][0], qa[ks][0], qa[ks][1], qa[ks][1], b0, b1);
          mma_16816<kBf16Mma>(sa[ks & 1][1], qa[ks][0], qa[ks][0], qa[ks][1], qa[ks][1], b2, b3);
        }
      } else {
        const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + tile_off<S>(row, kp * 2 + (lane >> 4)), r0, r1, r2, r3);
          const int k0 = 2 * kp, k1 = 2 * kp + 1;
          uint32_t f0l, f0h, f1l, f1h, f2l, f2h, f3l, f3h;
          e4m3x4_to_f16x4(r0, f0l, f0h);
          e4m3x4_to_f16x4(r1, f1l, f1h);
          e4m3x4_to_f16x4(r2, f2l, f2h);
          e4m3x4_to_f16x4(r3, f3l, f3h);
          mma_16816<false>(sa[0][0], qa[k0][0], qa[k0][0], qa[k0][1], qa[k0][1], f0l, f0h);
          mma_16816<false>(sa[0][1], qa[k0][0], qa[k0][0], qa[k0][1], qa[k0][1], f1l, f1h);
          mma_16816<false>(sa[1][0], qa[k1][0], qa[k1][0], qa[k1][1], qa[k1][1], f2l, f2h);
          mma_16816<false>(sa[1][1], qa[k1][0], qa[k1][0], qa[k1][1], qa[k1][1], f3l, f3h);
        }
      }
      const float s00 = sa[0][0][0] + sa[1][0][0], s01 = sa[0][0][1] + sa[1][0][1];
      const float s10 = sa[0][1][0] + sa[1][1][0], s11 = sa[0][1][1] + sa[1][1][1];

      // online softmax (log2 domain) over this lane's 4 tokens of row gq
      float zs = zrow;
      if constexpr (kFp8) zs *= ksc[i];
      float z[4] = {s00 * zs, s01 * zs, s10 * zs, s11 * zs};
      if (vt < kChunk) {
        if (2 * cq >= vt) z[0] = -INFINITY;
        if (2 * cq + 1 >= vt) z[1] = -INFINITY;
        if (8 + 2 * cq >= vt) z[2] = -INFINITY;
        if (9 + 2 * cq >= vt) z[3] = -INFINITY;
      }
      float mx = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const bool grow = mx > m_run + kLazyLog2;  // always true on a row's first chunk
      const float m_new = grow ? mx : m_run;
      const float alpha = grow ? ex2(m_run - m_new) : 1.f;
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[e] = ex2(z[e] - m_new);
      l_run = l_run * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
      m_run = m_new;
      float alpha_o = alpha;  // rescale of O
      bool grow_o = grow;
      if constexpr (kFp8) {
        // weights pr * 2^(lw + m_new - mw_new) = 2^(z + lw - mw_new) <= 2^kLazyLog2
        const float lw = vsc[i];
        const bool grow_w = mx + lw > mw_run + kLazyLog2;
        const float mw_new = grow_w ? mx + lw : mw_run;
        const bool none = mw_new == -INFINITY;
        alpha_o = (grow_w && !none) ? ex2(mw_run - mw_new) : 1.f;
        grow_o = grow_w;
        const float c = none ? 0.f : ex2(lw + m_new - mw_new) * vsg[i];
        mw_run = mw_new;
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] *= c;
      }
      if (__any_sync(0xffffffffu, grow_o)) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          o[t][0] *= alpha_o;
          o[t][1] *= alpha_o;
          o[t][2] *= alpha_o;
          o[t][3] *= alpha_o;
        }
      }
      // P as A fragment: rows 0..7 the 16-bit values, rows 8..15 the residuals
      uint32_t pa0, pa1, pa2, pa3;
      split2<kBf16Mma>(pr[0], pr[1], pa0, pa1);
      split2<kBf16Mma>(pr[2], pr[3], pa2, pa3);

      // O += P . V
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;  // token masks for b0 / b1 registers
      if (vt < kChunk) {
        mlo = (2 * cq < vt ? 0x0000ffffu : 0u) | (2 * cq + 1 < vt ? 0xffff0000u : 0u);
        mhi = (8 + 2 * cq < vt ? 0x0000ffffu : 0u) | (9 + 2 * cq < vt ? 0xffff0000u : 0u);
      }
      const int vrow = (lane & 7) + (((lane >> 3) & 1) << 3);
      if constexpr (!kFp8) {
#pragma unroll
        for (int jp = 0; jp < NT / 2; ++jp) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_t(vb + tile_off<S>(vrow, jp * 2 + (lane >> 4)), r0, r1, r2, r3);
          mma_16816<kBf16Mma>(o[2 * jp], pa0, pa1, pa2, pa3, r0 & mlo, r1 & mhi);
          mma_16816<kBf16Mma>(o[2 * jp + 1], pa0, pa1, pa2, pa3, r2 & mlo, r3 & mhi);
        }
      } else {
#pragma unroll
        for (int jp = 0; jp < NT / 4; ++jp) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_t(vb + tile_off<S>(vrow, jp * 2 + (lane >> 4)), r0, r1, r2, r3);
          r0 &= mlo;
          r1 &= mhi;
          r2 &= mlo;
          r3 &= mhi;
          // bytes of r: [tok 2c][d0], [tok 2c][d0+1], [tok 2c+1][d0], [tok 2c+1][d0+1]
          mma_16816<false>(o[4 * jp + 0], pa0, pa1, pa2, pa3,
                           e4m3x2_to_f16x2(__byte_perm(r0, 0, 0x0020)),
                           e4m3x2_to_f16x2(__byte_perm(r1, 0, 0x0020)));
          mma_16816<false>(o[4 * jp + 1], pa0, pa1, pa2, pa3,
                           e4m3x2_to_f16x2(__byte_perm(r0, 0, 0x0031)),
                           e4m3x2_to_f16x2(__byte_perm(r1, 0, 0x0031)));
          mma_16816<false>(o[4 * jp + 2], pa0, pa1, pa2, pa3,
                           e4m3x2_to_f16x2(__byte_perm(r2, 0, 0x0020)),
                           e4m3x2_to_f16x2(__byte_perm(r3, 0, 0x0020)));
          mma_16816<false>(o[4 * jp + 3], pa0, pa1, pa2, pa3,
                           e4m3x2_to_f16x2(__byte_perm(r2, 0, 0x0031)),
                           e4m3x2_to_f16x2(__byte_perm(r3, 0, 0x0031)));
        }
      }
    }
    __syncwarp();
    if (lane == 0 && li + STAGES < my_n) issue(li + STAGES);
  }

  if (failed) {
    // give the copies already in flight a bounded chance to land before the
    // shared memory is reused
    if (lane == 0) record_error(KV_ERR_TIMEOUT);
    for (int k = li; k < my_n && k < li + STAGES; ++k)
      (void)mbar_wait_bounded(wbar + (k % STAGES) * 8, (k / STAGES) & 1, kWaitLimitNs);
  }

  // ---- merge the warps
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();  // every warp is done with its stages: reuse them for the merge
  float* obuf = reinterpret_cast<float*>(smem);  // [WARPS][kMaxGroup][D]
  if (gq < p.group) {
    float* row = obuf + (warp * kMaxGroup + gq) * D;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      int d0, d1;
      if constexpr (!kFp8) {
        d0 = 8 * t + 2 * cq;
        d1 = d0 + 1;
      } else {
        d0 = 16 * (t >> 1) + 4 * cq + (t & 1);
        d1 = d0 + 2;
      }
      row[d0] = o[t][0] + o[t][2];
      row[d1] = o[t][1] + o[t][3];
    }
    if (cq == 0) {
      float* ml = mls + (warp * kMaxGroup + gq) * 4;
      ml[0] = m_run;
      ml[1] = l_run;
      ml[2] = kFp8 ? mw_run : m_run;
    }
  }
  __syncthreads();

  const bool split = p.num_parts > 1;
  for (int idx = threadIdx.x; idx < p.group * D; idx += WARPS * 32) {
    const int g = idx / D;
    const int d = idx - g * D;
    float Mz = -INFINITY, Mw = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      Mz = fmaxf(Mz, mls[(w * kMaxGroup + g) * 4 + 0]);
      Mw = fmaxf(Mw, mls[(w * kMaxGroup + g) * 4 + 2]);
    }
    float O = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float* ml = mls + (w * kMaxGroup + g) * 4;
      if (ml[0] != -INFINITY) L += ml[1] * ex2(ml[0] - Mz);
      if (ml[2] != -INFINITY) O += obuf[(w * kMaxGroup + g) * D + d] * ex2(ml[2] - Mw);
    }
    const int h = kvh * p.group + g;
    const int64_t sh = (int64_t)seq * p.num_q_heads + h;
    if (!split) {
      float r = 0.f;
      if (L > 0.f && Mw != -INFINITY) r = kFp8 ? (O / L) * ex2(Mw - Mz) : O / L;
      store_out(p.out, p.out_kind, sh * D + d, r);
    } else {
      const int64_t pi = sh * p.num_parts + part;
      p.part_o[pi * D + d] = O;
      if (d == 0) {
        p.part_ml[pi * 4 + 0] = Mz;
        p.part_ml[pi * 4 + 1] = L;
        p.part_ml[pi * 4 + 2] = Mw;
        p.part_ml[pi * 4 + 3] = 0.f;
      }
    }
  }
}

// Merge of split partials: for each (sequence, query head), with partition p
// holding (o_p, m_z,p, l_p, m_w,p) in the log2 domain,
//   Mz = max m_z,p,  L = sum l_p 2^(m_z,p - Mz),
//   Mw = max m_w,p,  O = sum o_p 2^(m_w,p - Mw),   out = (O / L) 2^(Mw - Mz).
// (For 16-bit caches m_w = m_z.)  One warp per (sequence, head); head_dim is
// 64 or 128.
__global__ void __launch_bounds__(256)
lse_reduce_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                  const int32_t* __restrict__ context_lens, void* out, int out_kind,
                  int num_q_heads, int head_dim, int num_parts, int part_tokens, int ctx_cap,
                  int batch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t idx = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (idx >= (int64_t)batch * num_q_heads) return;
  const int seq = (int)(idx / num_q_heads);
  int n = context_lens[seq];
  n = n < 0 ? 0 : (n > ctx_cap ? ctx_cap : n);
  const int np = max(1, (n + part_tokens - 1) / part_tokens);
  const float4* ml = reinterpret_cast<const float4*>(part_ml) + idx * num_parts;
  float Mz = -INFINITY, Mw = -INFINITY;
  for (int q = lane; q < np; q += 32) {
    const float4 v = ml[q];
    Mz = fmaxf(Mz, v.x);
    Mw = fmaxf(Mw, v.z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Mz = fmaxf(Mz, __shfl_xor_sync(0xffffffffu, Mz, o));
    Mw = fmaxf(Mw, __shfl_xor_sync(0xffffffffu, Mw, o));
  }
  float L = 0.f;
  for (int q = lane; q < np; q += 32) {
    const float4 v = ml[q];
    if (v.x != -INFINITY) L += v.y * ex2(v.x - Mz);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const bool empty = !(L > 0.f) || Mw == -INFINITY;
  const float scale = empty ? 0.f : ex2(Mw - Mz) / L;
  // each lane owns head_dim / 32 consecutive dims; partition weights are
  // computed once per 32 partitions and broadcast
  const int per = head_dim / 32;  // 2 or 4
  const float* po = part_o + idx * num_parts * head_dim + lane * per;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (!empty) {
    for (int q0 = 0; q0 < np; q0 += 32) {
      float wq = 0.f;
      if (q0 + lane < np) {
        const float mq = ml[q0 + lane].z;
        wq = mq == -INFINITY ? 0.f : ex2(mq - Mw);
      }
      const int nq = min(32, np - q0);
      for (int j = 0; j < nq; ++j) {
        const float wj = __shfl_sync(0xffffffffu, wq, j);
        const float* src = po + (int64_t)(q0 + j) * head_dim;
        if (per == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          acc[0] += wj * v.x;
          acc[1] += wj * v.y;
          acc[2] += wj * v.z;
          acc[3] += wj * v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          acc[0] += wj * v.x;
          acc[1] += wj * v.y;
        }
      }
    }
  }
  for (int k = 0; k < per; ++k) store_out(out, out_kind, idx * head_dim + lane * per + k, acc[k] * scale);
}

}  // namespace pagedkv
