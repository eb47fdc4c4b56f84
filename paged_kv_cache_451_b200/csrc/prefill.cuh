// Multi-token attention over the paged cache for sm_100a: the prompt (or a
// chunk of it, or a few drafted tokens) attends causally to everything the
// sequence has cached, its own new tokens included.
//
// Method: "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍", section
// "PagedAttention：把操作系统的虚拟内存搬进 GPU" (K/V in fixed-size blocks
// reached through a per-sequence block table) and section
// "连续批处理：别再等最慢的那个请求了" (prompts are processed before decoding
// continues; time to first token).  The pages give no kernel for this step.
// Reading taken: new token i of a sequence with n cached tokens, q_len of
// them new, sits at position n - q_len + i and attends to positions 0 .. that
// position.
//
// Unlike decode, this is a real dense contraction, so it runs on the
// fifth-generation tensor cores.  A work item is a pair of query tiles A, B
// of one (kv head, sequence); a query tile is 128 rows = 128 / g new tokens x
// the g query heads of one kv head's group, and both tiles share every K/V
// tile read.  The grid has one CTA per item, but CTAs persist (one per SM):
// a CTA that starts an item asks the hardware (cluster launch control) to
// cancel the launch of a CTA that has not started yet and takes over its
// item next, so the copies and first MMAs of the next item overlap the end
// of the current one and no CTA is set up per item.  Barrier phases run on
// counters across items.  Per 128-key tile j, with S and O of each query
// tile in tensor memory (TMEM, 4 x 128 columns):
//   S_j = Q . K_j^T          (tcgen05.mma, M 128, N 128, K = head_dim; Q and
//                            K_j in shared memory, 128-byte swizzled, K-major)
//   softmax rows in fp32 (one row per thread, warps 0-3 tile A, 4-7 tile B;
//   log2 domain, a lazily moved reference max, causal and sliding-window
//   masks only on the tiles that need them; pairs of keys through the
//   .f32x2 add / fma; S read 16 columns at a time with the next 16 in
//   flight); the probabilities P_j go back into S_j's TMEM columns as
//   16-bit values (bf16: value + rounding residual, about 16 significant
//   bits together)
//   O += P_j . V_j           (tcgen05.mma with A = P_j from TMEM, B = V_j from
//                            shared memory, MN-major; bf16: once per half)
// Warp 8 streams Q and the K/V tiles with 3-D TMA copies straight out of the
// paged pool (one 16-row box per 16 keys and 64 columns, placed so the tile
// lands in the canonical swizzled layout the MMA reads; each lane owns one
// box of every tile, so a tile's copies go out in one instruction: issued
// from a single thread they came out one every ~60 cycles and set the pace
// of the whole pipeline); warp 9 issues the
// MMAs from one thread in the order S_A(0) S_B(0) PV_A(0) S_A(1) PV_B(0)
// S_B(1) ..., so one tile's softmax runs while the tensor cores work on the
// other's.  Completion flows through mbarriers (TMA transaction counts,
// tcgen05.commit, thread arrives); every wait is bounded and aborts the CTA
// with KV_ERR_TIMEOUT.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>
#include <cstdint>
#include <type_traits>

#include "../../include/pagedkv.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace pagedkv {

constexpr int kPfRows = 128;        // query rows per tile (M of the MMA)
constexpr int kPfKeys = 128;        // keys per tile (N of Q.K^T, K of P.V)
constexpr int kPfTiles = 2;         // query tiles per CTA, sharing every K/V tile
constexpr int kPfThreads = 320;     // warps 0-7 softmax (4 per query tile), 8 copies, 9 MMA
constexpr uint32_t kPfTmemCols = 512;  // S_A, S_B (128 each) + O_A, O_B (<= 128 each)
constexpr uint64_t kPfWaitNs = 2000000000ull;
constexpr uint64_t kPfDrainNs = 50000000ull;  // copies and MMAs in flight finish in microseconds
constexpr int kPfSlots = 4;         // launch-control responses in flight or unread
// reference max moves only when a tile's max exceeds it by more than this
// many binades: probabilities stay <= 2^8, exact enough in 16 bits + residual
constexpr float kPfLazyLog2 = 8.f;

enum PrefillOutKind { PF_OUT_F16 = 0, PF_OUT_BF16 = 1, PF_OUT_F32 = 3 };

struct PrefillParams {
  const int32_t* cu_q;          // [batch + 1] first query row of each sequence
  const int32_t* block_tables;  // [batch][max_blocks]
  const int32_t* context_lens;  // [batch] cached tokens, the new ones included
  void* out;                    // [total_q][num_q_heads][D]
  int* err;                     // device error word
  int out_kind;
  int num_q_heads;
  int group;                    // query heads per kv head, <= 8
  int tokens_per_tile;          // 128 / group
  int num_q_pairs;              // pairs of query tiles per (kv head, sequence), max over sequences
  int kv_heads;
  int block_size;
  int num_blocks;
  int max_blocks;
  int total_q;
  int window;                   // > 0: each token attends only to its last `window` positions
  float scale_log2;             // softmax scale * log2(e), > 0
  int batch;
  int64_t num_items;            // num_q_pairs * kv_heads * batch
  // Shared-prefix mode (part_o != NULL): one virtual sequence whose new
  // tokens are the decode queries of the sequences sharing a prefix (one q
  // row each) and whose keys are the prefix's context_lens[0] tokens; every
  // row attends to all of them (no causal mask, no window), and the
  // epilogue writes split-K partials of partition 0 of the row's sequence
  // prefix_rows[row] (unnormalised O, its reference max and sum) in place
  // of an output row.
  float* part_o;                // [B][num_q_heads][num_parts][D]
  float* part_ml;               // [B][num_q_heads][num_parts][4]: m_z, l, m_w, 0
  const int32_t* prefix_rows;   // [total_q]
  int num_parts;
};

template <int D, int STAGES>
struct PrefillShape {
  static constexpr int NH = D / 64;            // 128-byte column blocks per row
  static constexpr int HALF = kPfRows * 128;   // one column block of a 128-row tile
  static constexpr int TILE = NH * HALF;       // a Q, K or V tile
  static constexpr int Q_OFF = 0;              // Q_A, Q_B
  static constexpr int K_OFF = Q_OFF + kPfTiles * TILE;
  static constexpr int V_OFF = K_OFF + STAGES * TILE;
  static constexpr int BAR_OFF = V_OFF + STAGES * TILE;
  // q full and q empty; K full/empty and V full/empty per stage; S full,
  // P full, P.V done and O free per query tile; the final MMA drain;
  // launch-control response full and read per slot
  static constexpr int NBAR = 2 + 4 * STAGES + 4 * kPfTiles + 1 + 2 * kPfSlots;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // TMEM base, abort flag
  static constexpr int RESP_OFF = (MISC_OFF + 16 + 15) / 16 * 16;  // 16-byte responses
  static constexpr int SMEM_BYTES = RESP_OFF + 16 * kPfSlots + 1024;  // + alignment slack
  static constexpr uint32_t S_COL = 0;                       // S_X at X * 128
  static constexpr uint32_t O_COL = kPfTiles * kPfKeys;      // O_X at 256 + X * D
  static_assert(kPfRows == kPfKeys, "Q, K and V tiles share one byte size");
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(O_COL + kPfTiles * D <= kPfTmemCols, "TMEM columns");
};

namespace pf {

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Non-suspending probe of a barrier phase (the waits here sit on the
// critical path between the MMA issuer and the softmax warps).
__device__ __forceinline__ bool probe(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Two fp32 values in one 64-bit register pair: sm_100 executes add, sub and
// fma on both halves with one instruction (.f32x2).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Wait for the phase with `parity`; give up when another role of the CTA
// has aborted, or after kPfWaitNs (then abort the CTA and record a timeout).
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                     int* err) {
  if (probe(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (probe(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kPfWaitNs) {
      *abort_flag = 1;
      atomicCAS(err, 0, KV_ERR_TIMEOUT);
      return false;
    }
  }
}

// Cluster launch control (sm_100): cancel the launch of a CTA of this grid
// that has not started and take over its work.  The 16-byte response lands
// in shared memory at `resp` and completes 16 transaction bytes on `bar`.
__device__ __forceinline__ void clc_try_cancel(uint32_t resp, uint32_t bar) {
  asm volatile(
      "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], "
      "[%1];" ::"r"(resp),
      "r"(bar)
      : "memory");
}

// The CTA index (x) a response names, or -1 when no launch was cancelled
// (every CTA of the grid has started: no work is left to take over).
__device__ __forceinline__ int64_t clc_item(uint32_t resp) {
  uint32_t ok, x = 0;
  asm volatile(
      "{\n\t.reg .b128 r;\n\t.reg .pred p;\n\t"
      "ld.shared.b128 r, [%2];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, r;\n\t}"
      : "=r"(ok), "+r"(x)
      : "r"(resp)
      : "memory");
  return ok ? (int64_t)x : -1;
}

// One work item: a pair of query tiles (A, B) of one (kv head, sequence).
struct Item {
  int s, kvh, q0, q_len, n, t0, kb, kend, ntiles;
  int ntok[kPfTiles], kendx[kPfTiles], ntx[kPfTiles];
};

// Geometry of item v.  Items run sequence by sequence (CTAs working side by
// side then read the same sequence's K/V tiles, from L2 after the first),
// and within a sequence heaviest first: its last pair of query tiles for
// every kv head, then the pairs before.  False
// when the item has no tokens, or its sequence's lengths are out of range
// (then `report` records KV_ERR_BOUNDS, once per sequence).
__device__ __forceinline__ bool item_at(const PrefillParams& p, int64_t v, bool report, Item& it) {
  const int64_t per_seq = (int64_t)p.kv_heads * p.num_q_pairs;
  it.s = (int)(v / per_seq);
  const int local = (int)(v - (int64_t)it.s * per_seq);
  const int qp = p.num_q_pairs - 1 - local / p.kv_heads;
  it.kvh = local % p.kv_heads;
  const int tq = p.tokens_per_tile;
  it.q0 = p.cu_q[it.s];
  it.q_len = p.cu_q[it.s + 1] - it.q0;
  it.n = p.context_lens[it.s];
  const bool prefix = p.part_o != nullptr;  // every row sees all n keys
  if (it.q0 < 0 || it.q_len < 0 || (!prefix && it.q_len > it.n) || (int64_t)it.q0 + it.q_len > p.total_q ||
      (int64_t)it.n > (int64_t)p.max_blocks * p.block_size ||
      it.q_len > p.num_q_pairs * kPfTiles * tq) {
    if (report && qp == p.num_q_pairs - 1 && it.kvh == 0) atomicCAS(p.err, 0, KV_ERR_BOUNDS);
    return false;
  }
  it.t0 = qp * kPfTiles * tq;
  if (it.t0 >= it.q_len) return false;
  // Key tiles start at kb: 0, or with a sliding window the 16-key chunk
  // holding the first position any row of the item sees (no block before
  // it is read: it may already be released).
  it.kb = p.window > 0 && !prefix ? max(0, it.n - it.q_len + it.t0 - p.window + 1) / 16 * 16 : 0;
#pragma unroll
  for (int x = 0; x < kPfTiles; ++x) {
    const int tx = it.t0 + x * tq;
    it.ntok[x] = tx < it.q_len ? min(tq, it.q_len - tx) : 0;
    it.kendx[x] = it.ntok[x] ? (prefix ? it.n : it.n - it.q_len + tx + it.ntok[x]) : 0;  // keys .. kend - 1
    it.ntx[x] = it.ntok[x] ? (it.kendx[x] - it.kb + kPfKeys - 1) / kPfKeys : 0;
  }
  it.kend = max(it.kendx[0], it.kendx[1]);
  it.ntiles = max(it.ntx[0], it.ntx[1]);  // K/V tiles read (tile B's when it has tokens)
  return true;
}

}  // namespace pf

template <bool kBf16, int D, int STAGES>
__global__ void __launch_bounds__(kPfThreads, 1)
paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap) {
  using S = PrefillShape<D, STAGES>;
  constexpr int NH = S::NH;
  constexpr bool kSplit = kBf16;  // bf16 probabilities carry their residual
  constexpr int KCH = kPfKeys / 16;  // 16-key boxes per tile

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  uint8_t* smem = smem_raw + (sbase - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = p.group, tq = p.tokens_per_tile;
  const int qrows = tq * g;

  const uint32_t bar0 = sbase + S::BAR_OFF;
  const uint32_t BQ = bar0;        // query tiles loaded
  const uint32_t QE = bar0 + 8u;   // query tiles free (every S of the item issued and done)
  auto KF = [&](int i) { return bar0 + 8u * (2 + i); };
  auto KE = [&](int i) { return bar0 + 8u * (2 + STAGES + i); };
  auto VF = [&](int i) { return bar0 + 8u * (2 + 2 * STAGES + i); };
  auto VE = [&](int i) { return bar0 + 8u * (2 + 3 * STAGES + i); };
  auto SF = [&](int x) { return bar0 + 8u * (2 + 4 * STAGES + x); };
  auto PF = [&](int x) { return bar0 + 8u * (2 + 4 * STAGES + kPfTiles + x); };
  auto PV = [&](int x) { return bar0 + 8u * (2 + 4 * STAGES + 2 * kPfTiles + x); };
  auto OF = [&](int x) { return bar0 + 8u * (2 + 4 * STAGES + 3 * kPfTiles + x); };
  const uint32_t FIN = bar0 + 8u * (2 + 4 * STAGES + 4 * kPfTiles);
  auto CF = [&](int i) { return FIN + 8u * (1 + i); };             // response i landed
  auto CR = [&](int i) { return FIN + 8u * (1 + kPfSlots + i); };  // response i read by all
  auto RESP = [&](int i) { return sbase + (uint32_t)S::RESP_OFF + 16u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::MISC_OFF + 8);

  if (threadIdx.x == 0) {
    mbar_init(BQ, 1);
    mbar_init(QE, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(KF(i), 1);
      mbar_init(KE(i), 1);
      mbar_init(VF(i), 1);
      mbar_init(VE(i), 1);
    }
    for (int x = 0; x < kPfTiles; ++x) {
      mbar_init(SF(x), 1);
      mbar_init(PF(x), kPfRows);
      mbar_init(PV(x), 1);
      mbar_init(OF(x), kPfRows);
    }
    mbar_init(FIN, 1);
    for (int i = 0; i < kPfSlots; ++i) {
      mbar_init(CF(i), 1);
      mbar_init(CR(i), 1 + kPfTiles * kPfRows / 32);  // the MMA warp + 8 softmax warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Query rows past tokens_per_tile * group are never written by the copies
  if (threadIdx.x < kPfTiles * kPfRows && (int)(threadIdx.x % kPfRows) >= qrows) {
    const int x = threadIdx.x / kPfRows, r = threadIdx.x % kPfRows;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      uint4* row = reinterpret_cast<uint4*>(smem + S::Q_OFF + x * S::TILE + h * S::HALF + r * 128);
#pragma unroll
      for (int i = 0; i < 8; ++i) row[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    pf::fence_proxy_async();
  }
  if (warp == 8) {
    __syncwarp();
    tc::alloc(smem_u32(tmem_slot), kPfTmemCols);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  // Work items of this CTA: item 0 is its own (blockIdx.x); item k >= 1 is
  // the CTA whose launch the copy warp cancelled when it began item k - 1
  // (response slot (k - 1) % kPfSlots; -1: none left).  Every role walks the
  // same items and keeps running counters, so barrier phases continue across
  // items: ic items with work, kc K/V tiles (stage kc % STAGES), per query
  // tile sc[x] S tiles and oc[x] items that used it.
  auto slot_of = [](uint32_t k) { return (int)((k - 1) % kPfSlots); };
  auto use_of = [](uint32_t k) { return ((k - 1) / kPfSlots) & 1u; };

  if (warp == 8) {
    // ------------------------------------------------------------ copies
    // The whole warp streams: lane c + KCH * h owns 16-key chunk c, column
    // block h of every tile (its block id, its box), so one instruction puts
    // a tile's NH * KCH box copies in flight; lane 0 sets the transaction
    // counts and asks for the next item.  Every lane takes the same waits
    // and branches.
    constexpr int NBOX = NH * KCH;  // 16 (head_dim 128) or 8 (64) boxes per tile
    const int c = lane % KCH, h = lane / KCH;
    const bool boxer = lane < NBOX;
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
    uint32_t ic = 0, kc = 0;
    uint32_t nk = 0, nv = 0;   // tiles whose K (V) copies were issued
    int64_t q_last = -1;       // index (in ic) of the last query copy issued
    uint32_t asked = 0, read = 0;  // items requested / responses read
    for (uint32_t k = 0;; ++k) {
      int64_t v = blockIdx.x;
      if (k > 0) {
        if (!__all_sync(0xffffffffu, pf::wait(CF(slot_of(k)), use_of(k), abort_flag, p.err))) break;
        read = k;
        v = pf::clc_item(RESP(slot_of(k)));
      }
      if (v < 0) break;  // every CTA of the grid has started: no item left
      // ask for item k + 1 now: the answer is back long before this item's
      // copies are issued.  Its slot was last used by item k + 1 - kPfSlots.
      if (k >= kPfSlots &&
          !__all_sync(0xffffffffu, pf::wait(CR(slot_of(k + 1)), use_of(k + 1) ^ 1u, abort_flag, p.err)))
        break;
      if (lane == 0) {
        mbar_arrive_expect_tx(CF(slot_of(k + 1)), 16u);
        pf::clc_try_cancel(RESP(slot_of(k + 1)), CF(slot_of(k + 1)));
      }
      asked = k + 1;
      pf::Item it;
      if (!pf::item_at(p, v, lane == 0, it)) continue;
      // the previous item's S MMAs must be done before its query tiles are replaced
      if (ic > 0 && !__all_sync(0xffffffffu, pf::wait(QE, (ic - 1) & 1, abort_flag, p.err))) break;
      if (lane == 0) mbar_arrive_expect_tx(BQ, (uint32_t)(kPfTiles * NH * qrows * 128));
      __syncwarp();
      q_last = ic;
      if (lane < kPfTiles * NH)
        tma_load_3d(sbase + S::Q_OFF + (lane / NH) * S::TILE + (lane % NH) * S::HALF, &qmap, BQ,
                    (lane % NH) * 64, it.kvh * g, it.q0 + it.t0 + (lane / NH) * tq);
      const int32_t* table = p.block_tables + (int64_t)it.s * p.max_blocks;
      bool stop = false;
      for (int j = 0; j < it.ntiles; ++j, ++kc) {
        const int st = kc % STAGES;
        const uint32_t use = kc / STAGES;
        const int key0 = it.kb + j * kPfKeys;
        const int nch = min(KCH, (it.kend - key0 + 15) / 16);
        const bool mine = boxer && c < nch;
        int blk = 0, row = 0;
        bool bad = false;
        if (mine) {
          const int key = key0 + 16 * c;
          blk = table[key / p.block_size];
          bad = blk < 0 || blk >= p.num_blocks;
          row = it.kvh * p.block_size + key % p.block_size;
        }
        if (__any_sync(0xffffffffu, bad)) {
          if (lane == 0) {
            atomicCAS(p.err, 0, KV_ERR_BOUNDS);
            *abort_flag = 1;
          }
          stop = true;
          break;
        }
        const uint32_t bytes = (uint32_t)(nch * NH * 16 * 128);
        if (use > 0 &&
            !__all_sync(0xffffffffu, pf::wait(KE(st), (use - 1) & 1, abort_flag, p.err))) {
          stop = true;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(KF(st), bytes);
        __syncwarp();
        if (mine)
          tma_load_3d(sbase + S::K_OFF + st * S::TILE + h * S::HALF + c * 2048, &kmap, KF(st),
                      h * 64, row, blk);
        nk = kc + 1;
        if (use > 0 &&
            !__all_sync(0xffffffffu, pf::wait(VE(st), (use - 1) & 1, abort_flag, p.err))) {
          stop = true;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(VF(st), bytes);
        __syncwarp();
        if (mine)
          tma_load_3d(sbase + S::V_OFF + st * S::TILE + h * S::HALF + c * 2048, &vmap, VF(st),
                      h * 64, row, blk);
        nv = kc + 1;
      }
      if (stop) break;
      ++ic;
    }
    if (lane == 0 && *abort_flag) {
      // let the copies and the launch-control answer in flight land before
      // the shared memory is released
      for (uint32_t kk = nk > STAGES ? nk - STAGES : 0; kk < nk; ++kk)
        (void)mbar_wait_bounded(KF(kk % STAGES), (kk / STAGES) & 1, kPfDrainNs);
      for (uint32_t kk = nv > STAGES ? nv - STAGES : 0; kk < nv; ++kk)
        (void)mbar_wait_bounded(VF(kk % STAGES), (kk / STAGES) & 1, kPfDrainNs);
      if (q_last >= 0) (void)mbar_wait_bounded(BQ, (uint32_t)q_last & 1, kPfDrainNs);
      if (asked > read) (void)mbar_wait_bounded(CF(slot_of(asked)), use_of(asked), kPfDrainNs);
    }
  } else if (warp == 9) {
    // --------------------------------------------------------------- MMA
    // Per item: S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) ...:
    // the softmax of one query tile runs while the tensor cores work on the
    // other's P.V and next S.
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_f16(kBf16, kPfRows, kPfKeys, false);
      constexpr uint32_t kIdO = tc::idesc_f16(kBf16, kPfRows, D, true);
      // Shared-memory descriptors of the Q, K and V regions, built once: the
      // start-address field (address >> 4, bits 0-13) of a position inside a
      // region is the region's plus (offset >> 4), as shared-memory addresses
      // stay below 256 KB and the field never carries; each MMA then costs
      // the issuing thread one add per operand.
      const uint64_t dQ = tc::desc_sw128(sbase + S::Q_OFF, 16, 1024);
      const uint64_t dK = tc::desc_sw128(sbase + S::K_OFF, 16, 1024);
      const uint64_t dV = tc::desc_sw128(sbase + S::V_OFF, S::HALF, 1024);
      auto issue_s = [&](int x, uint32_t kt) {
        const uint64_t q0 = dQ + (uint64_t)((x * S::TILE) >> 4);
        const uint64_t k0 = dK + (uint64_t)(((kt % STAGES) * S::TILE) >> 4);
        const uint32_t d = tmem + S::S_COL + x * kPfKeys;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * S::HALF + (kk % 4) * 32) >> 4;  // 16 columns per step
          tc::mma_ss(d, q0 + off, k0 + off, kIdS, kk > 0 ? 1u : 0u);
        }
        tc::commit(SF(x));
      };
      auto issue_pv = [&](int x, uint32_t kt, bool first) {
        const uint64_t v0 = dV + (uint64_t)(((kt % STAGES) * S::TILE) >> 4);
        const uint32_t aP = tmem + S::S_COL + x * kPfKeys, d = tmem + S::O_COL + x * D;
#pragma unroll
        for (int kk = 0; kk < KCH; ++kk) {
          // keys 16kk..16kk+15: their 16-bit values in columns 16kk..16kk+7,
          // (bf16) the residuals in the next 8
          const uint64_t bV = v0 + (uint64_t)((kk * 2048) >> 4);
          tc::mma_ts(d, aP + 16 * kk, bV, kIdO, (!first || kk > 0) ? 1u : 0u);
          if constexpr (kSplit) tc::mma_ts(d, aP + 16 * kk + 8, bV, kIdO, 1u);
        }
        tc::commit(PV(x));
      };
      uint32_t ic = 0, kc = 0, sc[kPfTiles] = {0, 0}, oc[kPfTiles] = {0, 0};
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        int64_t v = blockIdx.x;
        if (k > 0) {
          if (!pf::wait(CF(slot_of(k)), use_of(k), abort_flag, p.err)) break;
          v = pf::clc_item(RESP(slot_of(k)));
          mbar_arrive(CR(slot_of(k)));
        }
        if (v < 0) break;
        pf::Item it;
        if (!pf::item_at(p, v, false, it)) continue;
        ok = pf::wait(BQ, ic & 1, abort_flag, p.err) &&
             pf::wait(KF(kc % STAGES), (kc / STAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        tc::fence_after();
#pragma unroll
        for (int x = 0; x < kPfTiles; ++x)
          if (it.ntx[x] > 0) issue_s(x, kc);
        tc::commit(KE(kc % STAGES));
        if (it.ntiles == 1) tc::commit(QE);  // the item's last S: its query tiles may be replaced
        for (int j = 0; ok && j < it.ntiles; ++j) {
          const uint32_t kt = kc + j, kn = kt + 1;
          const int st = kt % STAGES;
          bool waited_k = false;
          if (!pf::wait(VF(st), (kt / STAGES) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int x = 0; x < kPfTiles; ++x) {
            if (j < it.ntx[x]) {
              // the first P.V of an item overwrites O_x: the previous item's
              // output must have been read
              if (j == 0 && oc[x] > 0 && !pf::wait(OF(x), (oc[x] - 1) & 1, abort_flag, p.err)) {
                ok = false;
                break;
              }
              if (!pf::wait(PF(x), (sc[x] + j) & 1, abort_flag, p.err)) {
                ok = false;
                break;
              }
              tc::fence_after();
              issue_pv(x, kt, j == 0);
            }
            if (j + 1 < it.ntx[x]) {
              if (!waited_k) {
                if (!pf::wait(KF(kn % STAGES), (kn / STAGES) & 1, abort_flag, p.err)) {
                  ok = false;
                  break;
                }
                tc::fence_after();
                waited_k = true;
              }
              issue_s(x, kn);
            }
          }
          if (!ok) break;
          tc::commit(VE(st));
          if (j + 1 < it.ntiles) {
            tc::commit(KE(kn % STAGES));
            if (j + 2 == it.ntiles) tc::commit(QE);
          }
        }
        if (!ok) break;
#pragma unroll
        for (int x = 0; x < kPfTiles; ++x) {
          sc[x] += it.ntx[x];
          oc[x] += it.ntx[x] > 0 ? 1 : 0;
        }
        kc += it.ntiles;
        ++ic;
      }
      // every MMA issued must finish before TMEM is released
      tc::commit(FIN);
      (void)mbar_wait_bounded(FIN, 0, kPfDrainNs);
    }
  } else {
    // ------------------------------------ softmax: one row a thread, warps
    // 0-3 own query tile A, warps 4-7 tile B
    const int x = warp / 4;
    const int r = threadIdx.x % kPfRows;
    const int tok = r / g, head = r - tok * g;
    const uint32_t lane_addr = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + S::S_COL + x * kPfKeys;
    const uint32_t tO = tmem + lane_addr + S::O_COL + x * D;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, kc = 0;  // this query tile's S tiles so far; K/V tiles so far
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
    int64_t v = blockIdx.x;
    if (k > 0) {
      ok = __all_sync(0xffffffffu, pf::wait(CF(slot_of(k)), use_of(k), abort_flag, p.err));
      if (!ok) break;
      v = pf::clc_item(RESP(slot_of(k)));
      __syncwarp();
      if (lane == 0) mbar_arrive(CR(slot_of(k)));
    }
    if (v < 0) break;
    pf::Item it;
    if (!pf::item_at(p, v, false, it)) continue;
    const int nt = x ? it.ntx[1] : it.ntx[0];  // selects keep the per-tile values in registers
    if (nt == 0) {
      kc += it.ntiles;
      continue;
    }
    const bool valid = r < qrows && tok < (x ? it.ntok[1] : it.ntok[0]);
    const bool prefix = p.part_o != nullptr;
    const int prow = valid && !prefix ? it.n - it.q_len + it.t0 + x * tq + tok
                                      : (x ? it.kendx[1] : it.kendx[0]) - 1;
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < nt; ++j) {
      ok = __all_sync(0xffffffffu, pf::wait(SF(x), (sc + j) & 1, abort_flag, p.err));
      if (!ok) break;
      tc::fence_after();
      const int lim = prow - it.kb - j * kPfKeys;  // columns wlo .. lim are visible
      const int wlo = p.window > 0 ? lim - p.window + 1 : INT_MIN;
      const bool masked = lim < kPfKeys - 1 || wlo > 0;
      // pass 1: the row max.  Only tiles on the causal diagonal mask
      // anything; a warp takes the masked code only when one of its rows needs it.
      const bool wmask = __any_sync(0xffffffffu, masked);
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
      {
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::ld32(tS + 32 * c, sr[c]);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::pin(sr[c]);
        auto row_max = [&](auto kMask) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float v0 = __uint_as_float(sr[c][i]), v1 = __uint_as_float(sr[c][i + 1]);
              if constexpr (decltype(kMask)::value) {
                if (32 * c + i > lim || 32 * c + i < wlo) v0 = -INFINITY;
                if (32 * c + i + 1 > lim || 32 * c + i + 1 < wlo) v1 = -INFINITY;
              }
              mx8[(i / 2) % 8] = pf::max3(mx8[(i / 2) % 8], v0, v1);
            }
        };
        if (wmask) row_max(std::true_type{});
        else row_max(std::false_type{});
      }
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx8[i] = fmaxf(mx8[i], mx8[i + w]);
      const float mt = mx8[0] * sl2;
      const bool grow = mt > m_ref + kPfLazyLog2;
      const float m_new = grow ? mt : m_ref;
      const float alpha = grow ? ex2(m_ref - m_new) : 1.f;
      __syncwarp();
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds P.V up to tile j - 1: wait for it, then rescale in TMEM
        ok = __all_sync(0xffffffffu, pf::wait(PV(x), (sc + j - 1) & 1, abort_flag, p.err));
        if (!ok) break;
        tc::fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tc::ld32(tO + 32 * c, o);
          tc::wait_ld();
          tc::pin(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::st32(tO + 32 * c, o);
        }
      }
      m_ref = m_new;
      // pass 2: P over S's own columns, 16 keys at a time: keys 16m + 2i,
      // 16m + 2i + 1 go to column 16m + i as a 16-bit pair, (bf16) their
      // rounding residuals to column 16m + 8 + i.  Pairs of keys run through
      // the .f32x2 instructions.
      const uint64_t sl2x2 = pf::f2(sl2, sl2), negm = pf::f2(-m_ref, -m_ref);
      uint64_t ls2[2] = {pf::f2(l * alpha, 0.f), pf::f2(0.f, 0.f)};
      auto probs = [&](auto kMask) {
        // 16 keys (16 columns of S) at a time; the next 16 are loading while
        // these are computed
        uint32_t sv0[16], sv1[16];
        auto chunk = [&](const uint32_t(&cur)[16], int m) {
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint64_t t = pf::fma2(pf::f2(__uint_as_float(cur[2 * i]), __uint_as_float(cur[2 * i + 1])),
                                        sl2x2, negm);
            float ta, tb;
            pf::f2_split(t, ta, tb);
            float a = ex2(ta), e = ex2(tb);
            if constexpr (decltype(kMask)::value) {
              if (16 * m + 2 * i > lim || 16 * m + 2 * i < wlo) a = 0.f;
              if (16 * m + 2 * i + 1 > lim || 16 * m + 2 * i + 1 < wlo) e = 0.f;
            }
            const uint64_t ae = pf::f2(a, e);
            ls2[i % 2] = pf::add2(ls2[i % 2], ae);
            if constexpr (kSplit) {
              hi[i] = pack2<true>(a, e);
              float ra, rb;
              pf::f2_split(pf::sub2(ae, pf::f2(__uint_as_float(hi[i] << 16),
                                               __uint_as_float(hi[i] & 0xffff0000u))), ra, rb);
              lo[i] = pack2<true>(ra, rb);
            } else {
              hi[i] = pack2<false>(a, e);
              lo[i] = 0u;
            }
          }
          tc::st8(tS + 16 * m, hi);
          if constexpr (kSplit) tc::st8(tS + 16 * m + 8, lo);
        };
        tc::ld16(tS, sv0);
        tc::wait_ld();
        tc::pin(sv0);
#pragma unroll 1
        for (int m = 0; m < kPfKeys / 16; m += 2) {
          tc::ld16(tS + 16 * (m + 1), sv1);
          chunk(sv0, m);
          tc::wait_ld();
          tc::pin(sv1);
          if (m + 2 < kPfKeys / 16) tc::ld16(tS + 16 * (m + 2), sv0);
          chunk(sv1, m + 1);
          if (m + 2 < kPfKeys / 16) {
            tc::wait_ld();
            tc::pin(sv0);
          }
        }
      };
      if (wmask) probs(std::true_type{});
      else probs(std::false_type{});
      {
        float s0, s1, s2, s3;
        pf::f2_split(ls2[0], s0, s1);
        pf::f2_split(ls2[1], s2, s3);
        l = (s0 + s1) + (s2 + s3);
      }
      tc::wait_st();
      if (j == nt - 1 && it.kend - it.kb - j * kPfKeys < kPfKeys) {
        // this tile's last K/V tile: zero the V rows past every key the CTA
        // reads (stale slots may hold any bits, and 0 * NaN is NaN); both
        // query tiles may write the same zeros
        const uint32_t kt = kc + j;
        const int st = kt % STAGES;
        ok = __all_sync(0xffffffffu, pf::wait(VF(st), (kt / STAGES) & 1, abort_flag, p.err));
        if (!ok) break;
        if (r >= it.kend - it.kb - j * kPfKeys) {
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            uint4* row = reinterpret_cast<uint4*>(smem + S::V_OFF + st * S::TILE + h * S::HALF + r * 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) row[i] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        pf::fence_proxy_async();
        __syncwarp();
      }
      tc::fence_before();
      mbar_arrive(PF(x));
    }
    if (ok) ok = __all_sync(0xffffffffu, pf::wait(PV(x), (sc + nt - 1) & 1, abort_flag, p.err));
    if (ok) {
      tc::fence_after();
      const float inv = 1.f / l;
      const int64_t orow =
          ((int64_t)(it.q0 + it.t0 + x * tq + tok) * p.num_q_heads + it.kvh * g + head) * D;
      // shared-prefix mode: partition 0 of the row's sequence, unnormalised
      int64_t prow_part = -1;
      if (prefix && valid) {
        const int64_t sq = p.prefix_rows[it.q0 + it.t0 + x * tq + tok];
        prow_part = (sq * p.num_q_heads + it.kvh * g + head) * p.num_parts;
        *reinterpret_cast<float4*>(p.part_ml + prow_part * 4) = make_float4(m_ref, l, m_ref, 0.f);
      }
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tc::ld32(tO + 32 * c, o);
        tc::wait_ld();
        tc::pin(o);
        if (prow_part >= 0) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow_part * D + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        } else if (valid && !prefix) {
          if (p.out_kind == PF_OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                   __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(
                  pack2<kBf16>(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                  pack2<kBf16>(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                  pack2<kBf16>(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                  pack2<kBf16>(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
          }
        }
        __syncwarp();
      }
      // O_x is read: the next item's first P.V may overwrite it
      tc::fence_before();
      mbar_arrive(OF(x));
    }
    sc += nt;
    kc += it.ntiles;
    }
  }

  // TMEM is released once every role is done with it
  tc::fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc::fence_after();
    tc::dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace pagedkv
