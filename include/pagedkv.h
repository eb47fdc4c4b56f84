/*
 * pagedkv — paged KV cache and PagedAttention decode for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point returns an int status (KV_OK or a negative
 * KV_ERR_* code); kv_last_error() gives a message for the calling thread's
 * last failure.  GPU entry points only enqueue work on the caller's stream
 * and never synchronise (except kv_get_device_error).  The library never
 * allocates device memory: the caller owns every device buffer and passes
 * raw pointers.  Host handles (kv_pool, kv_alloc, kv_sched) are owned by the
 * library between their create and destroy calls and are not thread-safe.
 *
 * The method follows the page "vLLM 推理加速原理详解：大模型服务吞吐量为何能
 * 提升 10 倍" (fudengji.cn), cited below by section:
 *   [PA]   "PagedAttention：把操作系统的虚拟内存搬进 GPU" — the KV cache is cut
 *          into fixed-size physical blocks; a per-sequence block table maps
 *          logically contiguous blocks to physically scattered ones; blocks
 *          are taken on demand; several logical blocks may share one physical
 *          block; the attention kernel reads K/V from the non-contiguous
 *          blocks.
 *   [CB]   "连续批处理：别再等最慢的那个请求了" — after every decode iteration,
 *          free the finished requests' blocks, read the free-block count,
 *          admit waiting requests first come first served while blocks allow
 *          (free_blocks > MIN_BLOCKS and can_allocate), then decode the
 *          running set.
 *   [PIT]  "vLLM 也不是银弹：真实部署中的坑" — FP8 KV cache as the remedy for
 *          long-context memory pressure; the whole cache is one preallocated
 *          pool.
 *   [MON]  "从零开始：vLLM 部署的实战建议", step four — running / waiting
 *          request counts and cache usage as the metrics to watch.
 *
 * Pool layout (the pages leave it open; this library fixes it): for each
 * layer, K and V are separate device arrays, each
 *     [num_blocks][kv_heads][block_size][head_dim]
 * elements, row-major, so one (block, kv head) tile of block_size x head_dim
 * elements is contiguous.  A token slot is block * block_size + offset.  For
 * FP8 pools each layer also has K and V scale arrays [num_blocks][kv_heads]
 * of fp32: the stored E4M3 code times its (block, head) scale is the value.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* kv_stream_t;

/* Element types.  KV_F32 is valid only as an attention output type. */
typedef enum { KV_F16 = 0, KV_BF16 = 1, KV_FP8_E4M3 = 2, KV_F32 = 3 } kv_dtype;

enum {
  KV_OK = 0,
  KV_ERR_ARG = -1,     /* invalid argument; nothing was enqueued */
  KV_ERR_OOM = -2,     /* the allocator has too few free blocks */
  KV_ERR_STATE = -3,   /* unknown / duplicate sequence, double free, unbound layer */
  KV_ERR_BOUNDS = -4,  /* device-reported: block id, slot or length out of range */
  KV_ERR_CUDA = -5,    /* a CUDA runtime / driver call failed */
  KV_ERR_TIMEOUT = -6  /* device-reported: a pipeline wait gave up (bounded spin) */
};

/* Preemption modes of the scheduling step (kv_sched_set_preemption). */
typedef enum { KV_PREEMPT_NONE = 0, KV_PREEMPT_SWAP = 1, KV_PREEMPT_RECOMPUTE = 2 } kv_preempt_mode;

typedef struct kv_pool kv_pool;
typedef struct kv_alloc kv_alloc;
typedef struct kv_sched kv_sched;
typedef struct kv_serve kv_serve;

/* Message for the calling thread's most recent failure ("" if none). */
const char* kv_last_error(void);
/* ABI version, currently 1. */
int kv_version(void);

/* ------------------------------------------------------------------ pool */

/* Describe a preallocated pool ([PA], [PIT]): num_layers layers of
 * num_blocks physical blocks of block_size token slots for kv_heads heads of
 * head_dim elements of `dtype` (KV_F16, KV_BF16 or KV_FP8_E4M3).
 * Supported: block_size 16, 32, 64, 128 or 256; head_dim 64 or 128;
 * num_blocks >= 1; 1 <= kv_heads; 1 <= num_layers <= 4096.  Host only; no
 * device work.  *out is owned by the caller until kv_pool_destroy.
 * Errors: KV_ERR_ARG for an unsupported geometry. */
int kv_pool_create(int block_size, int num_blocks, int kv_heads, int head_dim,
                   kv_dtype dtype, int num_layers, kv_pool** out);

/* Bytes the caller must allocate per layer for K (and the same again for
 * V), and for each FP8 scale array (0 for 16-bit pools).  Either pointer may
 * be NULL. */
int kv_pool_bytes(const kv_pool* pool, size_t* kv_bytes_per_layer,
                  size_t* scale_bytes_per_layer);

/* Attach caller-owned device memory to `layer`: k_base and v_base of
 * kv_bytes_per_layer bytes each, 16-byte aligned; k_scale and v_scale
 * [num_blocks][kv_heads] fp32 for FP8 pools (NULL otherwise).  Builds the
 * layer's TMA descriptors, so it needs a working CUDA driver; the pointers
 * must belong to the device that later launches use.  Rebinding replaces the
 * old pointers.  Errors: KV_ERR_ARG (bad layer, NULL or misaligned pointer,
 * scales missing for FP8), KV_ERR_CUDA (descriptor creation failed). */
int kv_pool_bind(kv_pool* pool, int layer, void* k_base, void* v_base, float* k_scale,
                 float* v_scale);

/* Decode launch configuration.  partition_tokens: context-partition length
 * for split decode, else a multiple of 16 in [16, 16384]; contexts longer
 * than one partition are split into partitions whose partial results are
 * merged by a log-sum-exp reduce (see paged_attention_decode).  0 chooses
 * automatically: partitions of at most 4096 tokens; if batch * kv_heads is
 * under three waves of resident CTAs, enough partitions (of at least 512
 * tokens) for four waves, raised (up to twice) until the last wave of
 * equal partitions is at least 85% full.  A context that fits one partition
 * is written directly and skips the reduce.  stages: shared-memory pipeline
 * depth per warp, 0 for automatic, else 2, 3, 4, 6 or 8; warps: warps per
 * CTA, 0 for automatic, else 4 or 8.  Automatic: 4 warps x 3 stages for
 * 8 KB and 4 KB stages (16-bit or FP8 with head_dim 128, 16-bit with 64;
 * 2 stages for 8 KB stages with GQA groups of 4 or more), 4 x 6 for 2 KB
 * stages.  A shape whose shared memory exceeds 227 KB per CTA is rejected
 * with KV_ERR_ARG.  Host only. */
int kv_pool_set_decode_config(kv_pool* pool, int partition_tokens, int stages, int warps);

int kv_pool_destroy(kv_pool* pool);

/* ------------------------------------------------------------ cache write */

/* Scatter new tokens' K and V into their slots ([PA]: blocks grow on demand,
 * each new token goes to the slot its sequence's table assigns).
 *   k_new, v_new   device [num_tokens][kv_heads][head_dim] of src_dtype
 *                  (KV_F16 or KV_BF16); for 16-bit pools src_dtype must be
 *                  the pool dtype and the bits are copied unchanged.
 *   slot_mapping   device int64 [num_tokens]; token t goes to block
 *                  slot / block_size, offset slot % block_size; slot < 0
 *                  skips the token.
 *   k_inv_scale, v_inv_scale   FP8 pools only: device fp32
 *                  [num_blocks][kv_heads]; each value is widened to fp32,
 *                  multiplied in fp32 by inv_scale[block][head], rounded to
 *                  E4M3 to nearest even and saturated to +-448 (NaN stays
 *                  NaN).  NULL for 16-bit pools.
 * Slots must be distinct (two tokens into one slot race).  A slot beyond the
 * pool is skipped and reported as KV_ERR_BOUNDS by kv_get_device_error.
 * num_tokens == 0 enqueues nothing.  Errors: KV_ERR_ARG, KV_ERR_STATE
 * (layer not bound), KV_ERR_CUDA (launch failed). */
int paged_kv_write(const kv_pool* pool, int layer, const void* k_new, const void* v_new,
                   kv_dtype src_dtype, const int64_t* slot_mapping, int num_tokens,
                   const float* k_inv_scale, const float* v_inv_scale, kv_stream_t stream);

/* ------------------------------------------------------------- block copy */

/* Copy-on-write support for shared blocks ([PA]: several logical blocks may
 * map to one physical block; a sequence that writes into a shared block
 * first gets a private copy).  pairs: device int32 [num_pairs][2] of
 * (src, dst) physical block ids.  For every bound layer, K and V (and the
 * FP8 scales) of block src are copied to block dst.  Pairs run in parallel:
 * every dst must be distinct and must not be any pair's src.  An id outside
 * the pool skips that pair and is reported as KV_ERR_BOUNDS by
 * kv_get_device_error.  num_pairs == 0 enqueues nothing.  Errors:
 * KV_ERR_ARG, KV_ERR_STATE (a layer not bound), KV_ERR_CUDA. */
int block_copy(const kv_pool* pool, const int32_t* pairs, int num_pairs, kv_stream_t stream);

/* -------------------------------------------------------- decode attention */

/* Scratch bytes paged_attention_decode needs for these sizes (0 when no
 * context is split).  Same partition policy as the decode call. */
size_t paged_attention_workspace_bytes(const kv_pool* pool, int batch, int num_q_heads,
                                       int max_context_len);

/* PagedAttention decode ([PA]): for every sequence s and query head h,
 *     out[s][h] = sum_t softmax_t(scale * q[s][h] . K_t) V_t
 * over the sequence's tokens t < context_lens[s], where token t is read at
 * block block_tables[s][t / block_size], offset t % block_size, kv head
 * h / (num_q_heads / kv_heads) (consecutive query heads share a kv head).
 * Softmax and accumulation run in fp32 with a running max and sum.
 *   q             device [batch][num_q_heads][head_dim] of q_dtype; for
 *                 16-bit pools q_dtype must be the pool dtype; FP8 pools
 *                 take KV_F16 or KV_BF16 queries.
 *   num_q_heads   a multiple of kv_heads with num_q_heads / kv_heads <= 8.
 *   block_tables  device int32 [batch][max_blocks_per_seq]; entries past
 *                 ceil(context_len / block_size) are not read.
 *   context_lens  device int32 [batch]; 0 gives an all-zero output row.
 *   max_context_len  host upper bound on every context_lens entry; it sizes
 *                 the launch.  A length above it, above
 *                 max_blocks_per_seq * block_size, or negative is clamped
 *                 and reported as KV_ERR_BOUNDS by kv_get_device_error, as is
 *                 a block id outside the pool (that block is skipped).
 *   out           device [batch][num_q_heads][head_dim] of out_dtype
 *                 (q_dtype or KV_F32).
 *   workspace     device scratch of workspace_bytes >=
 *                 paged_attention_workspace_bytes(...), 16-byte aligned;
 *                 may be NULL when that is 0.  Contexts longer than one
 *                 partition are split: each partition writes its unnormalised
 *                 output and its running maxima and sum there
 *                 (head_dim + 4 floats per (sequence, head, partition)),
 *                 followed by one int merge counter per (sequence, kv head),
 *                 and the partials are merged by log-sum-exp: by the last
 *                 partition CTA of each (sequence, kv head) to finish when a
 *                 16-bit pool's contexts split into at most 4 partitions,
 *                 else by a second kernel.  The call zeroes the counters on
 *                 the stream itself; the workspace needs no initialisation.
 *   seq_order     NULL, or device int32 [batch]: a permutation of 0..batch-1
 *                 giving the order in which sequences are scheduled onto the
 *                 GPU; outputs are unaffected.  Longest context first keeps
 *                 long sequences from starting last (a tail of idle SMs).
 *                 An entry outside [0, batch) is skipped and reported as
 *                 KV_ERR_BOUNDS.
 * batch == 0 enqueues nothing.  Errors: KV_ERR_ARG, KV_ERR_STATE (layer not
 * bound), KV_ERR_CUDA. */
int paged_attention_decode(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                           int num_q_heads, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* context_lens, int batch,
                           int max_context_len, float scale, void* out, kv_dtype out_dtype,
                           void* workspace, size_t workspace_bytes, const int32_t* seq_order,
                           kv_stream_t stream);

/* Sliding-window attention (the long-context remedy named among the
 * pitfalls of "vLLM 推理加速原理详解"; the page gives no definition): with
 * window > 0, paged_attention_decode attends, for a sequence of n tokens,
 * only to its last min(n, window) tokens (positions n - window .. n - 1), and
 * reads no block before the one holding position n - window, so blocks that
 * left the window may be released (kv_alloc_release_before).
 * paged_attention_prefill applies the same band to every new token (it
 * attends to its own last `window` positions) and reads no block wholly
 * before the first new token's window.  0 turns the window off.  Workspace
 * sizes follow the window.  Host only; KV_ERR_ARG for a negative window. */
int kv_pool_set_sliding_window(kv_pool* pool, int window);

/* Multi-token attention over the paged cache: the step that processes a
 * prompt, a chunk of one, or a few drafted tokens before decoding continues
 * ([PA], and the time-to-first-token discussion of the page's section
 * "连续批处理：别再等最慢的那个请求了"; the pages give no kernel for it).
 * Sequence s has n = context_lens[s] tokens in the cache, the last
 * q_len = cu_seqlens_q[s+1] - cu_seqlens_q[s] of which are its new tokens,
 * already written (paged_kv_write); new token i sits at position
 * n - q_len + i and attends causally to positions 0 .. n - q_len + i:
 *     out[r][h] = sum_{t <= pos} softmax_t(scale * q[r][h] . K_t) V_t,
 * r = cu_seqlens_q[s] + i, kv head h / (num_q_heads / kv_heads).  q_len = 1
 * is a decode step; q_len = n a whole prompt.  Runs on the tensor cores
 * (tcgen05) with fp32 accumulation and softmax.
 *   pool          f16 or bf16, head_dim 64 or 128 (others: KV_ERR_ARG).
 *   q             device [total_q][num_q_heads][head_dim] of the pool dtype,
 *                 16-byte aligned.
 *   cu_seqlens_q  device int32 [batch + 1], non-decreasing from 0;
 *                 total_q = cu_seqlens_q[batch] (host copy of it).
 *   max_q_len     host upper bound on every q_len; it sizes the launch.
 *   block_tables  device int32 [batch][max_blocks_per_seq].
 *   context_lens  device int32 [batch].  A sequence with q_len < 0,
 *                 q_len > n, q_len > max_q_len, rows past total_q, or
 *                 n > max_blocks_per_seq * block_size is skipped and
 *                 reported as KV_ERR_BOUNDS by kv_get_device_error, as is a
 *                 block id outside the pool (the CTA that meets it stops; the
 *                 rows of its current work item, and of the one it had
 *                 already claimed, are left unwritten).  A pipeline wait that
 *                 runs out (2 s) records KV_ERR_TIMEOUT the same way.
 *   scale         finite and > 0.
 *   out           device [total_q][num_q_heads][head_dim] of out_dtype (the
 *                 pool dtype or KV_F32), 16-byte aligned.
 * batch, total_q or max_q_len == 0 enqueues nothing.  No workspace.  Errors:
 * KV_ERR_ARG, KV_ERR_STATE (layer not bound), KV_ERR_CUDA.
 * The first call on a device (this one or paged_attention_decode_shared_prefix)
 * looks up the device address of the library's error word and keeps it until
 * the process exits; after cudaDeviceReset that address is stale, so a process
 * that resets a device must not call these two entry points on it again. */
int paged_attention_prefill(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                            int num_q_heads, const int32_t* cu_seqlens_q, int total_q,
                            int max_q_len, const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int batch, float scale, void* out,
                            kv_dtype out_dtype, kv_stream_t stream);

/* Bytes one host swap slot holds: for every layer, K then V, each the
 * block's kv_heads x block_size x head_dim elements followed (FP8) by its
 * kv_heads fp32 scales padded to 16 bytes. */
size_t kv_swap_block_bytes(const kv_pool* pool);

/* Swap copies for preemption, over the host link: the kernel reads or
 * writes the host swap space directly.  host_swap: pinned host memory
 * mapped into the device (e.g. cudaHostAlloc / a pinned torch tensor),
 * num_slots x kv_swap_block_bytes, 16-byte aligned.  pairs: device int32
 * [num_pairs][2], (device block, host slot) for kv_swap_out and (host slot,
 * device block) for kv_swap_in; every layer, K, V and FP8 scales move.  An
 * index out of range is skipped and reported as KV_ERR_BOUNDS by
 * kv_get_device_error.  Asynchronous on `stream`.  Errors: KV_ERR_ARG (host
 * memory not mapped, misaligned), KV_ERR_STATE (layer not bound),
 * KV_ERR_CUDA. */
int kv_swap_out(const kv_pool* pool, void* host_swap, int num_slots, const int32_t* pairs,
                int num_pairs, kv_stream_t stream);
int kv_swap_in(const kv_pool* pool, const void* host_swap, int num_slots, const int32_t* pairs,
               int num_pairs, kv_stream_t stream);

/* Decode for a batch in which some sequences share their first prefix_len
 * tokens through the same physical blocks (forked sequences, a common
 * system prompt or document; [PA]: blocks shared by reference count).  The
 * result is that of paged_attention_decode on the same arguments; only the
 * work is split: the shared prefix is attended once for all sharing
 * sequences on the tensor cores (their queries are the rows of one
 * multi-token pass over the prefix's blocks, no causal mask), each
 * sequence's own tokens by the decode kernel, and the two partial results
 * are merged by the log-sum-exp reduce.  The prefix's blocks are then read
 * once per kv head instead of once per sequence and kv head.
 *   Arguments as paged_attention_decode, plus:
 *   prefix_seqs    device int32 [num_sharers]: batch indices of the
 *                  sequences that share the prefix (each once).
 *   prefix_blocks  device int32 [prefix_len / block_size]: its blocks; for
 *                  every sharer s, block_tables[s][0 ..] starts with them and
 *                  context_lens[s] >= prefix_len (not checked: other tables
 *                  give another result).
 *   prefix_len     tokens of the prefix, whole blocks (0: plain decode).
 *   skip_lens      device int32 [batch]: prefix_len for the sharers, 0 for
 *                  every other sequence.
 *   workspace      device, 16-byte aligned, at least
 *                  paged_attention_shared_prefix_workspace_bytes(pool, batch,
 *                  num_q_heads, max_context_len, num_sharers) bytes (always
 *                  needed); q must be 16-byte aligned.
 *   Pools: f16 or bf16, no sliding window (others: KV_ERR_ARG).  Enqueues a
 *   row gather, one multi-token launch, the decode and the reduce on
 *   `stream`.  Device-side errors as paged_attention_decode (a sharer index
 *   outside the batch or a skip length that is not a multiple of 16 within
 *   the context: KV_ERR_BOUNDS). */
size_t paged_attention_shared_prefix_workspace_bytes(const kv_pool* pool, int batch, int num_q_heads,
                                                     int max_context_len, int num_sharers);
int paged_attention_decode_shared_prefix(const kv_pool* pool, int layer, const void* q, kv_dtype q_dtype,
                                         int num_q_heads, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens, int batch,
                                         int max_context_len, const int32_t* prefix_seqs, int num_sharers,
                                         const int32_t* prefix_blocks, int prefix_len,
                                         const int32_t* skip_lens, float scale, void* out,
                                         kv_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                         const int32_t* seq_order, kv_stream_t stream);

/* Largest scratch paged_attention_decode_noalloc can use (16 MiB). */
#define KV_NOALLOC_WORKSPACE_BYTES (16u << 20)

/* The same decode as paged_attention_decode, for callers that cannot
 * allocate device memory: a C host program or plugin that only receives the
 * pool and the tensors it is handed, code whose whole memory budget is
 * already given to the KV pool, or a hot path that must not call cudaMalloc
 * because it can synchronise the device.  Instead of a caller-provided
 * workspace, the split-K partials go to one scratch array that the library
 * defines in device memory at file scope, KV_NOALLOC_WORKSPACE_BYTES long;
 * every GPU that loads the library holds it until the process exits.  This
 * entry point allocates nothing and has no counterpart on the pages; it is an
 * interface convenience only.
 *   Arguments are those of paged_attention_decode without the workspace
 *   (and with sequences scheduled in batch order).
 *   Sizes whose paged_attention_workspace_bytes(...) exceeds
 *   KV_NOALLOC_WORKSPACE_BYTES are rejected with KV_ERR_ARG (use
 *   paged_attention_decode with your own workspace, or a partition setting
 *   that needs fewer partials).
 *   The first call on a device looks up the scratch array's device address
 *   (once per device, with that device current); make that first call before
 *   any stream capture.  The address is kept until the process exits: after
 *   cudaDeviceReset the library's device memory is reloaded elsewhere, so a
 *   process that resets a device must not call this entry point again on it.
 *   All calls share the one array, which keeps whatever the last call wrote;
 *   nothing in it has to start at zero, because every partial a call reads
 *   was written earlier in that same call.  Calls whose kernels can overlap
 *   on the GPU (other streams, other host threads) race on the array and
 *   must be serialised by the caller.
 * Errors: as paged_attention_decode, plus KV_ERR_CUDA if the scratch address
 * lookup fails. */
int paged_attention_decode_noalloc(const kv_pool* pool, int layer, const void* q,
                                   kv_dtype q_dtype, int num_q_heads,
                                   const int32_t* block_tables, int max_blocks_per_seq,
                                   const int32_t* context_lens, int batch, int max_context_len,
                                   float scale, void* out, kv_dtype out_dtype, kv_stream_t stream);

/* Self-test of the device-side failure path: enqueues one warp that waits,
 * with the same bounded wait the decode pipeline uses, on a barrier that
 * nothing completes.  After limit_ns nanoseconds (at most 10 s) the wait
 * gives up and the kernel records KV_ERR_TIMEOUT, which the next
 * kv_get_device_error returns; nothing is left in flight and the context
 * stays usable.  For tests and health checks. */
int kv_selftest_wait_timeout(uint64_t limit_ns, kv_stream_t stream);

/* Synchronise `stream`, then read and clear the current device's error word:
 * *err = KV_OK, KV_ERR_BOUNDS or KV_ERR_TIMEOUT (the first error any kernel
 * of this library recorded since the last call).  Errors: KV_ERR_CUDA. */
int kv_get_device_error(kv_stream_t stream, int* err);

/* ------------------------------------------------------ block allocator */

/* Refcounted free-list allocator of physical blocks ([PA]: blocks on demand,
 * any free block serves any request, shared blocks).  Deterministic: the free
 * list is FIFO (take from the head, freed blocks go to the tail in block-table
 * order); initial_free_order (a permutation of 0..num_blocks-1, or NULL for
 * ascending) sets its starting order.  Host only. */
int kv_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                    kv_alloc** out);
/* Number of free blocks ([CB] get_num_free_blocks). */
int kv_alloc_num_free(const kv_alloc* a, int* n);
/* *yes = 1 iff ceil(num_tokens / block_size) blocks are free ([CB] can_allocate). */
int kv_alloc_can_allocate(const kv_alloc* a, int num_tokens, int* yes);
/* New sequence holding ceil(num_tokens / block_size) fresh blocks ([CB]
 * allocate).  KV_ERR_STATE if seq_id exists, KV_ERR_OOM if too few blocks
 * (nothing changes). */
int kv_alloc_allocate(kv_alloc* a, int64_t seq_id, int num_tokens);
/* Reserve the slot of the sequence's next token: a new block when its token
 * count is a multiple of block_size; otherwise, if its last block is shared
 * (refcount > 1), a copy-on-write: a fresh block replaces it in this table
 * and (*cow_src, *cow_dst) name the copy the caller must run with block_copy
 * before writing.  cow_* are -1 when no copy is needed.  KV_ERR_OOM if a
 * block is needed and none is free (nothing changes). */
int kv_alloc_append_slot(kv_alloc* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                         int32_t* cow_dst);
/* child shares every block of parent (refcount + 1 each) and its length. */
int kv_alloc_fork(kv_alloc* a, int64_t parent, int64_t child);
/* Drop the sequence ([CB] free(block_table)): each of its blocks loses one
 * reference and returns to the free list at zero. */
int kv_alloc_free(kv_alloc* a, int64_t seq_id);
/* Copy the block table (at most cap entries) into out; *n = its length. */
int kv_alloc_block_table(const kv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n);
int kv_alloc_num_tokens(const kv_alloc* a, int64_t seq_id, int* n);
int kv_alloc_refcount(const kv_alloc* a, int32_t block, int* rc);
/* Free list in order (n_free entries) and all num_blocks refcounts; either
 * array may be NULL. */
int kv_alloc_snapshot(const kv_alloc* a, int32_t* free_list, int* n_free, int32_t* refcounts);
/* Lifetime counters: blocks taken, blocks returned, copy-on-write copies. */
int kv_alloc_counters(const kv_alloc* a, int64_t* allocated, int64_t* freed, int64_t* cow);
int kv_alloc_destroy(kv_alloc* a);

/* Prefix caching: requests that share a prompt prefix (a system prompt, a
 * document) reuse its KV blocks instead of recomputing them ("vLLM 推理加速
 * 原理详解", automatic prefix caching among the deployment settings and the
 * RAG throughput claim; the pages do not describe the lookup).  Reading
 * taken: only full blocks are cached; block i of a sequence is keyed by
 * FNV-1a-64 over (key of block i-1 as 8 little-endian bytes, then the block's
 * token ids as 4 little-endian bytes each), block -1's key being the FNV
 * offset basis 14695981039346656037; a hit also compares the stored parent
 * key and token ids, so a hash collision never shares a block.  Freed blocks
 * keep their key until the free list hands them out again (FIFO; a freed
 * sequence's blocks are appended deepest first), which evicts the key.
 * Host only, all O(block_size) per block.
 *
 * kv_alloc_enable_prefix_caching: switch caching on; only before any
 * sequence exists (else KV_ERR_STATE). */
int kv_alloc_enable_prefix_caching(kv_alloc* a);

/* Allocate a prompt of num_tokens token ids for seq_id: the longest run of
 * registered blocks matching the prompt from its first block is shared
 * (refcount + 1; a hit on a free block leaves the free list), at most
 * (num_tokens - 1) / block_size blocks so that the last prompt token is
 * always computed; the remaining blocks are taken fresh.  Writes the number
 * of cached tokens (hit blocks x block_size): the caller writes and attends
 * only tokens from there on.  The prompt's tokens are remembered for
 * kv_alloc_commit.  Without caching enabled nothing is shared.  Errors:
 * KV_ERR_ARG, KV_ERR_STATE (sequence exists), KV_ERR_OOM (nothing changes). */
int kv_alloc_allocate_prompt(kv_alloc* a, int64_t seq_id, const int32_t* tokens, int num_tokens,
                             int* num_cached_tokens);

/* kv_alloc_append_slot for a token whose id is known; the id is remembered
 * while the sequence's known tokens are contiguous from position 0. */
int kv_alloc_append_token(kv_alloc* a, int64_t seq_id, int32_t token, int64_t* slot,
                          int32_t* cow_src, int32_t* cow_dst);

/* Register (make findable) every full block of seq_id whose tokens are all
 * known and not registered yet; call once their KV has been written (or is
 * ordered before every later reader on the stream).  A block whose key is
 * already registered to another block stays unregistered.  num_registered
 * may be NULL. */
int kv_alloc_commit(kv_alloc* a, int64_t seq_id, int* num_registered);

/* Host swap space of num_slots block slots (FIFO free list), for the
 * scheduler's swap preemption.  KV_ERR_STATE while a sequence is swapped out. */
int kv_alloc_set_swap_space(kv_alloc* a, int num_slots);

/* Sliding window: release every block of seq_id wholly before position
 * min(token, n), n the sequence's token count (blocks 0 .. min(token, n) /
 * block_size - 1 not yet released), so the block that receives the next
 * token is never released; their table entries become -1 so logical block
 * indices stay put.  Shared blocks only lose this sequence's reference.
 * num_released may be NULL. */
int kv_alloc_release_before(kv_alloc* a, int64_t seq_id, int64_t token, int* num_released);

/* Cumulative hit blocks and evictions, and the number of registered blocks
 * (each pointer may be NULL). */
int kv_alloc_prefix_stats(const kv_alloc* a, int64_t* hit_blocks, int64_t* evictions,
                          int* cached_blocks);

/* --------------------------------------------------------- scheduling step */

/* Continuous-batching scheduler over an allocator ([CB]).  max_num_seqs caps
 * the running set; min_blocks is MIN_BLOCKS of the loop, or < 0 for "the
 * number of running sequences" (one block per running sequence kept in
 * reserve for its appended token; a request is admitted only if its prompt
 * blocks fit with that reserve, counting itself, still free).  The allocator
 * must outlive the scheduler. */
int kv_sched_create(kv_alloc* a, int max_num_seqs, int min_blocks, kv_sched** out);
/* Queue a request (FIFO) whose prompt has prompt_len tokens. */
int kv_sched_add_request(kv_sched* s, int64_t seq_id, int prompt_len);

/* A waiting request with its prompt token ids.  When the allocator has
 * prefix caching enabled, admission counts only the blocks the request takes
 * out of the free list (fresh ones plus free cached hits), allocates it with
 * kv_alloc_allocate_prompt, registers its full prompt blocks at once (the
 * step's cache write is ordered before any attention of the step), and the
 * step's slot_mapping holds only its uncached prompt tokens;
 * kv_sched_admitted_cached gives the cached token counts. */
int kv_sched_add_request_tokens(kv_sched* s, int64_t seq_id, const int32_t* tokens,
                                int num_tokens);
/* Put a sequence that already holds blocks (e.g. a fork) in the running set. */
int kv_sched_adopt(kv_sched* s, int64_t seq_id);

typedef struct {
  int batch;        /* running sequences after the step */
  int num_tokens;   /* slots to write: admitted prompts' tokens, then one per running seq */
  int num_cow;      /* copy-on-write pairs to run before the write */
  int num_admitted; /* requests moved from waiting to running */
  int max_blocks;   /* longest block table among the running sequences */
} kv_step_info;

/* One iteration in the page's order ([CB]): (1) the finished sequences
 * (each must be running) leave the running set and are freed; (2) read the
 * free count; (3) while requests wait, free > MIN_BLOCKS and fewer than
 * max_num_seqs run, the head request is admitted if its prompt fits (else it
 * stays at the head and admission stops); (4) one slot is appended for every
 * running sequence.  Outputs are kept until the next step; read them with
 * kv_sched_outputs.  KV_ERR_STATE (bad finished id) changes nothing;
 * KV_ERR_OOM means the appends of (4), run in batch order (with a window,
 * each followed by its sequence's release, whose blocks later appends may
 * take), would run out of blocks: (1)-(3) are applied, no slot is
 * appended. */
int kv_sched_step(kv_sched* s, const int64_t* finished_ids, int n_finished, kv_step_info* info);
/* Copy the last step's outputs to host arrays sized from kv_step_info (any
 * may be NULL): running_ids[batch]; block_tables[batch][table_width]
 * (table_width >= max_blocks, padded with -1); context_lens[batch] (tokens
 * after the append); slot_mapping[num_tokens]; cow_pairs[num_cow][2];
 * admitted_ids[num_admitted]. */
int kv_sched_outputs(const kv_sched* s, int64_t* running_ids, int32_t* block_tables,
                     int table_width, int32_t* context_lens, int64_t* slot_mapping,
                     int32_t* cow_pairs, int64_t* admitted_ids);
/* [MON]: running and waiting request counts, used and total blocks
 * (cache usage = used / total). */
/* Sliding window for the scheduling step: with window > 0, after its
 * append in step (4) every running sequence not admitted in this step
 * releases the blocks wholly before its last `window` positions
 * (kv_alloc_release_before), which a sliding-window decode never reads;
 * block tables then hold -1 for released entries.  0 (the default) keeps
 * every block.  KV_ERR_ARG for a negative window. */
int kv_sched_set_window(kv_sched* s, int window);

/* Preemption when the KV cache runs out ("vLLM 推理加速原理详解" names
 * preemption and swapping as what an undersized cache leads to; the
 * mechanism is this library's reading).  With a mode other than
 * KV_PREEMPT_NONE, each step first checks that the running set's appends fit
 * the free blocks; while they do not, the most recently scheduled running
 * sequence is preempted:
 *   KV_PREEMPT_SWAP: every block it holds alone moves to a host swap slot
 *     (kv_alloc_set_swap_space) and its device block is freed; blocks it
 *     shares stay, with its reference; it waits at the front of a swapped
 *     queue.  If the swap space lacks room it is recomputed instead.
 *   KV_PREEMPT_RECOMPUTE: its blocks are freed and it goes back to the front
 *     of the waiting queue with its whole context as the prompt.
 * In a step without preemption, swapped sequences come back first (first in,
 * first out) while their host-held blocks fit with the admission reserve;
 * new requests are admitted only when none is swapped out and nothing was
 * preempted in the step.  The caller runs
 * kv_swap_out for the step's swap-out pairs, then kv_swap_in for its swap-in
 * pairs, before the step's other kernels.  KV_PREEMPT_NONE (default): the
 * step fails with KV_ERR_OOM when the appends do not fit. */
int kv_sched_set_preemption(kv_sched* s, int mode);

/* Sizes of the last step's swap outputs, and the number of sequences now
 * swapped out (any pointer may be NULL). */
int kv_sched_swap_info(const kv_sched* s, int* num_swap_out, int* num_swap_in, int* num_preempted,
                       int* num_recomputed, int* num_swapped_in, int* num_swapped);

/* The last step's swap outputs (any pointer may be NULL):
 * swap_out_pairs[num_swap_out][2] (device block, host slot),
 * swap_in_pairs[num_swap_in][2] (host slot, device block), the ids swapped
 * out, recomputed (requeued) and swapped back in. */
int kv_sched_swap_outputs(const kv_sched* s, int32_t* swap_out_pairs, int32_t* swap_in_pairs,
                          int64_t* preempted_ids, int64_t* recomputed_ids, int64_t* swapped_in_ids);

/* Cached prompt tokens of each request admitted by the last step, in the
 * order of admitted_ids (0 without prefix caching). */
int kv_sched_admitted_cached(const kv_sched* s, int32_t* cached_tokens);

int kv_sched_stats(const kv_sched* s, int* running, int* waiting, int* used_blocks,
                   int* total_blocks);
int kv_sched_destroy(kv_sched* s);

/* ---------------------------------------------------------- serving step */

/* One continuous-batching iteration sequenced by the library ([CB]: free the
 * finished, admit first come first served, append one slot per running
 * sequence, then the step's kernels), so a serving loop makes two calls per
 * step (four with host staging) instead of one per array and kernel. */

/* Order in which the decode places the batch's sequences on the GPU (the
 * seq_order argument of paged_attention_decode; outputs do not depend on it).
 * BATCH: batch order (no permutation).  LONGEST: decreasing context length,
 * ties in batch order.  LONG_FIRST: the sequences longer than the batch mean,
 * longest first, then the rest in batch order. */
typedef enum { KV_ORDER_BATCH = 0, KV_ORDER_LONGEST = 1, KV_ORDER_LONG_FIRST = 2 } kv_order_policy;

/* Where a packed step's arrays sit in its buffer: byte offsets, each a
 * multiple of 16, or -1 for an array the step does not have. */
typedef struct {
  kv_step_info info;
  int table_width;      /* row stride of block_tables: max(info.max_blocks, 1) */
  int max_context_len;  /* longest context after the append (0: empty batch) */
  int num_swap_out;     /* swap-out pairs (kv_sched_swap_outputs) */
  int num_swap_in;      /* swap-in pairs */
  int prefill_tokens;   /* admitted prompts' uncached tokens, cu_seqlens[num_admitted] */
  int max_prefill_len;  /* most uncached tokens of one admitted prompt */
  int buffer;           /* kv_serve_schedule: the step's buffer set, 0 .. num_sets - 1 in turn; else 0 */
  int64_t bytes;        /* bytes of the buffer the step uses */
  int64_t slot_mapping;          /* int64[num_tokens] */
  int64_t block_tables;          /* int32[batch][table_width], padded with -1 */
  int64_t context_lens;          /* int32[batch] */
  int64_t seq_order;             /* int32[batch]; -1 under KV_ORDER_BATCH */
  int64_t cow_pairs;             /* int32[num_cow][2] */
  int64_t swap_out_pairs;        /* int32[num_swap_out][2] */
  int64_t swap_in_pairs;         /* int32[num_swap_in][2] */
  int64_t cu_seqlens;            /* int32[num_admitted + 1]: prefix sums of uncached prompt tokens */
  int64_t prefill_context_lens;  /* int32[num_admitted]: prompt lengths (context minus the appended token) */
} kv_step_layout;

/* Bytes a packed step can need with at most max_batch running sequences,
 * max_tokens written slots, tables of at most max_table_width blocks and
 * max_swap_pairs swap pairs each way (0 on a negative argument). */
size_t kv_step_packed_bytes(int max_batch, int max_tokens, int max_table_width, int max_swap_pairs);

/* kv_sched_step, then the step's device metadata written into buf (host
 * memory, 16-byte aligned, buf_bytes long) at the offsets returned in
 * *layout: the same arrays kv_sched_outputs / kv_sched_swap_outputs give,
 * the block tables at the step's own width, the scheduling order of
 * order_policy, and for the admitted prompts (the last num_admitted rows of
 * the running set) the cu_seqlens / context lengths paged_attention_prefill
 * takes.  running_ids (may be NULL) receives int64[batch].  Errors of
 * kv_sched_step are returned as they are (nothing changes for KV_ERR_STATE);
 * KV_ERR_ARG for a step whose tables are wider than max_table_width or whose
 * arrays do not fit buf: the scheduler step has then been taken and its
 * outputs stay readable with kv_sched_outputs. */
int kv_sched_step_packed(kv_sched* s, const int64_t* finished_ids, int n_finished, int order_policy,
                         int max_table_width, void* buf, size_t buf_bytes, int64_t* running_ids,
                         kv_step_layout* layout);

/* Decode scratch a serving loop needs for every batch of 1..max_batch
 * sequences with contexts up to max_context_len (the split policy divides
 * more finely when fewer sequences run). */
size_t kv_serve_workspace_bytes(const kv_pool* pool, int num_q_heads, int max_batch, int max_context_len);

/* Most buffer sets a serving loop cycles through. */
#define KV_SERVE_MAX_SETS 4

/* A serving loop over pool and sched (both must outlive it).  The caller owns
 * every buffer: num_sets (2 .. KV_SERVE_MAX_SETS) pinned host and as many
 * device metadata buffers of meta_bytes each (>= kv_step_packed_bytes(
 * max_batch, max_tokens, max_table_width, swap_slots), 16-byte aligned), the
 * decode workspace (>= kv_serve_workspace_bytes), and for swap preemption the
 * mapped pinned host swap space of swap_slots slots (kv_swap_out).
 * Consecutive steps use the sets in turn, and a step's uploads wait only for
 * the kernels of the step num_sets before it: with 2 sets, two steps cost at
 * least one upload plus one step's kernels; with 3 or more, uploads and
 * kernels of neighbouring steps overlap fully.  The loop creates three CUDA
 * events per set on the current device, which must stay current for its
 * calls.
 * num_q_heads, q_dtype (also the type of the new K/V rows) and scale are
 * those of the decode.  A loop holds per-step state: one host thread at a
 * time drives it (and its scheduler).  KV_ERR_ARG on bad arguments;
 * KV_ERR_CUDA if an event cannot be created. */
int kv_serve_create(kv_pool* pool, kv_sched* sched, int num_q_heads, kv_dtype q_dtype, float scale,
                    int order_policy, int max_batch, int max_tokens, int max_table_width, void* host_swap,
                    int swap_slots, int num_sets, void* const* host_meta, void* const* dev_meta,
                    size_t meta_bytes, void* workspace, size_t workspace_bytes, kv_serve** out);

/* The step's host half: waits (host) until the next set's pinned buffer's
 * last upload is done, runs kv_sched_step_packed into it, and enqueues on
 * upload_stream, after the kernels that last read the set's device buffer,
 * one copy of the packed bytes to that device buffer.  running_ids
 * (int64[max_batch], written only for a batch that fits) and layout may be
 * NULL.  KV_ERR_STATE if the previous step was never launched
 * (checked first: nothing changes); otherwise as kv_sched_step_packed, plus
 * KV_ERR_ARG when the step exceeds max_batch / max_tokens and KV_ERR_STATE
 * when it swaps without swap space (the scheduler step is then taken). */
int kv_serve_schedule(kv_serve* s, const int64_t* finished_ids, int n_finished, kv_stream_t upload_stream,
                      int64_t* running_ids, kv_step_layout* layout);

/* The step's kernels for one layer, on stream, after the step's metadata
 * upload: on the first call of a step kv_swap_out, kv_swap_in and block_copy
 * for all layers; then paged_kv_write of the step's num_tokens new rows
 * (k_new / v_new [num_tokens][kv_heads][head_dim] of q_dtype, FP8 pools'
 * inverse scales as in paged_kv_write), paged_attention_prefill of the
 * admitted prompts' uncached tokens when prefill_q / prefill_out are given
 * ([prefill_tokens][num_q_heads][head_dim], rows prompt by prompt), and
 * paged_attention_decode of the running set (q, out [batch][num_q_heads]
 * [head_dim]) in the loop's scheduling order.  Call once per layer after
 * each kv_serve_schedule.  KV_ERR_STATE with no step scheduled; KV_ERR_ARG
 * for a missing q / out (batch > 0) or k_new / v_new (tokens > 0), one of
 * prefill_q / prefill_out without the other, or a workspace smaller than the
 * step's decode needs (checked before anything is enqueued); otherwise the
 * first error of the entry points above (later ones are not enqueued). */
int kv_serve_launch(kv_serve* s, int layer, const void* q, const void* k_new, const void* v_new,
                    const float* k_inv_scale, const float* v_inv_scale, void* out, kv_dtype out_dtype,
                    const void* prefill_q, void* prefill_out, kv_stream_t stream);

/* Host input and output staging for a loop whose inputs come from host
 * memory.  The caller keeps num_sets sets of device input and output
 * buffers and uses set layout.buffer for a step.  kv_serve_upload (after
 * kv_serve_schedule, before the step's first launch) copies bytes from
 * pinned host memory to dev_dst on the step's upload stream, after the
 * kernels that last read that set (the step num_sets before); the step's
 * launches wait for it.  kv_serve_readback (after a launch) copies bytes from
 * dev_src to pinned host memory on readback_stream once the step's kernels
 * so far are done; the first launch of the next step that reuses the set
 * waits for it.  KV_ERR_STATE when called out of that
 * order, KV_ERR_ARG on NULL pointers with bytes > 0. */
int kv_serve_upload(kv_serve* s, void* dev_dst, const void* host_src, size_t bytes);
int kv_serve_readback(kv_serve* s, void* host_dst, const void* dev_src, size_t bytes, kv_stream_t readback_stream);

/* Waits for the loop's uploads, kernels and read-backs (host), then frees it. */
int kv_serve_destroy(kv_serve* s);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
