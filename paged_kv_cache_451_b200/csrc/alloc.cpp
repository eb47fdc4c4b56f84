// Refcounted free-list block allocator and continuous-batching step.
//
// Block rules: "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍",
// section "PagedAttention：把操作系统的虚拟内存搬进 GPU" — fixed-size physical
// blocks taken on demand, a per-sequence block table, any free block serves
// any request, several logical blocks may share one physical block.
// Scheduling loop: same page, section "连续批处理：别再等最慢的那个请求了" —
// free finished requests, read the free count, admit waiting requests first
// come first served while free_blocks > MIN_BLOCKS and can_allocate, then
// decode the running set.
//
// Policies the page leaves open, fixed here so runs are reproducible:
// FIFO free list (take from the head, return to the tail in table order);
// copy-on-write when appending into a block whose refcount is above one;
// head-of-line admission (a request that does not fit stays first and
// admission stops); MIN_BLOCKS defaults to the running count and a request
// is admitted only if its prompt blocks fit with that reserve (counting the
// request) left free, so the appends of the step cannot run out.

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <string>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "host_common.h"

namespace pagedkv {

namespace {
thread_local std::string g_msg;
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_msg = buf;
  return code;
}

int ok() {
  g_msg.clear();
  return KV_OK;
}

const char* last_error() { return g_msg.c_str(); }

}  // namespace pagedkv

using pagedkv::fail;
using pagedkv::ok;

struct SeqState {
  std::vector<int32_t> blocks;
  int64_t tokens = 0;
  std::vector<int32_t> toks;  // known token ids (prefix caching)
  int64_t registered = 0;     // leading blocks registered or skipped
};

// Prefix-caching key of one full block: FNV-1a (64-bit) over the parent
// key's 8 little-endian bytes, then the block's token ids as 4 little-endian
// bytes each (the FNV-1a definition: per byte, h ^= byte; h *= 1099511628211
// mod 2^64; from 14695981039346656037).
constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

inline uint64_t fnv_bytes(uint64_t h, uint64_t v, int nbytes) {
  for (int i = 0; i < nbytes; ++i) {
    h ^= (v >> (8 * i)) & 0xffu;
    h *= kFnvPrime;
  }
  return h;
}

inline uint64_t block_key(uint64_t parent, const int32_t* tokens, int n) {
  uint64_t h = fnv_bytes(kFnvOffset, parent, 8);
  for (int i = 0; i < n; ++i) h = fnv_bytes(h, (uint32_t)tokens[i], 4);
  return h;
}

struct CachedBlock {
  bool valid = false;
  uint64_t key = 0, parent = 0;
  std::vector<int32_t> tokens;
};

struct kv_alloc {
  int num_blocks = 0;
  int block_size = 0;
  // FIFO free list as an intrusive doubly linked list (O(1) removal of a
  // cached block that a prompt hits)
  std::vector<int32_t> prev, next;
  std::vector<char> is_free;
  int32_t head = -1, tail = -1;
  int64_t n_free = 0;
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, SeqState> seqs;
  int64_t n_alloc = 0, n_freed = 0, n_cow = 0;
  // prefix caching
  bool caching = false;
  std::unordered_map<uint64_t, int32_t> cached;
  std::vector<CachedBlock> key_of;
  int64_t n_hits = 0, n_evict = 0;
  // host swap space: FIFO free list of slots; a table entry -(2 + slot)
  // marks a block held in a host slot
  std::deque<int32_t> host_free;

  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }

  void push_back(int32_t b) {
    prev[b] = tail;
    next[b] = -1;
    if (tail >= 0) next[tail] = b; else head = b;
    tail = b;
    is_free[b] = 1;
    ++n_free;
  }

  void unlink(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
    prev[b] = next[b] = -1;
    is_free[b] = 0;
    --n_free;
  }

  void evict(int32_t b) {
    CachedBlock& c = key_of[b];
    if (!c.valid) return;
    auto it = cached.find(c.key);
    if (it != cached.end() && it->second == b) cached.erase(it);
    c.valid = false;
    c.tokens.clear();
    ++n_evict;
  }

  int32_t take() {
    int32_t b = head;
    unlink(b);
    if (caching) evict(b);
    refcount[b] = 1;
    ++n_alloc;
    return b;
  }

  void release(int32_t b) {
    if (--refcount[b] == 0) {
      push_back(b);
      ++n_freed;
    }
  }

  // Blocks one append to `s` needs: 1 for a new block or a copy, else 0.
  bool append_needs_block(const SeqState& s) const {
    if (s.tokens % block_size == 0) return true;
    return refcount[s.blocks.back()] > 1;
  }

  int append(SeqState& s, int64_t* slot, int32_t* cs, int32_t* cd) {
    int64_t pos = s.tokens;
    *cs = -1;
    *cd = -1;
    if (pos % block_size == 0) {
      if (n_free == 0) return KV_ERR_OOM;
      s.blocks.push_back(take());
    } else {
      int32_t last = s.blocks.back();
      if (refcount[last] > 1) {
        if (n_free == 0) return KV_ERR_OOM;
        int32_t fresh = take();
        --refcount[last];
        s.blocks.back() = fresh;
        *cs = last;
        *cd = fresh;
        ++n_cow;
      }
    }
    s.tokens = pos + 1;
    *slot = (int64_t)s.blocks[pos / block_size] * block_size + pos % block_size;
    return KV_OK;
  }

  int64_t swap_out_cost(const SeqState& st) const {
    int64_t c = 0;
    for (int32_t b : st.blocks) c += (b >= 0 && refcount[b] == 1) ? 1 : 0;
    return c;
  }

  int64_t swap_in_cost(const SeqState& st) const {
    int64_t c = 0;
    for (int32_t b : st.blocks) c += b <= -2 ? 1 : 0;
    return c;
  }

  // Move every block the sequence holds alone to a host slot; shared blocks
  // stay on the device with the reference kept.  Pairs (device, slot).
  void swap_out(SeqState& st, std::vector<int32_t>* pairs) {
    for (auto& b : st.blocks) {
      if (b >= 0 && refcount[b] == 1) {
        const int32_t slot = host_free.front();
        host_free.pop_front();
        pairs->push_back(b);
        pairs->push_back(slot);
        refcount[b] = 0;
        push_back(b);
        ++n_freed;
        b = -(2 + slot);
      }
    }
  }

  // Fresh device blocks for the host-held entries.  Pairs (slot, device).
  void swap_in(SeqState& st, std::vector<int32_t>* pairs) {
    for (auto& b : st.blocks) {
      if (b <= -2) {
        const int32_t slot = -b - 2;
        const int32_t nb = take();
        pairs->push_back(slot);
        pairs->push_back(nb);
        host_free.push_back(slot);
        b = nb;
      }
    }
  }

  // Whether the appends of `ids`, run in that order and each followed (for
  // a sequence not in `admitted`, with window > 0) by the release of the
  // blocks wholly before its last `window` positions, always find a free
  // block when they need one: a block boundary or a copy of a shared partly
  // filled last block takes one, a release whose block loses its last
  // reference returns one.  Changes nothing.
  bool appends_fit(const std::vector<int64_t>& ids, const std::unordered_set<int64_t>& admitted, int window) {
    int64_t f = n_free;
    std::unordered_map<int32_t, int32_t> rc;  // refcounts of shared blocks as the simulation changes them
    auto ref = [&](int32_t b) -> int32_t& {
      auto it = rc.find(b);
      if (it == rc.end()) it = rc.emplace(b, refcount[b]).first;
      return it->second;
    };
    for (int64_t r : ids) {
      const SeqState& st = seqs[r];
      const int64_t pos = st.tokens;
      if (pos % block_size == 0) {
        if (f == 0) return false;
        --f;
      } else {
        const int32_t last = st.blocks.back();
        if (refcount[last] > 1 || rc.count(last)) {  // refcounts only fall: an exclusive block stays so
          int32_t& c = ref(last);
          if (c > 1) {
            if (f == 0) return false;
            --f;
            --c;
          }
        }
      }
      if (window > 0 && !admitted.count(r)) {
        // the append's own block (index pos / block_size) is never released here
        const int64_t token = pos + 1 - window;
        const int64_t upto = std::min<int64_t>(token < 0 ? 0 : token / block_size, (int64_t)st.blocks.size());
        for (int64_t i = 0; i < upto; ++i) {
          const int32_t b = st.blocks[i];
          if (b < 0) continue;
          if (refcount[b] == 1 && !rc.count(b)) {
            ++f;
            rc.emplace(b, 0);
          } else if (--ref(b) == 0) {
            ++f;
          }
        }
      }
    }
    return true;
  }

  // Fresh blocks the appends of `seqs` take: one per sequence at a block
  // boundary, plus the copies of shared partly filled last blocks (at most
  // refcount - 1 per block).
  int64_t append_need(const std::vector<int64_t>& ids) {
    int64_t need = 0;
    std::unordered_map<int32_t, int64_t> shared;
    for (int64_t r : ids) {
      const SeqState& st = seqs[r];
      if (st.tokens % block_size == 0) {
        ++need;
      } else if (refcount[st.blocks.back()] > 1) {
        ++shared[st.blocks.back()];
      }
    }
    for (auto& kv : shared) {
      const int64_t copies = refcount[kv.first] - 1;
      need += kv.second < copies ? kv.second : copies;
    }
    return need;
  }

  // Blocks of the longest registered prefix of `tokens`, at most
  // (n - 1) / block_size of them (the last prompt token is always computed).
  void lookup(const int32_t* tokens, int n, std::vector<int32_t>* hits) const {
    hits->clear();
    if (!caching || n <= 0) return;
    const int cap = (n - 1) / block_size;
    uint64_t parent = kFnvOffset;
    for (int i = 0; i < cap; ++i) {
      const int32_t* t = tokens + (int64_t)i * block_size;
      const uint64_t k = block_key(parent, t, block_size);
      auto it = cached.find(k);
      if (it == cached.end()) break;
      const CachedBlock& c = key_of[it->second];
      if (!c.valid || c.key != k || c.parent != parent ||
          std::memcmp(c.tokens.data(), t, sizeof(int32_t) * block_size) != 0)
        break;
      hits->push_back(it->second);
      parent = k;
    }
  }

  // Free blocks an allocation of `tokens` removes from the free list.
  int64_t admission_cost(const int32_t* tokens, int n, std::vector<int32_t>* hits) const {
    lookup(tokens, n, hits);
    int64_t cost = blocks_for(n) - (int64_t)hits->size();
    for (int32_t b : *hits) cost += refcount[b] == 0 ? 1 : 0;
    return cost;
  }

  // Register every full block of `s` whose tokens are all known.
  int commit(SeqState& s) {
    if (!caching) return 0;
    const int64_t known = std::min<int64_t>((int64_t)s.toks.size(), s.tokens);
    const int64_t full = known / block_size;
    uint64_t parent = kFnvOffset;
    int added = 0;
    for (int64_t i = 0; i < full; ++i) {
      const int32_t* t = s.toks.data() + i * block_size;
      const uint64_t k = block_key(parent, t, block_size);
      if (i >= s.registered) {
        const int32_t b = s.blocks[i];
        if (b >= 0 && !cached.count(k) && !key_of[b].valid) {
          CachedBlock& c = key_of[b];
          c.valid = true;
          c.key = k;
          c.parent = parent;
          c.tokens.assign(t, t + block_size);
          cached.emplace(k, b);
          ++added;
        }
      }
      parent = k;
    }
    if (full > s.registered) s.registered = full;
    return added;
  }
};

extern "C" {

const char* kv_last_error(void) { return pagedkv::last_error(); }
int kv_version(void) { return 1; }

int kv_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                    kv_alloc** out) {
  if (!out) return fail(KV_ERR_ARG, "out is NULL");
  if (num_blocks <= 0 || block_size <= 0)
    return fail(KV_ERR_ARG, "num_blocks (%d) and block_size (%d) must be positive", num_blocks,
                block_size);
  kv_alloc* a = new (std::nothrow) kv_alloc();
  if (!a) return fail(KV_ERR_OOM, "host allocation failed");
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refcount.assign(num_blocks, 0);
  a->prev.assign(num_blocks, -1);
  a->next.assign(num_blocks, -1);
  a->is_free.assign(num_blocks, 0);
  a->key_of.resize(num_blocks);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return fail(KV_ERR_ARG, "initial_free_order is not a permutation of 0..%d", num_blocks - 1);
      }
      seen[b] = 1;
      a->push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) a->push_back(i);
  }
  *out = a;
  return ok();
}

int kv_alloc_destroy(kv_alloc* a) {
  delete a;
  return ok();
}

int kv_alloc_num_free(const kv_alloc* a, int* n) {
  if (!a || !n) return fail(KV_ERR_ARG, "NULL argument");
  *n = (int)a->n_free;
  return ok();
}

int kv_alloc_can_allocate(const kv_alloc* a, int num_tokens, int* yes) {
  if (!a || !yes || num_tokens < 0) return fail(KV_ERR_ARG, "bad argument");
  *yes = a->blocks_for(num_tokens) <= a->n_free;
  return ok();
}

int kv_alloc_allocate(kv_alloc* a, int64_t seq_id, int num_tokens) {
  if (!a || num_tokens < 0) return fail(KV_ERR_ARG, "bad argument");
  if (a->seqs.count(seq_id)) return fail(KV_ERR_STATE, "sequence %lld already exists", (long long)seq_id);
  int64_t need = a->blocks_for(num_tokens);
  if (need > a->n_free)
    return fail(KV_ERR_OOM, "need %lld blocks, %lld free", (long long)need, (long long)a->n_free);
  SeqState s;
  s.blocks.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->take());
  s.tokens = num_tokens;
  a->seqs.emplace(seq_id, std::move(s));
  return ok();
}

int kv_alloc_append_slot(kv_alloc* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                         int32_t* cow_dst) {
  if (!a || !slot || !cow_src || !cow_dst) return fail(KV_ERR_ARG, "NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  int rc = a->append(it->second, slot, cow_src, cow_dst);
  if (rc != KV_OK) return fail(rc, "no free block for sequence %lld", (long long)seq_id);
  return ok();
}

int kv_alloc_fork(kv_alloc* a, int64_t parent, int64_t child) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)parent);
  if (a->seqs.count(child)) return fail(KV_ERR_STATE, "sequence %lld already exists", (long long)child);
  SeqState s = it->second;
  for (int32_t b : s.blocks)
    if (b >= 0) ++a->refcount[b];
  a->seqs.emplace(child, std::move(s));
  return ok();
}

int kv_alloc_free(kv_alloc* a, int64_t seq_id) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  const auto& blocks = it->second.blocks;
  if (a->caching) {  // deepest block first: shared prefixes leave the cache last
    for (auto r = blocks.rbegin(); r != blocks.rend(); ++r) {
      if (*r >= 0) a->release(*r);
      else if (*r <= -2) a->host_free.push_back(-*r - 2);
    }
  } else {
    for (int32_t b : blocks) {
      if (b >= 0) a->release(b);
      else if (b <= -2) a->host_free.push_back(-b - 2);
    }
  }
  a->seqs.erase(it);
  return ok();
}

int kv_alloc_block_table(const kv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !out)) return fail(KV_ERR_ARG, "bad argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  const auto& b = it->second.blocks;
  *n = (int)b.size();
  for (int i = 0; i < cap && i < (int)b.size(); ++i) out[i] = b[i];
  return ok();
}

int kv_alloc_num_tokens(const kv_alloc* a, int64_t seq_id, int* n) {
  if (!a || !n) return fail(KV_ERR_ARG, "NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  *n = (int)it->second.tokens;
  return ok();
}

int kv_alloc_refcount(const kv_alloc* a, int32_t block, int* rc) {
  if (!a || !rc || block < 0 || block >= a->num_blocks) return fail(KV_ERR_ARG, "bad argument");
  *rc = a->refcount[block];
  return ok();
}

int kv_alloc_snapshot(const kv_alloc* a, int32_t* free_list, int* n_free, int32_t* refcounts) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  if (n_free) *n_free = (int)a->n_free;
  if (free_list) {
    int i = 0;
    for (int32_t b = a->head; b >= 0; b = a->next[b]) free_list[i++] = b;
  }
  if (refcounts) std::memcpy(refcounts, a->refcount.data(), sizeof(int32_t) * a->num_blocks);
  return ok();
}

int kv_alloc_enable_prefix_caching(kv_alloc* a) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  if (!a->seqs.empty()) return fail(KV_ERR_STATE, "enable prefix caching before any sequence exists");
  a->caching = true;
  return ok();
}

int kv_alloc_set_swap_space(kv_alloc* a, int num_slots) {
  if (!a || num_slots < 0) return fail(KV_ERR_ARG, "bad argument");
  for (const auto& kv : a->seqs)
    for (int32_t b : kv.second.blocks)
      if (b <= -2) return fail(KV_ERR_STATE, "a sequence is swapped out");
  a->host_free.clear();
  for (int i = 0; i < num_slots; ++i) a->host_free.push_back(i);
  return ok();
}

int kv_alloc_allocate_prompt(kv_alloc* a, int64_t seq_id, const int32_t* tokens, int num_tokens,
                             int* num_cached_tokens) {
  if (!a || num_tokens < 0 || (num_tokens > 0 && !tokens) || !num_cached_tokens)
    return fail(KV_ERR_ARG, "bad argument");
  if (a->seqs.count(seq_id)) return fail(KV_ERR_STATE, "sequence %lld already exists", (long long)seq_id);
  std::vector<int32_t> hits;
  const int64_t cost = a->admission_cost(tokens, num_tokens, &hits);
  if (cost > a->n_free)
    return fail(KV_ERR_OOM, "need %lld blocks, %lld free", (long long)cost, (long long)a->n_free);
  SeqState s;
  s.blocks.reserve(a->blocks_for(num_tokens));
  for (int32_t b : hits) {
    if (a->refcount[b] == 0) a->unlink(b);
    ++a->refcount[b];
    s.blocks.push_back(b);
  }
  a->n_hits += (int64_t)hits.size();
  const int64_t fresh = a->blocks_for(num_tokens) - (int64_t)hits.size();
  for (int64_t i = 0; i < fresh; ++i) s.blocks.push_back(a->take());
  s.tokens = num_tokens;
  s.toks.assign(tokens, tokens + num_tokens);
  s.registered = (int64_t)hits.size();
  a->seqs.emplace(seq_id, std::move(s));
  *num_cached_tokens = (int)hits.size() * a->block_size;
  return ok();
}

int kv_alloc_append_token(kv_alloc* a, int64_t seq_id, int32_t token, int64_t* slot,
                          int32_t* cow_src, int32_t* cow_dst) {
  if (!a || !slot || !cow_src || !cow_dst) return fail(KV_ERR_ARG, "NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  SeqState& st = it->second;
  const bool contiguous = (int64_t)st.toks.size() == st.tokens;
  int rc = a->append(st, slot, cow_src, cow_dst);
  if (rc != KV_OK) return fail(rc, "no free block for sequence %lld", (long long)seq_id);
  if (contiguous) st.toks.push_back(token);
  return ok();
}

int kv_alloc_commit(kv_alloc* a, int64_t seq_id, int* num_registered) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  const int n = a->commit(it->second);
  if (num_registered) *num_registered = n;
  return ok();
}

int kv_alloc_prefix_stats(const kv_alloc* a, int64_t* hit_blocks, int64_t* evictions,
                          int* cached_blocks) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  if (hit_blocks) *hit_blocks = a->n_hits;
  if (evictions) *evictions = a->n_evict;
  if (cached_blocks) *cached_blocks = (int)a->cached.size();
  return ok();
}

int kv_alloc_release_before(kv_alloc* a, int64_t seq_id, int64_t token, int* num_released) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  SeqState& st = it->second;
  // only positions the sequence holds: the block that receives its next
  // token is never released
  const int64_t held = std::min<int64_t>(token < 0 ? 0 : token, st.tokens);
  const int64_t upto = std::min<int64_t>(held / a->block_size, (int64_t)st.blocks.size());
  int released = 0;
  for (int64_t i = 0; i < upto; ++i) {
    if (st.blocks[i] < 0) continue;
    a->release(st.blocks[i]);
    st.blocks[i] = -1;
    ++released;
  }
  if (num_released) *num_released = released;
  return ok();
}

int kv_alloc_counters(const kv_alloc* a, int64_t* allocated, int64_t* freed, int64_t* cow) {
  if (!a) return fail(KV_ERR_ARG, "NULL allocator");
  if (allocated) *allocated = a->n_alloc;
  if (freed) *freed = a->n_freed;
  if (cow) *cow = a->n_cow;
  return ok();
}

}  // extern "C"

// ------------------------------------------------------------ scheduler

struct Request {
  int64_t id;
  int prompt_len;
  bool has_tokens;
  std::vector<int32_t> tokens;
};

struct kv_sched {
  kv_alloc* a = nullptr;
  int max_num_seqs = 0;
  int min_blocks = -1;
  int window = 0;  // > 0: release blocks that left the window after each step
  int preemption = KV_PREEMPT_NONE;
  std::deque<int64_t> swapped;
  std::vector<int32_t> out_swap_out, out_swap_in;  // flattened pairs
  std::vector<int64_t> out_preempted, out_recomputed, out_swapped_in;
  std::deque<Request> waiting;
  std::vector<int64_t> running;
  // outputs of the last step
  std::vector<int64_t> out_running;
  std::vector<int32_t> out_table_flat;  // the running sequences' tables, back to back
  std::vector<int64_t> out_table_off{0};  // row i is [off[i], off[i + 1]) of out_table_flat
  std::vector<int32_t> out_lens;
  std::vector<int64_t> out_slots;
  std::vector<int32_t> out_cow;
  std::vector<int64_t> out_admitted;
  std::vector<int32_t> out_cached;

  int min_blocks_now() const { return min_blocks < 0 ? (int)running.size() : min_blocks; }
};

extern "C" {

int kv_sched_create(kv_alloc* a, int max_num_seqs, int min_blocks, kv_sched** out) {
  if (!a || !out || max_num_seqs <= 0) return fail(KV_ERR_ARG, "bad argument");
  kv_sched* s = new (std::nothrow) kv_sched();
  if (!s) return fail(KV_ERR_OOM, "host allocation failed");
  s->a = a;
  s->max_num_seqs = max_num_seqs;
  s->min_blocks = min_blocks;
  *out = s;
  return ok();
}

int kv_sched_destroy(kv_sched* s) {
  delete s;
  return ok();
}

int kv_sched_add_request(kv_sched* s, int64_t seq_id, int prompt_len) {
  if (!s || prompt_len < 0) return fail(KV_ERR_ARG, "bad argument");
  s->waiting.push_back({seq_id, prompt_len, false, {}});
  return ok();
}

int kv_sched_add_request_tokens(kv_sched* s, int64_t seq_id, const int32_t* tokens, int num_tokens) {
  if (!s || num_tokens < 0 || (num_tokens > 0 && !tokens)) return fail(KV_ERR_ARG, "bad argument");
  s->waiting.push_back({seq_id, num_tokens, true, std::vector<int32_t>(tokens, tokens + num_tokens)});
  return ok();
}

int kv_sched_set_window(kv_sched* s, int window) {
  if (!s || window < 0) return fail(KV_ERR_ARG, "bad argument");
  s->window = window;
  return ok();
}

int kv_sched_adopt(kv_sched* s, int64_t seq_id) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (!s->a->seqs.count(seq_id)) return fail(KV_ERR_STATE, "sequence %lld is unknown", (long long)seq_id);
  for (int64_t r : s->running)
    if (r == seq_id) return fail(KV_ERR_STATE, "sequence %lld is already running", (long long)seq_id);
  s->running.push_back(seq_id);
  return ok();
}

int kv_sched_step(kv_sched* s, const int64_t* finished_ids, int n_finished, kv_step_info* info) {
  if (!s || !info || n_finished < 0 || (n_finished > 0 && !finished_ids))
    return fail(KV_ERR_ARG, "bad argument");
  kv_alloc* a = s->a;
  // validate before changing anything
  // the finished ids, sorted (a few per step): each must be running, once
  std::vector<int64_t> fin(finished_ids, finished_ids + n_finished);
  std::sort(fin.begin(), fin.end());
  for (size_t i = 1; i < fin.size(); ++i)
    if (fin[i] == fin[i - 1]) return fail(KV_ERR_STATE, "sequence %lld finished twice", (long long)fin[i]);
  auto finished = [&](int64_t r) { return std::binary_search(fin.begin(), fin.end(), r); };
  if (n_finished > 0) {
    size_t found = 0;
    for (int64_t r : s->running) found += finished(r);
    if (found != fin.size()) {
      std::vector<int64_t> run(s->running);
      std::sort(run.begin(), run.end());
      for (int64_t f : fin)
        if (!std::binary_search(run.begin(), run.end(), f))
          return fail(KV_ERR_STATE, "finished sequence %lld is not running", (long long)f);
    }
  }
  s->out_running.clear();
  s->out_table_flat.clear();
  s->out_table_off.assign(1, 0);
  s->out_lens.clear();
  s->out_slots.clear();
  s->out_cow.clear();
  s->out_admitted.clear();
  s->out_cached.clear();
  s->out_swap_out.clear();
  s->out_swap_in.clear();
  s->out_preempted.clear();
  s->out_recomputed.clear();
  s->out_swapped_in.clear();

  // (1) drop finished requests, return their blocks
  std::vector<int64_t> keep;
  keep.reserve(s->running.size());
  for (int64_t r : s->running)
    if (!finished(r)) keep.push_back(r);
  s->running.swap(keep);
  for (int i = 0; i < n_finished; ++i) kv_alloc_free(a, finished_ids[i]);

  // (1b) preemption: while the running set's appends do not fit, the most
  // recently scheduled running sequence leaves: swapped out (its exclusive
  // blocks to host slots; front of the swapped queue) or, without room in the
  // swap space or in recompute mode, freed and put back at the front of the
  // waiting queue with its whole context as the prompt
  if (s->preemption != KV_PREEMPT_NONE) {
    while (!s->running.empty() && a->append_need(s->running) > a->n_free) {
      const int64_t victim = s->running.back();
      s->running.pop_back();
      SeqState& st = a->seqs[victim];
      if (s->preemption == KV_PREEMPT_SWAP && a->swap_out_cost(st) <= (int64_t)a->host_free.size()) {
        a->swap_out(st, &s->out_swap_out);
        s->swapped.push_front(victim);
        s->out_preempted.push_back(victim);
      } else {
        const int n = (int)st.tokens;
        const bool known = (int64_t)st.toks.size() == st.tokens;
        std::vector<int32_t> toks = known ? st.toks : std::vector<int32_t>();
        kv_alloc_free(a, victim);
        s->waiting.push_front({victim, n, known, std::move(toks)});
        s->out_recomputed.push_back(victim);
      }
    }
    // (1c) swapped sequences come back first, first in first out, each if
    // its host-held blocks fit with the reserve left free; not in a step
    // that preempted
    while (s->out_preempted.empty() && s->out_recomputed.empty() && !s->swapped.empty() &&
           (int)s->running.size() < s->max_num_seqs) {
      const int64_t sid = s->swapped.front();
      SeqState& st = a->seqs[sid];
      const int64_t reserve = s->min_blocks_now() + (s->min_blocks < 0 ? 1 : 0);
      if (a->swap_in_cost(st) + reserve > a->n_free) break;
      s->swapped.pop_front();
      a->swap_in(st, &s->out_swap_in);
      s->running.push_back(sid);
      s->out_swapped_in.push_back(sid);
    }
  }

  // (2) free block count
  int64_t free_blocks = a->n_free;

  // (3) admit first come first served
  std::vector<int64_t> prompt_slots;
  std::vector<int32_t> hits;
  // nothing is admitted while a sequence is swapped out or in a step that
  // preempted
  while (!s->waiting.empty() && s->swapped.empty() && s->out_preempted.empty() &&
         s->out_recomputed.empty() && free_blocks > s->min_blocks_now() &&
         (int)s->running.size() < s->max_num_seqs) {
    const Request& req = s->waiting.front();
    const bool use_cache = a->caching && req.has_tokens;
    const int64_t need = use_cache ? a->admission_cost(req.tokens.data(), req.prompt_len, &hits)
                                   : a->blocks_for(req.prompt_len);
    const int64_t reserve = s->min_blocks_now() + (s->min_blocks < 0 ? 1 : 0);
    if (need > free_blocks || need + reserve > free_blocks) break;
    if (a->seqs.count(req.id)) return fail(KV_ERR_STATE, "sequence %lld already exists", (long long)req.id);
    const Request r = req;
    s->waiting.pop_front();
    int hit = 0;
    if (use_cache) {
      // the step's cache write runs before any attention of the step, so a
      // block registered now is written before a later admission reads it
      kv_alloc_allocate_prompt(a, r.id, r.tokens.data(), r.prompt_len, &hit);
      a->commit(a->seqs[r.id]);
    } else {
      kv_alloc_allocate(a, r.id, r.prompt_len);
      if (r.has_tokens) a->seqs[r.id].toks = r.tokens;
    }
    s->running.push_back(r.id);
    s->out_admitted.push_back(r.id);
    s->out_cached.push_back(hit);
    const SeqState& st = a->seqs[r.id];
    for (int t = hit; t < r.prompt_len; ++t)
      prompt_slots.push_back((int64_t)st.blocks[t / a->block_size] * a->block_size + t % a->block_size);
    free_blocks = a->n_free;
  }

  // (4) one slot per running sequence; check the whole batch fits first, in
  // the loop's own order (a window's releases free blocks for later appends)
  std::unordered_set<int64_t> admitted;
  if (s->window > 0) admitted.insert(s->out_admitted.begin(), s->out_admitted.end());
  {
    const int64_t need = a->append_need(s->running);
    if (need > a->n_free && !(s->window > 0 && a->appends_fit(s->running, admitted, s->window))) {
      info->batch = (int)s->running.size();
      info->num_tokens = info->num_cow = 0;
      info->num_admitted = (int)s->out_admitted.size();
      info->max_blocks = 0;
      return fail(KV_ERR_OOM, "appends need %lld blocks, %lld free", (long long)need,
                  (long long)a->n_free);
    }
  }
  s->out_slots = prompt_slots;
  int max_blocks = 0;
  for (int64_t r : s->running) {
    SeqState& st = a->seqs[r];
    int64_t slot;
    int32_t cs, cd;
    a->append(st, &slot, &cs, &cd);
    s->out_slots.push_back(slot);
    if (cs >= 0) {
      s->out_cow.push_back(cs);
      s->out_cow.push_back(cd);
    }
    if (s->window > 0 && !admitted.count(r)) {
      // this step's decode reads positions tokens - window .. tokens - 1: the
      // blocks wholly before them leave (a sequence admitted in this step
      // keeps its prompt blocks until the next step, after its prompt write)
      kv_alloc_release_before(a, r, st.tokens - s->window, nullptr);
    }
    s->out_running.push_back(r);
    s->out_table_flat.insert(s->out_table_flat.end(), st.blocks.begin(), st.blocks.end());
    s->out_table_off.push_back((int64_t)s->out_table_flat.size());
    s->out_lens.push_back((int32_t)st.tokens);
    if ((int)st.blocks.size() > max_blocks) max_blocks = (int)st.blocks.size();
  }
  info->batch = (int)s->running.size();
  info->num_tokens = (int)s->out_slots.size();
  info->num_cow = (int)s->out_cow.size() / 2;
  info->num_admitted = (int)s->out_admitted.size();
  info->max_blocks = max_blocks;
  return ok();
}

int kv_sched_outputs(const kv_sched* s, int64_t* running_ids, int32_t* block_tables,
                     int table_width, int32_t* context_lens, int64_t* slot_mapping,
                     int32_t* cow_pairs, int64_t* admitted_ids) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (block_tables) {
    const size_t n = s->out_table_off.size() - 1;
    for (size_t i = 0; i < n; ++i)
      if (s->out_table_off[i + 1] - s->out_table_off[i] > table_width)
        return fail(KV_ERR_ARG, "table_width %d < longest table %lld", table_width,
                    (long long)(s->out_table_off[i + 1] - s->out_table_off[i]));
    for (size_t i = 0; i < n; ++i) {
      int32_t* row = block_tables + i * (size_t)table_width;
      const int len = (int)(s->out_table_off[i + 1] - s->out_table_off[i]);
      if (len) std::memcpy(row, s->out_table_flat.data() + s->out_table_off[i], sizeof(int32_t) * len);
      for (int j = len; j < table_width; ++j) row[j] = -1;
    }
  }
  if (running_ids) std::memcpy(running_ids, s->out_running.data(), sizeof(int64_t) * s->out_running.size());
  if (context_lens) std::memcpy(context_lens, s->out_lens.data(), sizeof(int32_t) * s->out_lens.size());
  if (slot_mapping) std::memcpy(slot_mapping, s->out_slots.data(), sizeof(int64_t) * s->out_slots.size());
  if (cow_pairs) std::memcpy(cow_pairs, s->out_cow.data(), sizeof(int32_t) * s->out_cow.size());
  if (admitted_ids)
    std::memcpy(admitted_ids, s->out_admitted.data(), sizeof(int64_t) * s->out_admitted.size());
  return ok();
}

int kv_sched_stats(const kv_sched* s, int* running, int* waiting, int* used_blocks,
                   int* total_blocks) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (running) *running = (int)s->running.size();
  if (waiting) *waiting = (int)s->waiting.size();
  if (used_blocks) *used_blocks = s->a->num_blocks - (int)s->a->n_free;
  if (total_blocks) *total_blocks = s->a->num_blocks;
  return ok();
}

int kv_sched_set_preemption(kv_sched* s, int mode) {
  if (!s || (mode != KV_PREEMPT_NONE && mode != KV_PREEMPT_SWAP && mode != KV_PREEMPT_RECOMPUTE))
    return fail(KV_ERR_ARG, "bad argument");
  s->preemption = mode;
  return ok();
}

int kv_sched_swap_info(const kv_sched* s, int* num_swap_out, int* num_swap_in, int* num_preempted,
                       int* num_recomputed, int* num_swapped_in, int* num_swapped) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (num_swap_out) *num_swap_out = (int)s->out_swap_out.size() / 2;
  if (num_swap_in) *num_swap_in = (int)s->out_swap_in.size() / 2;
  if (num_preempted) *num_preempted = (int)s->out_preempted.size();
  if (num_recomputed) *num_recomputed = (int)s->out_recomputed.size();
  if (num_swapped_in) *num_swapped_in = (int)s->out_swapped_in.size();
  if (num_swapped) *num_swapped = (int)s->swapped.size();
  return ok();
}

int kv_sched_swap_outputs(const kv_sched* s, int32_t* swap_out_pairs, int32_t* swap_in_pairs,
                          int64_t* preempted_ids, int64_t* recomputed_ids, int64_t* swapped_in_ids) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (swap_out_pairs) std::copy(s->out_swap_out.begin(), s->out_swap_out.end(), swap_out_pairs);
  if (swap_in_pairs) std::copy(s->out_swap_in.begin(), s->out_swap_in.end(), swap_in_pairs);
  if (preempted_ids) std::copy(s->out_preempted.begin(), s->out_preempted.end(), preempted_ids);
  if (recomputed_ids) std::copy(s->out_recomputed.begin(), s->out_recomputed.end(), recomputed_ids);
  if (swapped_in_ids) std::copy(s->out_swapped_in.begin(), s->out_swapped_in.end(), swapped_in_ids);
  return ok();
}

int kv_sched_admitted_cached(const kv_sched* s, int32_t* cached_tokens) {
  if (!s) return fail(KV_ERR_ARG, "NULL scheduler");
  if (cached_tokens)
    for (size_t i = 0; i < s->out_cached.size(); ++i) cached_tokens[i] = s->out_cached[i];
  return ok();
}

}  // extern "C"
