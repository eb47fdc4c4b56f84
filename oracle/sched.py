"""Reference block allocator and scheduling step — TEST INFRASTRUCTURE ONLY.

Written from "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍":

* section "PagedAttention：把操作系统的虚拟内存搬进 GPU": the cache is cut into
  fixed-size physical blocks; each sequence's block table maps its logical
  blocks to physical ones; blocks are taken on demand as tokens are produced
  (no reservation for the maximum length); every block has the same size,
  so any free block serves any request; several logical blocks (prefix or
  beam sharing) may map to one physical block.
* section "连续批处理：别再等最慢的那个请求了" — the scheduling loop printed
  there: (1) drop finished requests and free their blocks, (2) read the
  number of free blocks, (3) while requests wait and the free count is above
  MIN_BLOCKS, pop the first waiting request and, if the block manager can
  allocate it, allocate and move it to the running set, (4) decode the
  running set.

Readings where the page leaves a step open:

* sharing implies a reference count per physical block; a block returns to
  the free list when its count reaches zero;
* the free list is FIFO: allocation takes from the head, freeing appends to
  the tail in block-table order (deterministic, so two implementations can be
  compared exactly);
* writing into a block whose count is above one first copies it
  (copy-on-write) into a fresh block, which replaces it in the writer's table;
* in step (3) the printed loop pops a request before testing it and never
  puts it back; the reading taken keeps FIFO order instead: a head request
  that cannot be allocated stays at the head and admission stops; the free
  count is re-read after each admission; admission also stops at
  ``max_num_seqs`` running sequences (the page's ``max_num_seqs`` setting);
* MIN_BLOCKS defaults to the number of running sequences: one block per
  running sequence is kept in reserve for this iteration's appended token.  A
  waiting request is admitted only if its prompt's blocks fit in the free
  blocks while that reserve (counting the request itself) stays free, so the
  appends of step (4) never run out of blocks;
* step (4) appends one token slot to every running sequence (admitted ones
  included) before the decode.
"""

from __future__ import annotations

from collections import deque


class OracleOOM(Exception):
    """No free block for a required allocation."""


class OracleStateError(Exception):
    """Unknown or duplicate sequence, or a block freed twice."""


def blocks_for(num_tokens: int, block_size: int) -> int:
    return -(-num_tokens // block_size)


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if initial_free_order is None else [int(b) for b in initial_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial free order must be a permutation of the blocks")
        self.free_list = deque(order)
        self.refcount = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.tokens: dict[int, int] = {}
        self.num_cow = 0
        self.num_alloc = 0
        self.num_freed = 0
        self.host_free = deque()

    # verbs named on the page
    def get_num_free_blocks(self) -> int:
        return len(self.free_list)

    def can_allocate(self, num_tokens: int) -> bool:
        return blocks_for(num_tokens, self.block_size) <= len(self.free_list)

    def _take(self) -> int:
        if not self.free_list:
            raise OracleOOM("no free block")
        b = self.free_list.popleft()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        self.num_alloc += 1
        return b

    def allocate(self, seq_id: int, num_tokens: int) -> None:
        if seq_id in self.tables:
            raise OracleStateError(f"sequence {seq_id} already exists")
        if num_tokens < 0:
            raise ValueError("negative token count")
        need = blocks_for(num_tokens, self.block_size)
        if need > len(self.free_list):
            raise OracleOOM("not enough free blocks")
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.tokens[seq_id] = num_tokens

    def free(self, seq_id: int) -> None:
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        for b in self.tables.pop(seq_id):
            if b <= -2:  # held in the host swap space
                self.host_free.append(-b - 2)
                continue
            if b < 0:  # already released (sliding window)
                continue
            if self.refcount[b] <= 0:
                raise OracleStateError(f"block {b} freed twice")
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_list.append(b)
                self.num_freed += 1
        del self.tokens[seq_id]

    # sharing and growth
    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables:
            raise OracleStateError(f"sequence {parent} is unknown")
        if child in self.tables:
            raise OracleStateError(f"sequence {child} already exists")
        self.tables[child] = list(self.tables[parent])
        self.tokens[child] = self.tokens[parent]
        for b in self.tables[child]:
            if b >= 0:
                self.refcount[b] += 1

    def append_slot(self, seq_id: int):
        """Reserve the slot of the sequence's next token.

        Returns (slot, cow_src, cow_dst); cow_* are -1 unless the last block
        was shared and had to be copied first.  slot = block * block_size +
        offset."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        table = self.tables[seq_id]
        pos = self.tokens[seq_id]
        cow_src = cow_dst = -1
        if pos % self.block_size == 0:
            table.append(self._take())
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                new = self._take()
                self.refcount[last] -= 1
                table[-1] = new
                cow_src, cow_dst = last, new
                self.num_cow += 1
        self.tokens[seq_id] = pos + 1
        slot = table[pos // self.block_size] * self.block_size + pos % self.block_size
        return slot, cow_src, cow_dst

    def release_before(self, seq_id: int, token: int) -> int:
        """Sliding window: release every block wholly before position
        min(token, n), n the sequence's token count (its table entry becomes
        -1; the table keeps its length so logical block indices stay put).
        Only positions the sequence holds count, so the block that receives
        its next token is never released.  Returns the number released."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        table = self.tables[seq_id]
        upto = min(min(max(token, 0), self.tokens[seq_id]) // self.block_size, len(table))
        n = 0
        for i in range(upto):
            b = table[i]
            if b < 0:
                continue
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_list.append(b)
                self.num_freed += 1
            table[i] = -1
            n += 1
        return n

    # ------------------------------------------------ swapping (preemption)
    # Reading taken (the pages only name "preemption and swapping" as what
    # happens when the KV cache runs out): a swapped-out sequence moves every
    # block it holds alone to a slot of a host swap space (FIFO free list of
    # slots) and returns the device block; a block it shares stays on the
    # device with its reference kept.  Its table entry for a host-held block
    # is -(2 + slot).  Swapping in takes fresh device blocks for those entries.

    def set_swap_space(self, num_slots: int) -> None:
        self.host_free = deque(range(int(num_slots)))

    def swap_out_cost(self, seq_id: int) -> int:
        return sum(1 for b in self.tables[seq_id] if b >= 0 and self.refcount[b] == 1)

    def swap_in_cost(self, seq_id: int) -> int:
        return sum(1 for b in self.tables[seq_id] if b <= -2)

    def swap_out(self, seq_id: int):
        """[(device block, host slot)] moved to host; device blocks freed."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        table = self.tables[seq_id]
        if self.swap_out_cost(seq_id) > len(getattr(self, "host_free", ())):
            raise OracleOOM("not enough host swap slots")
        pairs = []
        for i, b in enumerate(table):
            if b >= 0 and self.refcount[b] == 1:
                slot = self.host_free.popleft()
                pairs.append((b, slot))
                self.refcount[b] = 0
                self.free_list.append(b)
                self.num_freed += 1
                table[i] = -(2 + slot)
        return pairs

    def swap_in(self, seq_id: int):
        """[(host slot, device block)] brought back into fresh blocks."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        table = self.tables[seq_id]
        if self.swap_in_cost(seq_id) > len(self.free_list):
            raise OracleOOM("not enough free blocks")
        pairs = []
        for i, b in enumerate(table):
            if b <= -2:
                slot = -b - 2
                nb = self._take()
                pairs.append((slot, nb))
                self.host_free.append(slot)
                table[i] = nb
        return pairs

    def block_table(self, seq_id: int) -> list[int]:
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        return list(self.tables[seq_id])

    def snapshot(self):
        return list(self.free_list), list(self.refcount)


class Scheduler:
    """One scheduling iteration per :meth:`step`, in the page's order."""

    def __init__(self, bm: BlockManager, max_num_seqs: int, min_blocks: int | None = None,
                 window: int = 0):
        self.bm = bm
        self.max_num_seqs = max_num_seqs
        self.min_blocks = min_blocks  # None: number of running sequences
        # > 0: after its append, a running sequence releases the blocks wholly
        # before its last `window` positions (sliding-window decode reads no
        # earlier block); one admitted in this step keeps them until the next
        self.window = window
        # preemption when the running set's appends do not fit: None (the
        # step fails), "swap" or "recompute"
        self.preemption = None
        self.swapped: deque[int] = deque()
        self.waiting: deque[tuple[int, int]] = deque()
        self.running: list[int] = []

    def add_request(self, seq_id: int, prompt_len: int) -> None:
        self.waiting.append((seq_id, prompt_len, None))

    def add_request_tokens(self, seq_id: int, tokens) -> None:
        """A request whose prompt token ids are known (prefix caching)."""
        tokens = [int(t) for t in tokens]
        self.waiting.append((seq_id, len(tokens), tokens))

    def adopt(self, seq_id: int) -> None:
        """Put a sequence that already holds blocks (e.g. a fork) in the running set."""
        if seq_id not in self.bm.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        self.running.append(seq_id)

    def _min_blocks(self) -> int:
        return len(self.running) if self.min_blocks is None else self.min_blocks

    def step(self, finished_ids):
        # (1) remove finished requests and return their blocks
        finished = set(int(x) for x in finished_ids)
        for sid in finished:
            if sid not in self.running:
                raise OracleStateError(f"sequence {sid} is not running")
        self.running = [r for r in self.running if r not in finished]
        for sid in finished_ids:
            self.bm.free(int(sid))
        # (1b) preemption (reading taken; the pages only name it): while the
        # running set's appends do not fit, the most recently scheduled
        # running sequence leaves, swapped out (its exclusive blocks to host
        # slots; it waits at the front of the swapped queue) or, without room
        # in the swap space or in recompute mode, freed and put back at the
        # front of the waiting queue with its whole context as the prompt
        swap_out, swap_in, preempted, recomputed, swapped_in = [], [], [], [], []
        if self.preemption is not None:
            while self.running and self._append_need(self.running) > self.bm.get_num_free_blocks():
                victim = self.running.pop()
                if (self.preemption == "swap"
                        and self.bm.swap_out_cost(victim) <= len(getattr(self.bm, "host_free", ()))):
                    swap_out += self.bm.swap_out(victim)
                    self.swapped.appendleft(victim)
                    preempted.append(victim)
                else:
                    n = self.bm.tokens[victim]
                    toks = getattr(self.bm, "seq_tokens", {}).get(victim)
                    toks = list(toks) if toks is not None and len(toks) == n else None
                    self.bm.free(victim)
                    self.waiting.appendleft((victim, n, toks))
                    recomputed.append(victim)
            # (1c) swapped sequences come back first (first in, first out),
            # each if its host-held blocks fit with the reserve left free;
            # not in a step that preempted (nor is anything admitted then)
            while (not preempted and not recomputed and self.swapped
                   and len(self.running) < self.max_num_seqs):
                sid = self.swapped[0]
                reserve = self._min_blocks() + (1 if self.min_blocks is None else 0)
                if self.bm.swap_in_cost(sid) + reserve > self.bm.get_num_free_blocks():
                    break
                self.swapped.popleft()
                swap_in += self.bm.swap_in(sid)
                self.running.append(sid)
                swapped_in.append(sid)
        # (2) free block count
        free_blocks = self.bm.get_num_free_blocks()
        # (3) admit waiting requests, first come first served
        admitted = []
        cached = []
        prompt_slots = []
        caching = isinstance(self.bm, PrefixCachingBlockManager)
        while (self.waiting and not self.swapped and not preempted and not recomputed
               and free_blocks > self._min_blocks() and len(self.running) < self.max_num_seqs):
            sid, plen, toks = self.waiting[0]
            reserve = self._min_blocks() + (1 if self.min_blocks is None else 0)
            use_cache = caching and toks is not None
            need = self.bm.admission_cost(toks) if use_cache else blocks_for(plen, self.bm.block_size)
            if not (need <= free_blocks and need + reserve <= free_blocks):
                break
            if sid in self.bm.tables:
                raise OracleStateError(f"sequence {sid} already exists")
            self.waiting.popleft()
            if use_cache:
                hit = self.bm.allocate_prompt(sid, toks)
                # the step's cache write runs before any attention of the step,
                # so blocks registered now are written before a later admission
                # of this step reads them
                self.bm.commit(sid)
            else:
                self.bm.allocate(sid, plen)
                hit = 0
            self.running.append(sid)
            admitted.append(sid)
            cached.append(hit)
            table = self.bm.tables[sid]
            bs = self.bm.block_size
            prompt_slots.extend(table[t // bs] * bs + t % bs for t in range(hit, plen))
            free_blocks = self.bm.get_num_free_blocks()
        # (4) one new token slot per running sequence, then decode
        decode_slots, cow = [], []
        for sid in self.running:
            slot, cs, cd = self.bm.append_slot(sid)
            decode_slots.append(slot)
            if cs >= 0:
                cow.append((cs, cd))
            if self.window > 0 and sid not in admitted:
                self.bm.release_before(sid, self.bm.tokens[sid] - self.window)
        return {
            "running": list(self.running),
            "block_tables": [self.bm.block_table(s) for s in self.running],
            "context_lens": [self.bm.tokens[s] for s in self.running],
            "slot_mapping": prompt_slots + decode_slots,
            "cow_pairs": cow,
            "admitted": admitted,
            "cached": cached,
            "swap_out": swap_out,
            "swap_in": swap_in,
            "preempted": preempted,
            "recomputed": recomputed,
            "swapped_in": swapped_in,
        }

    def _append_need(self, seqs) -> int:
        """Fresh blocks the appends of `seqs` take: one per sequence at a
        block boundary, plus the copies of shared partly filled last blocks
        (at most refcount - 1 per block)."""
        bs = self.bm.block_size
        need, shared = 0, {}
        for sid in seqs:
            n, last = self.bm.tokens[sid], self.bm.tables[sid][-1] if self.bm.tables[sid] else -1
            if n % bs == 0:
                need += 1
            elif self.bm.refcount[last] > 1:
                shared[last] = shared.get(last, 0) + 1
        for b, k in shared.items():
            need += min(k, self.bm.refcount[b] - 1)
        return need

    def stats(self):
        used = self.bm.num_blocks - self.bm.get_num_free_blocks()
        return len(self.running), len(self.waiting), used, self.bm.num_blocks


# ------------------------------------------------------------ prefix caching
#
# "vLLM 推理加速原理详解" mentions automatic prefix caching (requests that
# share a system prompt reuse its KV blocks; the pitfalls section and the
# deployment flags) without describing the lookup.  Reading taken here:
#
# * only FULL blocks are cached; block i of a sequence is keyed by
#   key_i = FNV-1a-64(key_{i-1} as 8 little-endian bytes, then the block's
#   token ids as 4 little-endian bytes each), key_{-1} = the FNV offset basis
#   (the FNV-1a definition: for each byte, h ^= byte, h *= 1099511628211 mod
#   2^64, starting from 14695981039346656037);
# * a hit requires the stored parent key and token ids to equal the lookup's
#   (no sharing on a hash collision);
# * at admission the longest run of hits from block 0 is shared (refcount + 1;
#   a hit on a free block takes it out of the free list), capped so that at
#   least the prompt's last token is computed; the rest is allocated fresh;
# * a block is registered (becomes findable) when the caller commits its
#   tokens, i.e. once its KV has been written; a block whose key is already
#   registered to another block stays unregistered;
# * freed blocks keep their key; the free list stays FIFO, but a sequence's
#   blocks are appended deepest-first so that shared prefixes leave last;
#   taking a free block that still holds a key evicts that key.

FNV_OFFSET = 14695981039346656037
FNV_PRIME = 1099511628211
_MASK64 = (1 << 64) - 1


def fnv1a64(data: bytes, h: int = FNV_OFFSET) -> int:
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & _MASK64
    return h


def block_key(parent: int, tokens) -> int:
    data = int(parent).to_bytes(8, "little") + b"".join(
        (int(t) & 0xFFFFFFFF).to_bytes(4, "little") for t in tokens)
    return fnv1a64(data)


class PrefixCachingBlockManager(BlockManager):
    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        super().__init__(num_blocks, block_size, initial_free_order)
        self.cached: dict[int, int] = {}          # key -> block
        self.key_of: dict[int, tuple] = {}        # block -> (key, parent key, tokens)
        self.seq_tokens: dict[int, list[int]] = {}
        self.registered: dict[int, int] = {}      # seq -> leading blocks registered or skipped
        self.num_hits = 0
        self.num_evictions = 0

    def _take(self) -> int:
        if not self.free_list:
            raise OracleOOM("no free block")
        b = self.free_list[0]
        if b in self.key_of:
            key = self.key_of.pop(b)[0]
            if self.cached.get(key) == b:
                del self.cached[key]
            self.num_evictions += 1
        return super()._take()

    def _keys(self, tokens):
        bs = self.block_size
        keys, parent = [], FNV_OFFSET
        for i in range(len(tokens) // bs):
            blk = tuple(int(t) for t in tokens[i * bs:(i + 1) * bs])
            k = block_key(parent, blk)
            keys.append((k, parent, blk))
            parent = k
        return keys

    def lookup(self, tokens):
        """Blocks of the longest cached prefix of `tokens` (at most
        (len - 1) // block_size of them)."""
        cap = max(0, (len(tokens) - 1) // self.block_size)
        hits = []
        for k, parent, blk in self._keys(tokens)[:cap]:
            b = self.cached.get(k)
            if b is None or self.key_of.get(b) != (k, parent, blk):
                break
            hits.append(b)
        return hits

    def admission_cost(self, tokens) -> int:
        """Free blocks an allocate_prompt of `tokens` takes out of the free list."""
        hits = self.lookup(tokens)
        fresh = blocks_for(len(tokens), self.block_size) - len(hits)
        return fresh + sum(1 for b in hits if self.refcount[b] == 0)

    def allocate_prompt(self, seq_id: int, tokens) -> int:
        """Allocate a prompt, sharing its cached prefix; returns the number
        of cached tokens (the caller computes only the rest)."""
        if seq_id in self.tables:
            raise OracleStateError(f"sequence {seq_id} already exists")
        tokens = [int(t) for t in tokens]
        if self.admission_cost(tokens) > len(self.free_list):
            raise OracleOOM("not enough free blocks")
        hits = self.lookup(tokens)
        for b in hits:
            if self.refcount[b] == 0:
                self.free_list.remove(b)
            self.refcount[b] += 1
        self.num_hits += len(hits)
        fresh = blocks_for(len(tokens), self.block_size) - len(hits)
        self.tables[seq_id] = hits + [self._take() for _ in range(fresh)]
        self.tokens[seq_id] = len(tokens)
        self.seq_tokens[seq_id] = tokens
        self.registered[seq_id] = len(hits)
        return len(hits) * self.block_size

    def allocate(self, seq_id: int, num_tokens: int) -> None:
        super().allocate(seq_id, num_tokens)
        self.seq_tokens[seq_id] = []
        self.registered[seq_id] = 0

    def fork(self, parent: int, child: int) -> None:
        super().fork(parent, child)
        self.seq_tokens[child] = list(self.seq_tokens.get(parent, []))
        self.registered[child] = self.registered.get(parent, 0)

    def append_token(self, seq_id: int, token: int):
        """append_slot for a token whose id is known (recorded only while the
        sequence's known tokens are contiguous from position 0)."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        toks = self.seq_tokens.setdefault(seq_id, [])
        contiguous = len(toks) == self.tokens[seq_id]
        out = self.append_slot(seq_id)
        if contiguous:
            toks.append(int(token))
        return out

    def commit(self, seq_id: int) -> int:
        """Register every full block whose tokens are all known; returns how
        many blocks became findable."""
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        toks = self.seq_tokens.get(seq_id, [])
        keys = self._keys(toks[:self.tokens[seq_id]])
        table = self.tables[seq_id]
        done = self.registered.get(seq_id, 0)
        new = 0
        for i in range(done, len(keys)):
            k, parent, blk = keys[i]
            b = table[i]
            if b >= 0 and k not in self.cached and b not in self.key_of:
                self.cached[k] = b
                self.key_of[b] = (k, parent, blk)
                new += 1
        self.registered[seq_id] = max(done, len(keys))
        return new

    def free(self, seq_id: int) -> None:
        if seq_id not in self.tables:
            raise OracleStateError(f"sequence {seq_id} is unknown")
        for b in reversed(self.tables.pop(seq_id)):
            if b <= -2:
                self.host_free.append(-b - 2)
                continue
            if b < 0:
                continue
            if self.refcount[b] <= 0:
                raise OracleStateError(f"block {b} freed twice")
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_list.append(b)
                self.num_freed += 1
        del self.tokens[seq_id]
        self.seq_tokens.pop(seq_id, None)
        self.registered.pop(seq_id, None)
