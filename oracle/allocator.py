"""Reference block allocator (oracle; test infrastructure only).

Restates the bookkeeping of [P2] "PagedAttention：让 KV cache 按需生长":

* per request: block table (logical -> physical), written length, state --
  section "引用计数管理“谁还在读”，长度管理“哪里能写”";
* per physical block: refcount = number of live requests whose table holds it
  (not a token count) -- same section;
* a free queue of reallocatable blocks -- same section;
* append: fill the tail; when it is full take a block from the free queue and
  extend the table, earlier blocks never move -- section "写满一块，再拿下一块";
* release on finish/cancel: drop the table, refcount-1 on each block, blocks
  that reach 0 go back to the pool, no compaction -- section
  "请求结束，块就能交给下一位";
* fork shares every block (refcount+1); a write into a shared partial tail
  first allocates a new block, copies the valid slots, moves this request's
  mapping, then writes -- sections "只读时共用，要写入时再分开" and
  "一次写入，为什么会先少掉一个空闲块？";
* allocate-or-fail before any visible change; on failure the old mapping is
  untouched -- section "先确保分配成功，再改变可见状态";
* capacity is checked per request before publishing -- section
  "三个空闲块，四个请求同时跨边界";
* conservation: active unique + evictable cached + uncached free = pool --
  section "占用率只有 70%，为什么请求还是进不来？".

Readings where the page is silent (each also listed in the design notes):
* the free queue is FIFO: allocation pops the head, release pushes the tail,
  and a request's blocks are released in logical order;
* requests in one append call are served in the given order, each all or
  nothing; a sharer that sees refcount > 1 copies, the last holder writes in
  place;
* a copy-on-write copies exactly n mod B slots (the valid part of the tail);
* the cached set is off unless enabled; when on, a block whose refcount drops
  to 0 and that holds B valid tokens goes to the cached set (oldest first),
  partial blocks go to the free queue, and allocation evicts the oldest cached
  block only when the free queue is empty.

Prefix caching ([P2] sections "请求结束，块就能交给下一位" and
"引用计数管理“谁还在读”，长度管理“哪里能写”": released full blocks keep their
content key until evicted; [P2] section "只读时共用，要写入时再分开": a full-block
hit is shared without a copy; [P3] section 8: the key must name every input
that shaped the state -- the caller computes it, the allocator only stores it):
* ``set_block_key`` gives a full block of a live request a 64-bit content key
  (a key names one block; a block has one key);
* ``add_seq_prefix`` admits a request whose leading full blocks carry known
  keys: matching keys are taken in order until the first miss (a hit on a
  live block adds a reference, a hit on a cached block moves it back to
  active), the rest of the blocks come from the free queue; all or nothing;
* evicting a cached block (allocation with an empty free queue) drops its key.
"""
from __future__ import annotations

import collections
from typing import Dict, List, Optional, Sequence, Tuple

OK = 0
NO_BLOCKS = 1
INVALID = 2


class _Seq:
    __slots__ = ("table", "length")

    def __init__(self, table: List[int], length: int):
        self.table = table
        self.length = length


class RefAllocator:
    """Pure-Python block allocator; every operation is O(blocks touched)."""

    def __init__(self, num_blocks: int, block_size: int,
                 free_order: Optional[Sequence[int]] = None, enable_cache: bool = False):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad pool shape")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.enable_cache = bool(enable_cache)
        self.free = collections.deque(order)
        self.cached = collections.deque()
        self.ref = [0] * num_blocks
        self.seqs: Dict[int, _Seq] = {}
        self.counters = dict(allocs=0, frees=0, cow_copies=0, alloc_failures=0, evictions=0,
                             prefix_hits=0)
        self.key_of = {}      # block -> content key
        self.block_of = {}    # content key -> block

    # -- capacity -----------------------------------------------------------
    def available(self) -> int:
        return len(self.free) + (len(self.cached) if self.enable_cache else 0)

    def _take(self) -> int:
        if self.free:
            b = self.free.popleft()
        else:
            b = self.cached.popleft()
            self.counters["evictions"] += 1
            k = self.key_of.pop(b, None)
            if k is not None:
                del self.block_of[k]
        self.ref[b] = 1
        self.counters["allocs"] += 1
        return b

    # -- operations ---------------------------------------------------------
    def add_seq(self, seq_id: int, n_tokens: int) -> int:
        """Admit a request holding n_tokens of KV: ceil(n/B) new blocks or FAIL."""
        if seq_id in self.seqs or n_tokens < 0 or seq_id < 0:
            return INVALID
        need = -(-n_tokens // self.block_size)
        if need > self.available():
            self.counters["alloc_failures"] += 1
            return NO_BLOCKS
        table = [self._take() for _ in range(need)]
        self.seqs[seq_id] = _Seq(table, n_tokens)
        return OK

    def fork(self, parent: int, child: int) -> int:
        """child shares every block of parent (refcount + 1 each)."""
        if parent not in self.seqs or child in self.seqs or child < 0:
            return INVALID
        p = self.seqs[parent]
        for b in p.table:
            self.ref[b] += 1
        self.seqs[child] = _Seq(list(p.table), p.length)
        return OK

    def append(self, seq_ids: Sequence[int]) -> Tuple[int, List[int], List[Tuple[int, int, int]]]:
        """Reserve the slot of one new token for each request, in order.

        Returns (status, per-request statuses, copy list of (src, dst, n_valid)).
        status is OK when every request got its slot, NO_BLOCKS when at least
        one did not (that request is left exactly as it was), INVALID (and
        nothing changes) for an unknown or repeated id.
        """
        ids = [int(s) for s in seq_ids]
        if len(set(ids)) != len(ids) or any(s not in self.seqs for s in ids):
            return INVALID, [], []
        statuses: List[int] = []
        copies: List[Tuple[int, int, int]] = []
        B = self.block_size
        for sid in ids:
            s = self.seqs[sid]
            n = s.length
            if n % B == 0:
                # no tail yet, or the tail is full: a fresh block
                if self.available() < 1:
                    self.counters["alloc_failures"] += 1
                    statuses.append(NO_BLOCKS)
                    continue
                s.table.append(self._take())
            else:
                tail = s.table[-1]
                if self.ref[tail] > 1:
                    # shared partial tail: allocate, copy the valid part, remap
                    if self.available() < 1:
                        self.counters["alloc_failures"] += 1
                        statuses.append(NO_BLOCKS)
                        continue
                    new = self._take()
                    copies.append((tail, new, n % B))
                    self.ref[tail] -= 1
                    s.table[-1] = new
                    self.counters["cow_copies"] += 1
            s.length = n + 1
            statuses.append(OK)
        status = OK if all(x == OK for x in statuses) else NO_BLOCKS
        return status, statuses, copies

    def free_seq(self, seq_id: int) -> int:
        """Finish, cancel or preempt: release every block reference in logical order."""
        if seq_id not in self.seqs:
            return INVALID
        s = self.seqs.pop(seq_id)
        last = len(s.table) - 1
        for i, b in enumerate(s.table):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                full = i < last or (s.length > 0 and s.length % self.block_size == 0)
                if self.enable_cache and full:
                    self.cached.append(b)      # keeps its content key until evicted
                else:
                    self.free.append(b)
                    k = self.key_of.pop(b, None)
                    if k is not None:
                        del self.block_of[k]
                self.counters["frees"] += 1
        return OK

    def set_block_key(self, seq_id: int, logical_block: int, key: int) -> int:
        """Name the content of a full block of a live request (for later prefix hits)."""
        if seq_id not in self.seqs:
            return INVALID
        s = self.seqs[seq_id]
        if logical_block < 0 or (logical_block + 1) * self.block_size > s.length:
            return INVALID                      # only full blocks are shareable
        b = s.table[logical_block]
        key = int(key) & 0xFFFFFFFFFFFFFFFF
        owner = self.block_of.get(key)
        if owner is not None and owner != b:
            return INVALID                      # the key already names another block
        old = self.key_of.get(b)
        if old is not None and old != key:
            return INVALID                      # the block already has another key
        self.key_of[b] = key
        self.block_of[key] = b
        return OK

    def add_seq_prefix(self, seq_id: int, n_tokens: int, keys) -> Tuple[int, int]:
        """Admit a request reusing the cached blocks of its leading full blocks.

        Returns (status, number of leading blocks found in the cache).
        """
        keys = [int(k) & 0xFFFFFFFFFFFFFFFF for k in keys]
        if seq_id in self.seqs or n_tokens < 0 or seq_id < 0 or len(keys) * self.block_size > n_tokens:
            return INVALID, 0
        hits = []
        for k in keys:
            b = self.block_of.get(k)
            if b is None:
                break
            hits.append(b)
        need = -(-n_tokens // self.block_size) - len(hits)
        revived = sum(1 for b in hits if self.ref[b] == 0)
        if need > self.available() - (revived if self.enable_cache else 0):
            self.counters["alloc_failures"] += 1
            return NO_BLOCKS, 0
        for b in hits:
            if self.ref[b] == 0:
                self.cached.remove(b)
            self.ref[b] += 1
        self.counters["prefix_hits"] += len(hits)
        table = hits + [self._take() for _ in range(need)]
        self.seqs[seq_id] = _Seq(table, n_tokens)
        return OK, len(hits)

    # -- queries ------------------------------------------------------------
    def table(self, seq_id: int) -> List[int]:
        return list(self.seqs[seq_id].table)

    def length(self, seq_id: int) -> int:
        return self.seqs[seq_id].length

    def stats(self) -> Dict[str, int]:
        active = sum(1 for r in self.ref if r > 0)
        return dict(active=active, cached=len(self.cached), free=len(self.free),
                    pool=self.num_blocks, seqs=len(self.seqs), **self.counters)

    def check(self) -> bool:
        """Conservation plus a refcount recount from the live tables."""
        st = self.stats()
        if st["active"] + st["cached"] + st["free"] != self.num_blocks:
            return False
        recount = [0] * self.num_blocks
        for s in self.seqs.values():
            if len(s.table) != -(-s.length // self.block_size):
                return False
            for b in s.table:
                recount[b] += 1
        if recount != self.ref:
            return False
        idle = list(self.free) + list(self.cached)
        if len(set(idle)) != len(idle):
            return False
        if any(self.ref[b] != 0 for b in idle):
            return False
        # keys: a bijection between keyed blocks and their keys; free blocks carry none
        if any(self.block_of.get(k) != b for b, k in self.key_of.items()):
            return False
        if len(self.block_of) != len(self.key_of):
            return False
        return all(b not in self.key_of for b in self.free)
