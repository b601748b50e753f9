"""Host block manager: free list, reference counts, sequence block tables,
copy-on-write fork, prefix cache (TEST INFRASTRUCTURE: see ``oracle``).

Written from the allocator story of page "5.KV Cache 管理 & PagedAttention":

* Q9.1 ``BlockAllocator``: the free blocks are a list holding 0..N-1 in
  order; allocation pops the end of the list, freeing appends to it; an empty
  list is an out-of-memory error.
* Q9.4 ``RefCountBlockAllocator``: allocation sets the block's count to 1;
  ``incref`` / ``decref``; a block returns to the free list when its count
  reaches 0.
* Q10 ``ensure_capacity`` (also the multi-sequence manager of the same page):
  a sequence holds ceil(required / block_size) blocks, allocating the missing
  ones at the end of its table.
* Q12 ``append_token``: token position ``len`` goes to table[len // bs] at
  offset len % bs; a full (or missing) last block means a new block.
* Q18 ``COWBlockManager``: ``fork`` copies the parent's table and raises every
  block's count; writing into a block whose count is above 1 first copies it
  to a fresh block (the copy is returned as a (src, dst) pair for the device
  block copy), lowers the old block's count and points the table at the copy.
* Q20 ``PrefixCacheManager``: whole blocks of a prompt are looked up in a map
  from the prompt prefix to physical blocks; matched blocks are shared (count
  raised), the rest allocated fresh, and the new prompt's whole blocks are
  entered in the map.
* The LRU manager of the same page: when no block is free, the least recently
  used sequence is released.

Readings where the pages leave a step open (the C++ manager follows the same):

* A map entry holds one reference on its block, so a cached block stays valid
  after every sequence using it is gone.  An entry is keyed by (the entry of
  the previous block of the prompt, the block's tokens); entry ids are never
  reused, so the key identifies the whole prefix exactly.
* Allocation with an empty free list first evicts cache entries whose block
  only the cache holds, least recently used first (ties: oldest entry); then
  it fails.  (Sequence eviction is an explicit call, as on the page.)
* A write at offset 0 of a block the table already holds (reserved by
  ensure_capacity) uses that block; if it is shared, the sequence gets a fresh
  block without a copy (it holds no valid token yet).
* "Use" for LRU is a logical clock advanced by every call that touches a
  sequence or matches a cache entry.
"""

from __future__ import annotations


class BlockManagerError(Exception):
    pass


class OutOfBlocks(BlockManagerError):
    """No free block and nothing evictable.  A multi-token call that runs out
    keeps what it did before (like the pages' per-token loops): ``done``
    tokens were appended, with ``slots`` and ``copies`` for them."""

    def __init__(self, msg, done=0, slots=(), copies=()):
        super().__init__(msg)
        self.done, self.slots, self.copies = done, list(slots), list(copies)


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise BlockManagerError("bad sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_blocks = list(range(num_blocks))      # Q9.1
        self.ref_counts = [0] * num_blocks              # Q9.4
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.last_use: dict[int, int] = {}
        self.clock = 0
        # prefix cache: entry id -> [block, last_use]; (parent entry, tokens) -> entry id
        self.entries: dict[int, list[int]] = {}
        self.entry_key: dict[int, tuple] = {}
        self.index: dict[tuple, int] = {}
        self.next_entry = 1  # 0 = "no parent"

    # ------------------------------------------------------------ allocator
    def _tick(self) -> int:
        self.clock += 1
        return self.clock

    def _evict_one_cached(self) -> bool:
        best = None
        for eid, (blk, used) in self.entries.items():
            if self.ref_counts[blk] == 1 and (best is None or (used, eid) < best[0]):
                best = ((used, eid), eid)
        if best is None:
            return False
        eid = best[1]
        blk = self.entries.pop(eid)[0]
        del self.index[self.entry_key.pop(eid)]
        self.decref(blk)
        return True

    def allocate(self) -> int:
        if not self.free_blocks and not self._evict_one_cached():
            raise OutOfBlocks(f"no free block left in a pool of {self.num_blocks}")
        blk = self.free_blocks.pop()
        self.ref_counts[blk] = 1
        return blk

    def incref(self, blk: int) -> None:
        self.ref_counts[blk] += 1

    def decref(self, blk: int) -> None:
        self.ref_counts[blk] -= 1
        if self.ref_counts[blk] == 0:
            self.free_blocks.append(blk)

    def num_free(self) -> int:
        return len(self.free_blocks)

    # ------------------------------------------------------------ sequences
    def _seq(self, sid: int) -> list[int]:
        if sid not in self.tables:
            raise BlockManagerError(f"unknown sequence {sid}")
        self.last_use[sid] = self._tick()
        return self.tables[sid]

    def add_sequence(self, sid: int) -> None:
        if sid in self.tables:
            raise BlockManagerError(f"sequence {sid} exists")
        self.tables[sid] = []
        self.lens[sid] = 0
        self.last_use[sid] = self._tick()

    def free_sequence(self, sid: int) -> None:
        table = self._seq(sid)
        for blk in table:
            self.decref(blk)
        del self.tables[sid], self.lens[sid], self.last_use[sid]

    def ensure_capacity(self, sid: int, required_tokens: int) -> None:
        table = self._seq(sid)
        needed = (required_tokens + self.block_size - 1) // self.block_size
        while len(table) < needed:
            table.append(self.allocate())

    def append_tokens(self, sid: int, n: int):
        """Positions len..len+n-1: returns (slots, copy pairs (src, dst))."""
        table = self._seq(sid)
        bs = self.block_size
        slots, copies = [], []
        for k in range(n):
            pos = self.lens[sid]
            lb, off = divmod(pos, bs)
            try:
                if lb == len(table):
                    table.append(self.allocate())
                elif self.ref_counts[table[lb]] > 1:
                    old = table[lb]
                    new = self.allocate()
                    if off > 0:
                        copies.append((old, new))
                    self.decref(old)
                    table[lb] = new
            except OutOfBlocks as e:
                raise OutOfBlocks(str(e), k, slots, copies) from None
            slots.append(table[lb] * bs + off)
            self.lens[sid] = pos + 1
        return slots, copies

    def fork(self, parent: int, child: int) -> None:
        table = self._seq(parent)
        if child in self.tables:
            raise BlockManagerError(f"sequence {child} exists")
        for blk in table:
            self.incref(blk)
        self.tables[child] = list(table)
        self.lens[child] = self.lens[parent]
        self.last_use[child] = self._tick()

    def block_table(self, sid: int) -> list[int]:
        return list(self._seq(sid))

    def seq_len(self, sid: int) -> int:
        self._seq(sid)
        return self.lens[sid]

    def build_batch(self, sids, bt_stride: int):
        """[n, bt_stride] tables (-1 padded) and lengths of the given sequences."""
        tables, lens = [], []
        for sid in sids:
            t = self._seq(sid)
            if len(t) > bt_stride:
                raise BlockManagerError("table longer than bt_stride")
            tables.append(t + [-1] * (bt_stride - len(t)))
            lens.append(self.lens[sid])
        return tables, lens

    def evict_lru_sequence(self, exclude: int | None = None) -> int:
        """Release the least recently used sequence (not ``exclude``); returns its id."""
        cands = [(u, s) for s, u in self.last_use.items() if s != exclude]
        if not cands:
            raise OutOfBlocks("no sequence to evict")
        victim = min(cands)[1]
        table = self.tables.pop(victim)
        for blk in table:
            self.decref(blk)
        del self.lens[victim], self.last_use[victim]
        return victim

    # ------------------------------------------------------------ prefix cache
    def allocate_with_prefix(self, sid: int, tokens):
        """New sequence holding the prompt ``tokens``: whole blocks found in the
        cache are shared, the rest allocated; returns (matched tokens, slots of
        the positions from the match on)."""
        if sid in self.tables:
            raise BlockManagerError(f"sequence {sid} exists")
        bs = self.block_size
        tokens = list(tokens)
        table, parent = [], 0
        chain = []  # entry of every whole block of the prompt (matched or new)
        nfull = len(tokens) // bs
        for b in range(nfull):
            key = (parent, tuple(tokens[b * bs:(b + 1) * bs]))
            eid = self.index.get(key)
            if eid is None:
                break
            entry = self.entries[eid]
            entry[1] = self._tick()
            self.incref(entry[0])
            table.append(entry[0])
            chain.append(eid)
            parent = eid
        matched = len(table) * bs
        self.tables[sid] = table
        self.lens[sid] = len(tokens)
        self.last_use[sid] = self._tick()
        try:
            while len(table) < (len(tokens) + bs - 1) // bs:
                table.append(self.allocate())
        except OutOfBlocks:
            self.free_sequence(sid)
            raise
        for b in range(len(chain), nfull):  # enter the new whole blocks
            key = (parent, tuple(tokens[b * bs:(b + 1) * bs]))
            eid = self.next_entry
            self.next_entry += 1
            self.entries[eid] = [table[b], self._tick()]
            self.entry_key[eid] = key
            self.index[key] = eid
            self.incref(table[b])
            parent = eid
        slots = [table[p // bs] * bs + p % bs for p in range(matched, len(tokens))]
        return matched, slots

    def cached_blocks(self) -> int:
        return len(self.entries)
