"""Pins for the host block-manager oracle (oracle/block_manager.py) from the
pages' allocator scenarios and from invariants that hold after any sequence of
calls.  CPU only."""

import random

import pytest

from oracle.block_manager import BlockManager, BlockManagerError, OutOfBlocks


def test_free_list_pops_the_end():
    """Page "5.KV Cache 管理 & PagedAttention", Q9.1: free list 0..N-1, pop()
    from the end, freed blocks appended; an empty list is out of memory."""
    bm = BlockManager(4, 16)
    assert [bm.allocate() for _ in range(4)] == [3, 2, 1, 0]
    with pytest.raises(OutOfBlocks):
        bm.allocate()
    bm.decref(2)
    assert bm.num_free() == 1 and bm.allocate() == 2


def test_refcounts_free_only_at_zero():
    """Q9.4: a block shared twice goes back to the pool on the second decref."""
    bm = BlockManager(2, 16)
    b = bm.allocate()
    bm.incref(b)
    bm.decref(b)
    assert bm.num_free() == 1 and bm.ref_counts[b] == 1
    bm.decref(b)
    assert bm.num_free() == 2 and bm.ref_counts[b] == 0


def test_block_counts_of_the_worked_examples():
    """68 tokens need 5 blocks; 50 tokens need 4, the last holding 2 tokens
    (worked examples of the pages, 16-token blocks)."""
    bm = BlockManager(16, 16)
    bm.add_sequence(1)
    bm.ensure_capacity(1, 68)
    assert len(bm.block_table(1)) == 5
    bm.add_sequence(2)
    slots, copies = bm.append_tokens(2, 50)
    t = bm.block_table(2)
    assert len(t) == 4 and copies == []
    assert slots[49] == t[3] * 16 + 1 and slots[48] == t[3] * 16
    assert slots == [t[p // 16] * 16 + p % 16 for p in range(50)]


def test_append_token_uses_reserved_blocks_then_allocates():
    """Q10 then Q12: capacity reserved ahead is used before new blocks."""
    bm = BlockManager(8, 16)
    bm.add_sequence(7)
    bm.ensure_capacity(7, 20)
    reserved = bm.block_table(7)
    slots, _ = bm.append_tokens(7, 33)
    t = bm.block_table(7)
    assert t[:2] == reserved and len(t) == 3
    assert bm.seq_len(7) == 33 and slots[32] == t[2] * 16


def test_fork_then_write_copies_the_shared_partial_block():
    """Q18: the child shares the parent's blocks; its first write into the
    shared, partly filled last block copies that block (one copy pair), and
    the parent's table and tokens are untouched."""
    bm = BlockManager(8, 16)
    bm.add_sequence(0)
    bm.append_tokens(0, 40)
    parent = bm.block_table(0)
    bm.fork(0, 1)
    assert all(bm.ref_counts[b] == 2 for b in parent)
    slots, copies = bm.append_tokens(1, 1)
    child = bm.block_table(1)
    assert len(copies) == 1 and copies[0][0] == parent[2] and copies[0][1] == child[2]
    assert child[:2] == parent[:2] and child[2] != parent[2]
    assert bm.block_table(0) == parent and bm.seq_len(0) == 40 and bm.seq_len(1) == 41
    assert slots == [child[2] * 16 + 8]
    assert [bm.ref_counts[b] for b in parent] == [2, 2, 1] and bm.ref_counts[child[2]] == 1
    # the parent now owns its last block alone: no copy on its next write
    _, copies = bm.append_tokens(0, 1)
    assert copies == []


def test_fork_at_a_block_boundary_needs_no_copy():
    bm = BlockManager(8, 16)
    bm.add_sequence(0)
    bm.append_tokens(0, 48)
    bm.fork(0, 1)
    slots, copies = bm.append_tokens(1, 1)
    assert copies == [] and len(bm.block_table(1)) == 4 and slots[0] == bm.block_table(1)[3] * 16


def test_prefix_cache_shares_whole_blocks():
    """Q20: a second prompt with the same first 32 tokens shares those two
    blocks (counts raised), and gets fresh blocks for the rest; a prompt that
    differs in its first block shares nothing."""
    bm = BlockManager(16, 16)
    a = list(range(40))
    m, slots = bm.allocate_with_prefix(1, a)
    assert m == 0 and len(slots) == 40 and bm.cached_blocks() == 2
    ta = bm.block_table(1)
    b = a[:32] + [99] * 20
    m, slots = bm.allocate_with_prefix(2, b)
    tb = bm.block_table(2)
    assert m == 32 and tb[:2] == ta[:2] and tb[2] != ta[2]
    assert [bm.ref_counts[x] for x in ta[:2]] == [3, 3]        # two sequences + the cache
    assert slots == [tb[p // 16] * 16 + p % 16 for p in range(32, 52)]
    m, _ = bm.allocate_with_prefix(3, [5] + a[1:40])
    assert m == 0
    # a prefix that agrees in block 1 but not block 0 does not match block 1
    m, _ = bm.allocate_with_prefix(4, [7] * 16 + a[16:32])
    assert m == 0


def test_cache_eviction_when_the_pool_runs_out():
    """Blocks only the cache holds are evicted least recently used first,
    before allocation fails."""
    bm = BlockManager(4, 16)
    bm.allocate_with_prefix(1, list(range(48)))
    first = bm.block_table(1)
    bm.free_sequence(1)
    assert bm.num_free() == 1 and bm.cached_blocks() == 3
    bm.add_sequence(2)
    bm.append_tokens(2, 32)  # needs 2 blocks: the free one, then the oldest cache entry's
    assert bm.cached_blocks() == 2 and first[0] in bm.block_table(2)
    # a cached block still in use by a sequence is never evicted
    bm.allocate_with_prefix(3, list(range(32)))  # no match: block 0 of the prompt was evicted
    with pytest.raises(OutOfBlocks):
        bm.append_tokens(2, 64)


def test_lru_sequence_eviction():
    """The LRU manager releases the least recently used sequence."""
    bm = BlockManager(8, 16)
    for s in (1, 2, 3):
        bm.add_sequence(s)
        bm.append_tokens(s, 20)
    bm.append_tokens(1, 1)      # 1 used again
    assert bm.evict_lru_sequence(exclude=3) == 2
    assert bm.evict_lru_sequence() == 3
    with pytest.raises(BlockManagerError):
        bm.seq_len(2)


def _check_invariants(bm: BlockManager):
    refs = [0] * bm.num_blocks
    for t in bm.tables.values():
        for b in t:
            refs[b] += 1
    for blk, _ in bm.entries.values():
        refs[blk] += 1
    assert refs == bm.ref_counts
    free = set(bm.free_blocks)
    assert len(free) == len(bm.free_blocks)
    assert all((refs[b] == 0) == (b in free) for b in range(bm.num_blocks))
    for s, t in bm.tables.items():
        assert len(t) >= (bm.lens[s] + bm.block_size - 1) // bm.block_size


def test_invariants_under_random_calls():
    rnd = random.Random(5)
    bm = BlockManager(48, 16)
    live = []
    nxt = 0
    for _ in range(3000):
        op = rnd.random()
        try:
            if op < 0.2 or not live:
                bm.add_sequence(nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.45:
                bm.append_tokens(rnd.choice(live), rnd.randint(1, 20))
            elif op < 0.55:
                s = rnd.choice(live)
                bm.fork(s, nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.65:
                s = rnd.choice(live)
                bm.free_sequence(s)
                live.remove(s)
            elif op < 0.75:
                bm.ensure_capacity(rnd.choice(live), rnd.randint(0, 80))
            elif op < 0.9:
                toks = [rnd.randrange(3) for _ in range(rnd.randint(1, 70))]
                bm.allocate_with_prefix(nxt, toks)
                live.append(nxt)
                nxt += 1
            else:
                live.remove(bm.evict_lru_sequence())
        except OutOfBlocks:
            pass
        _check_invariants(bm)
    for s in list(live):
        bm.free_sequence(s)
    _check_invariants(bm)
    assert bm.num_free() + bm.cached_blocks() == 48
