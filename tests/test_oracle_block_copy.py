"""Pins for the block-copy oracle through the scenarios the pages describe:
copy-on-write after a fork and a swap-out / swap-in round trip.  CPU only."""

import numpy as np

from oracle import block_copy, cache_write, paging


def _pool(rng, nb=24, bs=16, hkv=2, d=8):
    k = rng.standard_normal((nb, bs, hkv, d)).astype(np.float16)
    v = rng.standard_normal((nb, bs, hkv, d)).astype(np.float16)
    return k, v


def test_copy_on_write_fork():
    """Page "5.KV Cache 管理 & PagedAttention", Q18: a child forked from a
    parent shares its blocks; writing the child's next token into the shared,
    partly filled last block first copies that block.  Afterwards the parent
    still reads its own tokens and the child reads the parent's plus its own."""
    rng = np.random.default_rng(0)
    bs = 16
    k, v = _pool(rng, bs=bs)
    parent_table, n = [5, 11, 2], 40                      # 40 tokens: last block partly filled
    before_k = paging.gather_sequence(k, parent_table, n).copy()
    before_v = paging.gather_sequence(v, parent_table, n).copy()
    child_table = list(parent_table)                       # fork: shared blocks
    ref = {b: 2 for b in parent_table}
    logical = n // bs
    shared = child_table[logical]
    assert ref[shared] > 1                                 # -> copy on write
    new_blk = 17
    block_copy.copy_blocks(k, v, k, v, [[shared, new_blk]])
    child_table[logical] = new_blk
    ref[shared] -= 1
    tok_k = rng.standard_normal((1, 2, 8)).astype(np.float16)
    tok_v = rng.standard_normal((1, 2, 8)).astype(np.float16)
    cache_write.reshape_and_cache(tok_k, tok_v, k, v, [paging.slot_of(child_table, n, bs)])
    np.testing.assert_array_equal(paging.gather_sequence(k, parent_table, n), before_k)
    np.testing.assert_array_equal(paging.gather_sequence(v, parent_table, n), before_v)
    np.testing.assert_array_equal(paging.gather_sequence(k, child_table, n + 1),
                                  np.concatenate([before_k, tok_k]))
    np.testing.assert_array_equal(paging.gather_sequence(v, child_table, n + 1),
                                  np.concatenate([before_v, tok_v]))


def test_swap_out_and_back_in():
    """Page "KV Cache 优化与内存管理深度解析", CPUSwap: swap_out copies a
    sequence's GPU blocks to CPU blocks; swap_in allocates (other) GPU blocks
    and loads them back.  The sequence then reads exactly what it had."""
    rng = np.random.default_rng(1)
    k, v = _pool(rng)
    table, n = [3, 9, 14, 0], 55
    before = paging.gather_sequence(k, table, n).copy()
    host_k = np.zeros((8, 16, 2, 8), np.float16)
    host_v = np.zeros_like(host_k)
    block_copy.copy_blocks(k, v, host_k, host_v, [[b, i] for i, b in enumerate(table)])  # swap out
    k[table] = np.nan                                      # the GPU blocks get reused
    new_table = [21, 7, 12, 19]
    block_copy.copy_blocks(host_k, host_v, k, v, [[i, b] for i, b in enumerate(new_table)])  # swap in
    np.testing.assert_array_equal(paging.gather_sequence(k, new_table, n), before)


def test_out_of_range_pairs_are_skipped_and_order_holds():
    rng = np.random.default_rng(2)
    k, v = _pool(rng, nb=6)
    k0 = k.copy()
    block_copy.copy_blocks(k, v, k, v, [[-1, 2], [1, 6], [9, 0]])
    np.testing.assert_array_equal(k, k0)
    block_copy.copy_blocks(k, v, k, v, [[1, 3], [2, 3]])   # later pair wins
    np.testing.assert_array_equal(k[3], k0[2])
