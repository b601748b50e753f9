"""Pins for the shared-prefix oracle: what forked sequences share (page "5.KV
Cache 管理 & PagedAttention", Q18 fork / copy-on-write), and that sharing
physical blocks leaves decode attention unchanged.  CPU only."""

import random

import numpy as np

from oracle import attention, block_copy, prefix_sharing
from paged_kv_cache_463_b200 import workloads as W


def test_fork_shares_every_whole_block():
    """Q18: the child's table is a copy of the parent's.  With 40 tokens the
    first two blocks are whole and shared; the third is partly filled, so it
    belongs to each member's suffix."""
    parent = [5, 11, 2]
    child = list(parent)
    assert prefix_sharing.common_prefix_blocks([parent, child], [40, 40]) == 2
    assert prefix_sharing.common_prefix_blocks([parent, child], [48, 48]) == 3


def test_copy_on_write_ends_the_shared_run():
    """After the child writes into the shared last block, that block is a
    private copy: the shared run stops before it."""
    parent = [5, 11, 2, 8]
    child = [5, 11, 17, 8]  # block 2 copied to 17 on write
    assert prefix_sharing.common_prefix_blocks([parent, child], [64, 64]) == 2
    # a member shorter than the run cuts it to its own whole blocks
    assert prefix_sharing.common_prefix_blocks([parent, parent], [64, 20]) == 1
    assert prefix_sharing.common_prefix_blocks([parent], [15]) == 0
    assert prefix_sharing.common_prefix_blocks([], []) == 0


def test_brute_force_on_random_tables():
    """Largest b for which every member's first b entries equal the first
    member's and every member holds b whole blocks, found by trying every b."""
    rnd = random.Random(3)
    for _ in range(300):
        m = rnd.randint(1, 4)
        base = [rnd.randrange(6) for _ in range(6)]
        rows = []
        for _ in range(m):
            r = list(base)
            for j in range(6):
                if rnd.random() < 0.15:
                    r[j] = rnd.randrange(6)
            rows.append(r)
        lens = [rnd.randint(0, 96) for _ in range(m)]
        best = 0
        for b in range(7):
            if all(r[:b] == rows[0][:b] for r in rows) and all(b * 16 <= n for n in lens):
                best = b
        assert prefix_sharing.common_prefix_blocks(rows, lens) == best


def test_sharing_blocks_does_not_change_attention():
    """Decode over tables that share prefix blocks equals decode over tables in
    which every member owns a private copy of those blocks (the state after a
    copy-on-write of each of them)."""
    rng = np.random.default_rng(7)
    nb, bs, hkv, d, hq = 40, 16, 2, 16, 4
    k = rng.standard_normal((nb, bs, hkv, d)).astype(np.float16)
    v = rng.standard_normal((nb, bs, hkv, d)).astype(np.float16)
    q = rng.standard_normal((3, hq, d)).astype(np.float16)
    prefix = [4, 9, 30]
    tables = [prefix + [1, 2], prefix + [3], prefix + [5, 6, 7]]
    lens = [3 * bs + 20, 3 * bs + 5, 3 * bs + 40]
    assert prefix_sharing.common_prefix_blocks(tables, lens) == 3
    shared = attention.decode_attention(q, k, v, tables, lens, 0.25, "f16", "f16")
    k2, v2 = k.copy(), v.copy()
    private = [list(t) for t in tables]
    fresh = iter(range(10, 30))
    for t in private[1:]:
        for j in range(3):
            dst = next(fresh)
            block_copy.copy_blocks(k2, v2, k2, v2, [[t[j], dst]])
            t[j] = dst
    assert prefix_sharing.common_prefix_blocks(private, lens) == 0
    alone = attention.decode_attention(q, k2, v2, private, lens, 0.25, "f16", "f16")
    np.testing.assert_array_equal(shared, alone)


def test_workload_groups_share_their_prefix():
    """The generator's groups (reference-counted prefix blocks, Q9.4 / Q18):
    members of one group share exactly the prefix; neighbours across a group
    boundary share nothing."""
    spec = W.scaled(W.SPEC_BY_NAME["shared-prefix-fp8"], num_seqs=12, prefix_groups=3, prefix_tokens=64,
                    seq_len_min=1, seq_len_max=40)
    lay = W.build_layout(spec)
    t = lay.block_tables.tolist()
    assert lay.group_start == [0, 4, 8, 12]
    for g in range(3):
        a, b = lay.group_start[g], lay.group_start[g + 1]
        assert lay.group_prefix_len[g] == 64
        assert prefix_sharing.common_prefix_blocks(t[a:b], lay.seq_lens[a:b]) == 4
        if g:
            assert prefix_sharing.common_prefix_blocks(t[a - 1:a + 1], lay.seq_lens[a - 1:a + 1]) == 0
    # every shared block's reference count is the group's size
    for g in range(3):
        for blk in t[lay.group_start[g]][:4]:
            assert lay.ref_counts[blk] == 4
