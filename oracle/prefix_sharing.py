"""Shared prefixes of forked sequences (TEST INFRASTRUCTURE: see ``oracle``).

Page "5.KV Cache 管理 & PagedAttention", Q18 (copy-on-write fork): forking a
sequence gives the child a copy of the parent's block table, so both name the
same physical blocks, whose reference counts go up; a block stops being shared
when one of them writes into it and receives a private copy.  Page
"paged-attention-and-vllm-inference" (prefix caching) reuses the blocks of a
cached prompt prefix in the same way.

What a set of sequences shares is therefore read off their block tables: the
leading table entries that name the same physical block in every member.  For
decode attention only whole blocks count as shared prefix here: a block is part
of the prefix when every member holds all block_size of its tokens (the
partially filled last block of a member, and everything after it, is that
member's own suffix).

Attention itself does not change: decode over a shared prefix is decode over
each member's full sequence (``attention.decode_attention``), which is what the
GPU results are compared against.
"""

from __future__ import annotations


def common_prefix_blocks(table_rows, seq_lens, block_size: int = 16) -> int:
    """Number of leading whole blocks that every member's table maps to the same
    physical block.  ``table_rows``: one list of block ids per member;
    ``seq_lens``: the members' lengths in tokens."""
    rows = [list(r) for r in table_rows]
    if not rows:
        return 0
    full = min(int(n) // block_size for n in seq_lens)  # blocks every member fills completely
    b = 0
    while b < full and all(r[b] == rows[0][b] for r in rows):
        b += 1
    return b
