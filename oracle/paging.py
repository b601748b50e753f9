"""Paged addressing: token position -> physical block and offset.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Sources:

* page "KV Cache 优化与内存管理深度解析：PagedAttention 原理与实践",
  class BlockTableDesign (table_structure, implementation): a sequence of n
  tokens occupies ceil(n / block_size) blocks; token t lives in logical block
  t // block_size at offset t % block_size, and the block table maps the
  logical block to a physical one; the last block may be partly filled;
* page "5.KV Cache 管理 & PagedAttention", Q8.3 (batched block table
  [B, max_blocks_per_seq], unused entries -1, plus each sequence's length),
  Q11 (read_kv_range: copy [start, end) of a sequence out of paged storage
  block by block into a contiguous buffer) and Q12 (append one token at
  (block_table[len // block_size], len % block_size)).

The cache layout is [num_blocks, block_size, num_kv_heads, head_dim] (the
paged_attention listing on page "paged-attention-and-vllm-inference").  A
"slot" is the flat token index physical_block * block_size + offset, i.e. the
token's row in the cache viewed as [num_blocks * block_size, ...].
"""

from __future__ import annotations

import numpy as np


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """Number of blocks a sequence of ``num_tokens`` tokens occupies."""
    return -(-int(num_tokens) // int(block_size))


def locate(block_table, pos: int, block_size: int) -> tuple[int, int]:
    """(physical block, offset inside it) of token position ``pos``."""
    logical = pos // block_size
    offset = pos % block_size
    return int(block_table[logical]), int(offset)


def slot_of(block_table, pos: int, block_size: int) -> int:
    """Flat cache row ("slot") holding token position ``pos``."""
    phys, off = locate(block_table, pos, block_size)
    return phys * block_size + off


def read_range(cache: np.ndarray, block_table, start: int, end: int) -> np.ndarray:
    """Tokens [start, end) of one sequence, copied out of paged storage.

    ``cache`` is [num_blocks, block_size, num_kv_heads, head_dim] raw storage;
    the result is [end - start, num_kv_heads, head_dim] in the same storage
    format.  Walks the positions block by block: from position ``pos`` it can
    read min(block_size - offset, end - pos) tokens out of the current
    physical block.
    """
    block_size = cache.shape[1]
    out = np.empty((end - start,) + cache.shape[2:], dtype=cache.dtype)
    pos, filled = start, 0
    while pos < end:
        phys, off = locate(block_table, pos, block_size)
        can_read = min(block_size - off, end - pos)
        out[filled:filled + can_read] = cache[phys, off:off + can_read]
        filled += can_read
        pos += can_read
    return out


def gather_sequence(cache: np.ndarray, block_table, seq_len: int) -> np.ndarray:
    """All ``seq_len`` cached tokens of one sequence, contiguous."""
    return read_range(cache, block_table, 0, int(seq_len))
