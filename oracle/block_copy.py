"""Block-granular copies between paged caches: copy-on-write and swap.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

* Copy-on-write fork (page "5.KV Cache 管理 & PagedAttention", Q18
  COWBlockManager.write_token): before a sequence writes into a physical block
  that other sequences still reference, the block is copied to a newly
  allocated one (copy_block(phy_idx, new_blk)) and the writer's table points to
  the copy.
* CPU swap (page "KV Cache 优化与内存管理深度解析", CPUSwap.implementation):
  swap_out moves a sequence's GPU blocks to CPU memory, swap_in allocates GPU
  blocks again and loads the data back.

Both are the same operation on whole blocks (every token slot, every KV head,
K and V): dst_cache[dst_block] = src_cache[src_block] for each (src, dst)
pair, in order.  A pair with a block outside either cache is skipped.
"""

from __future__ import annotations

import numpy as np


def copy_blocks(src_key, src_value, dst_key, dst_value, pairs) -> None:
    """In place on the dst arrays ([num_blocks, block_size, Hkv, D] raw storage)."""
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        if not (0 <= src < src_key.shape[0] and 0 <= dst < dst_key.shape[0]):
            continue
        dst_key[dst] = src_key[src]
        dst_value[dst] = src_value[src]
