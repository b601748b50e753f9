"""CPU oracle for paged decode attention and the paged cache write.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg
may import or run anything in this package.  The product path (the C-ABI
library under ``paged_kv_cache_463_b200/``) never imports it, and this package
never imports the product: the two share no kernels, headers, helpers, tables
or constants.  Only the seeded input generator
(``paged_kv_cache_463_b200/workloads.py``, which holds none of the method's
arithmetic) feeds both.

Everything here is plain, slow and written to be checked by eye against the
pages it cites:

* ``paging``      -- logical token position -> (physical block, offset) and
                     the contiguous re-assembly of a sequence's K/V
                     (page "5.KV Cache 管理 & PagedAttention", Q8, Q11, Q12;
                     page "KV Cache 优化与内存管理深度解析", BlockTableDesign).
* ``attention``   -- decode attention softmax(scale * q K^T) V in fp64, computed
                     directly over the re-assembled K/V in two explicit passes
                     (max, then exp/sum).  It does NOT use the online-softmax
                     recurrence that the GPU path uses.  ``prefill_attention``:
                     the same for several causal query rows per sequence
                     (prefill, chunked prefill).
* ``cache_write`` -- the per-token slot write (reshape_and_cache).
* ``block_copy``  -- whole-block copies (copy-on-write fork, CPU swap).
* ``prefix_sharing`` -- the whole blocks a group of forked sequences shares.
* ``block_manager`` -- the host allocator: free list, reference counts,
                     append / fork with copy-on-write, prefix cache, LRU release
                     (page "5.KV Cache 管理 & PagedAttention", Q9, Q10, Q12, Q18,
                     Q20).
* ``fp8_e4m3``    -- an OCP FP8 E4M3 codec written from the format definition.
* ``dtypes``      -- raw 16-bit / 8-bit storage -> fp64 values.
* ``kv_size``     -- the pages' closed-form KV-cache size.

Precision: all attention arithmetic is fp64 on the exactly decoded stored
values.  Pins (tests/test_oracle*.py) tie every function to something other
than itself: the pages' worked values, closed forms, invariants, and library
routines (torch SDPA, torch's fp8/bf16 casts) on special cases.
"""

from . import attention, block_copy, cache_write, dtypes, fp8_e4m3, kv_size, paging, prefix_sharing  # noqa: F401
