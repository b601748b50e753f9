/*
 * Host-side KV-cache block manager of libpaged_attn.so: the free list,
 * reference counts, per-sequence block tables, copy-on-write fork and prefix
 * cache that decide where each token's K/V lives (page "5.KV Cache 管理 &
 * PagedAttention", Q9 block allocator, Q10 ensure_capacity and the multi-
 * sequence manager, Q12 append_token, Q18 copy-on-write fork, Q20 prefix
 * cache, and the LRU manager of the same page).  Pure host code: no GPU is
 * touched.  Its outputs feed the device calls of paged_attn.h: slots for
 * reshape_and_cache, block tables and lengths for paged_attention_decode,
 * copy pairs for paged_copy_blocks.
 *
 * Semantics (all deterministic):
 *   - Blocks 0..num_blocks-1 start in a free list in that order; allocation
 *     takes the last entry, a block whose count drops to 0 is appended.
 *   - Allocation with an empty free list first evicts a prefix-cache entry
 *     whose block only the cache holds (least recently used, ties: oldest
 *     entry), then fails with PA_ERR_OUT_OF_BLOCKS.
 *   - Every call that names a sequence marks it used (a logical clock), as
 *     does a prefix-cache match of an entry; pa_bm_evict_lru_sequence
 *     releases the least recently used sequence.
 *   - Thread-safe: every call takes the manager's lock.
 * Status codes are those of paged_attn.h: PA_OK, PA_ERR_INVALID_ARG (null or
 * out-of-range argument, unknown or duplicate sequence id),
 * PA_ERR_OUT_OF_BLOCKS, PA_ERR_NO_MEMORY (host allocation failed).
 * Sequence ids are any int64 values chosen by the caller.
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* A manager of num_blocks physical blocks of block_size tokens (both > 0). */
int pa_bm_create(int num_blocks, int block_size, pa_block_manager** out);
int pa_bm_destroy(pa_block_manager* bm);

/* Free-list length; reference count of one block; number of prefix-cache
 * entries.  Results in *out. */
int pa_bm_num_free(pa_block_manager* bm, int* out);
int pa_bm_ref_count(pa_block_manager* bm, int block, int* out);
int pa_bm_cached_blocks(pa_block_manager* bm, int* out);

/* A new sequence with an empty table and length 0; release every block of a
 * sequence (count lowered by one each) and forget it. */
int pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id);
int pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* Q10: the sequence holds at least ceil(required_tokens / block_size) blocks
 * (missing ones allocated at the end of its table; the length is unchanged).
 * On PA_ERR_OUT_OF_BLOCKS the blocks allocated before the failure stay. */
int pa_bm_ensure_capacity(pa_block_manager* bm, int64_t seq_id, int64_t required_tokens);

/* Q12 / Q18: append num_tokens positions to a sequence.  slots[k] (caller
 * array of num_tokens) receives block * block_size + offset of position
 * len + k.  A write into a block other references share first moves the
 * sequence to a fresh block; if the block already held tokens of the
 * sequence, (src, dst) is appended to copy_pairs (caller array of num_tokens
 * pairs, int64 [n][2]) for paged_copy_blocks, and *num_copies counts them.
 * *num_appended receives how many positions were appended: num_tokens on
 * PA_OK, fewer on PA_ERR_OUT_OF_BLOCKS (those stay appended). */
int pa_bm_append_tokens(pa_block_manager* bm, int64_t seq_id, int num_tokens, int64_t* slots,
                        int64_t* copy_pairs, int* num_copies, int* num_appended);

/* One decode step's appends for a batch: one position for each of the n
 * sequences, in order (as n calls of pa_bm_append_tokens with one token).
 * slots [n]; copy_pairs [n][2] with the count in *num_copies; *num_appended
 * = n on PA_OK, or the number of sequences served before PA_ERR_OUT_OF_BLOCKS
 * (or before an unknown id, PA_ERR_INVALID_ARG). */
int pa_bm_append_batch(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slots, int64_t* copy_pairs,
                       int* num_copies, int* num_appended);

/* Q18: child (a new id) gets a copy of the parent's table and length; every
 * block's count is raised by one. */
int pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/* The sequence's length in tokens; its table (capacity entries at most;
 * *num_blocks receives the full table length even when it does not fit). */
int pa_bm_seq_len(pa_block_manager* bm, int64_t seq_id, int64_t* len);
int pa_bm_block_table(pa_block_manager* bm, int64_t seq_id, int32_t* out, int capacity, int* num_blocks);

/* Decode-call inputs for n sequences (in the order given): block_tables
 * [n][bt_stride] int32, -1 past each table; seq_lens [n] int32.
 * PA_ERR_INVALID_ARG if a table is longer than bt_stride or a length does
 * not fit int32. */
int pa_bm_build_batch(pa_block_manager* bm, const int64_t* seq_ids, int n, int32_t* block_tables, int bt_stride,
                      int32_t* seq_lens);

/* Release the least recently used sequence, other than exclude_id when
 * has_exclude is non-zero; its id in *victim.  PA_ERR_OUT_OF_BLOCKS when no
 * sequence qualifies. */
int pa_bm_evict_lru_sequence(pa_block_manager* bm, int64_t exclude_id, int has_exclude, int64_t* victim);

/* Q20: a new sequence holding the prompt tokens[0..num_tokens).  Its leading
 * whole blocks that match prefix-cache entries are shared; the rest are
 * allocated.  The prompt's whole blocks not yet cached become entries (each
 * entry holds one reference on its block).  *matched_tokens receives the
 * shared length (a multiple of block_size); slots (caller array of
 * num_tokens) receives the slots of positions matched_tokens..num_tokens-1,
 * their count in *num_slots: the positions the caller must still write.
 * On PA_ERR_OUT_OF_BLOCKS the sequence is not created (cache entries
 * evicted on the way stay evicted). */
int pa_bm_allocate_with_prefix(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                               int* matched_tokens, int64_t* slots, int* num_slots);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H_ */
