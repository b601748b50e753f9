/*
 * paged_attn.h -- C ABI of a B200 (sm_100a) library for the decode hot path of
 * PagedAttention: the per-step paged cache write and decode attention over a
 * block-paged KV cache.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers named *_cache, key, value, query, out, block_table(s), seq_lens,
 *   slot_mapping, k_out, v_out are DEVICE pointers into memory the caller owns
 *   (e.g. torch tensors); the library never frees or keeps them after a call
 *   returns.  `stream` is a cudaStream_t (NULL = legacy default stream).
 * - Calls validate their arguments on the host first; an invalid call returns
 *   a negative status and launches nothing.  Valid calls only enqueue work on
 *   `stream` and return PA_OK without synchronising.
 * - Data-dependent problems (a block id outside the pool, a slot outside the
 *   cache, a sequence longer than its table, a pipeline wait that ran out) are
 *   caught on the device: the offending access is skipped (or redirected to
 *   block 0), a bit is or-ed into the context's check word, and
 *   paged_attn_get_error() reports it.  Nothing traps, asserts or spins
 *   without bound.
 * - Layouts (row-major, element = the dtype named):
 *     query, out           [num_seqs, num_heads, head_dim]
 *     key_cache/value_cache [num_blocks, block_size, num_kv_heads, head_dim]
 *     block_tables         int32 [num_seqs, bt_stride]; entry j of row s is the
 *                          physical block holding tokens [16 j, 16 j + 16) of s;
 *                          entries past the sequence's last block are never read
 *                          (page "5.KV Cache 管理 & PagedAttention", Q8.3 uses -1)
 *     seq_lens             int32 [num_seqs], tokens cached for each sequence
 *                          (including the one written by this step)
 *     slot_mapping         int64 [num_tokens], slot = block * block_size + offset
 *   A context is used from one host thread at a time.
 */
#ifndef PAGED_ATTN_H_
#define PAGED_ATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes */
#define PA_OK 0
#define PA_ERR_INVALID_ARG (-1)  /* null pointer, bad shape/stride/alignment, size beyond the context's limits */
#define PA_ERR_UNSUPPORTED (-2)  /* dtype / head_dim / block_size combination not built */
#define PA_ERR_CUDA (-3)         /* a CUDA runtime call failed; paged_attn_last_error() has the message */
#define PA_ERR_DEVICE_CHECK (-4) /* a device-side check fired; paged_attn_last_check_bits() says which */
#define PA_ERR_NO_MEMORY (-5)    /* workspace allocation failed */
#define PA_ERR_SCRATCH_TOO_SMALL (-6) /* paged_attention_decode_noalloc: partials exceed PA_NOALLOC_SCRATCH_BYTES */
#define PA_ERR_OUT_OF_BLOCKS (-7)     /* block manager: no free block and nothing evictable (block_manager.h) */

/* ---- device check bits (paged_attn_last_check_bits) */
#define PA_CHECK_BAD_BLOCK 1    /* block-table entry outside [0, num_blocks): read block 0 instead */
#define PA_CHECK_BAD_SLOT 2     /* slot >= num_blocks * block_size: write skipped */
#define PA_CHECK_SEQ_TOO_LONG 4 /* seq_len > bt_stride * block_size, < 0, or beyond max_seq_len: clamped */
#define PA_CHECK_WAIT_TIMEOUT 8 /* a shared-memory pipeline wait gave up: that CTA's output is invalid */
#define PA_CHECK_BAD_PREFIX 16  /* shared-prefix decode: a group's description was unusable (see
                                   paged_attention_decode_shared_prefix) */

/* ---- element types */
typedef enum pa_dtype { PA_F16 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* partition_tokens special values */
#define PA_PARTITION_NONE 0  /* never split a sequence across CTAs */
#define PA_PARTITION_AUTO (-1)

/*
 * Fixed shape of one attention layer's cache and of the batches it serves.
 *   num_heads, num_kv_heads : query heads and KV heads; num_heads % num_kv_heads == 0.
 *                             Query head h reads KV head h / (num_heads / num_kv_heads)
 *                             (grouped-query attention, page "5.KV Cache 管理 &
 *                             PagedAttention", Q7 repeat_interleave; MHA when equal).
 *   head_dim                : 64, 128 or 256 for 16-bit caches; 128 or 256 for fp8.
 *   block_size              : tokens per physical block; 16 (the pages' default,
 *                             page "KV Cache 优化与内存管理深度解析", BlockSizeSelection).
 *   num_blocks              : physical blocks in each of key_cache / value_cache.
 *   q_dtype                 : PA_F16 or PA_BF16 (query, out and the new K/V rows).
 *   kv_dtype                : PA_F16 / PA_BF16 (must equal q_dtype) or PA_FP8_E4M3
 *                             (with q_dtype PA_F16); fp8 values carry one scale per
 *                             cache tensor (value = code * scale).
 *   max_num_seqs            : largest num_seqs a decode call may pass.
 *   max_blocks_per_seq      : largest ceil(max_seq_len / block_size) a call may pass.
 *   partition_tokens        : split-KV partition length (a multiple of block_size),
 *                             PA_PARTITION_NONE, or PA_PARTITION_AUTO: the decode
 *                             kernel picks, from the actual lengths, a power-of-two
 *                             multiple of 512 tokens (or no split) that keeps every
 *                             work item a modest fraction of one CTA's share.
 *   device                  : CUDA device ordinal the context and its calls use.
 *   flags                   : 0, or PA_FLAG_SHARED_PREFIX: also allocate the
 *                             shared-prefix workspace (max_num_seqs * num_heads *
 *                             ceil(max_blocks_per_seq / 32) * (head_dim + 2) floats,
 *                             plus max_num_seqs ints) that
 *                             paged_attention_decode_shared_prefix needs.
 */
#define PA_FLAG_SHARED_PREFIX 1
typedef struct pa_config {
  int num_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int num_blocks;
  int q_dtype;
  int kv_dtype;
  int max_num_seqs;
  int max_blocks_per_seq;
  int partition_tokens;
  int device;
  int flags;
} pa_config;

typedef struct pa_ctx pa_ctx;

/*
 * Create a context: validates `cfg`, allocates the split-KV workspace
 * (max_num_seqs * num_heads * max_partitions * (head_dim + 2) floats) and the
 * device check word on cfg->device.  On success *out owns them.
 * Returns PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_NO_MEMORY or
 * PA_ERR_CUDA (e.g. no GPU).  *out is NULL on failure.
 */
int paged_attn_create(const pa_config* cfg, pa_ctx** out);

/* Free the context's workspace.  Does not synchronise the caller's streams:
 * the caller must make sure no call on the context is still running. */
int paged_attn_destroy(pa_ctx* ctx);

/*
 * Paged cache write (page "5.KV Cache 管理 & PagedAttention", Q12 append_token:
 * the new token's K/V go to (block_table[len / block_size], len % block_size)).
 * For every token t in [0, num_tokens) with slot = slot_mapping[t] >= 0:
 *     key_cache[slot / block_size, slot % block_size, :, :] = key[t, :, :]
 *     value_cache[...]                                     = value[t, :, :]
 * key/value: [num_tokens, num_kv_heads, head_dim] of q_dtype, with row strides
 * key_token_stride / value_token_stride in elements (multiples of 8; pointers
 * 16-byte aligned).  16-bit caches receive the bytes unchanged.  An fp8 cache
 * receives E4M3(x / k_scale) (values: v_scale): IEEE fp32 division, round to
 * nearest even, saturating at +-448.  Slots < 0 are skipped; slots beyond the
 * cache set PA_CHECK_BAD_SLOT and are skipped.  Two tokens with the same slot
 * in one call: which one lands is unspecified.
 */
int reshape_and_cache(pa_ctx* ctx, const void* key, const void* value, int64_t key_token_stride,
                      int64_t value_token_stride, void* key_cache, void* value_cache,
                      const int64_t* slot_mapping, int num_tokens, float k_scale, float v_scale,
                      void* stream);

/*
 * Decode attention over the paged cache (page "5.KV Cache 管理 & PagedAttention",
 * Q4 decode_step step 4 and Q13; listing paged_attention on page
 * "paged-attention-and-vllm-inference"): for each sequence s < num_seqs and
 * query head h,
 *     out[s, h, :] = sum_j softmax_j(scale * q[s,h,:] . K[s,j,:]) V[s,j,:]
 * over the seq_lens[s] tokens j of s, K[s,j] = key_cache[block_tables[s, j/16],
 * j%16, h / (num_heads/num_kv_heads)].  fp8 caches are decoded as code*k_scale
 * and code*v_scale (k_scale, v_scale ignored for 16-bit caches).  Arithmetic is
 * fp32 (products of 16-bit operands on tensor cores); out is rounded once to
 * q_dtype.  seq_lens[s] == 0 gives a zero row.
 * max_seq_len: a host-side upper bound of seq_lens (sizes the partition grid
 * without a device->host read); 0 <= max_seq_len <= max_blocks_per_seq *
 * block_size.  Sequences longer than it, or than bt_stride * block_size, are
 * truncated and flagged (PA_CHECK_SEQ_TOO_LONG).
 * bt_stride: row stride of block_tables in entries (>= 1).
 * Pointers: out/query 16-byte aligned, caches 16-byte aligned.
 * Launches the decode kernel and then, as a programmatic dependent launch
 * on the same stream, the merge kernel whenever the call may split a
 * sequence: always with PA_PARTITION_AUTO (the split is chosen on the device,
 * and the merge kernel's CTAs for unsplit sequences exit at once), and with a
 * fixed partition shorter than max_seq_len.  PA_PARTITION_NONE, or a fixed
 * partition of at least max_seq_len tokens, launches the decode kernel alone.
 */
int paged_attention_decode(pa_ctx* ctx, void* out, const void* query, const void* key_cache,
                           const void* value_cache, const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int num_seqs, int max_seq_len, float scale, float k_scale,
                           float v_scale, void* stream);

/*
 * Decode attention for batches in which groups of sequences share the physical
 * blocks of a common prefix: sequences forked from one prompt (page "5.KV Cache
 * 管理 & PagedAttention", Q18: the fork copies the parent's block table and
 * raises the shared blocks' reference counts), or requests that reuse cached
 * prefix blocks (page "paged-attention-and-vllm-inference", prefix caching).
 * The result is the same as paged_attention_decode's on the same arguments
 * (rounding aside); only the order of work differs.  Each shared block is read
 * once per group and scored against the queries of all its members (one pass
 * over the prefixes); each sequence's private suffix is then decoded as usual,
 * and the two sets of partial results are combined by log-sum-exp.
 *
 * Groups (device int32 arrays):
 *   group_start[num_groups + 1]  : group g is sequences [group_start[g],
 *                                  group_start[g + 1]); non-decreasing, within
 *                                  [0, num_seqs].  Sequences before
 *                                  group_start[0] or from group_start[num_groups]
 *                                  on share nothing.
 *   group_prefix_len[num_groups] : tokens that group g's members share: a
 *                                  multiple of block_size (whole blocks), at most
 *                                  every member's seq_lens, at most
 *                                  max_prefix_len, and the members' block tables
 *                                  name the same physical blocks for it.  0: no
 *                                  shared prefix.
 * Host bounds: 1 <= num_groups <= num_seqs; 1 <= max_group_size <= num_seqs
 * (largest group); 0 <= max_prefix_len <= max_seq_len (largest prefix).
 * A group that breaks one of these rules (too many members, a prefix length
 * that is not a block multiple, longer than a member or than max_prefix_len,
 * or tables that differ over the prefix) sets PA_CHECK_BAD_PREFIX and its
 * members are decoded in full, without sharing (the output stays correct).  A
 * group_start that is decreasing or leaves [0, num_seqs] sets the same bit and
 * the affected sequences' outputs are unspecified.
 * The context must have been created with PA_FLAG_SHARED_PREFIX
 * (PA_ERR_UNSUPPORTED otherwise).  Launches the prefix pass, the decode pass
 * over the suffixes and the merge kernel, in stream order.
 */
int paged_attention_decode_shared_prefix(pa_ctx* ctx, void* out, const void* query, const void* key_cache,
                                         const void* value_cache, const int32_t* block_tables, int bt_stride,
                                         const int32_t* seq_lens, int num_seqs, int max_seq_len,
                                         const int32_t* group_start, const int32_t* group_prefix_len,
                                         int num_groups, int max_group_size, int max_prefix_len, float scale,
                                         float k_scale, float v_scale, void* stream);

/*
 * Multi-query paged attention: prefill and chunked prefill (page "5.KV Cache
 * 管理 & PagedAttention", Q6 MHAWithCache prefill branch: each query position
 * attends causally to the keys at its own and earlier positions; Q3.3 / Q19:
 * blockwise over the paged cache through the block table, with an online
 * softmax).  The chunk's K/V must already be in the cache (reshape_and_cache).
 * Sequence s holds seq_lens[s] cached tokens; its query rows are
 * query[query_start[s] .. query_start[s+1]) ([num_tokens, num_heads,
 * head_dim], q_dtype), the sequence's last q_len = query_start[s+1] -
 * query_start[s] positions, so row i is position p = seq_lens[s] - q_len + i:
 *     out[row, h, :] = sum_{j <= p} softmax_j(scale * q[row,h,:] . K[s,j,:]) V[s,j,:]
 * (q_len = seq_lens[s]: a whole prompt; 1: a decode step).  out has the
 * query's shape and dtype.  query_start: device int32 [num_seqs + 1],
 * non-decreasing, query_start[num_seqs] = num_tokens.  Host bounds:
 * max_query_len >= every q_len, max_seq_len >= every seq_len (both <=
 * max_blocks_per_seq * block_size).  A sequence with q_len > seq_len, or
 * longer than max_seq_len / bt_stride * block_size, or whose query rows fall
 * outside [0, num_tokens), sets PA_CHECK_SEQ_TOO_LONG (the rows of a
 * sequence with q_len > seq_len or rows outside the array are not written).
 * Arithmetic: 16-bit products accumulated in fp32 on the tensor cores (fp8
 * caches decoded to f16 first); one rounding of the output.
 * Returns PA_OK, PA_ERR_INVALID_ARG, PA_ERR_CUDA.
 */
int paged_attention_prefill(pa_ctx* ctx, void* out, const void* query, const void* key_cache, const void* value_cache,
                            const int32_t* block_tables, int bt_stride, const int32_t* seq_lens,
                            const int32_t* query_start, int num_seqs, int num_tokens, int max_query_len,
                            int max_seq_len, float scale, float k_scale, float v_scale, void* stream);

/*
 * Synchronise `stream`, read and clear the context's device check word.
 * Returns PA_OK when no check fired since the last call, PA_ERR_DEVICE_CHECK
 * otherwise (the bits are then in paged_attn_last_check_bits), PA_ERR_CUDA if
 * the synchronisation failed.
 */
int paged_attn_get_error(pa_ctx* ctx, void* stream);

/*
 * Failure-path test hook (the pages describe no counterpart; it exists so
 * that the device-side timeout exit can be exercised without any GPU fault).
 * The next paged_attention_decode or paged_attention_decode_shared_prefix on
 * this context runs its decode kernel with every pipeline wait bounded by
 * wait_limit_cycles SM clock cycles instead of the default (~2 s), and with
 * the first wait of each consumer warp aimed at a barrier that nothing ever
 * completes.  Every CTA of that launch therefore gives up after about
 * wait_limit_cycles, waits (with the default bound) for the copies it has in
 * flight, and exits; the call's output is invalid and paged_attn_get_error()
 * reports PA_CHECK_WAIT_TIMEOUT.  Later calls run normally.  One-shot.
 * wait_limit_cycles: [1000, the default limit].  Returns PA_OK or
 * PA_ERR_INVALID_ARG.
 */
int paged_attn_test_wait_timeout(pa_ctx* ctx, long long wait_limit_cycles);

/* Check bits seen by the last paged_attn_get_error (PA_CHECK_*). */
int paged_attn_last_check_bits(const pa_ctx* ctx);

/* Static description of a status code. */
const char* paged_attn_status_string(int status);

/* Message of the last PA_ERR_CUDA / validation failure on this context ("" if none). */
const char* paged_attn_last_error(const pa_ctx* ctx);

/*
 * Override the split-KV partition length for later decode calls:
 * PA_PARTITION_NONE, PA_PARTITION_AUTO, or a multiple of block_size no smaller
 * than the context's workspace allows (cfg.partition_tokens if positive, else 512).
 */
int paged_attn_set_partition_tokens(pa_ctx* ctx, int partition_tokens);

/* Read the context's partition setting for decode calls into
 * *partition_tokens: a length in tokens, PA_PARTITION_NONE (0), or
 * PA_PARTITION_AUTO (-1, chosen on the device per call from the lengths).
 * Returns PA_OK, or PA_ERR_INVALID_ARG for a null pointer. */
int paged_attn_get_partition_tokens(const pa_ctx* ctx, int* partition_tokens);

/*
 * Gather (page "5.KV Cache 管理 & PagedAttention", Q11 read_kv_range): copy
 * tokens [0, seq_len) of one sequence out of the paged caches into contiguous
 * k_out / v_out [seq_len, num_kv_heads, head_dim] (cache dtype, bytes
 * unchanged).  block_table_row: device int32 [>= ceil(seq_len / block_size)].
 * Entries outside the pool set PA_CHECK_BAD_BLOCK and yield zero rows.
 */
int paged_gather_kv(pa_ctx* ctx, void* k_out, void* v_out, const void* key_cache, const void* value_cache,
                    const int32_t* block_table_row, int seq_len, void* stream);

/*
 * Whole-block copies between paged caches, for copy-on-write and swap.
 * Copy-on-write (page "5.KV Cache 管理 & PagedAttention", Q18
 * COWBlockManager.write_token): before a sequence writes into a block other
 * sequences still share, the block is copied to a fresh one.  Swap (page "KV
 * Cache 优化与内存管理深度解析", CPUSwap): blocks move from GPU to CPU memory
 * and back into newly allocated GPU blocks.
 * For each pair i: dst_cache[pairs[i][1]] = src_cache[pairs[i][0]] for both K
 * and V (every token slot and KV head of the block; bytes unchanged).
 * Caches: [*_num_blocks, block_size, num_kv_heads, head_dim] of the context's
 * kv dtype, in any memory the device can address: device memory, or host
 * memory allocated pinned (cudaMallocHost / cudaHostAlloc), which the kernel
 * reads or writes directly over the host link.  block_pairs: int64
 * [num_pairs][2] (src, dst), device or pinned host memory.  A pair naming a
 * block outside its cache sets PA_CHECK_BAD_BLOCK and is skipped.  Pairs whose
 * blocks overlap (a block written by one pair and read or written by another)
 * give an unspecified result.  Pointers 16-byte aligned (pairs 8-byte).
 */
int paged_copy_blocks(pa_ctx* ctx, void* dst_key_cache, void* dst_value_cache, int64_t dst_num_blocks,
                      const void* src_key_cache, const void* src_value_cache, int64_t src_num_blocks,
                      const int64_t* block_pairs, int num_pairs, void* stream);

/*
 * Decode attention that allocates nothing (the pages describe no counterpart:
 * it exists for callers of this library that cannot allocate device memory,
 * e.g. hosts that hand out every byte of device memory from their own pool or
 * arena and forbid outside allocations, or serving loops that must not risk
 * an allocation failure, or the allocator's implicit device synchronisation,
 * in the middle of a step).
 *
 * Same computation, layouts and argument meanings as paged_attention_decode,
 * but without a context: the cache shape is passed directly (num_heads,
 * num_kv_heads, head_dim, block_size == 16, num_blocks, q_dtype, kv_dtype), and
 * the split-KV partials live in one fixed device array built into the library,
 * PA_NOALLOC_SCRATCH_BYTES (16 MiB) per GPU, held from the library's first use
 * on that GPU until the process exits.  The caller passes inputs and outputs.
 *
 * partition_tokens: 0 = one partition per sequence (needs no partials), else a
 * multiple of 16.  A call whose partials (num_seqs * num_heads * partitions *
 * (head_dim + 2) floats, with no split none), plus num_seqs ints rounded up
 * to 256 bytes and a 256-byte header, do not fit the array is refused with
 * PA_ERR_SCRATCH_TOO_SMALL before anything is launched.
 * check_bits: optional device int that receives PA_CHECK_* bits (or-ed in;
 * the caller clears it); NULL sends them to a word inside the array.
 * Runs on the calling thread's current CUDA device.  The first call on each
 * device does a one-time set-up there: it looks up the array's device
 * address, raises the shared-memory limit of every decode kernel the library
 * holds (all head_dim / dtype combinations), and clears the array's 256-byte
 * header (check word and work counters) with an asynchronous memset on
 * `stream`, ordered before that call's kernels on any kind of stream.  A
 * caller that captures streams into CUDA graphs should make this first call
 * before any capture.  Later calls change no host or device setting.
 * Every call on a device shares the array and finds it as the previous call
 * left it; calls whose kernels may overlap on the GPU (other streams or host
 * threads on the same device) race on it and must be serialised by the caller.
 * Never calls cudaMalloc, cudaFree or any allocating routine.
 * Returns PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED,
 * PA_ERR_SCRATCH_TOO_SMALL or PA_ERR_CUDA.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int paged_attention_decode_noalloc(void* out, const void* query, const void* key_cache, const void* value_cache,
                                   const int32_t* block_tables, int bt_stride, const int32_t* seq_lens, int num_seqs,
                                   int max_seq_len, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                   int num_blocks, int q_dtype, int kv_dtype, int partition_tokens, float scale,
                                   float k_scale, float v_scale, int* check_bits, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_H_ */
