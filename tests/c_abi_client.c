/*
 * A plain C99 client of libpaged_attn.so, built and run by
 * tests/test_c_client.py: the headers compile as C, the symbols link with C
 * linkage, and the host block manager works without Python.  Runs without a
 * GPU (the attention context is only asked to reject a bad configuration).
 *
 * The scenario follows page "5.KV Cache 管理 & PagedAttention": a sequence
 * grows (Q12), is forked and the child writes into a shared block
 * (Q18, copy-on-write), two prompts share cached blocks (Q20), and
 * sequences are released.  Every result is printed as one line
 * "<what> <values...>"; the test compares the lines with the oracle's.
 */
#include <stdio.h>
#include <string.h>

#include "block_manager.h"
#include "paged_attn.h"

static int fail(const char* what, int st) {
  printf("error %s %d\n", what, st);
  return 1;
}

static void print_append(const char* what, int st, const int64_t* slots, int na, const int64_t* pairs, int nc) {
  printf("%s %d slots", what, st);
  for (int k = 0; k < na; ++k) printf(" %lld", (long long)slots[k]);
  printf(" copies");
  for (int k = 0; k < nc; ++k) printf(" %lld:%lld", (long long)pairs[2 * k], (long long)pairs[2 * k + 1]);
  printf("\n");
}

static int append(pa_block_manager* bm, const char* what, int64_t sid, int n) {
  int64_t slots[64], pairs[128];
  int nc = 0, na = 0;
  if (n > 64) return fail(what, PA_ERR_INVALID_ARG);
  const int st = pa_bm_append_tokens(bm, sid, n, slots, pairs, &nc, &na);
  if (st != PA_OK && st != PA_ERR_OUT_OF_BLOCKS) return fail(what, st);
  print_append(what, st, slots, na, pairs, nc);
  return 0;
}

static int print_state(pa_block_manager* bm, const char* what, int num_blocks) {
  int nf = 0, cached = 0;
  if (pa_bm_num_free(bm, &nf) != PA_OK || pa_bm_cached_blocks(bm, &cached) != PA_OK) return fail(what, -1);
  printf("%s free %d cached %d refs", what, nf, cached);
  for (int b = 0; b < num_blocks; ++b) {
    int r = 0;
    if (pa_bm_ref_count(bm, b, &r) != PA_OK) return fail(what, -1);
    printf(" %d", r);
  }
  printf("\n");
  return 0;
}

int main(void) {
  enum { NB = 8, BS = 16 };
  pa_block_manager* bm = NULL;
  int st = pa_bm_create(NB, BS, &bm);
  if (st != PA_OK) return fail("create", st);

  /* a sequence of 20 tokens, then its fork writes one token of its own */
  if ((st = pa_bm_add_sequence(bm, 1)) != PA_OK) return fail("add", st);
  if (append(bm, "grow", 1, 20)) return 1;
  if ((st = pa_bm_fork(bm, 1, 2)) != PA_OK) return fail("fork", st);
  if (print_state(bm, "forked", NB)) return 1;
  if (append(bm, "child_write", 2, 1)) return 1;
  if (append(bm, "parent_write", 1, 1)) return 1;

  /* decode-call inputs for both */
  {
    const int64_t ids[2] = {1, 2};
    int32_t tables[2 * 4], lens[2];
    if ((st = pa_bm_build_batch(bm, ids, 2, tables, 4, lens)) != PA_OK) return fail("batch", st);
    printf("batch lens %d %d tables", lens[0], lens[1]);
    for (int k = 0; k < 8; ++k) printf(" %d", tables[k]);
    printf("\n");
  }

  /* one batched decode step's appends */
  {
    const int64_t ids[2] = {2, 1};
    int64_t slots[2], pairs[4];
    int nc = 0, na = 0;
    st = pa_bm_append_batch(bm, ids, 2, slots, pairs, &nc, &na);
    if (st != PA_OK && st != PA_ERR_OUT_OF_BLOCKS) return fail("append_batch", st);
    print_append("append_batch", st, slots, na, pairs, nc);
  }
  if (print_state(bm, "after_appends", NB)) return 1;

  /* release both, then two prompts sharing their first 32 tokens through the prefix cache */
  if ((st = pa_bm_free_sequence(bm, 1)) != PA_OK) return fail("free", st);
  if ((st = pa_bm_free_sequence(bm, 2)) != PA_OK) return fail("free", st);
  {
    int32_t a[40], b[36];
    int64_t slots[40];
    int matched = 0, ns = 0;
    for (int k = 0; k < 40; ++k) a[k] = 100 + k;
    for (int k = 0; k < 36; ++k) b[k] = k < 32 ? 100 + k : 900 + k;
    if ((st = pa_bm_allocate_with_prefix(bm, 3, a, 40, &matched, slots, &ns)) != PA_OK) return fail("prefix", st);
    printf("prefix_a matched %d slots", matched);
    for (int k = 0; k < ns; ++k) printf(" %lld", (long long)slots[k]);
    printf("\n");
    if ((st = pa_bm_allocate_with_prefix(bm, 4, b, 36, &matched, slots, &ns)) != PA_OK) return fail("prefix", st);
    printf("prefix_b matched %d slots", matched);
    for (int k = 0; k < ns; ++k) printf(" %lld", (long long)slots[k]);
    printf("\n");
  }
  if (print_state(bm, "prefixed", NB)) return 1;
  {
    int64_t victim = -1;
    if ((st = pa_bm_evict_lru_sequence(bm, 4, 1, &victim)) != PA_OK) return fail("evict", st);
    printf("evicted %lld\n", (long long)victim);
  }
  if (print_state(bm, "final", NB)) return 1;
  /* an unknown sequence is refused */
  printf("unknown %d\n", pa_bm_free_sequence(bm, 77));
  if ((st = pa_bm_destroy(bm)) != PA_OK) return fail("destroy", st);

  /* the attention context rejects a configuration whose head counts do not divide */
  {
    pa_config cfg;
    pa_ctx* ctx = NULL;
    memset(&cfg, 0, sizeof cfg);
    cfg.num_heads = 32;
    cfg.num_kv_heads = 5;
    cfg.head_dim = 128;
    cfg.block_size = 16;
    cfg.num_blocks = 64;
    cfg.q_dtype = PA_F16;
    cfg.kv_dtype = PA_F16;
    cfg.max_num_seqs = 4;
    cfg.max_blocks_per_seq = 8;
    cfg.partition_tokens = PA_PARTITION_AUTO;
    st = paged_attn_create(&cfg, &ctx);
    printf("create %d %s %d\n", st, paged_attn_status_string(st), ctx == NULL);
  }
  return 0;
}
