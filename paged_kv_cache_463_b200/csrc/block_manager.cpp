// Host block manager declared in include/block_manager.h: free list,
// reference counts, sequence tables, copy-on-write fork, prefix cache and LRU
// release (page "5.KV Cache 管理 & PagedAttention", Q9, Q10, Q12, Q18, Q20 and
// its LRU manager).  Host code only.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "block_manager.h"
#include "paged_attn.h"

#define PA_API extern "C" __attribute__((visibility("default")))

// An NVTX range around each block-manager call that changes its state or
// exports tables (no-ops unless a profiling tool is attached).
struct BmTraceRange {
  explicit BmTraceRange(const char* name) { nvtxRangePushA(name); }
  ~BmTraceRange() { nvtxRangePop(); }
  BmTraceRange(const BmTraceRange&) = delete;
  BmTraceRange& operator=(const BmTraceRange&) = delete;
};
#define BM_TRACE(name) const BmTraceRange bm_trace_range_(name)

namespace {

// Prefix-cache key: (entry of the previous block of the prompt, the block's tokens).
struct Key {
  int64_t parent;
  std::vector<int32_t> tokens;
  bool operator==(const Key& o) const { return parent == o.parent && tokens == o.tokens; }
};
struct KeyHash {
  size_t operator()(const Key& k) const {
    uint64_t h = 1469598103934665603ull ^ (uint64_t)k.parent;  // FNV-1a over the parent and tokens
    for (int32_t t : k.tokens) {
      h ^= (uint32_t)t;
      h *= 1099511628211ull;
    }
    return (size_t)h;
  }
};

struct Seq {
  std::vector<int32_t> table;
  int64_t len = 0;
  uint64_t last_use = 0;
};

struct Entry {
  int32_t block;
  uint64_t last_use;
  Key key;
};

struct OutOfBlocks {};

}  // namespace

struct pa_block_manager {
  std::mutex mu;
  int num_blocks = 0, block_size = 0;
  std::vector<int32_t> free_list;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  uint64_t clock = 0;
  std::unordered_map<int64_t, Entry> entries;  // entry id -> entry
  std::unordered_map<Key, int64_t, KeyHash> index;
  int64_t next_entry = 1;  // 0 = no parent

  uint64_t tick() { return ++clock; }

  bool evict_one_cached() {
    int64_t best = -1;
    uint64_t best_use = 0;
    for (const auto& kv : entries) {
      if (ref[kv.second.block] != 1) continue;
      if (best < 0 || kv.second.last_use < best_use || (kv.second.last_use == best_use && kv.first < best)) {
        best = kv.first;
        best_use = kv.second.last_use;
      }
    }
    if (best < 0) return false;
    auto it = entries.find(best);
    const int32_t blk = it->second.block;
    index.erase(it->second.key);
    entries.erase(it);
    decref(blk);
    return true;
  }
  int32_t allocate() {
    if (free_list.empty() && !evict_one_cached()) throw OutOfBlocks{};
    const int32_t b = free_list.back();
    free_list.pop_back();
    ref[b] = 1;
    return b;
  }
  void incref(int32_t b) { ++ref[b]; }
  void decref(int32_t b) {
    if (--ref[b] == 0) free_list.push_back(b);
  }
  // a known sequence, marked used; nullptr if unknown
  Seq* use(int64_t id) {
    auto it = seqs.find(id);
    if (it == seqs.end()) return nullptr;
    it->second.last_use = tick();
    return &it->second;
  }
};

#define BM_GUARD(bm)                      \
  if (!(bm)) return PA_ERR_INVALID_ARG;   \
  std::lock_guard<std::mutex> lock_((bm)->mu)

PA_API int pa_bm_create(int num_blocks, int block_size, pa_block_manager** out) {
  BM_TRACE("pa_bm_create");
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (!bm) return PA_ERR_NO_MEMORY;
  try {
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->free_list.resize(num_blocks);
    for (int i = 0; i < num_blocks; ++i) bm->free_list[i] = i;
    bm->ref.assign(num_blocks, 0);
  } catch (const std::bad_alloc&) {
    delete bm;
    return PA_ERR_NO_MEMORY;
  }
  *out = bm;
  return PA_OK;
}

PA_API int pa_bm_destroy(pa_block_manager* bm) {
  BM_TRACE("pa_bm_destroy");
  if (!bm) return PA_ERR_INVALID_ARG;
  delete bm;
  return PA_OK;
}

PA_API int pa_bm_num_free(pa_block_manager* bm, int* out) {
  BM_GUARD(bm);
  if (!out) return PA_ERR_INVALID_ARG;
  *out = (int)bm->free_list.size();
  return PA_OK;
}

PA_API int pa_bm_ref_count(pa_block_manager* bm, int block, int* out) {
  BM_GUARD(bm);
  if (!out || block < 0 || block >= bm->num_blocks) return PA_ERR_INVALID_ARG;
  *out = bm->ref[block];
  return PA_OK;
}

PA_API int pa_bm_cached_blocks(pa_block_manager* bm, int* out) {
  BM_GUARD(bm);
  if (!out) return PA_ERR_INVALID_ARG;
  *out = (int)bm->entries.size();
  return PA_OK;
}

PA_API int pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id) {
  BM_TRACE("pa_bm_add_sequence");
  BM_GUARD(bm);
  if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  try {
    Seq& s = bm->seqs[seq_id];
    s.last_use = bm->tick();
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}

PA_API int pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
  BM_TRACE("pa_bm_free_sequence");
  BM_GUARD(bm);
  Seq* s = bm->use(seq_id);
  if (!s) return PA_ERR_INVALID_ARG;
  for (int32_t b : s->table) bm->decref(b);
  bm->seqs.erase(seq_id);
  return PA_OK;
}

PA_API int pa_bm_ensure_capacity(pa_block_manager* bm, int64_t seq_id, int64_t required_tokens) {
  BM_TRACE("pa_bm_ensure_capacity");
  BM_GUARD(bm);
  if (required_tokens < 0) return PA_ERR_INVALID_ARG;
  Seq* s = bm->use(seq_id);
  if (!s) return PA_ERR_INVALID_ARG;
  const int64_t needed = (required_tokens + bm->block_size - 1) / bm->block_size;
  try {
    while ((int64_t)s->table.size() < needed) s->table.push_back(bm->allocate());
  } catch (const OutOfBlocks&) {
    return PA_ERR_OUT_OF_BLOCKS;
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}

PA_API int pa_bm_append_tokens(pa_block_manager* bm, int64_t seq_id, int num_tokens, int64_t* slots,
                               int64_t* copy_pairs, int* num_copies, int* num_appended) {
  BM_TRACE("pa_bm_append_tokens");
  BM_GUARD(bm);
  if (num_tokens < 0 || (num_tokens > 0 && (!slots || !copy_pairs)) || !num_copies || !num_appended)
    return PA_ERR_INVALID_ARG;
  *num_copies = 0;
  *num_appended = 0;
  Seq* s = bm->use(seq_id);
  if (!s) return PA_ERR_INVALID_ARG;
  const int bs = bm->block_size;
  try {
    for (int k = 0; k < num_tokens; ++k) {
      const int64_t pos = s->len;
      const int64_t lb = pos / bs, off = pos % bs;
      if (lb == (int64_t)s->table.size()) {
        s->table.push_back(bm->allocate());
      } else if (bm->ref[s->table[lb]] > 1) {
        const int32_t old = s->table[lb];
        const int32_t fresh = bm->allocate();
        if (off > 0) {
          copy_pairs[2 * *num_copies] = old;
          copy_pairs[2 * *num_copies + 1] = fresh;
          ++*num_copies;
        }
        bm->decref(old);
        s->table[lb] = fresh;
      }
      slots[k] = (int64_t)s->table[lb] * bs + off;
      s->len = pos + 1;
      *num_appended = k + 1;
    }
  } catch (const OutOfBlocks&) {
    return PA_ERR_OUT_OF_BLOCKS;
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}

PA_API int pa_bm_append_batch(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slots, int64_t* copy_pairs,
                              int* num_copies, int* num_appended) {
  BM_TRACE("pa_bm_append_batch");
  BM_GUARD(bm);
  if (n < 0 || (n > 0 && (!seq_ids || !slots || !copy_pairs)) || !num_copies || !num_appended)
    return PA_ERR_INVALID_ARG;
  *num_copies = 0;
  *num_appended = 0;
  const int bs = bm->block_size;
  try {
    for (int k = 0; k < n; ++k) {
      Seq* s = bm->use(seq_ids[k]);
      if (!s) return PA_ERR_INVALID_ARG;
      const int64_t pos = s->len;
      const int64_t lb = pos / bs, off = pos % bs;
      if (lb == (int64_t)s->table.size()) {
        s->table.push_back(bm->allocate());
      } else if (bm->ref[s->table[lb]] > 1) {
        const int32_t old = s->table[lb];
        const int32_t fresh = bm->allocate();
        if (off > 0) {
          copy_pairs[2 * *num_copies] = old;
          copy_pairs[2 * *num_copies + 1] = fresh;
          ++*num_copies;
        }
        bm->decref(old);
        s->table[lb] = fresh;
      }
      slots[k] = (int64_t)s->table[lb] * bs + off;
      s->len = pos + 1;
      *num_appended = k + 1;
    }
  } catch (const OutOfBlocks&) {
    return PA_ERR_OUT_OF_BLOCKS;
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}

PA_API int pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
  BM_TRACE("pa_bm_fork");
  BM_GUARD(bm);
  Seq* p = bm->use(parent_id);
  if (!p || bm->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
  try {
    Seq c;
    c.table = p->table;
    c.len = p->len;
    c.last_use = bm->tick();
    for (int32_t b : c.table) bm->incref(b);
    bm->seqs.emplace(child_id, std::move(c));
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}

PA_API int pa_bm_seq_len(pa_block_manager* bm, int64_t seq_id, int64_t* len) {
  BM_GUARD(bm);
  if (!len) return PA_ERR_INVALID_ARG;
  Seq* s = bm->use(seq_id);
  if (!s) return PA_ERR_INVALID_ARG;
  *len = s->len;
  return PA_OK;
}

PA_API int pa_bm_block_table(pa_block_manager* bm, int64_t seq_id, int32_t* out, int capacity, int* num_blocks) {
  BM_GUARD(bm);
  if (!num_blocks || capacity < 0 || (capacity > 0 && !out)) return PA_ERR_INVALID_ARG;
  Seq* s = bm->use(seq_id);
  if (!s) return PA_ERR_INVALID_ARG;
  const int n = (int)s->table.size();
  *num_blocks = n;
  if (capacity > 0 && n > 0) std::memcpy(out, s->table.data(), sizeof(int32_t) * (size_t)(n < capacity ? n : capacity));
  return PA_OK;
}

PA_API int pa_bm_build_batch(pa_block_manager* bm, const int64_t* seq_ids, int n, int32_t* block_tables, int bt_stride,
                             int32_t* seq_lens) {
  BM_TRACE("pa_bm_build_batch");
  BM_GUARD(bm);
  if (n < 0 || bt_stride < 1 || (n > 0 && (!seq_ids || !block_tables || !seq_lens))) return PA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    Seq* s = bm->use(seq_ids[i]);
    if (!s || (int64_t)s->table.size() > bt_stride || s->len > INT32_MAX) return PA_ERR_INVALID_ARG;
    int32_t* row = block_tables + (size_t)i * bt_stride;
    const int m = (int)s->table.size();
    for (int j = 0; j < bt_stride; ++j) row[j] = j < m ? s->table[j] : -1;
    seq_lens[i] = (int32_t)s->len;
  }
  return PA_OK;
}

PA_API int pa_bm_evict_lru_sequence(pa_block_manager* bm, int64_t exclude_id, int has_exclude, int64_t* victim) {
  BM_TRACE("pa_bm_evict_lru_sequence");
  BM_GUARD(bm);
  if (!victim) return PA_ERR_INVALID_ARG;
  bool found = false;
  uint64_t best_use = 0;
  int64_t best = 0;
  for (const auto& kv : bm->seqs) {
    if (has_exclude && kv.first == exclude_id) continue;
    if (!found || kv.second.last_use < best_use) {
      found = true;
      best_use = kv.second.last_use;
      best = kv.first;
    }
  }
  if (!found) return PA_ERR_OUT_OF_BLOCKS;
  for (int32_t b : bm->seqs[best].table) bm->decref(b);
  bm->seqs.erase(best);
  *victim = best;
  return PA_OK;
}

PA_API int pa_bm_allocate_with_prefix(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                      int* matched_tokens, int64_t* slots, int* num_slots) {
  BM_TRACE("pa_bm_allocate_with_prefix");
  BM_GUARD(bm);
  if (num_tokens < 0 || (num_tokens > 0 && (!tokens || !slots)) || !matched_tokens || !num_slots)
    return PA_ERR_INVALID_ARG;
  if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  const int bs = bm->block_size;
  const int nfull = num_tokens / bs;
  try {
    std::vector<int32_t> table;
    int64_t parent = 0;
    int matched_blocks = 0;
    Key key;
    for (int b = 0; b < nfull; ++b) {  // walk the cached chain
      key.parent = parent;
      key.tokens.assign(tokens + (size_t)b * bs, tokens + (size_t)(b + 1) * bs);
      auto it = bm->index.find(key);
      if (it == bm->index.end()) break;
      Entry& e = bm->entries.at(it->second);
      e.last_use = bm->tick();
      bm->incref(e.block);
      table.push_back(e.block);
      parent = it->second;
      ++matched_blocks;
    }
    Seq& s = bm->seqs[seq_id];
    s.table = table;
    s.len = num_tokens;
    s.last_use = bm->tick();
    try {
      while ((int)s.table.size() < (num_tokens + bs - 1) / bs) s.table.push_back(bm->allocate());
    } catch (const OutOfBlocks&) {
      Seq* again = bm->use(seq_id);  // release it like pa_bm_free_sequence (which marks it used first)
      for (int32_t b : again->table) bm->decref(b);
      bm->seqs.erase(seq_id);
      return PA_ERR_OUT_OF_BLOCKS;
    }
    for (int b = matched_blocks; b < nfull; ++b) {  // enter the prompt's new whole blocks
      Key k;
      k.parent = parent;
      k.tokens.assign(tokens + (size_t)b * bs, tokens + (size_t)(b + 1) * bs);
      const int64_t id = bm->next_entry++;
      Entry e{s.table[b], bm->tick(), k};
      bm->index.emplace(std::move(k), id);
      bm->entries.emplace(id, std::move(e));
      bm->incref(s.table[b]);
      parent = id;
    }
    const int matched = matched_blocks * bs;
    *matched_tokens = matched;
    *num_slots = num_tokens - matched;
    for (int p = matched; p < num_tokens; ++p) slots[p - matched] = (int64_t)s.table[p / bs] * bs + p % bs;
  } catch (const std::bad_alloc&) {
    return PA_ERR_NO_MEMORY;
  }
  return PA_OK;
}
