// Multi-query paged attention: prefill and chunked prefill.
//
// Page "5.KV Cache 管理 & PagedAttention", Q6 (MHAWithCache, prefill
// branch): every query position attends causally to the keys at its own and
// earlier positions; Q3.3 / Q19: the keys are read block by block from the
// paged cache through the sequence's block table, blockwise with an online
// softmax, after this chunk's K/V were written to the cache.  Sequence s has
// seq_lens[s] cached tokens and q_len = query_start[s+1] - query_start[s]
// query rows, its last q_len positions (q_len = seq_len: a whole prompt;
// smaller: a later chunk; 1: a decode step).
//
// One CTA per (row block, KV unit, sequence): the rows are the (query token,
// head) pairs of one KV unit, heads fastest, 128 per CTA, so a CTA covers
// 128 / h tokens of h query heads.  The keys it needs are those up to its
// last row's position (causal), in 64-token tensor-core steps of the shared
// stacked-attention core (prefix.cuh), each row masked at its own position;
// the CTA writes the final, normalised output rows.
#pragma once

#include "prefix.cuh"

namespace pa {

struct PrefillParams {
  void* out;                    // [T, Hq, D] query dtype
  const void* query;            // [T, Hq, D]
  const void* k_cache;          // [num_blocks, 16, Hkv, D]
  const void* v_cache;
  const int32_t* block_tables;  // [S, bt_stride]
  const int32_t* seq_lens;      // [S]
  const int32_t* query_start;   // [S + 1]
  int* err;
  int num_seqs;
  int num_tokens;   // rows of query / out
  int bt_stride;
  int num_heads;
  int group;
  int head_splits;
  int num_blocks;
  int max_blocks;   // ceil(max_seq_len / 16)
  float scale_log2;
  float v_scale;
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::REG_CTAS)
    paged_prefill_kernel(const PrefillParams p) {
  using Q = typename C::Q;
  constexpr int D = C::D;
  const int s = blockIdx.z;
  const int y = blockIdx.y;
  const int rb = gridDim.x - 1 - blockIdx.x;  // a sequence's row blocks heaviest (most keys) first
  const int kvh = y / p.head_splits;
  const int hs = y - kvh * p.head_splits;
  const int head0 = kvh * p.group + hs * kNH;
  const int hpu = min(kNH, p.group - hs * kNH);
  const int tpb = kPrefixRows / hpu;  // query tokens per CTA

  const int qs = p.query_start[s];
  const int q_len = p.query_start[s + 1] - qs;
  const int cap = min(p.bt_stride, p.max_blocks) * kBS;
  const int raw = p.seq_lens[s];
  const int len = raw < 0 ? 0 : min(raw, cap);
  const bool rows_ok = qs >= 0 && q_len >= 0 && qs + q_len <= p.num_tokens;  // inside query / out
  if (rb == 0 && y == 0 && threadIdx.x == 0 && (raw != len || !rows_ok || q_len > len))
    atomicOr(p.err, kCheckSeqTooLong);
  if (!rows_ok || q_len <= 0 || q_len > len || rb * tpb >= q_len) return;
  const int t1 = min(q_len, (rb + 1) * tpb);  // last query token of this CTA + 1
  const int kv_valid = len - q_len + t1;      // keys up to the last row's position

  struct Rows {
    const PrefillParams* p;
    int rb, tpb, hpu, head0, q_len, qs, pos0;  // pos0: position of query token 0
    __device__ bool at(int r, int& t, int& h) const {
      const int tl = r / hpu;
      if (tl >= tpb) return false;
      t = rb * tpb + tl;
      if (t >= q_len) return false;
      h = head0 + r % hpu;
      return true;
    }
    __device__ const void* q_row(int r) const {
      int t, h;
      if (!at(r, t, h)) return nullptr;
      return reinterpret_cast<const Q*>(p->query) + ((size_t)(qs + t) * p->num_heads + h) * D;
    }
    __device__ int limit(int r) const {  // causal: keys 0..pos
      int t, h;
      return at(r, t, h) ? pos0 + t + 1 : 1;
    }
    __device__ void store(int r, int c0, const float (&v)[16]) const {
      int t, h;
      if (!at(r, t, h)) return;
      Q* dst = reinterpret_cast<Q*>(p->out) + ((size_t)(qs + t) * p->num_heads + h) * D + c0;
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = pack2<C::kBf16>(v[2 * j], v[2 * j + 1]);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(dst + 8) = make_uint4(w[4], w[5], w[6], w[7]);
    }
    __device__ void store_ml(int, float, float) const {}
  };
  const Rows rw{&p, rb, tpb, hpu, head0, q_len, qs, len - q_len};
  const size_t row_stride = (size_t)(p.num_heads / p.group) * C::ROW_BYTES;
  const StackedJob job{p.block_tables + (size_t)s * p.bt_stride, (kv_valid + kBS - 1) / kBS, kv_valid,
                       p.num_blocks, static_cast<const uint8_t*>(p.k_cache) + (size_t)kvh * C::ROW_BYTES,
                       static_cast<const uint8_t*>(p.v_cache) + (size_t)kvh * C::ROW_BYTES, row_stride};
  stacked_attention<C>(job, rw, p.scale_log2, p.v_scale, p.err);
}

}  // namespace pa
