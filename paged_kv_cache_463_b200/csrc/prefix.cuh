// Shared-prefix pass of decode attention.
//
// Sequences forked from one prompt share the physical blocks of that prompt
// (page "5.KV Cache 管理 & PagedAttention", Q18 fork: the child's block table
// is a copy of the parent's and every shared block's reference count goes up;
// Q20 / page "paged-attention-and-vllm-inference", PrefixCacheManager: a
// cached prefix's blocks are reused by later requests).  Attention over a
// shared block is the same K/V against each member's query, so this pass loads
// every shared block once and scores it for all members at once; the members'
// private suffixes go through the regular decode kernel, and the merge kernel
// combines the two sets of (o, m, l) partials by log-sum-exp.
//
// Work: one CTA per (group, KV unit, 64 query rows, chunk of 32 prefix blocks).
// Query rows are (member sequence, query head of the unit) pairs, 8 per
// consumer warp (the MMA N), so one K/V tile feeds 64 rows.  Warp 0 streams
// the chunk's K/V tiles with TMA into an NS-stage ring (read from the group's
// first member's block table); warps 1..8 consume every stage (empty barrier
// count 8).  An fp8 E4M3 tile is converted once per block, by all 256 consumer
// threads, into a double-buffered f16 tile in the same 128-byte-swizzled
// layout, so that the 8 warps use the 16-bit MMA path on it.
#pragma once

#include "decode.cuh"

namespace pa {

enum : int { kCheckBadPrefix = 16 };

struct PrefixParams {
  const void* query;               // [S, Hq, D]
  const int32_t* block_tables;     // [S, bt_stride]
  const int32_t* seq_lens;         // [S]
  const int32_t* group_start;      // [num_groups + 1]: group g = sequences [start[g], start[g+1])
  const int32_t* group_prefix_len; // [num_groups]: shared tokens, a multiple of 16
  float* pre_o;                    // [S, Hq, max_chunks, D]
  float* pre_ml;                   // [S, Hq, max_chunks, 2]  (m in log2 units, l)
  int* seq_skip;                   // [S] out: leading blocks of each sequence this pass covers
  int* err;
  int num_seqs;
  int num_groups;
  int max_group_size;
  int max_prefix_blocks;  // ceil(max_prefix_len / 16) of the call (grid.x covers it)
  int bt_stride;
  int num_heads;
  int group;        // num_heads / num_kv_heads
  int head_splits;  // ceil(group / 8)
  int num_blocks;
  int max_blocks;   // ceil(max_seq_len / 16) of the call
  int max_chunks;   // prefix chunks a sequence may have (workspace extent)
  int row_blocks;   // grid.y = kv_units * row_blocks
  float scale_log2;
  float v_scale;
};

constexpr int kPrefixWarps = 8;                    // consumer warps
constexpr int kPrefixRows = kPrefixWarps * kNH;    // query rows per CTA

template <int D_, typename KV_, typename Q_, int NS_>
struct PrefixCfg {
  static constexpr int D = D_;
  using KV = KV_;
  using Q = Q_;
  static constexpr int NS = NS_;
  static constexpr bool kFp8 = sizeof(KV) == 1;
  static constexpr bool kBf16 = std::is_same<Q, __nv_bfloat16>::value;
  static constexpr int ROW_BYTES = D * (int)sizeof(KV);
  static constexpr int SUBTILES = ROW_BYTES / 128;
  static constexpr int TILE_BYTES = kBS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int F16_TILE = kBS * D * 2;      // converted tile (fp8 only)
  static constexpr int THREADS = 32 * (1 + kPrefixWarps);
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_CONV = NS * STAGE_BYTES;                  // 2 x (K, V) f16 tiles
  static constexpr int OFF_BAR = OFF_CONV + (kFp8 ? 4 * F16_TILE : 0);
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + 2 * NS * 8;
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle spans");
  static_assert(!kFp8 || std::is_same<Q, __half>::value, "fp8 caches pair with fp16 queries");
};

// Shared blocks of group g that the pass covers: the group's prefix in whole
// blocks, or 0 when the group's description cannot be used (then its members
// are decoded in full by the suffix pass).  Members' lengths and tables are
// checked separately, by one CTA per group.
__device__ __forceinline__ int group_prefix_blocks(const PrefixParams& p, int g, int first, int members) {
  if (first < 0 || members < 0 || first + members > p.num_seqs || members > p.max_group_size) return 0;
  const int len = p.group_prefix_len[g];
  const int cap = min(p.max_prefix_blocks, min(p.bt_stride, p.max_blocks));
  if (len < 0 || len % kBS != 0 || len / kBS > cap) return 0;
  return len / kBS;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) paged_prefix_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const PrefixParams p) {
  using Q = typename C::Q;
  constexpr int D = C::D, NS = C::NS;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_u32(smem);
  const uint32_t full0 = base + C::OFF_BAR, empty0 = full0 + NS * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int g = blockIdx.z;
  const int y = blockIdx.y / p.row_blocks;
  const int rb = blockIdx.y - y * p.row_blocks;
  const int chunk = blockIdx.x;
  const int first = p.group_start[g], members = p.group_start[g + 1] - first;
  const int pblk = group_prefix_blocks(p, g, first, members);

  if (blockIdx.x == 0 && blockIdx.y == 0) {
    // One CTA per group: the group's description, and the suffix offsets of
    // its members (plus those of the sequences before the first group / from
    // the last group's end on, which have no shared prefix).
    __shared__ int s_ok;
    const bool range_ok = first >= 0 && members >= 0 && first + members <= p.num_seqs;
    if (threadIdx.x == 0) {
      s_ok = 1;
      const int len = p.group_prefix_len[g];
      if (range_ok && len != 0 && pblk == 0) atomicOr(p.err, kCheckBadPrefix);
      if (!range_ok) atomicOr(p.err, kCheckBadPrefix);
    }
    __syncthreads();
    // every member is at least as long as the prefix and maps it to the same blocks
    for (int k = threadIdx.x; k < members * pblk; k += blockDim.x) {
      const int m = k / pblk, b = k - m * pblk;
      const int s = first + m;
      bool ok = p.seq_lens[s] >= pblk * kBS;
      if (m > 0)
        ok = ok && __ldg(p.block_tables + (size_t)s * p.bt_stride + b) ==
                       __ldg(p.block_tables + (size_t)first * p.bt_stride + b);
      if (!ok) s_ok = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !s_ok) atomicOr(p.err, kCheckBadPrefix);
    const int skip = s_ok ? pblk : 0;
    if (range_ok)
      for (int m = threadIdx.x; m < members; m += blockDim.x) p.seq_skip[first + m] = skip;
    if (g == 0) {
      const int lo = min(max(first, 0), p.num_seqs);
      for (int s = threadIdx.x; s < lo; s += blockDim.x) p.seq_skip[s] = 0;
    }
    if (g == p.num_groups - 1) {
      const int hi = max(min(first + members, p.num_seqs), 0);
      for (int s = hi + threadIdx.x; s < p.num_seqs; s += blockDim.x) p.seq_skip[s] = 0;
    }
  }

  const int kvh = y / p.head_splits;
  const int hs = y - kvh * p.head_splits;
  const int head0 = kvh * p.group + hs * kNH;
  const int hpu = min(kNH, p.group - hs * kNH);  // query heads of this KV unit
  const int rows = members * hpu;
  const int b0 = chunk * kPrefixChunkBlocks;
  const int nb = min(pblk, b0 + kPrefixChunkBlocks) - b0;
  if (nb <= 0 || rb * kPrefixRows >= rows) return;

  __shared__ int s_dead;  // a consumer warp's wait timed out: the others stop waiting too
  if (threadIdx.x == 0) {
    s_dead = 0;
    for (int i = 0; i < NS; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kPrefixWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // the group's blocks, as the first member's table names them
    int my = 0;
    if (lane < nb) {
      my = __ldg(p.block_tables + (size_t)first * p.bt_stride + b0 + lane);
      if (my < 0 || my >= p.num_blocks) {
        atomicOr(p.err, kCheckBadBlock);
        my = 0;
      }
    }
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    for (int i = 0; i < nb; ++i) {
      const int phys = __shfl_sync(0xffffffffu, my, i);
      int stop = 0;
      if (lane == 0) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait(empty0 + 8 * st, ((i / NS) - 1) & 1)) {
          atomicOr(p.err, kCheckWaitTimeout);
          stop = 1;
        } else {
          const uint32_t fb = full0 + 8 * st;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          const uint32_t kdst = base + C::OFF_RING + st * C::STAGE_BYTES;
#pragma unroll
          for (int sub = 0; sub < C::SUBTILES; ++sub) {
            const int x = kvh * D + sub * (128 / (int)sizeof(typename C::KV));
            tma_load_2d(kdst + sub * kBS * 128, &tmK, x, phys * kBS, fb);
            tma_load_2d(kdst + C::TILE_BYTES + sub * kBS * 128, &tmV, x, phys * kBS, fb);
          }
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int gid = lane >> 2, c4 = lane & 3;
  // query row n of this warp's 8 -> (sequence, head); false past the group's rows
  auto row_of = [&](int n, int& s, int& h) -> bool {
    const int r = rb * kPrefixRows + cw * kNH + n;
    if (r >= rows) return false;
    s = first + r / hpu;
    h = head0 + r % hpu;
    return true;
  };
  WarpAttn<D, false, C::kBf16> A;
  A.reset();
  {
    int s = 0, h = 0;
    const bool ok = row_of(gid, s, h);
    A.load_q(ok ? reinterpret_cast<const Q*>(p.query) + ((size_t)s * p.num_heads + h) * D : nullptr, c4);
  }
  // A timed-out wait (the check bit reports it) stops this warp's work, but it
  // keeps meeting the consumers' named barrier once per block, so that no
  // other warp waits for it there.
  bool dead = false;
  for (int i = 0; i < nb; ++i) {
    const int st = i % NS;
    if (!dead) {  // (warp-uniform)
      bool fail = *reinterpret_cast<volatile int*>(&s_dead) != 0;
      if (!fail) fail = !mbar_wait(full0 + 8 * st, (i / NS) & 1);
      dead = __any_sync(0xffffffffu, fail);
      if (dead && lane == 0) {
        atomicOr(p.err, kCheckWaitTimeout);
        s_dead = 1;
      }
    }
    const uint32_t kb = base + C::OFF_RING + st * C::STAGE_BYTES;
    uint32_t ka = kb, va = kb + C::TILE_BYTES;
    if constexpr (C::kFp8) {
      // The 256 consumer threads convert the K and V tiles (16 rows x D/16
      // 16-byte chunks each) into f16 tiles with the 16-bit layout; buffer
      // i & 1, so that converting block i + 1 never overwrites a tile a slower
      // warp still reads (the barrier below orders block i's reads before any
      // warp converts block i + 2).
      if (!dead) {
        const int t = threadIdx.x - 32;
        const int which = t >> 7;
        constexpr int CPR = D / 16;  // 16-byte fp8 chunks per row
        const uint32_t dst = base + C::OFF_CONV + ((i & 1) * 2 + which) * C::F16_TILE;
#pragma unroll
        for (int k = t & 127; k < kBS * CPR; k += 128) {
          const int r = k / CPR, cc = k - r * CPR;
          const uint4 v = lds128(kb + which * C::TILE_BYTES + tile_off(r, 16 * cc));
          uint32_t h[8];
          e4m3x4_to_f16x2x2(v.x, h[0], h[1]);
          e4m3x4_to_f16x2x2(v.y, h[2], h[3]);
          e4m3x4_to_f16x2x2(v.z, h[4], h[5]);
          e4m3x4_to_f16x2x2(v.w, h[6], h[7]);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + tile_off(r, 32 * cc)), "r"(h[0]),
                       "r"(h[1]), "r"(h[2]), "r"(h[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + tile_off(r, 32 * cc + 16)),
                       "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                       : "memory");
        }
      }
      named_bar_sync(1, kPrefixWarps * 32);  // converted tiles complete; the fp8 stage is free
      if (!dead && lane == 0) mbar_arrive(empty0 + 8 * st);
      ka = base + C::OFF_CONV + ((i & 1) * 2) * C::F16_TILE;
      va = ka + C::F16_TILE;
    }
    if (dead) continue;
    // the prefix covers whole blocks: all 16 tokens valid
    A.block(ka, va, kBS, p.scale_log2, lane);
    if constexpr (!C::kFp8) {
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
  }
  if (dead) return;
  float L0, L1;
  A.totals(L0, L1);
  int s0 = 0, h0 = 0, s1 = 0, h1 = 0;
  const bool ok0 = row_of(2 * c4, s0, h0), ok1 = row_of(2 * c4 + 1, s1, h1);
  const size_t row0 = ((size_t)s0 * p.num_heads + h0) * p.max_chunks + chunk;
  const size_t row1 = ((size_t)s1 * p.num_heads + h1) * p.max_chunks + chunk;
  store_partial<D, false>(A.o, A.m0, L0, L0 > 0.f ? p.v_scale / L0 : 0.f, ok0, A.m1, L1,
                          L1 > 0.f ? p.v_scale / L1 : 0.f, ok1, p.pre_o, p.pre_ml, row0, row1, lane);
}

}  // namespace pa
