// Paged decode attention for sm_100a.
//
// What it computes (page "5.KV Cache 管理 & PagedAttention", Q4 decode_step and
// Q13 / Q19; listing paged_attention on page "paged-attention-and-vllm-inference"):
// for every sequence s and query head h,
//     out[s,h,:] = softmax_j(scale * q[s,h,:] . K_s[j,:]) V_s
// over the seq_lens[s] cached tokens of s, whose K/V rows live in fixed-size
// physical blocks reached through block_tables[s, j / 16] at offset j % 16,
// with the KV head h / (num_heads / num_kv_heads) (grouped-query attention).
//
// Kernel design (B200):
//  * persistent grid (SMs x CTAs per SM).  Work is (sequence, KV unit =
//    KV head [x chunk of 8 query heads], range of 16-token blocks).  Two
//    ways of handing it out:
//      - stream-K (the default): CTAs form groups of kv_units, one CTA per
//        KV unit; the flattened (sequence, block) space is cut into equal
//        contiguous ranges, one per group, so every CTA has the same work and
//        the CTAs of a group read the same blocks (all KV heads of a token are
//        one contiguous row) at about the same time; a sequence cut by a
//        range boundary becomes several pieces, merged afterwards;
//      - tickets (an explicit partition length): items (sequence, partition,
//        KV unit) numbered in that order, handed out by an atomic counter;
//  * a CTA is two warps.  Warp 1 produces: for each item it bulk-copies the
//    item's query rows into a 2-slot shared-memory queue and streams each
//    16-token block's K and V tiles with 2-D TMA tensor loads (128-byte
//    swizzle, mbarrier byte counts, no multicast) into an NS-stage ring,
//    with a small metadata record per stage (item, valid tokens, first/last);
//    it runs ahead into the next item while the consumer finishes this one.
//    Warp 0 consumes, per block:
//      S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]   (mma.m16n8k16, K via ldmatrix)
//      online softmax in the log2 domain (running max m, sum l)
//      P^T packed to 16 bits and moved into the B-operand layout with movmatrix
//      O^T[D x 8] += V^T[D x 16 tok] . P^T[16 x 8]       (V via ldmatrix.trans)
//    fp8 E4M3 tiles are read with 128-bit shared loads and converted in
//    registers to f16 pairs (exact); the contraction order is permuted so
//    that every lane's operands are contiguous bytes; an item's fp8 tiles go
//    two by two through one step (one softmax update for 32 tokens);
//  * at an item's last block the consumer writes the output (one-partition
//    sequences) or (O / l, m, l) partials; paged_decode_merge_kernel, launched
//    as a programmatic dependent of this grid, combines split sequences with
//    the log-sum-exp rule
//      M = max_p m_p,  w_p = l_p 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace pa {

enum : int { kCheckBadBlock = 1, kCheckBadSlot = 2, kCheckSeqTooLong = 4, kCheckWaitTimeout = 8 };

constexpr int kBS = 16;  // tokens per physical block
constexpr int kNH = 8;   // query heads per item (MMA N)

// stage metadata flags (meta.w)
enum : int { kFirst = 1, kLast = 2, kEnd = 4 };

struct DecodeParams {
  void* out;                    // [S, Hq, D] query dtype
  const void* query;            // [S, Hq, D] query dtype
  const int32_t* block_tables;  // [S, bt_stride]
  const int32_t* seq_lens;      // [S]
  float* part_o;                // [S, Hq, max_parts, D]
  float* part_ml;               // [S, Hq, max_parts, 2]  (m in log2 units, l)
  int* err;                     // device check bits
  int* counters;                // [0] ticket, [1] finished CTAs (zero between launches)
  int num_seqs;
  int bt_stride;
  int num_heads;
  int group;        // num_heads / num_kv_heads
  int head_splits;  // ceil(group / 8)
  int kv_units;     // num_kv_heads * head_splits
  int num_blocks;   // physical pool size
  int max_blocks;        // ceil(max_seq_len / 16) of the call: lengths are clamped to it
  int force_partials;    // 1: one-partition sequences also write partials (a prefix pass adds terms)
  int partition_blocks;  // ticket mode: blocks per partition
  int auto_mode;         // 1: the kernel chooses tickets or stream-K (and the partition) from the lengths
  int min_piece_blocks;  // stream-K mode: shortest range a CTA group is given
  int* seq_merge;        // [S]: each sequence's merge work, written by CTA 0 for the merge kernel
  int max_parts;    // partitions a sequence may have (workspace extent)
  int q_slot_bytes; // min(group, 8) * head_dim * 2: one item's query rows
  int merge_hpc;    // merge kernel: query heads per CTA
  int merge_slices; // merge kernel: partition slices per head
  int merge_hpt;    // merge kernel: heads per thread (2 only with one slice)
  float scale_log2;  // softmax scale * log2(e) (* k_scale for fp8)
  float v_scale;     // 1, or the fp8 value scale
  // shared-prefix decode (all null / 0 otherwise): the prefix pass covered the
  // first seq_skip[s] blocks of sequence s; this pass covers the rest, and the
  // merge adds the prefix pass's ceil(seq_skip[s] / 32) partials per head
  const int* seq_skip = nullptr;  // [S]
  const float* pre_o = nullptr;   // [S, Hq, max_chunks, D]
  const float* pre_ml = nullptr;  // [S, Hq, max_chunks, 2]
  int max_chunks = 0;
  // failure-path test hook: every pipeline wait of the launch is bounded by
  // wait_limit cycles, and with debug_stall the consumer's first wait targets
  // a barrier that nothing completes, so the launch must take its timeout exit
  long long wait_limit = kWaitLimitCycles;
  int debug_stall = 0;
};

#ifndef PA_PREFIX_CHUNK_BLOCKS
#define PA_PREFIX_CHUNK_BLOCKS 32
#endif
constexpr int kPrefixChunkBlocks = PA_PREFIX_CHUNK_BLOCKS;  // blocks per partial of the prefix pass
// DecodeParams::seq_merge values: >= 0 = the decode partials to fold (plus
// the prefix pass's chunks in shared-prefix decode); or
constexpr int kMergeNone = -2;  // the decode kernel wrote the row (one unsplit item)
constexpr int kMergeZero = -1;  // no decode item covered the sequence: zero rows

// Clamp a sequence length to what its table row can address and to the
// call's max_seq_len bound (which sizes the partial workspace).
__device__ __forceinline__ int clamp_len(int len, const DecodeParams& p) {
  const int cap = min(p.bt_stride, p.max_blocks) * kBS;
  return len < 0 ? 0 : (len > cap ? cap : len);
}
// Partitions of a (clamped) length with `pb` blocks per partition; the
// workspace extent caps it.
__device__ __forceinline__ int num_partitions(int len, int pb, const DecodeParams& p) {
  const int nblk = (len + kBS - 1) / kBS;
  const int np = (nblk + pb - 1) / pb;
  return np < p.max_parts ? np : p.max_parts;
}

// Partition size (blocks) for near-uniform lengths in auto mode: the largest
// power-of-two multiple of the minimum such that one work item stays under
// 0.6 of one CTA's average share of the work (items then finish together), or
// no split at all if a whole sequence fits.
__device__ __forceinline__ int uniform_partition_blocks(const DecodeParams& p, long long sum_len, int max_len,
                                                        int ctas) {
  const int max_blk = (max_len + kBS - 1) / kBS;
  if (max_blk <= 0) return p.partition_blocks;
  const float budget = 0.6f * (float)p.kv_units * (float)sum_len / (float)ctas;  // tokens
  if ((float)max_len <= budget) return max(max_blk, p.partition_blocks);
  int pb = p.partition_blocks;
  while ((float)(2 * pb * kBS) <= budget && 2 * pb < max_blk) pb *= 2;
  return pb;
}

// Stream-K split of one sequence: its blocks occupy the global range
// [a, a + nblk) of the flattened (sequence, block) space, which is cut into
// equal ranges of `per_group` blocks, one per group of kv_units CTAs; the
// sequence's pieces are the groups g0..g1 that overlap it (the same pieces for
// every KV unit).
struct Pieces {
  int c0, count;
};
__device__ __forceinline__ Pieces unit_pieces(int a, int nblk, int per_group) {
  const int c0 = a / per_group;
  return {c0, (a + nblk - 1) / per_group - c0 + 1};
}

// Shared-memory layout of a decode CTA (offsets from a 1024-aligned base):
// ring[NS stages] | query slots[2] | mbarriers | exit record | stage metadata | prefix[S+1], lens[S]
// mbarriers: full[NS], empty[NS], qfull[2], qempty[2], and one that nothing
// completes (the target of the failure-path test hook).  Exit record: stages
// and query slots the consumer took, a flag set by a wait that ran out, and
// the two warps' scheduler slots.
__host__ __device__ constexpr int kDecodeBarriers(int ns) { return 2 * ns + 5; }
struct DecodeLayout {
  int ring, q, bar, exitrec, meta, prefix;
  __host__ __device__ DecodeLayout(int ns, int stage_bytes, int q_slot_bytes) {
    ring = 0;
    q = ns * stage_bytes;
    bar = q + 2 * q_slot_bytes;
    exitrec = (bar + kDecodeBarriers(ns) * 8 + 15) & ~15;
    meta = exitrec + 32;
    prefix = meta + ns * 16;
  }
  // bytes of dynamic shared memory for up to `max_seqs` sequences (+ alignment slack)
  __host__ __device__ size_t bytes(int max_seqs) const { return 1024 + prefix + 8 * (size_t)(max_seqs + 1); }
};

template <int D_, typename KV_, typename Q_, int NS_, int MIN_CTAS_ = 1>
struct DecodeCfg {
  static constexpr int D = D_;
  using KV = KV_;  // __half, __nv_bfloat16 or __nv_fp8_e4m3
  using Q = Q_;    // __half or __nv_bfloat16 (also the MMA operand type)
  static constexpr int NS = NS_;  // ring stages (one 16-token block each)
  static constexpr bool kFp8 = sizeof(KV) == 1;
  static constexpr bool kBf16 = std::is_same<Q, __nv_bfloat16>::value;
  static constexpr int ROW_BYTES = D * (int)sizeof(KV);
  static constexpr int SUBTILES = ROW_BYTES / 128;
  static constexpr int TILE_BYTES = kBS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int THREADS = 64;
  static constexpr int MIN_CTAS = MIN_CTAS_;  // register budget hint: CTAs that must fit on one SM
  static constexpr int NKT = D / 16;
  static constexpr int NDT = D / 16;
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle spans");
  static_assert(!kFp8 || std::is_same<Q, __half>::value, "fp8 caches pair with fp16 queries");
  static_assert(!std::is_same<KV, __half>::value || std::is_same<Q, __half>::value, "f16 cache needs f16 query");
  static_assert(!std::is_same<KV, __nv_bfloat16>::value || kBf16, "bf16 cache needs bf16 query");
  static DecodeLayout layout(int q_slot_bytes) { return DecodeLayout(NS, STAGE_BYTES, q_slot_bytes); }
};

// Byte offset of (row, byte-in-row) inside a [16 x ROW_BYTES] tile stored as
// 128-byte-wide sub-tiles with the TMA 128-byte swizzle (16-byte chunk index
// XOR row % 8).  `byte` is a multiple of 16 or lies inside one chunk.
__device__ __forceinline__ uint32_t tile_off(int row, int byte) {
  const int sub = byte >> 7;
  const int in = byte & 127;
  return (uint32_t)(sub * (kBS * 128) + row * 128 + ((((in >> 4) ^ (row & 7)) << 4) | (in & 15)));
}

// Store a warp's normalised partial rows (o / l as fp32, plus (m, l)) for
// output columns 2*c4 (row0) and 2*c4 + 1 (row1), straight from registers.
template <int D, bool FP8>
__device__ __forceinline__ void store_partial(const float (&o)[D / 16][4], float m0, float L0, float i0, bool ok0,
                                              float m1, float L1, float i1, bool ok1, float* part_o, float* part_ml,
                                              size_t row0, size_t row1, int lane) {
  const int gid = lane >> 2;
  float* d0 = part_o + row0 * D;
  float* d1 = part_o + row1 * D;
#pragma unroll
  for (int t = 0; t < D / 16; ++t) {
    if constexpr (!FP8) {
      if (ok0) {
        d0[16 * t + gid] = o[t][0] * i0;
        d0[16 * t + gid + 8] = o[t][2] * i0;
      }
      if (ok1) {
        d1[16 * t + gid] = o[t][1] * i1;
        d1[16 * t + gid + 8] = o[t][3] * i1;
      }
    } else {  // adjacent dims: one 8-byte store per column
      const int d = (D / 8) * gid + 2 * t;
      if (ok0) *reinterpret_cast<float2*>(d0 + d) = make_float2(o[t][0] * i0, o[t][2] * i0);
      if (ok1) *reinterpret_cast<float2*>(d1 + d) = make_float2(o[t][1] * i1, o[t][3] * i1);
    }
  }
  if (gid == 0) {
    if (ok0) *reinterpret_cast<float2*>(part_ml + row0 * 2) = make_float2(m0, L0);
    if (ok1) *reinterpret_cast<float2*>(part_ml + row1 * 2) = make_float2(m1, L1);
  }
}

// One warp's attention state for 8 query columns (MMA N) over a stream of
// 16-token K/V tiles in shared memory, and the per-tile math:
//   S^T[16 tok x 8] = K[16 x D] . Q^T[D x 8]          (mma.m16n8k16)
//   online softmax in the log2 domain with lazy rescaling
//   O^T[D x 8] += V^T[D x 16 tok] . P^T[16 x 8]        (P^T via movmatrix)
// Lane (gid = lane / 4, c4 = lane % 4) holds query column gid's fragments and
// the output columns 2*c4, 2*c4 + 1.  FP8 tiles (E4M3) are converted to f16 in
// registers, with the contraction order permuted so that a lane's operand
// bytes are contiguous.
template <int D, bool FP8, bool BF16>
struct WarpAttn {
  static constexpr int NKT = D / 16;
  static constexpr int NDT = D / 16;
  uint32_t qf[NKT][2];
  float o[NDT][4];
  float m0, m1, l0, l1;
  // fp8 V rows of the current tile: lane row gid owns dims [D/8*gid,
  // D/8*gid + D/8) of tokens 2c4, 2c4+1, 2c4+8, 2c4+9; output tile t holds
  // dims D/8*gid + 2t (MMA row gid) and +1 (row gid+8)
  uint4 vr[4][FP8 ? D / 128 : 1];

  __device__ __forceinline__ void load_v8(uint32_t vb, int gid, int c4) {
    constexpr int LB = D / 8;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = 2 * c4 + (r & 1) + ((r >> 1) << 3);
#pragma unroll
      for (int u = 0; u < LB / 16; ++u) vr[r][u] = lds128(vb + tile_off(row, LB * gid + 16 * u));
    }
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int t = 0; t < NDT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  }

  // Q^T as MMA B fragments from this lane's query column (row gid of the
  // warp's 8); `row` == nullptr gives a zero column.  16-bit elements.
  __device__ __forceinline__ void load_q(const void* row, int c4) {
    const uint8_t* q = reinterpret_cast<const uint8_t*>(row);
#pragma unroll
    for (int j = 0; j < NKT; ++j) {
      if constexpr (!FP8) {
        qf[j][0] = q ? *reinterpret_cast<const uint32_t*>(q + 2 * (16 * j + 2 * c4)) : 0u;
        qf[j][1] = q ? *reinterpret_cast<const uint32_t*>(q + 2 * (16 * j + 2 * c4 + 8)) : 0u;
      } else {
        // permuted contraction order: lane column c4 owns dims [D/4*c4, D/4*c4 + D/4)
        const uint2 v = q ? *reinterpret_cast<const uint2*>(q + 2 * ((D / 4) * c4 + 4 * j)) : make_uint2(0u, 0u);
        qf[j][0] = v.x;
        qf[j][1] = v.y;
      }
    }
  }

  // Lazy rescaling with this lane's own maxima bm0 / bm1 of its two columns:
  // the reference max only moves (and O, l are rescaled) when some head's
  // new scores exceed it by more than 2^kLazy; otherwise weights up to 2^kLazy
  // are accumulated as they are (exact in fp32, and well inside the 16-bit P
  // range).  A head's running max is the same in all lanes of its column, so
  // "some lane's own scores exceed it" is the same test as "the column max
  // does": the column reductions are only needed when it passes.
  __device__ __forceinline__ void update_max(float bm0, float bm1) {
    constexpr float kLazy = 8.f;
    const bool grow = (bm0 > m0 + kLazy) || (bm1 > m1 + kLazy);
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
      }
      const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
      const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      l0 *= al0;
      l1 *= al1;
#pragma unroll
      for (int t = 0; t < NDT; ++t) {
        o[t][0] *= al0;
        o[t][1] *= al1;
        o[t][2] *= al0;
        o[t][3] *= al1;
      }
    }
  }

  // fp8: S^T partial sums (two accumulation chains) of the K tile at kb.
  __device__ __forceinline__ void scores8(uint32_t kb, float (&sa)[4], float (&sb)[4], int gid, int c4) {
    constexpr int LB = D / 4;  // bytes of a K row owned by one lane
    constexpr int LC = LB / 16;
    uint4 kr[2][LC];
#pragma unroll
    for (int u = 0; u < LC; ++u) {
      kr[0][u] = lds128(kb + tile_off(gid, LB * c4 + 16 * u));
      kr[1][u] = lds128(kb + tile_off(gid + 8, LB * c4 + 16 * u));
    }
    const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&kr[0][0]);
    const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&kr[1][0]);
#pragma unroll
    for (int j = 0; j < NKT; ++j) {
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_f16x2x2(w0[j], a0, a2);
      e4m3x4_to_f16x2x2(w1[j], a1, a3);
      if (j & 1)
        mma_16816<false>(sb, a0, a1, a2, a3, qf[j][0], qf[j][1]);
      else
        mma_16816<false>(sa, a0, a1, a2, a3, qf[j][0], qf[j][1]);
    }
  }

  // fp8: O^T += V^T P^T with the V rows held in vr (rows past `valid` zeroed
  // first: they may hold NaN/Inf).
  __device__ __forceinline__ void pv8(int valid, uint32_t pb0, uint32_t pb1, int c4) {
    constexpr int LC = D / 128;
    if (valid < kBS) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = 2 * c4 + (r & 1) + ((r >> 1) << 3);
        if (row >= valid) {
#pragma unroll
          for (int u = 0; u < LC; ++u) vr[r][u] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(&vr[0][0]);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(&vr[1][0]);
    const uint32_t* r2 = reinterpret_cast<const uint32_t*>(&vr[2][0]);
    const uint32_t* r3 = reinterpret_cast<const uint32_t*>(&vr[3][0]);
#pragma unroll
    for (int w = 0; w < NDT / 2; ++w) {
      uint32_t a0, a1, a2, a3;
      // tile 2w: bytes 0,1 of word w; tile 2w+1: bytes 2,3
      e4m3x4_to_f16x2x2(prmt(r0[w], r1[w], 0x5140u), a0, a1);
      e4m3x4_to_f16x2x2(prmt(r2[w], r3[w], 0x5140u), a2, a3);
      mma_16816<false>(o[2 * w], a0, a1, a2, a3, pb0, pb1);
      e4m3x4_to_f16x2x2(prmt(r0[w], r1[w], 0x7362u), a0, a1);
      e4m3x4_to_f16x2x2(prmt(r2[w], r3[w], 0x7362u), a2, a3);
      mma_16816<false>(o[2 * w + 1], a0, a1, a2, a3, pb0, pb1);
    }
  }

  // fp8: two consecutive tiles of one item (the first full, the second with
  // valid2 tokens) with one softmax step over their 32 tokens.
  __device__ __forceinline__ void block2(uint32_t kb1, uint32_t vb1, uint32_t kb2, uint32_t vb2, int valid2,
                                         float sl, int lane) {
    const int gid = lane >> 2, c4 = lane & 3;
    float s1a[4] = {0.f, 0.f, 0.f, 0.f}, s1b[4] = {0.f, 0.f, 0.f, 0.f};
    float s2a[4] = {0.f, 0.f, 0.f, 0.f}, s2b[4] = {0.f, 0.f, 0.f, 0.f};
    scores8(kb1, s1a, s1b, gid, c4);
    load_v8(vb1, gid, c4);
    scores8(kb2, s2a, s2b, gid, c4);
    const float x0 = (s1a[0] + s1b[0]) * sl, x1 = (s1a[1] + s1b[1]) * sl;
    const float x2 = (s1a[2] + s1b[2]) * sl, x3 = (s1a[3] + s1b[3]) * sl;
    const float y0 = gid < valid2 ? (s2a[0] + s2b[0]) * sl : -INFINITY;
    const float y1 = gid < valid2 ? (s2a[1] + s2b[1]) * sl : -INFINITY;
    const float y2 = gid + 8 < valid2 ? (s2a[2] + s2b[2]) * sl : -INFINITY;
    const float y3 = gid + 8 < valid2 ? (s2a[3] + s2b[3]) * sl : -INFINITY;
    update_max(fmaxf(fmaxf(x0, x2), fmaxf(y0, y2)), fmaxf(fmaxf(x1, x3), fmaxf(y1, y3)));
    const float p0 = ex2(x0 - m0), p1 = ex2(x1 - m1), p2 = ex2(x2 - m0), p3 = ex2(x3 - m1);
    const float q0 = ex2(y0 - m0), q1 = ex2(y1 - m1), q2 = ex2(y2 - m0), q3 = ex2(y3 - m1);
    l0 += (p0 + p2) + (q0 + q2);
    l1 += (p1 + p3) + (q1 + q3);
    const uint32_t pb0 = movmatrix_trans(pack2<false>(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack2<false>(p2, p3));
    const uint32_t qb0 = movmatrix_trans(pack2<false>(q0, q1));
    const uint32_t qb1 = movmatrix_trans(pack2<false>(q2, q3));
    pv8(kBS, pb0, pb1, c4);
    load_v8(vb2, gid, c4);
    pv8(valid2, qb0, qb1, c4);
  }

  // One 16-token tile: K at kb, V at vb (shared addresses, 128-byte swizzled
  // [16 x D] tiles); tokens >= valid are masked out.  sl = softmax scale x log2(e).
  __device__ __forceinline__ void block(uint32_t kb, uint32_t vb, int valid, float sl, int lane) {
    const int gid = lane >> 2, c4 = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    // ---- S^T = K Q^T
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (!FP8) {
#pragma unroll
      for (int j = 0; j < NKT; ++j) {
        const int tok = ri + ((mi & 1) << 3);
        const int dim = 16 * j + ((mi >> 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + tile_off(tok, dim * 2), a0, a1, a2, a3);
        if (j & 1)
          mma_16816<BF16>(sb, a0, a1, a2, a3, qf[j][0], qf[j][1]);
        else
          mma_16816<BF16>(sa, a0, a1, a2, a3, qf[j][0], qf[j][1]);
      }
    } else {
      constexpr int LB = D / 4;  // bytes of a K row owned by one lane
      constexpr int LC = LB / 16;
      uint4 kr[2][LC];
#pragma unroll
      for (int u = 0; u < LC; ++u) {
        kr[0][u] = lds128(kb + tile_off(gid, LB * c4 + 16 * u));
        kr[1][u] = lds128(kb + tile_off(gid + 8, LB * c4 + 16 * u));
      }
      load_v8(vb, gid, c4);  // the V loads overlap the S contraction and the softmax
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&kr[0][0]);
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&kr[1][0]);
#pragma unroll
      for (int j = 0; j < NKT; ++j) {
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_f16x2x2(w0[j], a0, a2);
        e4m3x4_to_f16x2x2(w1[j], a1, a3);
        if (j & 1)
          mma_16816<false>(sb, a0, a1, a2, a3, qf[j][0], qf[j][1]);
        else
          mma_16816<false>(sa, a0, a1, a2, a3, qf[j][0], qf[j][1]);
      }
    }
    // ---- online softmax (log2 domain); rows of S^T are tokens gid, gid+8
    const float x0 = gid < valid ? (sa[0] + sb[0]) * sl : -INFINITY;
    const float x1 = gid < valid ? (sa[1] + sb[1]) * sl : -INFINITY;
    const float x2 = gid + 8 < valid ? (sa[2] + sb[2]) * sl : -INFINITY;
    const float x3 = gid + 8 < valid ? (sa[3] + sb[3]) * sl : -INFINITY;
    update_max(fmaxf(x0, x2), fmaxf(x1, x3));
    const float p0 = ex2(x0 - m0), p1 = ex2(x1 - m1), p2 = ex2(x2 - m0), p3 = ex2(x3 - m1);
    l0 += p0 + p2;
    l1 += p1 + p3;
    const uint32_t pb0 = movmatrix_trans(pack2<BF16>(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack2<BF16>(p2, p3));
    // ---- O^T += V^T P^T
    if constexpr (!FP8) {
      if (valid == kBS) {
#pragma unroll
        for (int t = 0; t < NDT; ++t) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(vb + tile_off(ri + ((mi >> 1) << 3), (16 * t + ((mi & 1) << 3)) * 2), a0, a1, a2, a3);
          mma_16816<BF16>(o[t], a0, a1, a2, a3, pb0, pb1);
        }
      } else {  // zero V of tokens past the end (they may hold NaN/Inf)
        const uint32_t mlo = (2 * c4 < valid ? 0x0000ffffu : 0u) | (2 * c4 + 1 < valid ? 0xffff0000u : 0u);
        const uint32_t mhi = (2 * c4 + 8 < valid ? 0x0000ffffu : 0u) | (2 * c4 + 9 < valid ? 0xffff0000u : 0u);
#pragma unroll
        for (int t = 0; t < NDT; ++t) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(vb + tile_off(ri + ((mi >> 1) << 3), (16 * t + ((mi & 1) << 3)) * 2), a0, a1, a2, a3);
          mma_16816<BF16>(o[t], a0 & mlo, a1 & mlo, a2 & mhi, a3 & mhi, pb0, pb1);
        }
      }
    } else {
      pv8(valid, pb0, pb1, c4);
    }
  }

  // Full softmax sums of this lane's two columns (l summed over the 16 token rows).
  __device__ __forceinline__ void totals(float& L0, float& L1) const {
    L0 = l0;
    L1 = l1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      L0 += __shfl_xor_sync(0xffffffffu, L0, off);
      L1 += __shfl_xor_sync(0xffffffffu, L1, off);
    }
  }

  // Output dim of (tile t, MMA row half hi) for this lane: 16-bit path
  // 16t + gid + 8hi; fp8 path D/8*gid + 2t + hi.
  __device__ __forceinline__ static int dim(int t, int hi, int gid) {
    if constexpr (!FP8) return 16 * t + gid + 8 * hi;
    else return (D / 8) * gid + 2 * t + hi;
  }
};

// The launch's work hand-out, computed by one warp of every CTA (all 32
// lanes call this) from the clamped lengths: lens[S] and the exclusive prefix
// prefix[S+1] of items (ticket mode) or blocks (stream-K mode) in shared
// memory.  In auto mode the hand-out is chosen from the lengths: near-uniform
// lengths (all within 10 %) -> tickets with large partitions (items finish
// together; the memory system stays saturated), varying lengths -> stream-K
// ranges (no stragglers).  A zero-length sequence is one item with no blocks
// in ticket mode (so its zero output gets written) and has no blocks in
// stream-K mode (the merge kernel writes its zero output).  CTA 0 records the
// choice for the merge kernel.
struct HandOut {
  int pb;       // ticket mode: blocks per partition
  int per_cta;  // stream-K mode: blocks per CTA group
  bool sk;
};
__device__ __forceinline__ HandOut decode_hand_out(const DecodeParams& p, int* prefix, int* lens, int lane) {
  const int S = p.num_seqs;
  int pb = p.partition_blocks, per_cta = 0;
  bool sk = false;

  bool bad = false;
  long long sum_len = 0;
  int min_len = 0x7fffffff, max_len = 0;
  // The lengths (and suffix offsets) of up to 256 sequences are loaded
  // before any is stored to shared memory: loads queued behind each chunk's
  // stores would cost one memory round trip per 32 sequences.
  constexpr int HB = 8;
  for (int b0 = 0; b0 < S; b0 += 32 * HB) {
    int raw[HB], skip[HB];
#pragma unroll
    for (int k = 0; k < HB; ++k) {
      const int s = b0 + 32 * k + lane;
      raw[k] = s < S ? __ldg(p.seq_lens + s) : 0;
      skip[k] = (p.seq_skip && s < S) ? __ldg(p.seq_skip + s) : 0;
    }
#pragma unroll
    for (int k = 0; k < HB; ++k) {
      const int s = b0 + 32 * k + lane;
      if (s < S) {
        int len = clamp_len(raw[k], p);
        bad |= raw[k] != len;
        if (p.seq_skip) len = max(0, len - skip[k] * kBS);  // the private suffix
        lens[s] = len;
        sum_len += len;
        min_len = min(min_len, len);
        max_len = max(max_len, len);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sum_len += __shfl_xor_sync(0xffffffffu, sum_len, off);
    min_len = min(min_len, __shfl_xor_sync(0xffffffffu, min_len, off));
    max_len = max(max_len, __shfl_xor_sync(0xffffffffu, max_len, off));
  }
  if (p.auto_mode) {
    const bool uniform = (long long)min_len * 10 >= (long long)max_len * 9;
    sk = !uniform && (int)gridDim.x >= p.kv_units;
    if (!sk) pb = uniform_partition_blocks(p, sum_len, max_len, gridDim.x);
  }
  __syncwarp();
  // exclusive prefix of the per-sequence counts: 8 chunks of 32 scanned side
  // by side (independent shuffle chains), then chained by their totals
  int carry = 0;
  for (int b0 = 0; b0 < S; b0 += 32 * HB) {
    int x[HB];
#pragma unroll
    for (int k = 0; k < HB; ++k) {
      const int s = b0 + 32 * k + lane;
      int n = 0;
      if (s < S) {
        const int len = lens[s];
        const int nblk = (len + kBS - 1) / kBS;
        if (sk) {
          n = nblk;
        } else {
          bad |= (nblk + pb - 1) / pb > p.max_parts;
          n = max(1, num_partitions(len, pb, p)) * p.kv_units;
        }
      }
      x[k] = n;
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int k = 0; k < HB; ++k) {
        const int y = __shfl_up_sync(0xffffffffu, x[k], off);
        if (lane >= off) x[k] += y;
      }
    }
#pragma unroll
    for (int k = 0; k < HB; ++k) {
      const int s = b0 + 32 * k + lane;
      if (s < S) prefix[s + 1] = carry + x[k];
      carry += __shfl_sync(0xffffffffu, x[k], 31);
    }
  }
  if (lane == 0) prefix[0] = 0;
  if (blockIdx.x == 0 && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, kCheckSeqTooLong);
  if (sk) {
    const int groups = max(1, (int)gridDim.x / p.kv_units);
    per_cta = max(p.min_piece_blocks, (carry + groups - 1) / groups);  // blocks per CTA group
  }
  if (blockIdx.x == 0) {  // each sequence's merge work under this launch's hand-out
    __syncwarp();
    const bool shared = p.seq_skip != nullptr;
    for (int s = lane; s < S; s += 32) {
      const int len = lens[s];
      const int nblk = (len + kBS - 1) / kBS;
      // decode partials: stream-K pieces, or fixed partitions
      const int np = sk ? (nblk == 0 ? 0 : unit_pieces(prefix[s], nblk, per_cta).count) : num_partitions(len, pb, p);
      p.seq_merge[s] = (!shared && sk && nblk == 0) ? kMergeZero : (shared || np > 1) ? np : kMergeNone;
    }
  }
  return {pb, per_cta, sk};
}

// A work item: sequence, partition (piece) index and count, KV unit, block range.
struct Item {
  int s, y, part, np, len, b0, nb, off;  // off: table entries before the suffix
};

// Items of a launch's hand-out (decode_hand_out), as the producer warp of a
// CTA enumerates them.
struct WorkItems {
  const DecodeParams& p;
  const int* prefix;  // [S + 1] (shared memory)
  const int* lens;    // [S]
  int pb, per_cta, sk_group;

  __device__ int last_seq_at(int v) const {  // last s with prefix[s] <= v (skips empty sequences)
    int lo = 0, hi = p.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  // ticket mode: item t of the (sequence, partition, KV unit) enumeration
  __device__ Item ticket(int t) const {
    Item it;
    it.s = last_seq_at(t);
    const int r = t - prefix[it.s];
    it.part = r / p.kv_units;
    it.y = r - it.part * p.kv_units;
    it.len = lens[it.s];
    it.np = max(1, num_partitions(it.len, pb, p));
    const int nblk = (it.len + kBS - 1) / kBS;
    it.b0 = it.part * pb;
    it.nb = max(0, min(nblk, it.b0 + pb) - it.b0);
    it.off = p.seq_skip ? __ldg(p.seq_skip + it.s) : 0;
    return it;
  }
  // stream-K mode: this CTA's KV unit of the sequence under global block g, up to `end`
  __device__ Item streamk(int g, int end) const {
    Item it;
    it.s = last_seq_at(g);
    it.len = lens[it.s];
    const int nblk = (it.len + kBS - 1) / kBS;
    it.y = (int)blockIdx.x - sk_group * p.kv_units;
    it.b0 = g - prefix[it.s];
    it.nb = min(nblk - it.b0, end - g);
    const Pieces pc = unit_pieces(prefix[it.s], nblk, per_cta);
    it.part = sk_group - pc.c0;
    it.np = pc.count;
    it.off = p.seq_skip ? __ldg(p.seq_skip + it.s) : 0;
    return it;
  }
  // Lane j's block-table entry of chunk c (blocks 32c + j) of an item; out-of-pool ids are flagged.
  __device__ int table_chunk(const Item& it, int c, int lane) const {
    const int i = 32 * c + lane;
    int b = 0;
    if (i < it.nb) {
      b = __ldg(p.block_tables + (size_t)it.s * p.bt_stride + it.off + it.b0 + i);
      if (b < 0 || b >= p.num_blocks) {
        atomicOr(p.err, kCheckBadBlock);
        b = 0;
      }
    }
    return b;
  }
};

template <class C>
__global__ void __launch_bounds__(64, C::MIN_CTAS) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const DecodeParams p) {
  using Q = typename C::Q;
  constexpr int D = C::D, NS = C::NS;
  extern __shared__ uint8_t smem_dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.num_seqs;
  // the merge kernel (launched as a programmatic dependent) may be scheduled
  // now; it waits for this grid's completion before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const DecodeLayout L(NS, C::STAGE_BYTES, p.q_slot_bytes);
  const uint32_t base_u32 = smem_u32(smem);
  const uint32_t full0 = base_u32 + L.bar, empty0 = full0 + NS * 8, qfull0 = full0 + 2 * NS * 8, qempty0 = qfull0 + 16;
  const uint32_t never = qempty0 + 16;  // no thread ever arrives on it
  // [0] stages, [1] q slots, [2] timed out, [4] [5] the warps' slots
  volatile int* exitrec = reinterpret_cast<volatile int*>(smem + L.exitrec);
  const long long wl = p.wait_limit;
  int4* meta = reinterpret_cast<int4*>(smem + L.meta);
  int* prefix = reinterpret_cast<int*>(smem + L.prefix);  // [S + 1]
  int* lens = prefix + (S + 1);                             // [S], clamped

  // Roles by scheduler.  The SM gives each warp a slot, slot w is issued
  // from by scheduler w % 4, and the two warps of a CTA take adjacent slots:
  // with warp 0 as the consumer everywhere, all of an SM's consumer warps
  // (the ones doing the math) end up on two of its four schedulers.  The
  // consumer is instead the warp whose slot has bit 0 equal to bit 2, which
  // puts the consumers of four consecutive CTAs on schedulers 0, 2, 1, 3
  // (warp 0 if the rule does not pick exactly one).  Either choice computes
  // the same; only the speed depends on it.
  if (lane == 0) {
    unsigned int w;
    asm volatile("mov.u32 %0, %%warpid;" : "=r"(w));
    exitrec[4 + warp] = (int)w;
  }
  __syncthreads();
  const int slot0 = exitrec[4], slot1 = exitrec[5];
  const bool pick0 = (slot0 & 1) == ((slot0 >> 2) & 1), pick1 = (slot1 & 1) == ((slot1 >> 2) & 1);
  const bool producer = warp != ((pick1 && !pick0) ? 1 : 0);

  int pb = p.partition_blocks, per_cta = 0;
  bool sk = false;
  if (producer) {
    const HandOut h = decode_hand_out(p, prefix, lens, lane);
    pb = h.pb;
    per_cta = h.per_cta;
    sk = h.sk;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecodeBarriers(NS); ++i) mbar_init(full0 + 8 * i, 1);
    fence_mbar_init();
    exitrec[0] = exitrec[1] = exitrec[2] = 0;
  }
  __syncthreads();
  const int total = prefix[S];  // items (ticket mode) or blocks (stream-K mode)
  // Copies this CTA's producer has issued (lane 0 counts): ring stages armed
  // and query slots filled, in order.  After a wait runs out, the ones the
  // consumer did not take are waited for before the CTA exits.
  int armed = 0, q_armed = 0;

  if (producer) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int stage_i = 0, item_i = 0, stop = 0;
    // Claim stage `stage_i` (lane 0): wait until the consumer released its last use.
    auto claim = [&](int& st) -> bool {
      st = stage_i % NS;
      if (stage_i >= NS && !mbar_wait(empty0 + 8 * st, ((stage_i / NS) - 1) & 1, wl)) {
        atomicOr(p.err, kCheckWaitTimeout);
        exitrec[2] = 1;
        return false;
      }
      return true;
    };
    const WorkItems items{p, prefix, lens, pb, per_cta, (int)blockIdx.x / p.kv_units};
    const int sk_group = items.sk_group;
    auto decode = [&](int t) { return items.ticket(t); };
    auto decode_sk = [&](int g, int end) { return items.streamk(g, end); };
    auto load_chunk = [&](const Item& it, int c) { return items.table_chunk(it, c, lane); };
    // Work cursor: a ticket (ticket mode) or a global block index (stream-K
    // mode, over this CTA's range [blockIdx.x * per_cta, g_end)).
    // Software pipeline: the next item's ticket is claimed four blocks before
    // this item's end (late enough to keep the hand-out dynamic, early enough
    // to hide the atomic's latency) and its first block-table chunk is loaded
    // one block later.
    // Stream-K: group g = blockIdx / kv_units covers [g * per_cta, (g + 1) * per_cta)
    // of the (sequence, block) space, each CTA of the group for its own KV unit
    // (CTAs beyond the last whole group get no work).
    const bool sk_idle = sk && sk_group >= max(1, (int)gridDim.x / p.kv_units);
    const int g_end = sk ? (int)min((long long)total, ((long long)sk_group + 1) * per_cta) : 0;
    auto has = [&](int t) { return sk ? (!sk_idle && t < g_end) : t < total; };
    int t_cur = 0, t_next = 0;
    if (sk) {
      t_cur = (int)min((long long)sk_group * per_cta, (long long)total);
    } else {
      if (lane == 0) t_cur = atomicAdd(&p.counters[0], 1);
      t_cur = __shfl_sync(0xffffffffu, t_cur, 0);
    }
    Item cur = {}, nxt = {};
    int chunk = 0, nchunk = 0;
    if (has(t_cur)) {
      cur = sk ? decode_sk(t_cur, g_end) : decode(t_cur);
      chunk = load_chunk(cur, 0);
    }
    while (has(t_cur) && !stop) {
      const int kvh = cur.y / p.head_splits;
      const int hs = cur.y - kvh * p.head_splits;
      const int head0 = kvh * p.group + hs * kNH;
      const int nheads = min(kNH, p.group - hs * kNH);
      const int meta_z = cur.part | (cur.np << 16);
      bool claimed = false, fetched = false;
      // claim / prefetch near the item's end (at once for items shorter than that)
      auto lookahead = [&](int i) {
        if (!claimed && i >= cur.nb - 4) {
          if (!sk && lane == 0) t_next = atomicAdd(&p.counters[0], 1);
          claimed = true;
        }
        if (!fetched && i >= cur.nb - 3) {
          t_next = sk ? t_cur + cur.nb : __shfl_sync(0xffffffffu, t_next, 0);
          if (has(t_next)) {
            nxt = sk ? decode_sk(t_next, g_end) : decode(t_next);
            nchunk = load_chunk(nxt, 0);
          }
          fetched = true;
        }
      };
      if (lane == 0) {  // this item's query rows -> q slot
        const int qs = item_i & 1;
        if (item_i >= 2 && !mbar_wait(qempty0 + 8 * qs, ((item_i >> 1) - 1) & 1, wl)) {
          atomicOr(p.err, kCheckWaitTimeout);
          exitrec[2] = 1;
          stop = 1;
        } else {
          const uint32_t bytes = nheads * D * 2;
          mbar_arrive_expect_tx(qfull0 + 8 * qs, bytes);
          bulk_load(base_u32 + L.q + qs * p.q_slot_bytes,
                    reinterpret_cast<const uint8_t*>(p.query) + ((size_t)cur.s * p.num_heads + head0) * D * 2, bytes,
                    qfull0 + 8 * qs);
          ++q_armed;
        }
      }
      stop = __shfl_sync(0xffffffffu, stop, 0);
      if (stop) break;
      ++item_i;
      if (cur.nb == 0) {  // empty sequence: a metadata-only stage
        if (lane == 0) {
          int st;
          if (!claim(st)) {
            stop = 1;
          } else {
            meta[st] = make_int4(cur.s, cur.y, meta_z, kFirst | kLast);
            mbar_arrive(full0 + 8 * st);
            ++armed;
          }
        }
        ++stage_i;
        stop = __shfl_sync(0xffffffffu, stop, 0);
      }
      const int nchunks = (cur.nb + 31) / 32;
      for (int c = 0; c < nchunks && !stop; ++c) {
        const int ahead = (c + 1 < nchunks) ? load_chunk(cur, c + 1) : 0;
        const int cnt = min(32, cur.nb - 32 * c);
        for (int j = 0; j < cnt; ++j) {
          const int phys = __shfl_sync(0xffffffffu, chunk, j);
          const int i = 32 * c + j;
          if (lane == 0) {
            int st;
            if (!claim(st)) {
              stop = 1;
            } else {
              const int valid = min(kBS, cur.len - (cur.b0 + i) * kBS);
              const int flags = (i == 0 ? kFirst : 0) | (i == cur.nb - 1 ? kLast : 0) | (valid << 8);
              meta[st] = make_int4(cur.s, cur.y, meta_z, flags);
              const uint32_t fb = full0 + 8 * st;
              mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
              const uint32_t kdst = base_u32 + L.ring + st * C::STAGE_BYTES;
              const uint32_t vdst = kdst + C::TILE_BYTES;
              const int yy = phys * kBS;
#pragma unroll
              for (int sub = 0; sub < C::SUBTILES; ++sub) {
                const int x = kvh * D + sub * (128 / (int)sizeof(typename C::KV));
                tma_load_2d(kdst + sub * kBS * 128, &tmK, x, yy, fb);
                tma_load_2d(vdst + sub * kBS * 128, &tmV, x, yy, fb);
              }
              ++armed;
            }
          }
          ++stage_i;
          stop = __shfl_sync(0xffffffffu, stop, 0);
          if (stop) break;
          lookahead(i);
        }
        chunk = ahead;
      }
      lookahead(cur.nb);  // items with no blocks, or a loop cut short
      t_cur = t_next;
      cur = nxt;
      chunk = nchunk;
    }
    if (!stop && lane == 0) {  // end marker
      int st;
      if (claim(st)) {
        meta[st] = make_int4(0, 0, 0, kEnd);
        mbar_arrive(full0 + 8 * st);
        ++armed;
      }
    }
  } else {
    // ---------------------------------------------------------------- consumer
    const int gid = lane >> 2, c4 = lane & 3;
    WarpAttn<D, C::kFp8, C::kBf16> A;
    A.reset();
    int stage_i = 0, item_i = 0;
    int blk = 0;  // block of the current item (fp8 pairing)
    int cur_s = 0, cur_head0 = 0, cur_nheads = 0, cur_part = 0, cur_np = 1;

    while (true) {
      const int st = stage_i % NS;
      // (test hook: the first wait targets the barrier nothing completes)
      const bool stall = p.debug_stall && stage_i == 0;
      // (all lanes wait; the warp leaves together even if the limit ran out
      // for some lanes only)
      if (!__all_sync(0xffffffffu,
                      mbar_wait(stall ? never : full0 + 8 * st, stall ? 0u : (uint32_t)((stage_i / NS) & 1), wl))) {
        atomicOr(p.err, kCheckWaitTimeout);
        exitrec[2] = 1;
        break;
      }
      const int4 md = meta[st];
      if (md.w & kEnd) break;
      if (md.w & kFirst) {
        // new item: its query rows, fresh softmax state
        cur_s = md.x;
        const int kvh = md.y / p.head_splits;
        const int hs = md.y - kvh * p.head_splits;
        cur_head0 = kvh * p.group + hs * kNH;
        cur_nheads = min(kNH, p.group - hs * kNH);
        cur_part = md.z & 0xffff;
        cur_np = md.z >> 16;
        const int qs = item_i & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(qfull0 + 8 * qs, (item_i >> 1) & 1, wl))) {
          atomicOr(p.err, kCheckWaitTimeout);
          exitrec[2] = 1;
          break;
        }
        A.load_q(gid < cur_nheads ? smem + L.q + qs * p.q_slot_bytes + gid * D * 2 : nullptr, c4);
        // the slot's next writer is a bulk copy (async proxy): order these
        // generic-proxy reads before it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qempty0 + 8 * qs);
        ++item_i;
        A.reset();
      }
      const int valid = (md.w >> 8) & 0xff;
      if (md.w & kFirst) blk = 0;
      // fp8: blocks 2k and 2k+1 of an item go through one step (one softmax
      // update for 32 tokens).  The pairing depends only on the block's
      // position in its item, so results do not depend on timing.
      bool two = false;
      int st2 = 0;
      if constexpr (C::kFp8) {
        if (!(md.w & kLast) && !(blk & 1)) {
          st2 = (stage_i + 1) % NS;
          if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * st2, ((stage_i + 1) / NS) & 1, wl))) {
            atomicOr(p.err, kCheckWaitTimeout);
            exitrec[2] = 1;
            break;
          }
          two = true;
        }
      }
      blk += two ? 2 : 1;
      int last = md.w & kLast;
      if (two) {
        const int4 md2 = meta[st2];
        const uint32_t kb = base_u32 + L.ring + st * C::STAGE_BYTES;
        const uint32_t kb2 = base_u32 + L.ring + st2 * C::STAGE_BYTES;
        A.block2(kb, kb + C::TILE_BYTES, kb2, kb2 + C::TILE_BYTES, (md2.w >> 8) & 0xff, p.scale_log2, lane);
        fence_proxy_async_smem();  // (the stages' next writer is TMA)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(empty0 + 8 * st);
          mbar_arrive(empty0 + 8 * st2);
        }
        stage_i += 2;
        last = md2.w & kLast;
      } else {
        if (valid > 0) {
          const uint32_t kb = base_u32 + L.ring + st * C::STAGE_BYTES;
          A.block(kb, kb + C::TILE_BYTES, valid, p.scale_log2, lane);
        }
        fence_proxy_async_smem();  // (the stage's next writer is TMA)
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * st);
        ++stage_i;
      }

      if (last) {
        // ---- finish the item straight from registers; lane (gid, c4) holds
        // heads 2c4, 2c4+1 of 2 dims per tile
        float L0, L1;
        A.totals(L0, L1);
        const int h0 = 2 * c4, h1 = 2 * c4 + 1;
        const float i0 = L0 > 0.f ? p.v_scale / L0 : 0.f;
        const float i1 = L1 > 0.f ? p.v_scale / L1 : 0.f;
        const bool ok0 = h0 < cur_nheads, ok1 = h1 < cur_nheads;
        if (cur_np == 1 && !p.force_partials) {
          Q* d0 = reinterpret_cast<Q*>(p.out) + ((size_t)cur_s * p.num_heads + cur_head0 + h0) * D;
          Q* d1 = d0 + D;
#pragma unroll
          for (int t = 0; t < C::NDT; ++t) {
            if (ok0) {
              d0[A.dim(t, 0, gid)] = Q(A.o[t][0] * i0);
              d0[A.dim(t, 1, gid)] = Q(A.o[t][2] * i0);
            }
            if (ok1) {
              d1[A.dim(t, 0, gid)] = Q(A.o[t][1] * i1);
              d1[A.dim(t, 1, gid)] = Q(A.o[t][3] * i1);
            }
          }
        } else {
          const size_t row0 = ((size_t)cur_s * p.num_heads + cur_head0 + h0) * p.max_parts + cur_part;
          const size_t row1 = row0 + p.max_parts;
          store_partial<D, C::kFp8>(A.o, A.m0, L0, i0, ok0, A.m1, L1, i1, ok1, p.part_o, p.part_ml, row0, row1,
                                    lane);
        }
      }
    }
    if (lane == 0) {  // what this warp took, for the timeout exit below
      exitrec[0] = stage_i;
      exitrec[1] = item_i;
    }
  }

  __syncthreads();
  // After a wait ran out, the consumer stopped taking stages while TMA and
  // bulk copies the producer issued may still be landing in this CTA's shared
  // memory: wait (bounded by the default limit) for every stage and query slot
  // armed but not taken, so that no copy outlives the CTA.  At most NS stages
  // and 2 slots are outstanding, each in its own ring position.
  if (producer && lane == 0 && exitrec[2]) {
    for (int k = exitrec[0]; k < armed; ++k) mbar_wait(full0 + 8 * (k % NS), (k / NS) & 1);
    for (int i = exitrec[1]; i < q_armed; ++i) mbar_wait(qfull0 + 8 * (i & 1), (i >> 1) & 1);
  }
  // the last CTA to finish resets the counters for the next launch
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&p.counters[1], 1);
    if (prev == (int)gridDim.x - 1) {
      atomicExch(&p.counters[0], 0);
      atomicExch(&p.counters[1], 0);
      __threadfence();
    }
  }
}

// Log-sum-exp merge of split sequences.  A CTA of 256 threads covers
// `merge_hpc` consecutive query heads of one sequence; its threads are
// (head, partition slice, 4-dim chunk) triples, `merge_slices` slices taking
// every merge_slices-th partial.  Each thread folds its partials into a
// running (max M, weight sum W, weighted sum) in one pass, four partials'
// loads in flight (few registers, so that a whole batch's merge CTAs are
// resident at once), and the slices are folded together in shared memory
// with the same rule; out = weighted sum / W.  A head's partials are the
// decode pass's np partitions, followed, in shared-prefix decode, by the
// prefix pass's chunks; np comes from the decode kernel (seq_merge), read in
// one load.  Launched as a programmatic dependent of the decode kernel: it
// may be scheduled early and waits for the decode grid to finish before
// reading.
template <typename Q, int D, bool BF16>
__global__ void __launch_bounds__(256, 4) paged_decode_merge_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int CH = D / 4;  // float4 chunks per head
  constexpr int B = 4;       // partials per batch
  __shared__ float4 red[256];
  __shared__ float2 redm[256];
  const int hpc = p.merge_hpc, slices = p.merge_slices;
  const int hblocks = (p.num_heads + hpc - 1) / hpc;
  const int s = blockIdx.x / hblocks;
  const int h0 = (blockIdx.x - s * hblocks) * hpc;
  const bool shared = p.seq_skip != nullptr;
  const int code = p.seq_merge[s];
  const int skip = shared ? p.seq_skip[s] : 0;
  if (code == kMergeNone) return;  // written by the decode kernel
  if (code == kMergeZero) {        // empty sequence: zero rows (no decode item covered it)
    for (int i = threadIdx.x; i < hpc * D; i += blockDim.x) {
      const int h = h0 + i / D;
      if (h < p.num_heads) reinterpret_cast<Q*>(p.out)[((size_t)s * p.num_heads + h) * D + i % D] = Q(0.0f);
    }
    return;
  }
  const int np = code;
  const int nc = shared ? (skip + kPrefixChunkBlocks - 1) / kPrefixChunkBlocks : 0;  // prefix partials
  const int nt = np + nc;
  // partial q of head h: decode partition q < np, else prefix chunk q - np
  auto ml_of = [&](int h, int q) -> const float* {
    return q < np ? p.part_ml + (((size_t)s * p.num_heads + h) * p.max_parts + q) * 2
                  : p.pre_ml + (((size_t)s * p.num_heads + h) * p.max_chunks + (q - np)) * 2;
  };
  auto o_of = [&](int h, int q) -> const float* {
    return q < np ? p.part_o + (((size_t)s * p.num_heads + h) * p.max_parts + q) * D
                  : p.pre_o + (((size_t)s * p.num_heads + h) * p.max_chunks + (q - np)) * D;
  };
  const int c = threadIdx.x % CH;
  const int rest = threadIdx.x / CH;
  // fold a summary (m, w, a4), w = sum l 2^(m_q - m) and a4 = sum l 2^(m_q - m) o_q, into (M, W, acc)
  auto fold = [](float& M, float& W, float4& acc, float m, float w, const float4& a4) {
    if (!(w > 0.f)) return;
    const float mn = fmaxf(M, m);
    const float a = ex2(M - mn), b = ex2(m - mn);
    acc.x = fmaf(b, a4.x, acc.x * a);
    acc.y = fmaf(b, a4.y, acc.y * a);
    acc.z = fmaf(b, a4.z, acc.z * a);
    acc.w = fmaf(b, a4.w, acc.w * a);
    W = fmaf(W, a, w * b);
    M = mn;
  };
  auto write = [&](int h, const float4& acc, float W) {
    const float inv = W > 0.f ? 1.f / W : 0.f;  // no weighted partial: a zero row
    Q* dst = reinterpret_cast<Q*>(p.out) + ((size_t)s * p.num_heads + h) * D + 4 * c;
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack2<BF16>(acc.x * inv, acc.y * inv), pack2<BF16>(acc.z * inv, acc.w * inv));
  };
  if (p.merge_hpt == 2) {
    // one slice, two heads per thread (rest and rest + hpass of the CTA's
    // heads): both heads' partial loads in flight together, two partials of
    // each per batch
    const int hpass = (int)blockDim.x / CH;
    const int ha = h0 + rest, hb = h0 + rest + hpass;
    const bool aa = rest < hpc && ha < p.num_heads, ab = rest + hpass < hpc && hb < p.num_heads;
    float Ma = -INFINITY, Wa = 0.f, Mb = -INFINITY, Wb = 0.f;
    float4 acca = make_float4(0.f, 0.f, 0.f, 0.f), accb = acca;
    for (int q0 = 0; q0 < nt; q0 += 2) {
      float2 mlq[4];
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // u: (head b?, partial q0 + (u & 1))
        const int q = q0 + (u & 1);
        const bool isb = u >> 1;
        const bool ok = q < nt && (isb ? ab : aa);
        const int hh = isb ? hb : ha;
        mlq[u] = ok ? *reinterpret_cast<const float2*>(ml_of(hh, q)) : make_float2(-INFINITY, 0.f);
        v[u] = ok ? *reinterpret_cast<const float4*>(o_of(hh, q) + 4 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // a partial (o, m, l) is the summary (m, l, l o)
        const float l = mlq[u].y;
        const float4 a4 = make_float4(l * v[u].x, l * v[u].y, l * v[u].z, l * v[u].w);
        if (u >> 1) fold(Mb, Wb, accb, mlq[u].x, l, a4);
        else fold(Ma, Wa, acca, mlq[u].x, l, a4);
      }
    }
    if (aa) write(ha, acca, Wa);
    if (ab) write(hb, accb, Wb);
    return;
  }
  const int slice = rest % slices, hl = rest / slices;
  const int h = h0 + hl;
  const bool active = hl < hpc && h < p.num_heads;
  float M = -INFINITY, W = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // fold in a summary (m, w, a4) with w = sum l 2^(m_q - m) and a4 = sum l 2^(m_q - m) o_q
  auto combine = [&](float m, float w, const float4& a4) {
    if (!(w > 0.f)) return;
    const float mn = fmaxf(M, m);
    const float a = ex2(M - mn), b = ex2(m - mn);
    acc.x = fmaf(b, a4.x, acc.x * a);
    acc.y = fmaf(b, a4.y, acc.y * a);
    acc.z = fmaf(b, a4.z, acc.z * a);
    acc.w = fmaf(b, a4.w, acc.w * a);
    W = fmaf(W, a, w * b);
    M = mn;
  };
  if (active) {
    for (int q0 = slice; q0 < nt; q0 += B * slices) {
      float2 mlq[B];
      float4 v[B];
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int q = q0 + u * slices;
        const bool ok = q < nt;
        mlq[u] = ok ? *reinterpret_cast<const float2*>(ml_of(h, q)) : make_float2(-INFINITY, 0.f);
        v[u] = ok ? *reinterpret_cast<const float4*>(o_of(h, q) + 4 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < B; ++u) {  // a partial (o, m, l) is the summary (m, l, l o)
        const float l = mlq[u].y;
        combine(mlq[u].x, l, make_float4(l * v[u].x, l * v[u].y, l * v[u].z, l * v[u].w));
      }
    }
  }
  if (slices > 1) {
    red[threadIdx.x] = acc;
    redm[threadIdx.x] = make_float2(M, W);
    __syncthreads();
    if (slice == 0 && active) {
      for (int k = 1; k < slices; ++k) {
        const float2 mw = redm[threadIdx.x + k * CH];
        combine(mw.x, mw.y, red[threadIdx.x + k * CH]);
      }
    }
  }
  if (slice == 0 && active) write(h, acc, W);
}

}  // namespace pa
