// Shared-prefix pass of decode attention.
//
// Sequences forked from one prompt share the physical blocks of that prompt
// (page "5.KV Cache 管理 & PagedAttention", Q18 fork: the child's block table
// is a copy of the parent's and every shared block's reference count goes up;
// page "paged-attention-and-vllm-inference", prefix caching: a cached
// prefix's blocks are reused by later requests).  Attention over a shared
// block is the same K/V against each member's query, so this pass loads every
// shared block once and scores it for all members at once; the members'
// private suffixes go through the regular decode kernel, and the merge kernel
// combines the two sets of (o, m, l) partials by log-sum-exp.
//
// With all members' query heads of one KV head stacked, attention over the
// prefix is a dense contraction: for a step of T = 32 tokens (SB = 2 blocks),
// S[128 rows x T] = Q K^T, then O[128 x D] += P V.  Both run on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// one CTA per (group, KV unit, 128 query rows, chunk of 32 prefix blocks).
// The core, `stacked_attention`, is shared with the multi-query (prefill)
// kernel.  It keeps B step buffers (a step's K and V operands in shared
// memory, 128-byte swizzled, K K-major and V MN-major; its S, then P, in
// tensor memory); its roles:
//   warps 4..7  one loading warp per step buffer: wait for the P V that last
//               read the buffer, fill the step's K and V operands from the
//               cache (16-bit: 16-byte cp.async straight into the operand;
//               fp8: from the warp's raw staging slot, fetched with cp.async
//               while it waited, converted to f16), write zero V rows past
//               the valid keys, and issue the step's S (lane 0; a thread
//               issues a tcgen05.mma only every ~80 cycles, so the steps' S
//               come from four threads);
//   warp 8      issues O += P V for a step once the softmax has written its
//               P (P read from tensor memory as the A operand);
//   warps 0..3  one query row per thread: read the step's S row from TMEM,
//               online softmax in the log2 domain (lazy: O is rescaled in
//               TMEM only when a row's maximum grows by more than 2^8), write
//               P (16-bit pairs) back over the first T/2 columns of the same
//               S buffer; at the end read O, normalise, hand the row to the
//               caller's store.
#pragma once

#include "decode.cuh"
#include "umma.cuh"

namespace pa {

enum : int { kCheckBadPrefix = 16 };

struct PrefixParams {
  const void* query;               // [S, Hq, D]
  const void* k_cache;             // [num_blocks, 16, Hkv, D]
  const void* v_cache;
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

constexpr int kPrefixRows = 128;  // query rows per CTA (the MMA M)


// Shared memory per SM, for capping residency.
constexpr int kSmemPerSM = 233472;

template <int D_, typename KV_, typename Q_, int SB_, int B_>
struct PrefixCfg {
  static constexpr int D = D_;
  using KV = KV_;
  using Q = Q_;
  static constexpr int SB = SB_;   // blocks per step
  static constexpr int T = SB * kBS;  // tokens per step (the S MMA's N, the P V MMA's K)
  static constexpr int B = B_;     // step buffers (S and P in TMEM, K and V in shared memory): how far the steps run ahead
  static constexpr int NW = B < 4 ? B : 4;  // loading warps: one per step buffer
  static constexpr bool kFp8 = sizeof(KV) == 1;
  static constexpr bool kBf16 = std::is_same<Q, __nv_bfloat16>::value;
  static constexpr int ROW_BYTES = D * (int)sizeof(KV);  // one token's K (or V) row of one KV head in the cache
  static constexpr int CH = ROW_BYTES / 16;               // its 16-byte chunks
  // Step buffer layout (both K and V, 16-bit operands, 128-byte
  // swizzle): [D / 64 sub-tiles][T rows x 128 B], so that a sub-tile is a
  // K-major (K) or MN-major (V) MMA operand with 8-row atoms 1024 bytes apart.
  static constexpr int BUF_SUB = T * 128;          // bytes between a step buffer's sub-tiles
  static constexpr int BUF_BYTES = T * D * 2;      // one step buffer of K or V
  static constexpr int Q_BYTES = kPrefixRows * D * 2;  // 128-byte swizzled, D/64 sub-tiles of 128 rows
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;    // [B] step buffers
  static constexpr int OFF_V = OFF_K + B * BUF_BYTES;
  // fp8: each loading warp's raw staging of one step (its K rows, then its V rows, cache layout)
  static constexpr int RAW_BYTES = kFp8 ? 2 * T * ROW_BYTES : 0;
  static constexpr int OFF_RAW = OFF_V + B * BUF_BYTES;  // [NW]
  static constexpr int OFF_BAR = OFF_RAW + NW * RAW_BYTES;
  // s_full[B] p_full[B] pv_done[B] fin q_ready
  static constexpr int NBARS = 3 * B + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;  // tmem base, dead flag
  static constexpr int TMEM_COLS = D + B * T <= 128 ? 128 : (D + B * T <= 256 ? 256 : 512);
  // O: D columns; S buffers: T columns each, a step's P over the first T/2 of its buffer
  static constexpr int O_COL = 0, S_COL = D;
  static constexpr int MAX_CTAS = 512 / TMEM_COLS;  // CTAs whose TMEM fits one SM
  static constexpr int LAYOUT_BYTES = 1024 + OFF_MISC + 16;
  // at least this much shared memory, so that no more than MAX_CTAS CTAs are resident
  static constexpr int MIN_BYTES = kSmemPerSM / (MAX_CTAS + 1) + 1024;
  static constexpr int SMEM_BYTES = LAYOUT_BYTES > MIN_BYTES ? LAYOUT_BYTES : MIN_BYTES;
  static constexpr int THREADS = 288;  // softmax warps 0..3, loading warps 4..7, P V warp 8
  // register budget: as many CTAs per SM as tensor and shared memory allow, up to two
  static constexpr int SMEM_CTAS = kSmemPerSM / (SMEM_BYTES + 1024);
  static constexpr int FIT_CTAS = MAX_CTAS < SMEM_CTAS ? MAX_CTAS : SMEM_CTAS;
  static constexpr int REG_CTAS = FIT_CTAS < 2 ? FIT_CTAS : 2;
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle spans");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  static_assert(T % 32 == 0 && T <= 256, "step tokens (P is stored 16 columns at a time)");
  static_assert(B % NW == 0 && SB <= 32, "each step buffer has one loading warp");
  static_assert(!kFp8 || std::is_same<Q, __half>::value, "fp8 caches pair with fp16 queries");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  // byte offset of (row, byte-in-row) in a 128-byte-swizzled tile of `rows` rows
  __device__ static uint32_t sw128(int rows, int row, int byte) {
    return (uint32_t)((byte >> 7) * (rows * 128) + row * 128 + (((((byte & 127) >> 4) ^ (row & 7)) << 4) | (byte & 15)));
  }
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

// A block range's contribution to 128 stacked query rows on the tensor
// cores (the roles described at the top of this file).  `job` names the
// range: the block-table entries of its nb blocks, the number of its tokens
// that exist (later ones are masked and their V zeroed) and the KV head.
// `rows` maps the CTA's 128 rows to queries and outputs:
//   const void* q_row(r)          query row (16-bit, D values) or nullptr (zero row)
//   int limit(r)                  keys of the range row r sees (a prefix of it)
//   void store(r, c0, v[16])      normalised output dims c0..c0+15 (times v_scale)
//   void store_ml(r, m, l)        the row's max (log2 units) and sum
// Called by all C::THREADS threads of the CTA; returns after tensor memory is freed.
struct StackedJob {
  const int32_t* table;  // nb block ids
  int nb;
  int kv_valid;          // tokens 0..kv_valid-1 of the range exist
  int num_blocks;        // physical pool size (ids outside it are flagged and replaced by block 0)
  const uint8_t* k_head;  // this KV head's row of token 0 of block 0 in the K and V caches
  const uint8_t* v_head;
  size_t row_stride;      // bytes between consecutive token rows of the cache
};

template <class C, class Rows>
__device__ __forceinline__ void stacked_attention(const StackedJob& job, const Rows& rows, float scale_log2,
                                                  float v_scale, int* err) {
  constexpr int D = C::D, B = C::B, SB = C::SB, T = C::T, NW = C::NW, CH = C::CH;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_u32(smem);
  const uint32_t sfull0 = base + C::OFF_BAR, pfull0 = sfull0 + 8 * B, pvdone0 = pfull0 + 8 * B, fin = pvdone0 + 8 * B,
                 qready = fin + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* dead = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = job.nb;
  const int nsteps = (nb + SB - 1) / SB;

  // ---- set-up: barriers, tensor memory, the query tile (128-byte swizzled):
  // its copies are in flight while the loading warps start on the first
  // steps' K and V; only the first S waits for it
  if (threadIdx.x == 0) {
    for (int i = 0; i < B; ++i) {
      mbar_init(sfull0 + 8 * i, 1);  // tcgen05.commit after the step's S
      mbar_init(pfull0 + 8 * i, 4);  // the four softmax warps
      mbar_init(pvdone0 + 8 * i, 1);  // tcgen05.commit after the step's P V
    }
    mbar_init(fin, 1 + NW);  // the MMA-issuing threads: the loading warps' (S) and warp 8's (P V)
    mbar_init(qready, 4);    // the query tile has landed (the four softmax warps' rows)
    *dead = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp < 4) {  // row r's D values: every 16-byte chunk in flight at once (cp.async)
    const int r = threadIdx.x;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(rows.q_row(r));
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint32_t dst = base + C::OFF_Q + C::sw128(kPrefixRows, r, 16 * c);
      if (src)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + 16 * c) : "memory");
      else
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < 4) {  // (barrier initialisation is visible to every thread by now)
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    fence_proxy_async_smem();  // this thread's query row -> visible to the tensor core
    __syncwarp();
    if (lane == 0) mbar_arrive(qready);
  }

  // A failed (timed-out) wait marks the CTA dead: every role then stops at
  // its next wait that does not complete at once.
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*dead) return false;
    if (mbar_wait(bar, parity)) return true;
    atomicOr(err, kCheckWaitTimeout);
    *dead = 1;
    return false;
  };
  // The same, voted across the warp, for waits that all 32 lanes make: the
  // warp takes the failure path together even if the limit ran out for some
  // lanes only (they meet again at warp-wide operations further on).
  auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, wait(bar, parity));
  };

  if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------------- loads, S
    // Step u (tokens u*T .. u*T+T-1 of the range) uses step buffer cb = u % B
    // (its K and V operands in shared memory, its S and P in TMEM), which
    // step u - B used: that step's P V must have completed.  Loading warp
    // w < NW takes the steps u = w mod NW, one at a time: it fills the
    // step's K and V operands, waits for its own copies, and its lane 0
    // issues the step's S (one thread issues a tcgen05.mma only every ~80
    // cycles, so the steps' S come from NW threads).  The buffers thus
    // refill independently of each other; every buffer has one loading warp,
    // which therefore never waits on a barrier more than one phase ahead.
    // Lane l moves the cache's 16-byte chunks l, l + 32, ... of the step's T
    // rows (consecutive lanes: consecutive chunks of a row):
    //   16-bit: straight into the operand (cp.async);
    //   fp8: into the warp's raw staging slot (cp.async), as soon as the
    //   warp has converted its previous step, so that the fetch overlaps the
    //   wait for the step's buffer; then converted to f16 (exact) into the
    //   operand.
    // V rows past the valid keys become zeros (P is 0 there, and 0 * garbage
    // could be NaN); so do the K rows of blocks past the range (masked).
    constexpr int PER = T * CH / 32;  // chunks per lane per tensor and step
    static_assert(T * CH % 32 == 0, "whole chunks per lane");
    constexpr uint32_t idS = umma_idesc_f16(kPrefixRows, T, C::kBf16);
    const uint32_t qa = base + C::OFF_Q;
    const int w = warp - 4;
    // block-table entries of a step: lane j < SB holds block u * SB + j
    auto table_entry = [&](int u) -> int {
      const int i = u * SB + lane;
      int phys = 0;
      if (lane < SB && i < nb) {
        phys = __ldg(job.table + i);
        if (phys < 0 || phys >= job.num_blocks) {
          atomicOr(err, kCheckBadBlock);
          phys = 0;
        }
      }
      return phys;
    };
    int entry = w < NW && w < nsteps ? table_entry(w) : 0;
    // 16-bit interior steps: lane l's chunks k = 0..PER-1 are row lrow + RPK k
    // of the step, 16-byte chunk lcc of the row (RPK = 32 / CH rows per k, so
    // chunk k lies in block (RPK k) / 16 whatever the lane); the cache offset
    // within a block and the shared-memory offset are per-lane constants plus
    // compile-time terms, the swizzle term cycling with period 8 / RPK
    constexpr int RPK = 32 / CH;
    static_assert(C::kFp8 || (32 % CH == 0 && 8 % RPK == 0), "whole rows per chunk index");
    constexpr int NXT = 8 / RPK;
    const int lrow = lane / CH, lcc = lane % CH;
    const uint32_t lsrc = (uint32_t)lrow * (uint32_t)job.row_stride + 16u * lcc;
    const uint32_t lbase = (uint32_t)((lcc >> 3) * (T * 128) + lrow * 128);
    uint32_t xt[NXT];
#pragma unroll
    for (int i = 0; i < NXT; ++i) xt[i] = (uint32_t)(((lcc & 7) ^ ((lrow + RPK * i) & 7)) << 4);
    bool q_landed = false;
    // fp8: step u's K rows (blocks of the range) and V rows (valid tokens)
    // into this warp's raw staging slot, cache layout; lane l: chunks l, l + 32, ...
    auto fetch_raw = [&](int u) {
      const uint32_t raw = base + C::OFF_RAW + w * C::RAW_BYTES;
      int ph[SB];  // the step's block ids (one shuffle per block)
#pragma unroll
      for (int j = 0; j < SB; ++j) ph[j] = __shfl_sync(0xffffffffu, entry, j);
      const bool interior = (u + 1) * SB <= nb && (u + 1) * T <= job.kv_valid;  // every block and row present
#pragma unroll
      for (int kq = 0; kq < 2 * PER; ++kq) {
        const int which = kq >= PER, c = lane + 32 * (kq - which * PER);
        const int row = c / CH, cc = c % CH, j = row / kBS, r = row % kBS;
        const int phys = ph[j];
        const size_t src = ((size_t)phys * kBS + r) * job.row_stride + 16 * cc;
        const bool have = interior || (which ? u * T + row < job.kv_valid : u * SB + j < nb);
        if (have)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(raw + which * (T * C::ROW_BYTES) +
                                                                      row * C::ROW_BYTES + 16 * cc),
                       "l"((which ? job.v_head : job.k_head) + src) : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if constexpr (C::kFp8) {
      if (w < NW && w < nsteps) {
        fetch_raw(w);
        if (w + NW < nsteps) entry = table_entry(w + NW);
      }
    }
#pragma unroll 1
    for (int u = w; w < NW && u < nsteps; u += NW) {
      const int cb = u % B;
      if (u >= B && !wait_all(pvdone0 + 8 * cb, ((u - B) / B) & 1)) break;  // step u - B is done with the buffer
      const uint32_t kbuf = base + C::OFF_K + cb * C::BUF_BYTES, vbuf = base + C::OFF_V + cb * C::BUF_BYTES;
      if constexpr (!C::kFp8) {
        int ph[SB];  // the step's block ids (one shuffle per block)
#pragma unroll
        for (int j = 0; j < SB; ++j) ph[j] = __shfl_sync(0xffffffffu, entry, j);
        if ((u + 1) * SB <= nb && (u + 1) * T <= job.kv_valid) {
          // interior step: every block and every row exists
          const uint8_t* kb[SB];
          const uint8_t* vb[SB];
#pragma unroll
          for (int j = 0; j < SB; ++j) {
            const size_t b = (size_t)ph[j] * kBS * job.row_stride + lsrc;
            kb[j] = job.k_head + b;
            vb[j] = job.v_head + b;
          }
#pragma unroll
          for (int k = 0; k < PER; ++k) {
            const int j = (RPK * k) / kBS, ro = (RPK * k) % kBS;  // block, row offset beyond lrow (compile-time)
            const uint32_t so = (uint32_t)ro * (uint32_t)job.row_stride;
            const uint32_t off = lbase + RPK * k * 128 + xt[k % NXT];
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(kbuf + off), "l"(kb[j] + so)
                         : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(vbuf + off), "l"(vb[j] + so)
                         : "memory");
          }
        } else {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int c = lane + 32 * k;
          const int row = c / CH, cc = c % CH;  // token u * T + row of the range, 16-byte chunk cc
          const int j = row / kBS, r = row % kBS;
          const int phys = ph[j];
          const uint32_t off = C::sw128(T, row, 16 * cc);
          const size_t src = ((size_t)phys * kBS + r) * job.row_stride + 16 * cc;
          if (u * SB + j < nb)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(kbuf + off), "l"(job.k_head + src)
                         : "memory");
          else
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(kbuf + off), "r"(0u) : "memory");
          if (u * T + row < job.kv_valid)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(vbuf + off), "l"(job.v_head + src)
                         : "memory");
          else
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vbuf + off), "r"(0u) : "memory");
        }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (u + NW < nsteps) entry = table_entry(u + NW);  // (in flight while the copies land)
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      } else {
        // the step's raw rows were fetched into this warp's staging slot ahead of time
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        const uint32_t raw = base + C::OFF_RAW + w * C::RAW_BYTES;
        // chunks read in batches of up to 16 (independent loads in flight), then converted and stored
        constexpr int NB = 2 * PER < 16 ? 2 * PER : 16;
        static_assert((2 * PER) % NB == 0, "whole batches");
        const bool interior = (u + 1) * SB <= nb && (u + 1) * T <= job.kv_valid;  // every block and row present
#pragma unroll
        for (int b0 = 0; b0 < 2 * PER; b0 += NB) {
          uint4 v[NB];
#pragma unroll
          for (int q = 0; q < NB; ++q) {
            const int kq = b0 + q, which = kq >= PER, c = lane + 32 * (kq - which * PER);
            const int row = c / CH, cc = c % CH;
            v[q] = lds128(raw + which * (T * C::ROW_BYTES) + row * C::ROW_BYTES + 16 * cc);
          }
#pragma unroll
          for (int q = 0; q < NB; ++q) {
            const int kq = b0 + q, which = kq >= PER, c = lane + 32 * (kq - which * PER);
            const int row = c / CH, cc = c % CH, j = row / kBS;
            const bool have = interior || (which ? u * T + row < job.kv_valid : u * SB + j < nb);
            uint32_t h[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (have) {
              e4m3x4_to_f16x2x2(v[q].x, h[0], h[1]);
              e4m3x4_to_f16x2x2(v[q].y, h[2], h[3]);
              e4m3x4_to_f16x2x2(v[q].z, h[4], h[5]);
              e4m3x4_to_f16x2x2(v[q].w, h[6], h[7]);
            }
            const uint32_t dst = which ? vbuf : kbuf;
            sts128(dst + C::sw128(T, row, 32 * cc), make_uint4(h[0], h[1], h[2], h[3]));
            sts128(dst + C::sw128(T, row, 32 * cc + 16), make_uint4(h[4], h[5], h[6], h[7]));
          }
        }
      }
      fence_proxy_async_smem();  // this lane's operand writes -> visible to the tensor core
      __syncwarp();
      if (!q_landed) {  // the query tile, once
        if (!wait_all(qready, 0)) break;
        q_landed = true;
      }
      if (lane == 0) {  // S = Q K^T of step u into S buffer cb, over 16-wide slices of D
        tc_fence_after();
        // a slice's descriptor is the operand's with its byte offset / 16 added to the start-address field
        const uint64_t a0 = umma_desc(qa, 16, 1024, kUmmaSwizzle128), b0 = umma_desc(kbuf, 16, 1024, kUmmaSwizzle128);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = a0 + (uint64_t)((((k >> 2) * (kPrefixRows * 128) + (k & 3) * 32)) >> 4);
          const uint64_t b = b0 + (uint64_t)((((k >> 2) * C::BUF_SUB + (k & 3) * 32)) >> 4);
          umma_f16(tmem + C::S_COL + cb * T, a, b, idS, k > 0);
        }
        umma_commit(sfull0 + 8 * cb);
      }
      if constexpr (C::kFp8) {  // this warp's next step: its raw rows land while that step waits for its buffer
        if (u + NW < nsteps) {
          fetch_raw(u + NW);
          if (u + 2 * NW < nsteps) entry = table_entry(u + 2 * NW);
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight when the CTA exits
    if (w < NW && lane == 0) {  // every MMA this thread issued has completed before tensor memory is released
      umma_commit(fin);
      mbar_wait(fin, 0);
    }
  } else if (warp == 8) {
    // ---------------------------------------------------------------- P V issue
    // O += P V for each step once the softmax has written its P (P read
    // from tensor memory as the A operand, V MN-major from the step's
    // buffer); the commit frees the step buffer.
    if (lane == 0) {
      constexpr uint32_t idO = umma_idesc_f16(kPrefixRows, D, C::kBf16, /*b_mn_major=*/true);
#pragma unroll 1
      for (int u = 0; u < nsteps; ++u) {
        const int cb = u % B;
        if (!wait(pfull0 + 8 * cb, (u / B) & 1)) break;
        tc_fence_after();
        const uint32_t pt = tmem + C::S_COL + cb * T;
        const uint32_t va = base + C::OFF_V + cb * C::BUF_BYTES;
        const uint64_t v0 = umma_desc(va, C::BUF_SUB, 1024, kUmmaSwizzle128);
#pragma unroll
        for (int k = 0; k < T / 16; ++k) {  // 16-token slices (one block each)
          const uint64_t b = v0 + (uint64_t)((k * (kBS * 128)) >> 4);
          umma_f16_ts(tmem + C::O_COL, pt + 8 * k, b, idO, (u > 0 || k > 0) ? 1 : 0);
        }
        umma_commit(pvdone0 + 8 * cb);
      }
      umma_commit(fin);  // every MMA this thread issued has completed before tensor memory is released
      mbar_wait(fin, 0);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax (warps 0..3)
    const int r = threadIdx.x;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lanes
    const int lim = min(rows.limit(r), job.kv_valid);  // keys this row sees, from the range start
    const int wlim = __reduce_min_sync(0xffffffffu, lim);  // the warp's fewest
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int u = 0; u < nsteps && ok; ++u) {
      const int cb = u % B;
      ok = wait_all(sfull0 + 8 * cb, (u / B) & 1);
      if (!ok) break;
      tc_fence_after();
      // The step's T scores, TC at a time in registers: with T > TC a first
      // pass over the chunks (last to first) takes the maximum, a second
      // (first to last, the first chunk still in registers) the exponentials.
      constexpr int TC = T < 32 ? T : 32, NCH = T / TC;
      static_assert(T % TC == 0, "whole chunks");
      const int valid = min(T, lim - u * T);  // keys of this step the row sees
      // Steps before the diagonal, where every row of the warp sees every key
      // and the scale is positive, take the max of the raw scores and fold
      // the scale into the exponent's FMA; the others scale and mask first.
      const bool plain = scale_log2 > 0.f && wlim >= (u + 1) * T;  // (every row of the warp sees every key)
      const float xs = plain ? scale_log2 : 1.f;  // exponent = x * xs - m
      float x[TC];
      auto load = [&](int ch) {
        if constexpr (TC == 32) {
          uint32_t sv[32];
          tmem_ld32(trow + C::S_COL + cb * T + ch * TC, sv);
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(sv[j]);
        } else {
#pragma unroll
          for (int c0 = 0; c0 < TC; c0 += 16) {
            uint32_t sv[16];
            tmem_ld16(trow + C::S_COL + cb * T + ch * TC + c0, sv);
#pragma unroll
            for (int j = 0; j < 16; ++j) x[c0 + j] = __uint_as_float(sv[j]);
          }
        }
        tmem_wait_ld();
        if (!plain) {
#pragma unroll
          for (int j = 0; j < TC; ++j) x[j] = ch * TC + j < valid ? x[j] * scale_log2 : -INFINITY;
        }
      };
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent max chains
#pragma unroll
      for (int ch = NCH - 1; ch >= 0; --ch) {
        load(ch);
#pragma unroll
        for (int j = 0; j < TC; j += 2) mx[(j >> 1) & 3] = max3f(mx[(j >> 1) & 3], x[j], x[j + 1]);
      }
      const float bm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * xs;
      // lazy rescaling: move the reference max (and rescale l, O) only when
      // this step's max exceeds it by more than 2^8
      const bool grow = bm > m + 8.f;
      if (u > 0 && __any_sync(0xffffffffu, grow)) {
        ok = wait_all(pvdone0 + 8 * ((u - 1) % B), ((u - 1) / B) & 1);  // O holds every earlier step
        if (!ok) break;
        tc_fence_after();
        const float al = grow ? ex2(m - bm) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(trow + C::O_COL + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * al);
          tmem_st16(trow + C::O_COL + c0, o);
        }
        tmem_wait_st();
        l *= al;
      }
      if (grow) m = bm;
      // P of row r as 16-bit pairs over the first T/2 columns of this S
      // buffer: chunk ch's P goes to columns ch * TC / 2 .., which held
      // scores of chunk ch / 2 <= ch, already read.  It is the A operand of
      // the step's P V; the buffer's next S is issued only after that P V.
      float2 sm[2] = {{0.f, 0.f}, {0.f, 0.f}};  // four independent sum chains, two per instruction
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        if (ch > 0) load(ch);
#pragma unroll
        for (int c0 = 0; c0 < TC / 2; c0 += 16) {
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {  // keys 2(c0+q), 2(c0+q)+1: exponents two per instruction
            const float2 e = fma2(make_float2(x[2 * (c0 + q)], x[2 * (c0 + q) + 1]), make_float2(xs, xs),
                                  make_float2(-m, -m));
            const float2 pp = make_float2(ex2(e.x), ex2(e.y));
            sm[q & 1] = add2(sm[q & 1], pp);
            pk[q] = pack2<C::kBf16>(pp.x, pp.y);
          }
          tmem_st16(trow + C::S_COL + cb * T + ch * (TC / 2) + c0, pk);
        }
      }
      l += (sm[0].x + sm[1].x) + (sm[0].y + sm[1].y);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull0 + 8 * cb);
    }
    if (ok) ok = wait_all(pvdone0 + 8 * ((nsteps - 1) % B), ((nsteps - 1) / B) & 1);  // the last P V
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? v_scale / l : 0.f;
      constexpr int OB = D < 64 ? D : 64;  // O columns read per wait
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += OB) {
        uint32_t o[OB / 16][16];
#pragma unroll
        for (int k = 0; k < OB / 16; ++k) tmem_ld16(trow + C::O_COL + c0 + 16 * k, o[k]);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < OB / 16; ++k) {
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(o[k][j]) * inv;
          rows.store(r, c0 + 16 * k, v);
        }
      }
      rows.store_ml(r, m, l);
    }
  }

  // ---- tear-down: every tcgen05 operation has completed (the MMA-issuing
  // threads waited for their last commits; loads were waited for); release TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::REG_CTAS)
    paged_prefix_kernel(const PrefixParams p) {
  using Q = typename C::Q;
  constexpr int D = C::D;

  const int g = blockIdx.z;
  const int chunk = blockIdx.x;
  const int first = p.group_start[g], members = p.group_start[g + 1] - first;
  const int pblk = group_prefix_blocks(p, g, first, members);

  // The last row of the grid checks the groups (its x = 0 CTA per group),
  // beside the CTAs that attend over the prefixes.
  if (blockIdx.y == gridDim.y - 1) {
    if (blockIdx.x != 0) return;
    // One CTA per group: the group's description, and the suffix offsets of
    // its members (plus those of the sequences before the first group / from
    // the last group's end on, which have no shared prefix).
    __shared__ int s_ok;
    const bool range_ok = first >= 0 && members >= 0 && first + members <= p.num_seqs;
    if (threadIdx.x == 0) {
      s_ok = 1;
      const int len = p.group_prefix_len[g];
      if (!range_ok || (len != 0 && pblk == 0)) atomicOr(p.err, kCheckBadPrefix);
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
    return;
  }
  const int y = blockIdx.y / p.row_blocks;
  const int rb = blockIdx.y - y * p.row_blocks;

  const int kvh = y / p.head_splits;
  const int hs = y - kvh * p.head_splits;
  const int head0 = kvh * p.group + hs * kNH;
  const int hpu = min(kNH, p.group - hs * kNH);  // query heads of this KV unit
  const int rows = members * hpu;                 // (member, head) rows of this KV unit
  const int b0 = chunk * kPrefixChunkBlocks;
  const int nb = min(pblk, b0 + kPrefixChunkBlocks) - b0;
  if (nb <= 0 || rb * kPrefixRows >= rows) return;

  // query row r of this CTA: (member, head) pair idx = rb * 128 + r of the
  // group (heads fastest); partials go to prefix chunk `chunk`
  struct Rows {
    const PrefixParams* p;
    int rb, rows, first, hpu, head0, chunk;
    __device__ bool at(int r, int& s, int& h) const {
      const int idx = rb * kPrefixRows + r;
      if (idx >= rows) return false;
      s = first + idx / hpu;
      h = head0 + idx % hpu;
      return true;
    }
    __device__ const void* q_row(int r) const {
      int s, h;
      if (!at(r, s, h)) return nullptr;
      return reinterpret_cast<const Q*>(p->query) + ((size_t)s * p->num_heads + h) * D;
    }
    __device__ int limit(int) const { return 1 << 30; }  // whole blocks: every key of the range
    __device__ size_t row(int s, int h) const { return ((size_t)s * p->num_heads + h) * p->max_chunks + chunk; }
    __device__ void store(int r, int c0, const float (&v)[16]) const {
      int s, h;
      if (!at(r, s, h)) return;
      float* dst = p->pre_o + row(s, h) * D + c0;
#pragma unroll
      for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
    __device__ void store_ml(int r, float m, float l) const {
      int s, h;
      if (at(r, s, h)) *reinterpret_cast<float2*>(p->pre_ml + row(s, h) * 2) = make_float2(m, l);
    }
  };
  const Rows rw{&p, rb, rows, first, hpu, head0, chunk};
  const size_t row_stride = (size_t)(p.num_heads / p.group) * C::ROW_BYTES;
  const StackedJob job{p.block_tables + (size_t)first * p.bt_stride + b0, nb, nb * kBS, p.num_blocks,
                       static_cast<const uint8_t*>(p.k_cache) + (size_t)kvh * C::ROW_BYTES,
                       static_cast<const uint8_t*>(p.v_cache) + (size_t)kvh * C::ROW_BYTES, row_stride};
  stacked_attention<C>(job, rw, p.scale_log2, p.v_scale, p.err);
}

}  // namespace pa
