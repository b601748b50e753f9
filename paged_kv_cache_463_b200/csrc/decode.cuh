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
//  * one CTA per (KV partition, KV head [x query-head chunk of 8], sequence);
//  * warp NC is the producer: it reads the partition's block-table entries
//    (one per lane, shuffled out), and lane 0 streams each 16-token block's K
//    and V tiles into an NS-deep shared-memory ring with 2-D TMA tensor loads
//    (128-byte swizzle, completion counted on an mbarrier, no multicast);
//  * warps 0..NC-1 consume whole blocks round-robin, each keeping its own
//    running max / sum / output (online softmax in the log2 domain):
//      S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]     (mma.m16n8k16, K via ldmatrix)
//      P^T = exp2(S^T - m) packed to 16 bits, moved into the B-operand layout
//            with movmatrix (an 8x8 transpose in registers)
//      O^T[D x 8] += V^T[D x 16 tok] . P^T[16 x 8]         (V via ldmatrix.trans)
//    fp8 E4M3 tiles are read with 128-bit shared loads and converted in
//    registers to f16 pairs (exact); the contraction index order is permuted
//    so that every lane's operands are contiguous bytes;
//  * the consumer warps merge their (m, l, O) through shared memory; a
//    sequence that fits one partition writes its output directly, otherwise
//    (O / l, m, l) go to the workspace and paged_decode_merge_kernel combines
//    the partitions with the log-sum-exp rule:
//      M = max_p m_p,  w_p = l_p 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace pa {

enum : int { kCheckBadBlock = 1, kCheckBadSlot = 2, kCheckSeqTooLong = 4, kCheckWaitTimeout = 8 };

constexpr int kBS = 16;  // tokens per physical block
constexpr int kNH = 8;   // query heads per CTA (MMA N)

struct DecodeParams {
  void* out;                    // [S, Hq, D] query dtype
  const void* query;            // [S, Hq, D] query dtype
  const int32_t* block_tables;  // [S, bt_stride]
  const int32_t* seq_lens;      // [S]
  float* part_o;                // [S, Hq, max_parts, D]
  float* part_ml;               // [S, Hq, max_parts, 2]  (m in log2 units, l)
  int* err;                     // device check bits
  int num_seqs;
  int bt_stride;
  int num_heads;
  int group;        // num_heads / num_kv_heads
  int head_splits;  // ceil(group / 8)
  int num_blocks;   // physical pool size
  int partition_blocks;
  int max_parts;    // grid x of the partition kernel
  float scale_log2;  // softmax scale * log2(e) (* k_scale for fp8)
  float v_scale;     // 1, or the fp8 value scale
};

// Partitions a sequence of `len` tokens is split into (after the same clamps
// the partition kernel applies).
__device__ __forceinline__ int clamp_len(int len, const DecodeParams& p) {
  const int cap = p.bt_stride * kBS;
  return len < 0 ? 0 : (len > cap ? cap : len);
}
__device__ __forceinline__ int num_partitions(int len, const DecodeParams& p) {
  const int nblk = (len + kBS - 1) / kBS;
  const int np = (nblk + p.partition_blocks - 1) / p.partition_blocks;
  return np < p.max_parts ? np : p.max_parts;
}

template <int D_, typename KV_, typename Q_, int NC_, int NS_>
struct DecodeCfg {
  static constexpr int D = D_;
  using KV = KV_;  // __half, __nv_bfloat16 or __nv_fp8_e4m3
  using Q = Q_;    // __half or __nv_bfloat16 (also the MMA operand type)
  static constexpr int NC = NC_;  // consumer warps
  static constexpr int NS = NS_;  // ring stages (one block each)
  static constexpr bool kFp8 = sizeof(KV) == 1;
  static constexpr bool kBf16 = std::is_same<Q, __nv_bfloat16>::value;
  static constexpr int ROW_BYTES = D * (int)sizeof(KV);
  static constexpr int SUBTILES = ROW_BYTES / 128;
  static constexpr int TILE_BYTES = kBS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int THREADS = (NC + 1) * 32;
  static constexpr int RED_STRIDE = D + 4;
  static constexpr int RED_BYTES = NC * kNH * RED_STRIDE * 4;
  static constexpr int RING_BYTES = NS * STAGE_BYTES > RED_BYTES ? NS * STAGE_BYTES : RED_BYTES;
  static constexpr int BAR_BYTES = 2 * NS * 8;
  static constexpr int ML_BYTES = (NC + 1) * kNH * 2 * 4;
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + ML_BYTES;
  static constexpr int NKT = D / 16;
  static constexpr int NDT = D / 16;
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle spans");
  static_assert(!kFp8 || std::is_same<Q, __half>::value, "fp8 caches pair with fp16 queries");
  static_assert(!std::is_same<KV, __half>::value || std::is_same<Q, __half>::value, "f16 cache needs f16 query");
  static_assert(!std::is_same<KV, __nv_bfloat16>::value || kBf16, "bf16 cache needs bf16 query");
};

// Byte offset of (row, byte-in-row) inside a [16 x ROW_BYTES] tile stored as
// 128-byte-wide sub-tiles with the TMA 128-byte swizzle (16-byte chunk index
// XOR row % 8).  `byte` is a multiple of 16 or lies inside one chunk.
__device__ __forceinline__ uint32_t tile_off(int row, int byte) {
  const int sub = byte >> 7;
  const int in = byte & 127;
  return (uint32_t)(sub * (kBS * 128) + row * 128 + ((((in >> 4) ^ (row & 7)) << 4) | (in & 15)));
}

__device__ __forceinline__ uint32_t ld_u32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }

template <class C>
__global__ void __launch_bounds__(C::THREADS) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const DecodeParams p) {
  using Q = typename C::Q;
  constexpr int D = C::D, NC = C::NC, NS = C::NS;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
  uint64_t* empty = full + NS;
  float* red_ml = reinterpret_cast<float*>(empty + NS);  // [NC + 1][kNH][2]

  const int part = blockIdx.x;
  const int kvh = blockIdx.y / p.head_splits;
  const int hsplit = blockIdx.y - kvh * p.head_splits;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int raw_len = p.seq_lens[s];
  const int len = clamp_len(raw_len, p);
  const int nblk = (len + kBS - 1) / kBS;
  const int nparts = num_partitions(len, p);
  if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0 &&
      (raw_len != len || (nblk + p.partition_blocks - 1) / p.partition_blocks > p.max_parts))
    atomicOr(p.err, kCheckSeqTooLong);

  const int head0 = kvh * p.group + hsplit * kNH;
  const int nheads = min(kNH, p.group - hsplit * kNH);
  if (part >= nparts) {
    if (nparts == 0 && part == 0) {  // empty sequence: zero output rows
      Q* o = reinterpret_cast<Q*>(p.out) + ((size_t)s * p.num_heads + head0) * D;
      for (int i = threadIdx.x; i < nheads * D; i += blockDim.x) o[i] = Q(0.0f);
    }
    return;
  }
  const int b0 = part * p.partition_blocks;
  const int nb = min(nblk, b0 + p.partition_blocks) - b0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t ring_u32 = smem_u32(ring);

  if (warp == NC) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    const int32_t* bt = p.block_tables + (size_t)s * p.bt_stride + b0;
    int stop = 0;
    for (int i0 = 0; i0 < nb && !stop; i0 += 32) {
      int my = 0;
      if (i0 + lane < nb) {
        my = __ldg(bt + i0 + lane);
        if (my < 0 || my >= p.num_blocks) {
          atomicOr(p.err, kCheckBadBlock);
          my = 0;
        }
      }
      const int cnt = min(32, nb - i0);
      for (int j = 0; j < cnt; ++j) {
        const int phys = __shfl_sync(0xffffffffu, my, j);
        const int i = i0 + j;
        const int st = i % NS;
        if (lane == 0) {
          if (i >= NS && !mbar_wait(smem_u32(&empty[st]), ((i / NS) - 1) & 1)) {
            atomicOr(p.err, kCheckWaitTimeout);
            stop = 1;
          } else {
            const uint32_t fb = smem_u32(&full[st]);
            mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
            const uint32_t kdst = ring_u32 + st * C::STAGE_BYTES;
            const uint32_t vdst = kdst + C::TILE_BYTES;
            const int y = phys * kBS;
#pragma unroll
            for (int sub = 0; sub < C::SUBTILES; ++sub) {
              const int x = kvh * D + sub * (128 / (int)sizeof(typename C::KV));
              tma_load_2d(kdst + sub * kBS * 128, &tmK, x, y, fb);
              tma_load_2d(vdst + sub * kBS * 128, &tmV, x, y, fb);
            }
          }
        }
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (stop) break;
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gid = lane >> 2, c4 = lane & 3;
  const bool head_ok = gid < nheads;
  const Q* qrow = reinterpret_cast<const Q*>(p.query) + ((size_t)s * p.num_heads + head0 + (head_ok ? gid : 0)) * D;

  // Q^T as MMA B fragments (k = head_dim, n = query head).
  uint32_t qf[C::NKT][2];
#pragma unroll
  for (int j = 0; j < C::NKT; ++j) {
    if constexpr (!C::kFp8) {
      qf[j][0] = head_ok ? ld_u32(qrow + 16 * j + 2 * c4) : 0u;
      qf[j][1] = head_ok ? ld_u32(qrow + 16 * j + 2 * c4 + 8) : 0u;
    } else {
      // permuted contraction order: lane column c4 owns dims [D/4*c4, D/4*c4 + D/4),
      // k-step j uses 4 consecutive ones of them
      const uint2 v = head_ok ? *reinterpret_cast<const uint2*>(qrow + (D / 4) * c4 + 4 * j) : make_uint2(0u, 0u);
      qf[j][0] = v.x;
      qf[j][1] = v.y;
    }
  }

  float o[C::NDT][4];
#pragma unroll
  for (int t = 0; t < C::NDT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int mi = lane >> 3, ri = lane & 7;
  bool dead = false;

  for (int i = warp; i < nb; i += NC) {
    const int st = i % NS;
    if (!mbar_wait(smem_u32(&full[st]), (i / NS) & 1)) {
      atomicOr(p.err, kCheckWaitTimeout);
      dead = true;
      break;
    }
    const int valid = min(kBS, len - (b0 + i) * kBS);
    const uint32_t kb = ring_u32 + st * C::STAGE_BYTES;
    const uint32_t vb = kb + C::TILE_BYTES;

    // ---- S^T = K Q^T
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (!C::kFp8) {
#pragma unroll
      for (int j = 0; j < C::NKT; ++j) {
        const int tok = ri + ((mi & 1) << 3);
        const int dim = 16 * j + ((mi >> 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + tile_off(tok, dim * 2), a0, a1, a2, a3);
        if (j & 1)
          mma_16816<C::kBf16>(sb, a0, a1, a2, a3, qf[j][0], qf[j][1]);
        else
          mma_16816<C::kBf16>(sa, a0, a1, a2, a3, qf[j][0], qf[j][1]);
      }
    } else {
      constexpr int LB = D / 4;        // bytes of a K row owned by one lane
      constexpr int LC = LB / 16;      // 16-byte chunks of it
      uint4 kr[2][LC];
#pragma unroll
      for (int u = 0; u < LC; ++u) {
        kr[0][u] = lds128(kb + tile_off(gid, LB * c4 + 16 * u));
        kr[1][u] = lds128(kb + tile_off(gid + 8, LB * c4 + 16 * u));
      }
#pragma unroll
      for (int j = 0; j < C::NKT; ++j) {
        const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&kr[0][0]);
        const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&kr[1][0]);
        const uint32_t x = w0[j], y = w1[j];
        const uint32_t a0 = e4m3x2_to_f16x2(x), a2 = e4m3x2_to_f16x2(x >> 16);
        const uint32_t a1 = e4m3x2_to_f16x2(y), a3 = e4m3x2_to_f16x2(y >> 16);
        if (j & 1)
          mma_16816<false>(sb, a0, a1, a2, a3, qf[j][0], qf[j][1]);
        else
          mma_16816<false>(sa, a0, a1, a2, a3, qf[j][0], qf[j][1]);
      }
    }

    // ---- online softmax (log2 domain); rows of S^T are tokens gid, gid+8
    const float sl = p.scale_log2;
    const float x0 = gid < valid ? (sa[0] + sb[0]) * sl : -INFINITY;
    const float x1 = gid < valid ? (sa[1] + sb[1]) * sl : -INFINITY;
    const float x2 = gid + 8 < valid ? (sa[2] + sb[2]) * sl : -INFINITY;
    const float x3 = gid + 8 < valid ? (sa[3] + sb[3]) * sl : -INFINITY;
    float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
    }
    const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
    const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p0 = ex2(x0 - mn0), p1 = ex2(x1 - mn1), p2 = ex2(x2 - mn0), p3 = ex2(x3 - mn1);
    l0 = fmaf(l0, al0, p0 + p2);
    l1 = fmaf(l1, al1, p1 + p3);
#pragma unroll
    for (int t = 0; t < C::NDT; ++t) {
      o[t][0] *= al0;
      o[t][1] *= al1;
      o[t][2] *= al0;
      o[t][3] *= al1;
    }
    const uint32_t pb0 = movmatrix_trans(pack2<C::kBf16>(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack2<C::kBf16>(p2, p3));

    // ---- O^T += V^T P^T
    if constexpr (!C::kFp8) {
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (valid < kBS) {  // zero V of tokens past the end (may hold NaN/Inf)
        mlo = (2 * c4 < valid ? 0x0000ffffu : 0u) | (2 * c4 + 1 < valid ? 0xffff0000u : 0u);
        mhi = (2 * c4 + 8 < valid ? 0x0000ffffu : 0u) | (2 * c4 + 9 < valid ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int t = 0; t < C::NDT; ++t) {
        const int tok = ri + ((mi >> 1) << 3);
        const int dim = 16 * t + ((mi & 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vb + tile_off(tok, dim * 2), a0, a1, a2, a3);
        mma_16816<C::kBf16>(o[t], a0 & mlo, a1 & mlo, a2 & mhi, a3 & mhi, pb0, pb1);
      }
    } else {
      // lane row gid owns dims [D/8*gid, D/8*gid + D/8) of tokens 2c4, 2c4+1, 2c4+8, 2c4+9;
      // output tile t holds dims D/8*gid + 2t (MMA row gid) and +1 (row gid+8)
      constexpr int LB = D / 8;
      constexpr int LC = LB / 16;
      uint4 vr[4][LC];
      const int rows[4] = {2 * c4, 2 * c4 + 1, 2 * c4 + 8, 2 * c4 + 9};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int u = 0; u < LC; ++u) {
          uint4 v = lds128(vb + tile_off(rows[r], LB * gid + 16 * u));
          if (rows[r] >= valid) v = make_uint4(0u, 0u, 0u, 0u);
          vr[r][u] = v;
        }
      }
#pragma unroll
      for (int t = 0; t < C::NDT; ++t) {
        const int w = t >> 1;
        const uint32_t sel = (t & 1) ? 0x7362u : 0x5140u;
        const uint32_t xa = reinterpret_cast<const uint32_t*>(&vr[0][0])[w];
        const uint32_t ya = reinterpret_cast<const uint32_t*>(&vr[1][0])[w];
        const uint32_t xb = reinterpret_cast<const uint32_t*>(&vr[2][0])[w];
        const uint32_t yb = reinterpret_cast<const uint32_t*>(&vr[3][0])[w];
        const uint32_t lo = prmt(xa, ya, sel), hi = prmt(xb, yb, sel);
        const uint32_t a0 = e4m3x2_to_f16x2(lo), a1 = e4m3x2_to_f16x2(lo >> 16);
        const uint32_t a2 = e4m3x2_to_f16x2(hi), a3 = e4m3x2_to_f16x2(hi >> 16);
        mma_16816<false>(o[t], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
  }

  // ---------------------------------------------------------------- combine
  // full l over this warp's tokens (rows gid of all lanes with the same c4)
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (dead) {  // a timed-out warp contributes nothing
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  }
  if (gid == 0) {
    red_ml[(warp * kNH + 2 * c4) * 2 + 0] = m0;
    red_ml[(warp * kNH + 2 * c4) * 2 + 1] = l0;
    red_ml[(warp * kNH + 2 * c4 + 1) * 2 + 0] = m1;
    red_ml[(warp * kNH + 2 * c4 + 1) * 2 + 1] = l1;
  }
  // every consumer is done reading the ring and its m/l are visible
  if constexpr (NC > 1) named_bar_sync(1, NC * 32); else __syncwarp();

  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < NC; ++w) {
    M0 = fmaxf(M0, red_ml[(w * kNH + 2 * c4) * 2]);
    M1 = fmaxf(M1, red_ml[(w * kNH + 2 * c4 + 1) * 2]);
  }
  const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
  const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
  if (warp == 0 && gid == 0) {
    float L0 = 0.f, L1 = 0.f;
#pragma unroll
    for (int w = 0; w < NC; ++w) {
      const float mw0 = red_ml[(w * kNH + 2 * c4) * 2], lw0 = red_ml[(w * kNH + 2 * c4) * 2 + 1];
      const float mw1 = red_ml[(w * kNH + 2 * c4 + 1) * 2], lw1 = red_ml[(w * kNH + 2 * c4 + 1) * 2 + 1];
      if (mw0 != -INFINITY) L0 += lw0 * ex2(mw0 - M0);
      if (mw1 != -INFINITY) L1 += lw1 * ex2(mw1 - M1);
    }
    red_ml[(NC * kNH + 2 * c4) * 2 + 0] = M0;
    red_ml[(NC * kNH + 2 * c4) * 2 + 1] = L0;
    red_ml[(NC * kNH + 2 * c4 + 1) * 2 + 0] = M1;
    red_ml[(NC * kNH + 2 * c4 + 1) * 2 + 1] = L1;
  }
  float* red = reinterpret_cast<float*>(ring) + warp * kNH * C::RED_STRIDE;
  float* r0 = red + (2 * c4) * C::RED_STRIDE;
  float* r1 = red + (2 * c4 + 1) * C::RED_STRIDE;
#pragma unroll
  for (int t = 0; t < C::NDT; ++t) {
    if constexpr (!C::kFp8) {
      r0[16 * t + gid] = o[t][0] * f0;
      r1[16 * t + gid] = o[t][1] * f1;
      r0[16 * t + gid + 8] = o[t][2] * f0;
      r1[16 * t + gid + 8] = o[t][3] * f1;
    } else {
      const int d = (D / 8) * gid + 2 * t;
      *reinterpret_cast<float2*>(r0 + d) = make_float2(o[t][0] * f0, o[t][2] * f0);
      *reinterpret_cast<float2*>(r1 + d) = make_float2(o[t][1] * f1, o[t][3] * f1);
    }
  }
  if constexpr (NC > 1) named_bar_sync(1, NC * 32); else __syncwarp();

  // ---------------------------------------------------------------- output
  const float* all = reinterpret_cast<const float*>(ring);
  const int tid = threadIdx.x;
  for (int idx = tid; idx < nheads * (D / 4); idx += NC * 32) {
    const int n = idx / (D / 4);
    const int d = 4 * (idx - n * (D / 4));
    float4 acc = *reinterpret_cast<const float4*>(all + n * C::RED_STRIDE + d);
#pragma unroll
    for (int w = 1; w < NC; ++w) {
      const float4 v = *reinterpret_cast<const float4*>(all + (w * kNH + n) * C::RED_STRIDE + d);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const float Mn = red_ml[(NC * kNH + n) * 2 + 0];
    const float Ln = red_ml[(NC * kNH + n) * 2 + 1];
    const float inv = Ln > 0.f ? p.v_scale / Ln : 0.f;
    const int h = head0 + n;
    if (nparts == 1) {
      Q* dst = reinterpret_cast<Q*>(p.out) + ((size_t)s * p.num_heads + h) * D + d;
      const uint32_t lo = pack2<C::kBf16>(acc.x * inv, acc.y * inv);
      const uint32_t hi = pack2<C::kBf16>(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    } else {
      const size_t row = ((size_t)s * p.num_heads + h) * p.max_parts + part;
      *reinterpret_cast<float4*>(p.part_o + row * D + d) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      if (d == 0) *reinterpret_cast<float2*>(p.part_ml + row * 2) = make_float2(Mn, Ln);
    }
  }
}

// Log-sum-exp merge of the partitions of every (sequence, head) that was
// split; one warp per (sequence, head).
template <typename Q, int D, bool BF16>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const DecodeParams p) {
  const int wg = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wg >= p.num_seqs * p.num_heads) return;
  const int s = wg / p.num_heads, h = wg - s * p.num_heads;
  const int np = num_partitions(clamp_len(p.seq_lens[s], p), p);
  if (np <= 1) return;
  const size_t row0 = ((size_t)s * p.num_heads + h) * p.max_parts;
  const float* ml = p.part_ml + row0 * 2;
  const float* po = p.part_o + row0 * D;
  float M = -INFINITY;
  for (int q = lane; q < np; q += 32) M = fmaxf(M, ml[2 * q]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  constexpr int PER = D / 32;  // dims per lane
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  float W = 0.f;
  for (int q = 0; q < np; ++q) {
    const float2 mlq = *reinterpret_cast<const float2*>(ml + 2 * q);
    const float w = mlq.y > 0.f ? mlq.y * ex2(mlq.x - M) : 0.f;
    W += w;
    const float* src = po + (size_t)q * D + lane * PER;
#pragma unroll
    for (int k = 0; k < PER; k += 2) {
      const float2 v = *reinterpret_cast<const float2*>(src + k);
      acc[k] = fmaf(w, v.x, acc[k]);
      acc[k + 1] = fmaf(w, v.y, acc[k + 1]);
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  Q* dst = reinterpret_cast<Q*>(p.out) + ((size_t)s * p.num_heads + h) * D + lane * PER;
#pragma unroll
  for (int k = 0; k < PER; k += 2) *reinterpret_cast<uint32_t*>(dst + k) = pack2<BF16>(acc[k] * inv, acc[k + 1] * inv);
}

}  // namespace pa
