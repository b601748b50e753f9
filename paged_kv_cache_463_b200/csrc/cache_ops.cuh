// Paged cache write ("reshape_and_cache") and a paged -> contiguous gather.
//
// Cache write (page "5.KV Cache 管理 & PagedAttention", Q12 append_token): the
// new K/V row of token t goes to physical block slot[t] / block_size at offset
// slot[t] % block_size; a negative slot is skipped.  For an fp8 E4M3 cache the
// value stored is the E4M3 encoding (round to nearest even, saturating at
// +-448) of x / scale computed in IEEE fp32.
//
// Gather (Q11 read_kv_range): tokens [0, seq_len) of one sequence copied out
// of paged storage into a contiguous [seq_len, Hkv, D] buffer, bytes unchanged.
//
// Block copy (page "5.KV Cache 管理 & PagedAttention", Q18 copy-on-write: a
// shared block is copied before a sequence writes into it; page "KV Cache
// 优化与内存管理深度解析", CPUSwap: blocks move between GPU and CPU memory):
// dst_cache[dst] = src_cache[src] for each (src, dst) pair, whole blocks (all
// token slots and KV heads, K and V).  Either cache may be pinned host memory,
// which the kernel reaches directly over the host link.
//
// All are pure data movement: one thread moves 16-byte vectors.
#pragma once

#include "decode.cuh"

namespace pa {

struct CacheWriteParams {
  const void* key;    // [T, Hkv, D] source dtype, token stride key_stride elements
  const void* value;
  long long key_stride, value_stride;
  void* key_cache;    // [NB, bs, Hkv, D]
  void* value_cache;
  const long long* slot_mapping;  // [T]
  long long num_slots;            // NB * bs
  int num_tokens;
  int row_elems;                  // Hkv * D
  float k_scale, v_scale;
  int* err;
};

// 16-bit source -> same 16-bit cache: byte copy.
__global__ void __launch_bounds__(256) reshape_and_cache_copy_kernel(const CacheWriteParams p) {
  const int vec_per_row = p.row_elems / 8;  // 8 x 16-bit = 16 bytes
  const long long total = (long long)p.num_tokens * vec_per_row;
  const bool is_v = blockIdx.y == 1;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(is_v ? p.value : p.key);
  uint16_t* dst = reinterpret_cast<uint16_t*>(is_v ? p.value_cache : p.key_cache);
  const long long stride = is_v ? p.value_stride : p.key_stride;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(idx / vec_per_row);
    const int v = (int)(idx - (long long)t * vec_per_row);
    const long long slot = p.slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= p.num_slots) {
      atomicOr(p.err, kCheckBadSlot);
      continue;
    }
    const uint4 x = *reinterpret_cast<const uint4*>(src + t * stride + v * 8);
    *reinterpret_cast<uint4*>(dst + slot * p.row_elems + v * 8) = x;
  }
}

template <bool SRC_BF16>
__device__ __forceinline__ float to_f32(uint16_t bits) {
  if constexpr (SRC_BF16) {
    return __uint_as_float(static_cast<uint32_t>(bits) << 16);
  } else {
    return __half2float(__ushort_as_half(bits));
  }
}

// 16-bit source -> fp8 E4M3 cache: x / scale (IEEE fp32 division), RNE, satfinite.
template <bool SRC_BF16>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(const CacheWriteParams p) {
  const int vec_per_row = p.row_elems / 8;
  const long long total = (long long)p.num_tokens * vec_per_row;
  const bool is_v = blockIdx.y == 1;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(is_v ? p.value : p.key);
  uint8_t* dst = reinterpret_cast<uint8_t*>(is_v ? p.value_cache : p.key_cache);
  const long long stride = is_v ? p.value_stride : p.key_stride;
  const float sc = is_v ? p.v_scale : p.k_scale;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(idx / vec_per_row);
    const int v = (int)(idx - (long long)t * vec_per_row);
    const long long slot = p.slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= p.num_slots) {
      atomicOr(p.err, kCheckBadSlot);
      continue;
    }
    const uint4 x = *reinterpret_cast<const uint4*>(src + t * stride + v * 8);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t out[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __fdiv_rn(to_f32<SRC_BF16>(static_cast<uint16_t>(w[k] & 0xffffu)), sc);
      const float b = __fdiv_rn(to_f32<SRC_BF16>(static_cast<uint16_t>(w[k] >> 16)), sc);
      const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
      const uint32_t pair = static_cast<uint32_t>(two);
      if (k & 1)
        out[k >> 1] |= pair << 16;
      else
        out[k >> 1] = pair;
    }
    *reinterpret_cast<uint2*>(dst + slot * p.row_elems + v * 8) = make_uint2(out[0], out[1]);
  }
}

struct GatherParams {
  void* k_out;  // [seq_len, Hkv, D] cache dtype
  void* v_out;
  const void* key_cache;
  const void* value_cache;
  const int32_t* block_table;  // [>= ceil(seq_len / bs)]
  int seq_len;
  int row_bytes;               // Hkv * D * element size
  int num_blocks;
  int* err;
};

__global__ void __launch_bounds__(256) paged_gather_kernel(const GatherParams p) {
  const int vec_per_row = p.row_bytes / 16;
  const long long total = (long long)p.seq_len * vec_per_row;
  const bool is_v = blockIdx.y == 1;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(is_v ? p.value_cache : p.key_cache);
  uint8_t* dst = reinterpret_cast<uint8_t*>(is_v ? p.v_out : p.k_out);
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / vec_per_row);
    const int v = (int)(idx - (long long)pos * vec_per_row);
    const int phys = p.block_table[pos / kBS];
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (phys < 0 || phys >= p.num_blocks) {
      atomicOr(p.err, kCheckBadBlock);
    } else {
      const long long row = (long long)phys * kBS + (pos % kBS);
      x = *reinterpret_cast<const uint4*>(src + row * p.row_bytes + v * 16);
    }
    *reinterpret_cast<uint4*>(dst + (long long)pos * p.row_bytes + v * 16) = x;
  }
}

struct CopyBlocksParams {
  void* dst_key;
  void* dst_value;
  const void* src_key;
  const void* src_value;
  const long long* pairs;  // [num_pairs, 2]: (src block, dst block)
  int num_pairs;
  int block_vecs;          // 16-byte vectors per block and tensor
  long long src_blocks, dst_blocks;
  int* err;
};

// CTAs stride over the pairs; the threads of a CTA copy one block's 16-byte
// vectors, four independent copies in flight per thread.  blockIdx.y selects
// K (0) or V (1).
__global__ void __launch_bounds__(256) paged_copy_blocks_kernel(const CopyBlocksParams p) {
  const bool is_v = blockIdx.y == 1;
  const uint4* src = reinterpret_cast<const uint4*>(is_v ? p.src_value : p.src_key);
  uint4* dst = reinterpret_cast<uint4*>(is_v ? p.dst_value : p.dst_key);
  for (int pair = blockIdx.x; pair < p.num_pairs; pair += gridDim.x) {
    const long long sb = p.pairs[2 * pair], db = p.pairs[2 * pair + 1];
    if (sb < 0 || sb >= p.src_blocks || db < 0 || db >= p.dst_blocks) {
      if (threadIdx.x == 0) atomicOr(p.err, kCheckBadBlock);
      continue;
    }
    const uint4* s = src + sb * p.block_vecs;
    uint4* d = dst + db * p.block_vecs;
    for (int w0 = threadIdx.x; w0 < p.block_vecs; w0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int w = w0 + u * blockDim.x;
        if (w < p.block_vecs) v[u] = s[w];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int w = w0 + u * blockDim.x;
        if (w < p.block_vecs) d[w] = v[u];
      }
    }
  }
}

}  // namespace pa
