// Host side of the C ABI declared in include/paged_attn.h: argument
// validation, the split-KV workspace, TMA tensor maps over the caches, and
// kernel dispatch.  All compute is in decode.cuh / cache_ops.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include <nvtx3/nvToolsExt.h>

#include "paged_attn.h"
#include "cache_ops.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "prefix.cuh"

#define PA_API extern "C" __attribute__((visibility("default")))

// An NVTX range around each C-ABI call that touches the GPU, named after the
// call (seen by Nsight Systems and by ncu --nvtx; without a tool attached the
// push and pop do nothing).  The allocation-free entry point has none: it
// leaves every host-side resource alone too.
struct PaTraceRange {
  explicit PaTraceRange(const char* name) { nvtxRangePushA(name); }
  ~PaTraceRange() { nvtxRangePop(); }
  PaTraceRange(const PaTraceRange&) = delete;
  PaTraceRange& operator=(const PaTraceRange&) = delete;
};
#define PA_TRACE(name) const PaTraceRange pa_trace_range_(name)

namespace {

using pa::DecodeCfg;
using pa::DecodeParams;

struct KernelSet {
  const void* decode = nullptr;
  // the same decode kernel with a one-stage-shallower ring (16-bit head_dim
  // 128), used where it fits more CTAs per SM (choose_decode)
  const void* decode_shallow = nullptr;
  int ns_shallow = 0;
  const void* merge = nullptr;
  const void* prefix = nullptr;   // shared-prefix pass
  const void* prefill = nullptr;  // multi-query (prefill) attention, same CTA shape as the prefix pass
  int threads = 0;
  int ns = 0, stage_bytes = 0;  // ring shape (the rest of the layout depends on the call)
  int prefix_threads = 0, prefix_smem = 0;
  size_t smem(int q_slot_bytes, int max_seqs) const {
    return pa::DecodeLayout(ns, stage_bytes, q_slot_bytes).bytes(max_seqs);
  }
};

// CS: the shallower-ring decode configuration, or void.
template <class C, class P, class CS>
KernelSet make_set() {
  KernelSet k;
  k.decode = reinterpret_cast<const void*>(&pa::paged_decode_kernel<C>);
  if constexpr (!std::is_void<CS>::value) {
    static_assert(CS::STAGE_BYTES == C::STAGE_BYTES && CS::THREADS == C::THREADS, "same ring stages and CTA");
    k.decode_shallow = reinterpret_cast<const void*>(&pa::paged_decode_kernel<CS>);
    k.ns_shallow = CS::NS;
  }
  k.merge = reinterpret_cast<const void*>(&pa::paged_decode_merge_kernel<typename C::Q, C::D, C::kBf16>);
  k.prefix = reinterpret_cast<const void*>(&pa::paged_prefix_kernel<P>);
  k.prefill = reinterpret_cast<const void*>(&pa::paged_prefill_kernel<P>);
  k.threads = C::THREADS;
  k.ns = C::NS;
  k.stage_bytes = C::STAGE_BYTES;
  k.prefix_threads = P::THREADS;
  k.prefix_smem = P::SMEM_BYTES;
  return k;
}

// Resident decode CTAs per SM for a call shape; with a shallower-ring
// variant, take it when more of its CTAs fit (bytes in flight per SM: CTAs x
// stages).  Results do not depend on the ring depth.  Both kernels' shared
// memory limits must have been raised.
cudaError_t choose_decode(KernelSet* ks, int q_slot, int max_seqs, int* per_sm) {
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, ks->decode, ks->threads,
                                                                ks->smem(q_slot, max_seqs));
  if (e != cudaSuccess || !ks->decode_shallow) return e;
  KernelSet alt = *ks;
  alt.decode = ks->decode_shallow;
  alt.ns = ks->ns_shallow;
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, alt.decode, alt.threads, alt.smem(q_slot, max_seqs));
  if (e != cudaSuccess) return e;
  if (n > *per_sm) {
    *ks = alt;
    *per_sm = n;
  }
  return cudaSuccess;
}

// Every kernel of the library asks for the same (maximum shared-memory)
// L1/shared split, so consecutive launches (cache write -> decode -> merge)
// never make the SMs switch configuration between kernels.
cudaError_t pin_carveout(const void* fn) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t pin_all_carveouts(const KernelSet& ks) {
  const void* fns[] = {ks.decode, ks.decode_shallow ? ks.decode_shallow : ks.decode, ks.merge, ks.prefix, ks.prefill,
                       reinterpret_cast<const void*>(&pa::reshape_and_cache_copy_kernel),
                       reinterpret_cast<const void*>(&pa::reshape_and_cache_fp8_kernel<true>),
                       reinterpret_cast<const void*>(&pa::reshape_and_cache_fp8_kernel<false>),
                       reinterpret_cast<const void*>(&pa::paged_gather_kernel),
                       reinterpret_cast<const void*>(&pa::paged_copy_blocks_kernel)};
  for (const void* f : fns) {
    cudaError_t e = pin_carveout(f);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The merge kernel as a programmatic dependent of the decode kernel just
// launched on `s`: its CTAs may be scheduled while the decode grid drains and
// wait (griddepcontrol.wait) for the decode grid before reading partials.
// Merge CTA shape: more partitions -> more partition slices per head, fewer
// heads per CTA (256 threads = heads x slices x head_dim/4 chunks).
void merge_shape(int head_dim, int parts, int num_heads, int* hpc, int* slices, int* hpt) {
  const int ch = head_dim / 4;
  int sl = 1;
  while (sl < 8 && sl * 16 <= parts) sl *= 2;  // <= 15 partitions: 1 slice, ... , >= 128: 8
  while (sl > 1 && ch * sl > 256) sl /= 2;
  int h = 256 / (ch * sl);
  if (h > pa::kNH) h = pa::kNH;
  if (h > num_heads) h = num_heads;
  if (h < 1) h = 1;
  // one slice and many heads: two heads per thread (half the CTAs: a large
  // batch's merge in one wave instead of two)
  const int t = (sl == 1 && h == 256 / ch && num_heads >= 2 * h) ? 2 : 1;
  *hpc = h * t;
  *slices = sl;
  *hpt = t;
}

cudaError_t launch_merge(const KernelSet& ks, const pa::DecodeParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.num_seqs * ((p.num_heads + p.merge_hpc - 1) / p.merge_hpc)));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  pa::DecodeParams pp = p;
  void* args[] = {&pp};
  return cudaLaunchKernelExC(&cfg, ks.merge, args);
}

// Shortest block range a CTA is given in stream-K mode (256 tokens), which
// bounds the pieces a sequence can be cut into.
constexpr int kMinPieceBlocks = 16;

// query rows one item copies: min(group, 8) heads of head_dim 16-bit values
int q_slot_bytes(int num_heads, int num_kv_heads, int head_dim) {
  const int g = num_heads / num_kv_heads;
  return (g < pa::kNH ? g : pa::kNH) * head_dim * 2;
}

// Ring depth (16-token blocks in flight per CTA) per (head_dim, cache type).
#ifndef PA_NS_16B_64
#define PA_NS_16B_64 8
#endif
#ifndef PA_NS_16B_128
#define PA_NS_16B_128 3
#endif
#ifndef PA_NS_16B_256
#define PA_NS_16B_256 3
#endif
#ifndef PA_NS_FP8_128
#define PA_NS_FP8_128 4
#endif
#ifndef PA_NS_FP8_256
#define PA_NS_FP8_256 4
#endif
template <int D, typename KV, typename Q>
struct Tuned;
// (head_dim, cache type) -> ring depth, and the CTAs per SM the register
// budget must allow (matching what shared memory allows).
#ifndef PA_MIN_CTAS_FP8_128
#define PA_MIN_CTAS_FP8_128 8
#endif
// The tensor-core passes (shared prefixes, prefill): blocks per step and
// step buffers.  head_dim 64 / 128: 32-key steps with four step buffers (the
// steps run up to three ahead of the softmax, and four warps load and issue
// S for them), which still leave room (tensor and shared memory) for two
// CTAs per SM, so that two softmax warps share each scheduler; 64-key steps
// with two buffers measured slower (a buffer's refill then sits on the
// critical path).  head_dim 256: 32-key steps, two buffers (one CTA per SM).
#ifndef PA_PX_SB
#define PA_PX_SB 2
#endif
#ifndef PA_PX_B
#define PA_PX_B 4
#endif
template <> struct Tuned<64, __half, __half> {
  using C = DecodeCfg<64, __half, __half, PA_NS_16B_64, 8>;
  using CS = void;
  using P = pa::PrefixCfg<64, __half, __half, PA_PX_SB, PA_PX_B>;
};
template <> struct Tuned<128, __half, __half> {
  using C = DecodeCfg<128, __half, __half, PA_NS_16B_128, 8>;
  using CS = DecodeCfg<128, __half, __half, PA_NS_16B_128 - 1, 8>;
  using P = pa::PrefixCfg<128, __half, __half, PA_PX_SB, PA_PX_B>;
};
template <> struct Tuned<256, __half, __half> {
  using C = DecodeCfg<256, __half, __half, PA_NS_16B_256, 3>;
  using CS = void;
  using P = pa::PrefixCfg<256, __half, __half, 2, 2>;
};
template <> struct Tuned<64, __nv_bfloat16, __nv_bfloat16> {
  using C = DecodeCfg<64, __nv_bfloat16, __nv_bfloat16, PA_NS_16B_64, 8>;
  using CS = void;
  using P = pa::PrefixCfg<64, __nv_bfloat16, __nv_bfloat16, PA_PX_SB, PA_PX_B>;
};
template <> struct Tuned<128, __nv_bfloat16, __nv_bfloat16> {
  using C = DecodeCfg<128, __nv_bfloat16, __nv_bfloat16, PA_NS_16B_128, 8>;
  using CS = DecodeCfg<128, __nv_bfloat16, __nv_bfloat16, PA_NS_16B_128 - 1, 8>;
  using P = pa::PrefixCfg<128, __nv_bfloat16, __nv_bfloat16, PA_PX_SB, PA_PX_B>;
};
template <> struct Tuned<256, __nv_bfloat16, __nv_bfloat16> {
  using C = DecodeCfg<256, __nv_bfloat16, __nv_bfloat16, PA_NS_16B_256, 3>;
  using CS = void;
  using P = pa::PrefixCfg<256, __nv_bfloat16, __nv_bfloat16, 2, 2>;
};
template <> struct Tuned<128, __nv_fp8_e4m3, __half> {
  using C = DecodeCfg<128, __nv_fp8_e4m3, __half, PA_NS_FP8_128, PA_MIN_CTAS_FP8_128>;
  using CS = void;
  using P = pa::PrefixCfg<128, __nv_fp8_e4m3, __half, PA_PX_SB, PA_PX_B>;
};
template <> struct Tuned<256, __nv_fp8_e4m3, __half> {
  using C = DecodeCfg<256, __nv_fp8_e4m3, __half, PA_NS_FP8_256, 4>;
  using CS = void;
  using P = pa::PrefixCfg<256, __nv_fp8_e4m3, __half, 2, 2>;
};

bool select_kernels(int head_dim, int q_dtype, int kv_dtype, KernelSet* ks) {
#define PA_CASE(D, KVT, QT) \
  *ks = make_set<typename Tuned<D, KVT, QT>::C, typename Tuned<D, KVT, QT>::P, typename Tuned<D, KVT, QT>::CS>(); \
  return true
  if (kv_dtype == PA_F16 && q_dtype == PA_F16) {
    if (head_dim == 64) { PA_CASE(64, __half, __half); }
    if (head_dim == 128) { PA_CASE(128, __half, __half); }
    if (head_dim == 256) { PA_CASE(256, __half, __half); }
  }
  if (kv_dtype == PA_BF16 && q_dtype == PA_BF16) {
    if (head_dim == 64) { PA_CASE(64, __nv_bfloat16, __nv_bfloat16); }
    if (head_dim == 128) { PA_CASE(128, __nv_bfloat16, __nv_bfloat16); }
    if (head_dim == 256) { PA_CASE(256, __nv_bfloat16, __nv_bfloat16); }
  }
  if (kv_dtype == PA_FP8_E4M3 && q_dtype == PA_F16) {
    if (head_dim == 128) { PA_CASE(128, __nv_fp8_e4m3, __half); }
    if (head_dim == 256) { PA_CASE(256, __nv_fp8_e4m3, __half); }
  }
#undef PA_CASE
  return false;
}

int elem_bytes(int dt) { return dt == PA_FP8_E4M3 ? 1 : 2; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

struct pa_ctx {
  pa_config cfg{};
  int device = 0;
  int num_sms = 0;
  int ctas_per_sm = 1;
  int max_parts = 0;            // workspace partitions per (seq, head)
  int min_partition_tokens = 0; // smallest partition the workspace allows
  int partition_tokens = 0;     // current setting (PA_PARTITION_* or > 0)
  float* part_o = nullptr;
  float* part_ml = nullptr;
  int* err = nullptr;           // [0] check word, [1..2] decode kernel counters (DecodeParams::counters)
  int* seq_merge = nullptr;     // [max_num_seqs] each sequence's merge work (decode -> merge)
  // shared-prefix decode (PA_FLAG_SHARED_PREFIX)
  int max_chunks = 0;           // prefix partials per (seq, head)
  float* pre_o = nullptr;
  float* pre_ml = nullptr;
  int* seq_skip = nullptr;      // [max_num_seqs] prefix blocks per sequence (prefix pass -> decode, merge)
  int* err_host = nullptr;      // pinned
  int grid = 0;                 // persistent grid: SMs x resident CTAs
  int last_bits = 0;
  long long test_wait_limit = 0;  // > 0: the next decode launch takes the failure path (test hook)
  KernelSet ks;
  std::unordered_map<const void*, CUtensorMap> maps;
  std::string msg;
};

namespace {

int fail(pa_ctx* ctx, int status, const char* what) {
  if (ctx) ctx->msg = what;
  return status;
}

int cuda_fail(pa_ctx* ctx, cudaError_t e, const char* where) {
  if (ctx) ctx->msg = std::string(where) + ": " + cudaGetErrorString(e);
  return PA_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 2-D view of a cache as [num_blocks * block_size rows, num_kv_heads * head_dim
// elements]; box = one 128-byte-wide, block_size-tall sub-tile, 128-byte swizzle.
int tensor_map(pa_ctx* ctx, const void* base, CUtensorMap* out) {
  auto it = ctx->maps.find(base);
  if (it != ctx->maps.end()) {
    *out = it->second;
    return PA_OK;
  }
  auto enc = encode_fn();
  if (!enc) return fail(ctx, PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const pa_config& c = ctx->cfg;
  const int eb = elem_bytes(c.kv_dtype);
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)c.num_kv_heads * c.head_dim, (cuuint64_t)c.num_blocks * c.block_size};
  cuuint64_t strides[1] = {(cuuint64_t)c.num_kv_heads * c.head_dim * eb};
  cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)c.block_size};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return fail(ctx, PA_ERR_CUDA, buf);
  }
  if (ctx->maps.size() >= 512) ctx->maps.clear();
  ctx->maps.emplace(base, m);
  *out = m;
  return PA_OK;
}



}  // namespace

PA_API const char* paged_attn_status_string(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_DEVICE_CHECK: return "device-side check fired";
    case PA_ERR_NO_MEMORY: return "out of device memory";
    case PA_ERR_SCRATCH_TOO_SMALL: return "split-KV partials exceed the no-alloc scratch (PA_NOALLOC_SCRATCH_BYTES)";
    case PA_ERR_OUT_OF_BLOCKS: return "no free KV-cache block (block manager)";
    default: return "unknown status";
  }
}

PA_API const char* paged_attn_last_error(const pa_ctx* ctx) { return ctx ? ctx->msg.c_str() : ""; }

PA_API int paged_attn_last_check_bits(const pa_ctx* ctx) { return ctx ? ctx->last_bits : 0; }

PA_API int paged_attn_create(const pa_config* cfg, pa_ctx** out) {
  PA_TRACE("paged_attn_create");
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return PA_ERR_INVALID_ARG;
  const pa_config c = *cfg;
  if (c.num_heads <= 0 || c.num_kv_heads <= 0 || c.num_heads % c.num_kv_heads != 0 || c.num_blocks <= 0 ||
      c.max_num_seqs <= 0 || c.max_blocks_per_seq <= 0 || (c.flags & ~PA_FLAG_SHARED_PREFIX) != 0 ||
      c.device < 0)
    return PA_ERR_INVALID_ARG;
  if (c.block_size != pa::kBS) return PA_ERR_UNSUPPORTED;
  if ((long long)c.num_blocks * c.block_size > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  if (c.partition_tokens < PA_PARTITION_AUTO || (c.partition_tokens > 0 && c.partition_tokens % c.block_size))
    return PA_ERR_INVALID_ARG;
  if (c.q_dtype < PA_F16 || c.q_dtype > PA_BF16 || c.kv_dtype < PA_F16 || c.kv_dtype > PA_FP8_E4M3)
    return PA_ERR_INVALID_ARG;
  KernelSet ks;
  if (!select_kernels(c.head_dim, c.q_dtype, c.kv_dtype, &ks)) return PA_ERR_UNSUPPORTED;
  if ((long long)c.num_kv_heads * c.head_dim * elem_bytes(c.kv_dtype) % 16 != 0) return PA_ERR_UNSUPPORTED;

  cudaError_t e = cudaSetDevice(c.device);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  pa_ctx* ctx = new pa_ctx();
  ctx->cfg = c;
  ctx->device = c.device;
  ctx->ks = ks;
  ctx->partition_tokens = c.partition_tokens;
  ctx->min_partition_tokens = c.partition_tokens > 0 ? c.partition_tokens : 512;
  const int max_tokens = c.max_blocks_per_seq * c.block_size;
  // partials per (sequence, head): fixed partitions of >= min_partition_tokens,
  // or stream-K pieces of >= kMinPieceBlocks blocks (+1 for a range boundary)
  const int ticket_parts = (max_tokens + ctx->min_partition_tokens - 1) / ctx->min_partition_tokens;
  const int sk_parts = (c.max_blocks_per_seq + kMinPieceBlocks - 1) / kMinPieceBlocks + 1;
  ctx->max_parts = ticket_parts > sk_parts ? ticket_parts : sk_parts;

  int st = PA_OK;
  do {
    if ((e = cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, c.device)) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaDeviceGetAttribute");
      break;
    }
    int optin = 0;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c.device)) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaDeviceGetAttribute");
      break;
    }
    if (ks.smem(q_slot_bytes(c.num_heads, c.num_kv_heads, c.head_dim), c.max_num_seqs) > (size_t)optin) {
      st = fail(ctx, PA_ERR_UNSUPPORTED, "max_num_seqs too large for the decode kernel's shared memory");
      break;
    }
    if ((e = cudaFuncSetAttribute(ks.decode, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) != cudaSuccess ||
        (ks.decode_shallow &&
         (e = cudaFuncSetAttribute(ks.decode_shallow, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) !=
             cudaSuccess) ||
        (e = cudaFuncSetAttribute(ks.prefix, cudaFuncAttributeMaxDynamicSharedMemorySize, ks.prefix_smem)) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(ks.prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, ks.prefix_smem)) !=
            cudaSuccess ||
        (e = pin_all_carveouts(ks)) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaFuncSetAttribute");
      break;
    }
    if ((e = choose_decode(&ctx->ks, q_slot_bytes(c.num_heads, c.num_kv_heads, c.head_dim), c.max_num_seqs,
                           &ctx->ctas_per_sm)) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
      break;
    }
    if (ctx->ctas_per_sm < 1) {
      st = fail(ctx, PA_ERR_UNSUPPORTED, "decode kernel does not fit on an SM");
      break;
    }
    const size_t rows = (size_t)c.max_num_seqs * c.num_heads * ctx->max_parts;
    if (cudaMalloc(&ctx->part_o, rows * c.head_dim * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&ctx->part_ml, rows * 2 * sizeof(float)) != cudaSuccess) {
      cudaGetLastError();
      st = PA_ERR_NO_MEMORY;
      break;
    }
    ctx->grid = ctx->num_sms * ctx->ctas_per_sm;
    if ((e = cudaMalloc(&ctx->seq_merge, c.max_num_seqs * sizeof(int))) != cudaSuccess) {
      cudaGetLastError();
      st = PA_ERR_NO_MEMORY;
      break;
    }

    if (c.flags & PA_FLAG_SHARED_PREFIX) {
      ctx->max_chunks = (c.max_blocks_per_seq + pa::kPrefixChunkBlocks - 1) / pa::kPrefixChunkBlocks;
      const size_t prow = (size_t)c.max_num_seqs * c.num_heads * ctx->max_chunks;
      if (cudaMalloc(&ctx->pre_o, prow * c.head_dim * sizeof(float)) != cudaSuccess ||
          cudaMalloc(&ctx->pre_ml, prow * 2 * sizeof(float)) != cudaSuccess ||
          cudaMalloc(&ctx->seq_skip, c.max_num_seqs * sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        st = PA_ERR_NO_MEMORY;
        break;
      }
    }
    if ((e = cudaMalloc(&ctx->err, 8 * sizeof(int))) != cudaSuccess ||
        (e = cudaMemset(ctx->err, 0, 8 * sizeof(int))) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaMalloc(check word)");
      break;
    }
    if ((e = cudaMallocHost(&ctx->err_host, sizeof(int))) != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaMallocHost");
      break;
    }
  } while (false);
  if (st != PA_OK) {
    paged_attn_destroy(ctx);
    return st;
  }
  *out = ctx;
  return PA_OK;
}

PA_API int paged_attn_destroy(pa_ctx* ctx) {
  PA_TRACE("paged_attn_destroy");
  if (!ctx) return PA_ERR_INVALID_ARG;
  cudaSetDevice(ctx->device);
  if (ctx->part_o) cudaFree(ctx->part_o);
  if (ctx->part_ml) cudaFree(ctx->part_ml);
  if (ctx->err) cudaFree(ctx->err);
  if (ctx->seq_merge) cudaFree(ctx->seq_merge);
  if (ctx->pre_o) cudaFree(ctx->pre_o);
  if (ctx->pre_ml) cudaFree(ctx->pre_ml);
  if (ctx->seq_skip) cudaFree(ctx->seq_skip);
  if (ctx->err_host) cudaFreeHost(ctx->err_host);
  delete ctx;
  return PA_OK;
}

PA_API int paged_attn_set_partition_tokens(pa_ctx* ctx, int partition_tokens) {
  if (!ctx) return PA_ERR_INVALID_ARG;
  if (partition_tokens == PA_PARTITION_NONE || partition_tokens == PA_PARTITION_AUTO) {
    ctx->partition_tokens = partition_tokens;
    return PA_OK;
  }
  if (partition_tokens < ctx->min_partition_tokens || partition_tokens % ctx->cfg.block_size)
    return fail(ctx, PA_ERR_INVALID_ARG, "partition_tokens below the workspace minimum or not a block multiple");
  ctx->partition_tokens = partition_tokens;
  return PA_OK;
}

PA_API int paged_attn_get_partition_tokens(const pa_ctx* ctx, int* partition_tokens) {
  if (!ctx || !partition_tokens) return PA_ERR_INVALID_ARG;
  *partition_tokens = ctx->partition_tokens;
  return PA_OK;
}

PA_API int reshape_and_cache(pa_ctx* ctx, const void* key, const void* value, int64_t key_token_stride,
                             int64_t value_token_stride, void* key_cache, void* value_cache,
                             const int64_t* slot_mapping, int num_tokens, float k_scale, float v_scale,
                             void* stream) {
  PA_TRACE("reshape_and_cache");
  if (!ctx) return PA_ERR_INVALID_ARG;
  const pa_config& c = ctx->cfg;
  if (num_tokens < 0) return fail(ctx, PA_ERR_INVALID_ARG, "num_tokens < 0");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping)
    return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
  const int row = c.num_kv_heads * c.head_dim;
  if (key_token_stride < row || value_token_stride < row || key_token_stride % 8 || value_token_stride % 8)
    return fail(ctx, PA_ERR_INVALID_ARG, "token strides must be >= num_kv_heads*head_dim and multiples of 8");
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(slot_mapping, 8))
    return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
  const bool fp8 = c.kv_dtype == PA_FP8_E4M3;
  if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return fail(ctx, PA_ERR_INVALID_ARG, "fp8 scales must be finite and > 0");
  cudaSetDevice(ctx->device);
  pa::CacheWriteParams p;
  p.key = key;
  p.value = value;
  p.key_stride = key_token_stride;
  p.value_stride = value_token_stride;
  p.key_cache = key_cache;
  p.value_cache = value_cache;
  p.slot_mapping = reinterpret_cast<const long long*>(slot_mapping);
  p.num_slots = (long long)c.num_blocks * c.block_size;
  p.num_tokens = num_tokens;
  p.row_elems = row;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.err = ctx->err;
  const long long vecs = (long long)num_tokens * (row / 8);
  const int threads = 256;
  long long blocks = (vecs + threads - 1) / threads;
  const long long cap = (long long)ctx->num_sms * 8;
  if (blocks > cap) blocks = cap;
  dim3 grid((unsigned)blocks, 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!fp8)
    pa::reshape_and_cache_copy_kernel<<<grid, threads, 0, s>>>(p);
  else if (c.q_dtype == PA_BF16)
    pa::reshape_and_cache_fp8_kernel<true><<<grid, threads, 0, s>>>(p);
  else
    pa::reshape_and_cache_fp8_kernel<false><<<grid, threads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(ctx, e, "reshape_and_cache launch");
}

namespace {

// The shared-prefix part of a decode call (absent for plain decode).
struct PrefixArgs {
  const int32_t* group_start;
  const int32_t* group_prefix_len;
  int num_groups, max_group_size, max_prefix_len;
};

int decode_impl(pa_ctx* ctx, void* out, const void* query, const void* key_cache, const void* value_cache,
                const int32_t* block_tables, int bt_stride, const int32_t* seq_lens, int num_seqs, int max_seq_len,
                float scale, float k_scale, float v_scale, void* stream, const PrefixArgs* pre) {
  if (!ctx) return PA_ERR_INVALID_ARG;
  const pa_config& c = ctx->cfg;
  if (num_seqs < 0 || num_seqs > c.max_num_seqs) return fail(ctx, PA_ERR_INVALID_ARG, "num_seqs out of range");
  if (num_seqs == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens)
    return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
  if (bt_stride < 1) return fail(ctx, PA_ERR_INVALID_ARG, "bt_stride < 1");
  if (max_seq_len < 0 || max_seq_len > c.max_blocks_per_seq * c.block_size)
    return fail(ctx, PA_ERR_INVALID_ARG, "max_seq_len outside [0, max_blocks_per_seq*block_size]");
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4))
    return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
  if (!std::isfinite(scale)) return fail(ctx, PA_ERR_INVALID_ARG, "scale not finite");
  const bool fp8 = c.kv_dtype == PA_FP8_E4M3;
  if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return fail(ctx, PA_ERR_INVALID_ARG, "fp8 scales must be finite and > 0");
  const int group = c.num_heads / c.num_kv_heads;
  const int head_splits = (group + pa::kNH - 1) / pa::kNH;
  const int kv_units = c.num_kv_heads * head_splits;
  int prefix_chunks = 0, row_blocks = 0;
  if (pre) {
    if (!(c.flags & PA_FLAG_SHARED_PREFIX))
      return fail(ctx, PA_ERR_UNSUPPORTED, "context created without PA_FLAG_SHARED_PREFIX");
    if (!pre->group_start || !pre->group_prefix_len) return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
    if (!aligned(pre->group_start, 4) || !aligned(pre->group_prefix_len, 4))
      return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
    if (pre->num_groups < 1 || pre->num_groups > num_seqs || pre->num_groups > 65535)
      return fail(ctx, PA_ERR_INVALID_ARG, "num_groups outside [1, num_seqs]");
    if (pre->max_group_size < 1 || pre->max_group_size > num_seqs)
      return fail(ctx, PA_ERR_INVALID_ARG, "max_group_size outside [1, num_seqs]");
    if (pre->max_prefix_len < 0 || pre->max_prefix_len > max_seq_len)
      return fail(ctx, PA_ERR_INVALID_ARG, "max_prefix_len outside [0, max_seq_len]");
    const int pblocks = pre->max_prefix_len / c.block_size;
    prefix_chunks = (pblocks + pa::kPrefixChunkBlocks - 1) / pa::kPrefixChunkBlocks;
    const int rows_per_unit = pre->max_group_size * (group < pa::kNH ? group : pa::kNH);
    row_blocks = (rows_per_unit + pa::kPrefixRows - 1) / pa::kPrefixRows;
    if ((long long)kv_units * row_blocks + 1 > 65535)
      return fail(ctx, PA_ERR_UNSUPPORTED, "max_group_size too large for the prefix grid");
  }
  cudaSetDevice(ctx->device);

  CUtensorMap mk, mv;
  int st = tensor_map(ctx, key_cache, &mk);
  if (st != PA_OK) return st;
  if ((st = tensor_map(ctx, value_cache, &mv)) != PA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  if (pre) {  // shared blocks first: their partials, and each sequence's suffix offset
    pa::PrefixParams q;
    q.query = query;
    q.k_cache = key_cache;
    q.v_cache = value_cache;
    q.block_tables = block_tables;
    q.seq_lens = seq_lens;
    q.group_start = pre->group_start;
    q.group_prefix_len = pre->group_prefix_len;
    q.pre_o = ctx->pre_o;
    q.pre_ml = ctx->pre_ml;
    q.seq_skip = ctx->seq_skip;
    q.err = ctx->err;
    q.num_seqs = num_seqs;
    q.num_groups = pre->num_groups;
    q.max_group_size = pre->max_group_size;
    q.max_prefix_blocks = pre->max_prefix_len / c.block_size;
    q.bt_stride = bt_stride;
    q.num_heads = c.num_heads;
    q.group = group;
    q.head_splits = head_splits;
    q.num_blocks = c.num_blocks;
    q.max_blocks = max_seq_len > 0 ? (max_seq_len + c.block_size - 1) / c.block_size : 1;
    q.max_chunks = ctx->max_chunks;
    q.row_blocks = row_blocks;
    q.scale_log2 = (float)((double)scale * 1.4426950408889634 * (fp8 ? (double)k_scale : 1.0));
    q.v_scale = fp8 ? v_scale : 1.0f;
    void* qargs[] = {&q};
    // grid.y: the attention CTAs, plus one row whose x = 0 CTA checks each group
    const dim3 grid((unsigned)(prefix_chunks > 0 ? prefix_chunks : 1), (unsigned)(kv_units * row_blocks + 1),
                    (unsigned)pre->num_groups);
    cudaError_t e = cudaLaunchKernel(ctx->ks.prefix, grid, dim3(ctx->ks.prefix_threads), qargs,
                                     ctx->ks.prefix_smem, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "prefix launch");
  }

  // PA_PARTITION_AUTO: stream-K ranges (the split follows from the balance);
  // otherwise fixed partitions handed out by tickets
  const bool is_auto = ctx->partition_tokens == PA_PARTITION_AUTO;
  const int max_blocks = (max_seq_len + c.block_size - 1) / c.block_size;
  // auto: the device picks tickets (partitions >= min_partition_tokens) or
  // stream-K ranges (pieces >= kMinPieceBlocks) per call; the workspace holds
  // either.  `parts` only shapes the merge kernel.
  const int pt = is_auto ? ctx->min_partition_tokens : ctx->partition_tokens;
  const int part_blocks = pt > 0 ? pt / c.block_size : (max_blocks > 0 ? max_blocks : 1);
  int parts = (max_blocks + part_blocks - 1) / part_blocks;
  if (parts < 1) parts = 1;
  if (parts > ctx->max_parts) return fail(ctx, PA_ERR_INVALID_ARG, "too many partitions for the workspace");
  if (is_auto && ctx->grid >= kv_units) {
    const long long groups = ctx->grid / kv_units;
    long long per_group = ((long long)num_seqs * (max_blocks > 0 ? max_blocks : 1) + groups - 1) / groups;
    if (per_group < kMinPieceBlocks) per_group = kMinPieceBlocks;
    const int sk_parts = (int)((max_blocks + per_group - 1) / per_group) + 1;
    if (sk_parts > parts) parts = sk_parts < ctx->max_parts ? sk_parts : ctx->max_parts;
  }

  DecodeParams p;
  p.out = out;
  p.query = query;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.part_o = ctx->part_o;
  p.part_ml = ctx->part_ml;
  p.err = ctx->err;
  p.counters = ctx->err + 1;
  p.num_seqs = num_seqs;
  p.bt_stride = bt_stride;
  p.num_heads = c.num_heads;
  p.group = group;
  p.head_splits = head_splits;
  p.kv_units = kv_units;
  p.q_slot_bytes = q_slot_bytes(c.num_heads, c.num_kv_heads, c.head_dim);
  p.num_blocks = c.num_blocks;
  p.max_blocks = max_blocks > 0 ? max_blocks : 1;
  p.force_partials = pre ? 1 : 0;
  p.partition_blocks = part_blocks;
  p.auto_mode = is_auto ? 1 : 0;
  p.min_piece_blocks = kMinPieceBlocks;
  p.seq_merge = ctx->seq_merge;
  p.max_parts = ctx->max_parts;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634 * (fp8 ? (double)k_scale : 1.0));
  p.v_scale = fp8 ? v_scale : 1.0f;
  if (pre) {
    p.seq_skip = ctx->seq_skip;
    p.pre_o = ctx->pre_o;
    p.pre_ml = ctx->pre_ml;
    p.max_chunks = ctx->max_chunks;
  }

  if (ctx->test_wait_limit > 0) {  // one-shot failure-path test hook
    p.wait_limit = ctx->test_wait_limit;
    p.debug_stall = 1;
    ctx->test_wait_limit = 0;
  }

  merge_shape(c.head_dim, parts + prefix_chunks, c.num_heads, &p.merge_hpc, &p.merge_slices, &p.merge_hpt);
  void* args[] = {&mk, &mv, &p};
  cudaError_t e = cudaLaunchKernel(ctx->ks.decode, dim3(ctx->grid), dim3(ctx->ks.threads), args,
                                   ctx->ks.smem(q_slot_bytes(c.num_heads, c.num_kv_heads, c.head_dim), c.max_num_seqs), s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "decode launch");
  if ((pre || is_auto || parts > 1) && (e = launch_merge(ctx->ks, p, s)) != cudaSuccess)
    return cuda_fail(ctx, e, "merge launch");
  return PA_OK;
}

}  // namespace

PA_API int paged_attention_decode(pa_ctx* ctx, void* out, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* block_tables, int bt_stride,
                                  const int32_t* seq_lens, int num_seqs, int max_seq_len, float scale,
                                  float k_scale, float v_scale, void* stream) {
  PA_TRACE("paged_attention_decode");
  return decode_impl(ctx, out, query, key_cache, value_cache, block_tables, bt_stride, seq_lens, num_seqs,
                     max_seq_len, scale, k_scale, v_scale, stream, nullptr);
}

PA_API int paged_attention_decode_shared_prefix(pa_ctx* ctx, void* out, const void* query, const void* key_cache,
                                                const void* value_cache, const int32_t* block_tables,
                                                int bt_stride, const int32_t* seq_lens, int num_seqs,
                                                int max_seq_len, const int32_t* group_start,
                                                const int32_t* group_prefix_len, int num_groups,
                                                int max_group_size, int max_prefix_len, float scale,
                                                float k_scale, float v_scale, void* stream) {
  PA_TRACE("paged_attention_decode_shared_prefix");
  const PrefixArgs pre = {group_start, group_prefix_len, num_groups, max_group_size, max_prefix_len};
  return decode_impl(ctx, out, query, key_cache, value_cache, block_tables, bt_stride, seq_lens, num_seqs,
                     max_seq_len, scale, k_scale, v_scale, stream, &pre);
}

PA_API int paged_attention_prefill(pa_ctx* ctx, void* out, const void* query, const void* key_cache,
                                   const void* value_cache, const int32_t* block_tables, int bt_stride,
                                   const int32_t* seq_lens, const int32_t* query_start, int num_seqs, int num_tokens,
                                   int max_query_len, int max_seq_len, float scale, float k_scale, float v_scale,
                                   void* stream) {
  PA_TRACE("paged_attention_prefill");
  if (!ctx) return PA_ERR_INVALID_ARG;
  const pa_config& c = ctx->cfg;
  if (num_seqs < 0 || num_seqs > 65535) return fail(ctx, PA_ERR_INVALID_ARG, "num_seqs outside [0, 65535]");
  if (num_tokens < 0 || max_query_len < 0) return fail(ctx, PA_ERR_INVALID_ARG, "negative size");
  if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !query_start)
    return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
  if (bt_stride < 1) return fail(ctx, PA_ERR_INVALID_ARG, "bt_stride < 1");
  if (max_seq_len < 1 || max_seq_len > c.max_blocks_per_seq * c.block_size)
    return fail(ctx, PA_ERR_INVALID_ARG, "max_seq_len outside [1, max_blocks_per_seq*block_size]");
  if (max_query_len > max_seq_len) return fail(ctx, PA_ERR_INVALID_ARG, "max_query_len > max_seq_len");
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) || !aligned(query_start, 4))
    return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
  if (!std::isfinite(scale)) return fail(ctx, PA_ERR_INVALID_ARG, "scale not finite");
  const bool fp8 = c.kv_dtype == PA_FP8_E4M3;
  if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return fail(ctx, PA_ERR_INVALID_ARG, "fp8 scales must be finite and > 0");
  cudaSetDevice(ctx->device);
  pa::PrefillParams p;
  p.out = out;
  p.query = query;
  p.k_cache = key_cache;
  p.v_cache = value_cache;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.query_start = query_start;
  p.err = ctx->err;
  p.num_seqs = num_seqs;
  p.num_tokens = num_tokens;
  p.bt_stride = bt_stride;
  p.num_heads = c.num_heads;
  p.group = c.num_heads / c.num_kv_heads;
  p.head_splits = (p.group + pa::kNH - 1) / pa::kNH;
  p.num_blocks = c.num_blocks;
  p.max_blocks = (max_seq_len + c.block_size - 1) / c.block_size;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634 * (fp8 ? (double)k_scale : 1.0));
  p.v_scale = fp8 ? v_scale : 1.0f;
  const int hmax = p.group < pa::kNH ? p.group : pa::kNH;
  const int tpb = pa::kPrefixRows / hmax;  // query tokens per CTA (fewest: the widest KV unit)
  const dim3 grid((unsigned)((max_query_len + tpb - 1) / tpb), (unsigned)(c.num_kv_heads * p.head_splits),
                  (unsigned)num_seqs);
  void* args[] = {&p};
  cudaError_t e = cudaLaunchKernel(ctx->ks.prefill, grid, dim3(ctx->ks.prefix_threads), args, ctx->ks.prefix_smem,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(ctx, e, "prefill launch");
}

PA_API int paged_attn_get_error(pa_ctx* ctx, void* stream) {
  PA_TRACE("paged_attn_get_error");
  if (!ctx) return PA_ERR_INVALID_ARG;
  cudaSetDevice(ctx->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ctx->err_host, ctx->err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->err, 0, sizeof(int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "paged_attn_get_error");
  ctx->last_bits = *ctx->err_host;
  if (ctx->last_bits & PA_CHECK_WAIT_TIMEOUT) {
    // a launch that gave up may have left its work counters non-zero
    if ((e = cudaMemsetAsync(ctx->err + 1, 0, 2 * sizeof(int), s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
      return cuda_fail(ctx, e, "paged_attn_get_error(counter reset)");
  }
  return ctx->last_bits ? PA_ERR_DEVICE_CHECK : PA_OK;
}

PA_API int paged_attn_test_wait_timeout(pa_ctx* ctx, long long wait_limit_cycles) {
  if (!ctx) return PA_ERR_INVALID_ARG;
  if (wait_limit_cycles < 1000 || wait_limit_cycles > pa::kWaitLimitCycles)
    return fail(ctx, PA_ERR_INVALID_ARG, "wait_limit_cycles outside [1000, default limit]");
  ctx->test_wait_limit = wait_limit_cycles;
  return PA_OK;
}

PA_API int paged_gather_kv(pa_ctx* ctx, void* k_out, void* v_out, const void* key_cache, const void* value_cache,
                           const int32_t* block_table_row, int seq_len, void* stream) {
  PA_TRACE("paged_gather_kv");
  if (!ctx) return PA_ERR_INVALID_ARG;
  const pa_config& c = ctx->cfg;
  if (seq_len < 0 || seq_len > c.max_blocks_per_seq * c.block_size)
    return fail(ctx, PA_ERR_INVALID_ARG, "seq_len out of range");
  if (seq_len == 0) return PA_OK;
  if (!k_out || !v_out || !key_cache || !value_cache || !block_table_row)
    return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(k_out, 16) || !aligned(v_out, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16))
    return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
  cudaSetDevice(ctx->device);
  pa::GatherParams p;
  p.k_out = k_out;
  p.v_out = v_out;
  p.key_cache = key_cache;
  p.value_cache = value_cache;
  p.block_table = block_table_row;
  p.seq_len = seq_len;
  p.row_bytes = c.num_kv_heads * c.head_dim * elem_bytes(c.kv_dtype);
  p.num_blocks = c.num_blocks;
  p.err = ctx->err;
  const long long vecs = (long long)seq_len * (p.row_bytes / 16);
  long long blocks = (vecs + 255) / 256;
  if (blocks > (long long)ctx->num_sms * 8) blocks = (long long)ctx->num_sms * 8;
  pa::paged_gather_kernel<<<dim3((unsigned)blocks, 2), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(ctx, e, "paged_gather_kv launch");
}

// ---------------------------------------------------------------------------
// Decode without any allocation.
//
// Some callers cannot call cudaMalloc at all: hosts that hand out device
// memory only from their own pool or arena and forbid outside allocations
// (an inference server that budgets every byte of HBM up front), or callers
// that must not risk an allocation failure, or the allocator's implicit
// device synchronisation, in the middle of a serving step.  For them this
// entry point needs no context: the split-KV partials live in one file-scope
// device array of fixed size, which every GPU that loads this library holds
// until the process exits.
//
// The array is shared by every call on a device and keeps whatever the last
// call left in it.  Only its 256-byte header (the check word and the decode
// kernel's work-ticket counters) must start at zero: the first call on a
// device clears it on the caller's stream, ahead of its own kernels, and
// every launch leaves the counters at zero again.  Every partial that the
// merge reads is written earlier in the same call; the check word is only
// ever or-ed into.  Two calls whose kernels overlap on the GPU (different
// streams, or different host threads, on one device) race on the array.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoallocDevices = 64;
constexpr size_t kNoallocHeader = 256;  // bytes reserved at the front (check word, work counters)

struct NoallocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int num_sms = 0;
  int smem_optin = 0;
};
NoallocDevice g_noalloc_dev[kMaxNoallocDevices];
std::mutex g_noalloc_mu;

// Every (head_dim, q_dtype, kv_dtype) the library has decode kernels for.
constexpr int kDecodeCombos[][3] = {{64, PA_F16, PA_F16},        {128, PA_F16, PA_F16},
                                    {256, PA_F16, PA_F16},       {64, PA_BF16, PA_BF16},
                                    {128, PA_BF16, PA_BF16},     {256, PA_BF16, PA_BF16},
                                    {128, PA_F16, PA_FP8_E4M3},  {256, PA_F16, PA_FP8_E4M3}};

// First call on `dev` (the current device): the device address of the
// scratch array (its name in host code is only a host-side handle; kernels
// must be given the address cudaGetSymbolAddress returns with the device
// current), the shared-memory limit and carve-out of every decode and merge
// kernel, and the header cleared on `stream`, so that the caller's first
// kernels, queued after it on the same stream, see zero counters whatever
// kind of stream it is.  Later calls only read the cached record.
int noalloc_setup(int dev, cudaStream_t stream, NoallocDevice* out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return PA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return PA_ERR_CUDA;
    for (const auto& c : kDecodeCombos) {
      KernelSet ks;
      if (!select_kernels(c[0], c[1], c[2], &ks)) return PA_ERR_CUDA;
      if (cudaFuncSetAttribute(ks.decode, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) !=
              cudaSuccess ||
          pin_carveout(ks.decode) != cudaSuccess || pin_carveout(ks.merge) != cudaSuccess)
        return PA_ERR_CUDA;
      if (ks.decode_shallow &&
          (cudaFuncSetAttribute(ks.decode_shallow, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) !=
               cudaSuccess ||
           pin_carveout(ks.decode_shallow) != cudaSuccess))
        return PA_ERR_CUDA;
    }
    if (cudaMemsetAsync(p, 0, kNoallocHeader, stream) != cudaSuccess) return PA_ERR_CUDA;
    d.scratch = static_cast<unsigned char*>(p);
    d.ready = true;
  }
  *out = d;
  return PA_OK;
}

// Same 2-D view and box as tensor_map(), encoded on the stack each call.
int encode_cache_map(const void* base, int kv_dtype, int num_kv_heads, int head_dim, int num_blocks, CUtensorMap* m) {
  auto enc = encode_fn();
  if (!enc) return PA_ERR_CUDA;
  const int eb = elem_bytes(kv_dtype);
  cuuint64_t dims[2] = {(cuuint64_t)num_kv_heads * head_dim, (cuuint64_t)num_blocks * pa::kBS};
  cuuint64_t strides[1] = {(cuuint64_t)num_kv_heads * head_dim * eb};
  cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)pa::kBS};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

PA_API int paged_attention_decode_noalloc(void* out, const void* query, const void* key_cache,
                                          const void* value_cache, const int32_t* block_tables, int bt_stride,
                                          const int32_t* seq_lens, int num_seqs, int max_seq_len, int num_heads,
                                          int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                          int q_dtype, int kv_dtype, int partition_tokens, float scale,
                                          float k_scale, float v_scale, int* check_bits, void* stream) {
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || num_blocks <= 0 || num_seqs < 0 ||
      bt_stride < 1 || max_seq_len < 0 || partition_tokens < 0)
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBS) return PA_ERR_UNSUPPORTED;
  if (partition_tokens % block_size) return PA_ERR_INVALID_ARG;
  if ((long long)num_blocks * block_size > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  KernelSet ks;
  if (!select_kernels(head_dim, q_dtype, kv_dtype, &ks)) return PA_ERR_UNSUPPORTED;
  if ((long long)num_kv_heads * head_dim * elem_bytes(kv_dtype) % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) || (check_bits && !aligned(check_bits, 4)))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  const bool fp8 = kv_dtype == PA_FP8_E4M3;
  if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return PA_ERR_INVALID_ARG;

  // Size the split before touching the device: refuse what the array cannot hold.
  const int max_blocks = (max_seq_len + block_size - 1) / block_size;
  const int part_blocks = partition_tokens > 0 ? partition_tokens / block_size : (max_blocks > 0 ? max_blocks : 1);
  int parts = (max_blocks + part_blocks - 1) / part_blocks;
  if (parts < 1) parts = 1;
  const size_t rows = (size_t)num_seqs * num_heads * parts;
  const size_t codes = ((size_t)num_seqs * sizeof(int) + 255) / 256 * 256;  // the merge's per-sequence work
  const size_t ml_bytes = (rows * 2 * sizeof(float) + 255) / 256 * 256;
  const size_t need = kNoallocHeader + codes + (parts > 1 ? ml_bytes + rows * head_dim * sizeof(float) : 0);
  if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_SCRATCH_TOO_SMALL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoallocDevices) return PA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  NoallocDevice nd;
  int st = noalloc_setup(dev, s, &nd);
  if (st != PA_OK) return st;
  unsigned char* scratch = nd.scratch;
  const int num_sms = nd.num_sms;
  if (ks.smem(q_slot_bytes(num_heads, num_kv_heads, head_dim), num_seqs) > (size_t)nd.smem_optin)
    return PA_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (choose_decode(&ks, q_slot_bytes(num_heads, num_kv_heads, head_dim), num_seqs, &per_sm) != cudaSuccess ||
      per_sm < 1)
    return PA_ERR_CUDA;
  const size_t smem = ks.smem(q_slot_bytes(num_heads, num_kv_heads, head_dim), num_seqs);

  CUtensorMap mk, mv;
  if ((st = encode_cache_map(key_cache, kv_dtype, num_kv_heads, head_dim, num_blocks, &mk)) != PA_OK) return st;
  if ((st = encode_cache_map(value_cache, kv_dtype, num_kv_heads, head_dim, num_blocks, &mv)) != PA_OK) return st;

  DecodeParams p;
  p.out = out;
  p.query = query;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.seq_merge = reinterpret_cast<int*>(scratch + kNoallocHeader);
  p.part_ml = reinterpret_cast<float*>(scratch + kNoallocHeader + codes);
  p.part_o = reinterpret_cast<float*>(scratch + kNoallocHeader + codes + ml_bytes);
  p.err = check_bits ? check_bits : reinterpret_cast<int*>(scratch);
  p.counters = reinterpret_cast<int*>(scratch) + 4;
  p.num_seqs = num_seqs;
  p.bt_stride = bt_stride;
  p.num_heads = num_heads;
  p.group = num_heads / num_kv_heads;
  p.head_splits = (p.group + pa::kNH - 1) / pa::kNH;
  p.kv_units = num_kv_heads * p.head_splits;
  p.q_slot_bytes = q_slot_bytes(num_heads, num_kv_heads, head_dim);
  p.num_blocks = num_blocks;
  p.max_blocks = max_blocks > 0 ? max_blocks : 1;
  p.force_partials = 0;
  p.partition_blocks = part_blocks;
  p.auto_mode = 0;
  p.min_piece_blocks = kMinPieceBlocks;
  p.max_parts = parts;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634 * (fp8 ? (double)k_scale : 1.0));
  p.v_scale = fp8 ? v_scale : 1.0f;

  merge_shape(head_dim, parts, num_heads, &p.merge_hpc, &p.merge_slices, &p.merge_hpt);
  void* args[] = {&mk, &mv, &p};
  if (cudaLaunchKernel(ks.decode, dim3(num_sms * per_sm), dim3(ks.threads), args, smem, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (parts > 1 && launch_merge(ks, p, s) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

PA_API int paged_copy_blocks(pa_ctx* ctx, void* dst_key_cache, void* dst_value_cache, int64_t dst_num_blocks,
                             const void* src_key_cache, const void* src_value_cache, int64_t src_num_blocks,
                             const int64_t* block_pairs, int num_pairs, void* stream) {
  PA_TRACE("paged_copy_blocks");
  if (!ctx) return PA_ERR_INVALID_ARG;
  const pa_config& c = ctx->cfg;
  if (num_pairs < 0) return fail(ctx, PA_ERR_INVALID_ARG, "num_pairs < 0");
  if (num_pairs == 0) return PA_OK;
  if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || !block_pairs)
    return fail(ctx, PA_ERR_INVALID_ARG, "null pointer");
  if (dst_num_blocks <= 0 || src_num_blocks <= 0) return fail(ctx, PA_ERR_INVALID_ARG, "block counts must be > 0");
  if (!aligned(dst_key_cache, 16) || !aligned(dst_value_cache, 16) || !aligned(src_key_cache, 16) ||
      !aligned(src_value_cache, 16) || !aligned(block_pairs, 8))
    return fail(ctx, PA_ERR_INVALID_ARG, "misaligned pointer");
  cudaSetDevice(ctx->device);
  pa::CopyBlocksParams p;
  p.dst_key = dst_key_cache;
  p.dst_value = dst_value_cache;
  p.src_key = src_key_cache;
  p.src_value = src_value_cache;
  p.pairs = reinterpret_cast<const long long*>(block_pairs);
  p.num_pairs = num_pairs;
  p.block_vecs = c.block_size * c.num_kv_heads * c.head_dim * elem_bytes(c.kv_dtype) / 16;
  p.src_blocks = src_num_blocks;
  p.dst_blocks = dst_num_blocks;
  p.err = ctx->err;
  long long blocks = num_pairs;
  const long long cap = (long long)ctx->num_sms * 16;
  if (blocks > cap) blocks = cap;
  pa::paged_copy_blocks_kernel<<<dim3((unsigned)blocks, 2), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(ctx, e, "paged_copy_blocks launch");
}
