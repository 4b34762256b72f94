// decode_noalloc.cu -- decode + combine in one call that allocates no device memory.
//
// Some callers cannot allocate device memory for the split partials themselves: a
// framework that owns every device allocation may not expose a scratch allocator to
// an attention op, and a caller in the middle of capturing a CUDA graph cannot call
// cudaMalloc. For them the partials live in a static array compiled into this
// library. The caller still passes every input and output buffer.
//
// The array is shared by all calls on a device and keeps the last call's contents.
// Nothing in it needs clearing: every call rewrites all of the partials it reads.
// Two calls that overlap on the GPU (different streams, or host threads without
// ordering between their streams) race on it.
// With num_splits == 1 there are no partials: the decode kernel writes the output and
// log-sum-exp itself, in one launch, and the array is not touched.
#include <atomic>
#include <mutex>

#include "../../include/gemma_attn.h"
#include "common.cuh"
#include "kernels.h"

namespace gattn {
namespace {

constexpr size_t kNoAllocBytes = GEMMA_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocMaxDevices = 64;

// Split partials (fp32 O, then fp32 log-sum-exp) of gemma_attn_decode_noalloc. Each GPU
// that loads the library holds these bytes until the process exits. In host code this
// name is only a stand-in for the symbol, never a device address: host code passes the
// address that cudaGetSymbolAddress returns for the current device.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::atomic<void*> g_noalloc_addr[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device; looked up once per device.
int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GEMMA_ATTN_ERR_DEVICE;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return GEMMA_ATTN_ERR_UNSUPPORTED;
  void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    p = g_noalloc_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return GEMMA_ATTN_ERR_DEVICE;
      g_noalloc_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return GEMMA_ATTN_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace gattn

extern "C" int gemma_attn_decode_noalloc(const gemma_attn_params* params, const void* q, const void* new_k,
                                         const void* new_v, const void* k_cache, const void* v_cache,
                                         int32_t cache_layout, int32_t cache_capacity,
                                         const int32_t* cache_seqlens, int32_t batch, int32_t n_q,
                                         int32_t max_cache_len, int32_t num_splits, void* out, float* lse,
                                         void* stream_) {
  using namespace gattn;
  if (!params) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (params->kind == GEMMA_ATTN_BIDIR) return GEMMA_ATTN_ERR_UNSUPPORTED;  // prefill only
  if (params->kind != GEMMA_ATTN_LOCAL && params->kind != GEMMA_ATTN_GLOBAL) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (params->num_q_heads <= 0 || params->num_kv_heads <= 0 || params->num_q_heads % params->num_kv_heads)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  const int d = params->head_dim;
  if (d != 32 && d != 64 && d != 128 && d != 256 && d != 512) return GEMMA_ATTN_ERR_UNSUPPORTED;
  if (params->kind == GEMMA_ATTN_LOCAL && params->window < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (!(params->rope_p >= 0.f && params->rope_p <= 1.f) || !(params->rope_base > 0.f) ||
      !(params->softmax_scale > 0.f))
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (params->out_dtype != GEMMA_ATTN_OUT_BF16 && params->out_dtype != GEMMA_ATTN_OUT_F32)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  const bool global = params->kind == GEMMA_ATTN_GLOBAL;
  if (!q || !new_k || !k_cache || !cache_seqlens || !out) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (global != (new_v == nullptr) || global != (v_cache == nullptr)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (batch < 1 || n_q < 1 || num_splits < 1 || max_cache_len < 0 || cache_capacity < 1)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  const bool keys_rotated = (cache_layout & GEMMA_ATTN_CACHE_KEYS_ROTATED) != 0;
  if (keys_rotated && global) return GEMMA_ATTN_ERR_INVALID_ARG;  // the K=V tensor is also the values
  cache_layout &= ~GEMMA_ATTN_CACHE_KEYS_ROTATED;
  if (cache_layout != GEMMA_ATTN_CACHE_CONTIGUOUS && cache_layout != GEMMA_ATTN_CACHE_RING)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_layout == GEMMA_ATTN_CACHE_RING && (global || cache_capacity != params->window))
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_layout == GEMMA_ATTN_CACHE_CONTIGUOUS && cache_capacity < max_cache_len)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  const int group = params->num_q_heads / params->num_kv_heads;
  if (group * n_q > decode_max_rows(params->head_dim)) return GEMMA_ATTN_ERR_UNSUPPORTED;
  if (((uintptr_t)q | (uintptr_t)new_k | (uintptr_t)new_v | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15u)
    return GEMMA_ATTN_ERR_MISALIGNED;

  // One split: the decode kernel writes out and lse itself (the combine of a single
  // partial is the identity) and nothing is staged. Otherwise partials for
  // num_splits x rows: fp32 O [splits, rows, d] then fp32 lse [splits, rows].
  const bool direct = num_splits == 1;
  const size_t rows = (size_t)batch * n_q * params->num_q_heads;
  const size_t o_bytes = align256((size_t)num_splits * rows * d * sizeof(float));
  const size_t l_bytes = align256((size_t)num_splits * rows * sizeof(float));
  float* partial_o = nullptr;
  float* partial_lse = nullptr;
  if (!direct) {
    if (o_bytes + l_bytes > kNoAllocBytes) return GEMMA_ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc != GEMMA_ATTN_OK) return rc;
    partial_o = static_cast<float*>(scratch);
    partial_lse = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + o_bytes);
  }

  DecodeArgs a{};
  if (direct) {
    a.out = out;
    a.out_lse = lse;
    a.out_f32 = params->out_dtype == GEMMA_ATTN_OUT_F32;
  }
  a.q = static_cast<const uint16_t*>(q);
  a.new_k = static_cast<const uint16_t*>(new_k);
  a.new_v = static_cast<const uint16_t*>(new_v);
  a.k_cache = static_cast<const uint16_t*>(k_cache);
  a.v_cache = static_cast<const uint16_t*>(v_cache);
  a.cache_seqlens = cache_seqlens;
  a.partial_o = partial_o;
  a.partial_lse = partial_lse;
  a.batch = batch; a.n_q = n_q; a.num_q_heads = params->num_q_heads; a.num_kv_heads = params->num_kv_heads;
  a.head_dim = d; a.is_local = global ? 0 : 1; a.window = global ? 0 : params->window;
  a.ring = cache_layout == GEMMA_ATTN_CACHE_RING; a.capacity = cache_capacity; a.num_splits = num_splits;
  a.keys_rotated = keys_rotated ? 1 : 0;
  a.r = rotated_pairs(params->rope_p, d);
  a.log2_base = log2((double)params->rope_base);
  a.softmax_scale = params->softmax_scale;
  if (!decode_supported(a)) return GEMMA_ATTN_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (launch_decode(a, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  if (direct) return GEMMA_ATTN_OK;

  CombineArgs c;
  c.partial_o = partial_o; c.partial_lse = partial_lse; c.out = out; c.lse = lse;
  c.num_splits = num_splits; c.rows = (int)rows; c.head_dim = d;
  c.out_f32 = params->out_dtype == GEMMA_ATTN_OUT_F32;
  if (launch_combine(c, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  return GEMMA_ATTN_OK;
}
