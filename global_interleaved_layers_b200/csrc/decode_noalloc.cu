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
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

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
  set_launch_count(0);
  if (!out) return GEMMA_ATTN_ERR_INVALID_ARG;
  DecodeArgs a{};
  int rc = decode_prepare(params, q, new_k, new_v, k_cache, v_cache, cache_layout, cache_capacity, cache_seqlens,
                          batch, n_q, max_cache_len, num_splits, &a);
  if (rc != GEMMA_ATTN_OK) return rc;
  // Every call, whatever its split count, looks the array's address up first, so that
  // the first call on a device does the lookup (outside any stream capture the caller
  // starts later).
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != GEMMA_ATTN_OK) return rc;

  // One split: the decode kernel writes out and lse itself (the combine of a single
  // partial is the identity) and nothing is staged. Otherwise partials for
  // num_splits x rows: fp32 O [splits, rows, d] then fp32 lse [splits, rows].
  const bool direct = num_splits == 1;
  const int d = params->head_dim;
  const size_t rows = (size_t)batch * n_q * params->num_q_heads;
  const size_t o_bytes = align256((size_t)num_splits * rows * d * sizeof(float));
  const size_t l_bytes = align256((size_t)num_splits * rows * sizeof(float));
  const bool f32 = params->out_dtype == GEMMA_ATTN_OUT_F32;
  if (direct) {
    a.out = out;
    a.out_lse = lse;
    a.out_f32 = f32 ? 1 : 0;
  } else {
    if (o_bytes + l_bytes > kNoAllocBytes) return GEMMA_ATTN_ERR_WORKSPACE;
    a.partial_o = static_cast<float*>(scratch);
    a.partial_lse = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + o_bytes);
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (launch_decode(a, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  if (direct) {
    set_launch_count(1);
    return GEMMA_ATTN_OK;
  }

  CombineArgs c;
  c.partial_o = a.partial_o; c.partial_lse = a.partial_lse; c.out = out; c.lse = lse;
  c.num_splits = num_splits; c.rows = (int)rows; c.head_dim = d;
  c.out_f32 = f32 ? 1 : 0;
  if (launch_combine(c, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  set_launch_count(2);
  return GEMMA_ATTN_OK;
}
