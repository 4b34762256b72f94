// append.cu -- write the new tokens' K (and V) rows into a decode cache.
//
// After a decode / verify step has read the new tokens from new_k / new_v beside the
// cache, their rows join the cache: token i of sequence b sits at position
// p = cache_seqlens[b] + i and goes to slot p mod W of a window ring (local layers) or to
// row p of a contiguous cache (global layers: the single K=V tensor, "Visual guide to
// Gemma 4", sections "K=V technique" and "GQA": the KV cache holds one projected tensor
// per KV head). A ring whose keys are kept rotated receives the key rotated for p (the
// first r pairs, (j, j + d/2), angle p * base^(-2j/d): section "p-RoPE"); values and
// K=V rows are stored as given.
//
// One warp per (sequence, new token, KV head) row: lanes copy 16-byte chunks; for a
// rotated key, lane l takes the chunk pairs (c, c + d/16) holding pairs 8c .. 8c + 7, so
// both halves of each pair are in its registers.
#include "common.cuh"
#include "kernels.h"

namespace gattn {

namespace {

__device__ __forceinline__ void unpack8_bf16(const uint4& w, float* f) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(ws[k] << 16);
    f[2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

}  // namespace

__global__ void cache_append_kernel(AppendArgs a) {
  const int warp_global = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int rows = a.batch * a.n_q * a.num_kv_heads;
  if (warp_global >= rows) return;
  const int kvh = warp_global % a.num_kv_heads;
  const int i = (warp_global / a.num_kv_heads) % a.n_q;
  const int b = warp_global / (a.num_kv_heads * a.n_q);
  const int len = a.cache_seqlens[b];
  const int pos = len + i;
  if (len < 0 || (!a.ring && pos >= a.capacity)) {  // no room: record it, write nothing
    if (lane == 0) atomicOr(&g_status, kStatusSeqlen);
    return;
  }
  // A ring keeps the newest `capacity` positions: with more new tokens than slots, token
  // i and token i + capacity map to the same slot, and only the later one is written.
  if (a.ring && i < a.n_q - a.capacity) return;
  const int slot = a.ring ? pos % a.capacity : pos;
  const size_t src_row = (((size_t)b * a.n_q + i) * a.num_kv_heads + kvh) * a.head_dim;
  const size_t dst_row = (((size_t)b * a.num_kv_heads + kvh) * a.capacity + slot) * a.head_dim;
  const int chunks = a.head_dim / 8;  // 16-byte chunks per row
  // values (separate-V layers) and un-rotated keys: plain copies
  if (a.v_cache != nullptr)
    for (int c = lane; c < chunks; c += 32)
      *reinterpret_cast<uint4*>(a.v_cache + dst_row + c * 8) = *reinterpret_cast<const uint4*>(a.new_v + src_row + c * 8);
  if (!a.keys_rotated || a.r == 0) {
    for (int c = lane; c < chunks; c += 32)
      *reinterpret_cast<uint4*>(a.k_cache + dst_row + c * 8) = *reinterpret_cast<const uint4*>(a.new_k + src_row + c * 8);
    return;
  }
  const int halfc = chunks / 2;  // chunk c of the first half pairs with chunk c + halfc
  for (int c = lane; c < halfc; c += 32) {
    float x0[8], x1[8], y0[8], y1[8];
    unpack8_bf16(*reinterpret_cast<const uint4*>(a.new_k + src_row + c * 8), x0);
    unpack8_bf16(*reinterpret_cast<const uint4*>(a.new_k + src_row + (c + halfc) * 8), x1);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 8 * c + e;
      if (j < a.r) {
        float cs, sn;
        rope_cos_sin((double)pos, rope_inv_freq_turns(j, a.head_dim, a.log2_base), &cs, &sn);
        y0[e] = x0[e] * cs - x1[e] * sn;
        y1[e] = x0[e] * sn + x1[e] * cs;
      } else {
        y0[e] = x0[e];
        y1[e] = x1[e];
      }
    }
    *reinterpret_cast<uint4*>(a.k_cache + dst_row + c * 8) = pack8_bf16(y0);
    *reinterpret_cast<uint4*>(a.k_cache + dst_row + (c + halfc) * 8) = pack8_bf16(y1);
  }
}

cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream) {
  const long long rows = (long long)a.batch * a.n_q * a.num_kv_heads;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;  // 8 rows per block
  const long long blocks = (rows * 32 + threads - 1) / threads;
  cache_append_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gattn
