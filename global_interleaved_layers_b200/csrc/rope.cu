// rope.cu -- rotated side copy of the 64-dim chunks that p-RoPE touches.
//
// p-RoPE rotates only the r = floor(p*d/2) highest-frequency pairs (j, j + d/2) and
// passes the rest through ("Visual guide to Gemma 4", section "p-RoPE"). The prefill
// kernel reads every chunk that contains a rotated dimension from this copy and all
// other chunks (and all value chunks) from the caller's un-rotated tensor. For head
// dims below 64 the copy is also the zero-padded operand the 64-wide tiles need.
#include "common.cuh"
#include "kernels.h"

namespace gattn {

// One thread per (token, output column); the angle is computed once and applied to
// every head of that token.
__global__ void rope_side_kernel(RopeArgs a) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)a.tokens * a.n_out;
  if (idx >= total) return;
  const int tok = (int)(idx / a.n_out);
  const int o = (int)(idx % a.n_out);
  // o-th copied column -> dimension of the (padded) head
  int want = o / 64, chunk = 0;
  for (int c = 0; c < 32; ++c) {
    if ((a.chunk_mask >> c) & 1u) {
      if (want == 0) { chunk = c; break; }
      --want;
    }
  }
  const int dim = chunk * 64 + (o % 64);
  const int half = a.d / 2;
  uint16_t* dst = a.dst + (size_t)tok * a.heads * a.n_out + o;
  const uint16_t* src = a.src + (size_t)tok * a.heads * a.d;
  if (dim >= a.d) {
    for (int h = 0; h < a.heads; ++h) dst[(size_t)h * a.n_out] = 0;
    return;
  }
  const int j = dim < half ? dim : dim - half;
  if (j >= a.r) {
    for (int h = 0; h < a.heads; ++h) dst[(size_t)h * a.n_out] = src[(size_t)h * a.d + dim];
    return;
  }
  float c, s;
  rope_cos_sin((double)a.positions[tok], rope_inv_freq_turns(j, a.d, a.log2_base), &c, &s);
  for (int h = 0; h < a.heads; ++h) {
    const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(src + (size_t)h * a.d);
    const float x0 = __bfloat162float(row[j]);
    const float x1 = __bfloat162float(row[j + half]);
    const float y = dim < half ? (x0 * c - x1 * s) : (x0 * s + x1 * c);
    __nv_bfloat16 yb = __float2bfloat16_rn(y);
    dst[(size_t)h * a.n_out] = *reinterpret_cast<uint16_t*>(&yb);
  }
}

cudaError_t launch_rope_side(const RopeArgs& a, cudaStream_t stream) {
  const long long total = (long long)a.tokens * a.n_out;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  rope_side_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gattn
