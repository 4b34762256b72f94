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

namespace {

// Column of the side copy that holds head dimension `dim`, or -1 when dim's 64-dim chunk
// is not copied.
__device__ __forceinline__ int side_col(uint32_t chunk_mask, int dim) {
  const int c = dim >> 6;
  if (!((chunk_mask >> c) & 1u)) return -1;
  return __popc(chunk_mask & ((1u << c) - 1u)) * 64 + (dim & 63);
}

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

// Rotates (or copies) the 8 pairs j0..j0+7 of every head of one token of one tensor,
// four heads at a time so that eight 16-byte loads are in flight before any store.
__device__ __forceinline__ void rope_heads(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                           int heads, int tok, int d, int n_out, int j0, int col0, int col1,
                                           bool pad, const float* c, const float* s) {
  const int half = d / 2;
  for (int h0 = 0; h0 < heads; h0 += 4) {
    uint4 a[4], b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (h0 + k < heads) {
        const uint16_t* p = src + ((size_t)tok * heads + h0 + k) * d;
        a[k] = __ldg(reinterpret_cast<const uint4*>(p + j0));
        b[k] = __ldg(reinterpret_cast<const uint4*>(p + j0 + half));
      }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (h0 + k < heads) {
        uint16_t* q = dst + ((size_t)tok * heads + h0 + k) * n_out;
        float x0[8], x1[8], y0[8], y1[8];
        unpack8(a[k], x0);
        unpack8(b[k], x1);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          y0[e] = x0[e] * c[e] - x1[e] * s[e];
          y1[e] = x0[e] * s[e] + x1[e] * c[e];
        }
        if (col0 >= 0) *reinterpret_cast<uint4*>(q + col0) = pack8(y0);
        if (col1 >= 0) *reinterpret_cast<uint4*>(q + col1) = pack8(y1);
        if (pad)
          for (int z = d; z < 64; z += 8) *reinterpret_cast<uint4*>(q + z) = make_uint4(0, 0, 0, 0);
      }
  }
}

// One thread per (token, group of 8 consecutive pairs j0..j0+7): it computes the 8
// angles once and rotates those pairs in every head of the token, for the queries and
// (in the same launch) the keys, with 16-byte loads and stores of both halves (dims
// j0.. and j0 + d/2 ..).
__global__ void rope_side_kernel(RopeArgs a) {
  const int half = a.d / 2;
  const int groups = a.groups_active;  // later groups have no dim in the copied chunks
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.tokens * groups) return;
  const int tok = (int)(idx / groups);
  const int j0 = (int)(idx % groups) * 8;
  const int col0 = side_col(a.chunk_mask, j0);
  const int col1 = side_col(a.chunk_mask, j0 + half);
  const bool pad = a.d < 64 && j0 == 0;  // this thread also zeroes the padding columns d .. 63
  if (col0 < 0 && col1 < 0 && !pad) return;  // neither half of these pairs is in the copy
  float c[8], s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    c[e] = 1.f;
    s[e] = 0.f;
    if (j0 + e < a.r) rope_cos_sin((double)a.positions[tok], rope_inv_freq_turns(j0 + e, a.d, a.log2_base), &c[e], &s[e]);
  }
  rope_heads(a.src, a.dst, a.heads, tok, a.d, a.n_out, j0, col0, col1, pad, c, s);
  if (a.heads2 > 0) rope_heads(a.src2, a.dst2, a.heads2, tok, a.d, a.n_out, j0, col0, col1, pad, c, s);
}

// 2D rotation for the vision encoder's patches ("Visual guide to Gemma 4", section
// "Vision encoder": the embedding split in two parts that encode the horizontal and the
// vertical position separately): dims [0, d/2) rotated by w, dims [d/2, d) by h, each
// half as a d/2-dim rotation with pairs (j, j + d/4) and theta_j = base^(-2j/(d/2)).
// One thread per (token, half, group of 8 pairs of that half): it computes the 8 angles
// once and rotates those pairs in every head of the queries and the keys; every dim of
// a row is rotated, so the copy holds whole rows.
__global__ void rope2d_side_kernel(Rope2dArgs a) {
  const int quarter = a.d / 4;               // pairs per half
  const int groups = a.d / 32;               // groups of 8 pairs per half
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.tokens * 2 * groups) return;
  const int tok = (int)(idx / (2 * groups));
  const int part = (int)((idx / groups) % 2);  // 0: first half, position w; 1: second half, position h
  const int j0 = (int)(idx % groups) * 8;
  const int pos = a.positions_hw[2 * tok + (part == 0 ? 1 : 0)];
  float c[8], s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) rope_cos_sin((double)pos, rope_inv_freq_turns(j0 + e, a.d / 2, a.log2_base), &c[e], &s[e]);
  const int col0 = part * (a.d / 2) + j0, col1 = col0 + quarter;
  for (int t = 0; t < 2; ++t) {
    const uint16_t* src = t == 0 ? a.src : a.src2;
    uint16_t* dst = t == 0 ? a.dst : a.dst2;
    const int heads = t == 0 ? a.heads : a.heads2;
    for (int h = 0; h < heads; ++h) {
      const size_t row = ((size_t)tok * heads + h) * a.d;
      float x0[8], x1[8], y0[8], y1[8];
      unpack8(*reinterpret_cast<const uint4*>(src + row + col0), x0);
      unpack8(*reinterpret_cast<const uint4*>(src + row + col1), x1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        y0[e] = x0[e] * c[e] - x1[e] * s[e];
        y1[e] = x0[e] * s[e] + x1[e] * c[e];
      }
      *reinterpret_cast<uint4*>(dst + row + col0) = pack8(y0);
      *reinterpret_cast<uint4*>(dst + row + col1) = pack8(y1);
    }
  }
}

cudaError_t launch_rope2d_side(const Rope2dArgs& a, cudaStream_t stream) {
  const long long total = (long long)a.tokens * 2 * (a.d / 32);
  if (total == 0) return cudaSuccess;
  const int threads = 128;
  rope2d_side_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rope_side(const RopeArgs& a, cudaStream_t stream) {
  const long long total = (long long)a.tokens * a.groups_active;
  if (total == 0 || a.n_out == 0) return cudaSuccess;
  const int threads = 128;
  const long long blocks = (total + threads - 1) / threads;
  rope_side_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gattn
