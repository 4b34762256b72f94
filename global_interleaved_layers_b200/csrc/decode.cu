// decode.cu -- split-KV decode / speculative verify, and the log-sum-exp combine.
//
// n_q new query tokens per sequence attend to the sequence's cached keys plus the
// new tokens themselves. Local layers read a window-slot ring (token p in slot
// p mod W); global layers read a contiguous cache holding the single K=V tensor
// ("Visual guide to Gemma 4", sections "K=V technique" and "GQA": the KV cache is
// what GQA and K=V shrink). Keys are stored un-rotated: the copy used for scores
// is rotated on load (p-RoPE: only the first r pairs), values are used as loaded.
//
// The visible keys of a sequence, ordered by position, are cut into `num_splits`
// contiguous ranges; one CTA handles (sequence, KV head, split) for all query
// heads of that KV head and all n_q tokens, and writes an unnormalised partial
// (O / l and the log-sum-exp) that the combine kernel merges.
#include "common.cuh"
#include "kernels.h"

namespace gattn {

namespace {
constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kRowsPerWarp = 8;
}

// Each warp owns up to 8 query rows (a row = one query head for one new token) and
// a strided subset of the split's keys. A lane holds H = D/64 consecutive dims from
// each half of the head (dims lane*H.. and D/2 + lane*H..), so both members of every
// rotary pair sit in the same lane.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(DecodeArgs a) {
  constexpr int HALF = D / 2;
  constexpr int H = (HALF >= 32) ? HALF / 32 : 1;   // dims per half per lane
  constexpr int ACTIVE = (HALF >= 32) ? 32 : HALF;  // lanes holding dims
  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int group = a.num_q_heads / a.num_kv_heads;
  const int G = group * a.n_q;                       // query rows of this CTA
  const int nrg = (G + kRowsPerWarp - 1) / kRowsPerWarp;
  const int streams = kDecWarps / nrg;               // warps per row group (>= 1)
  const int rg = warp % nrg;
  const int stream_id = warp / nrg;
  const bool warp_active = warp < nrg * streams;

  const int len = a.cache_seqlens[b];
  const int first = a.is_local ? max(0, len - a.window + 1) : 0;  // oldest position any query sees
  const int nk = (len - first) + a.n_q;
  const int per = (nk + a.num_splits - 1) / a.num_splits;
  const int v_lo = split * per;
  const int v_hi = min(nk, v_lo + per);

  extern __shared__ float dsm[];
  float* qs = dsm;                                   // [G][D] rotated, scaled queries
  float* red = qs + (size_t)G * D;                   // [warps][8][D + 2] partial states

  const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
  // ---- rotated queries into shared memory
  for (int idx = threadIdx.x; idx < G * HALF; idx += kDecThreads) {
    const int g = idx / HALF, j = idx % HALF;
    const int i = g / group, hh = g % group;
    const int qpos = len + i;
    const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(
        a.q + (((size_t)b * a.n_q + i) * a.num_q_heads + kvh * group + hh) * D);
    float x0 = __bfloat162float(qrow[j]), x1 = __bfloat162float(qrow[j + HALF]);
    float y0 = x0, y1 = x1;
    if (j < a.r) {
      float c, s;
      rope_cos_sin((double)qpos, rope_inv_freq_turns(j, D, a.log2_base), &c, &s);
      y0 = x0 * c - x1 * s;
      y1 = x0 * s + x1 * c;
    }
    qs[g * D + j] = y0 * scale_log2;
    qs[g * D + j + HALF] = y1 * scale_log2;
  }
  __syncthreads();

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][2 * H];
#pragma unroll
  for (int g = 0; g < kRowsPerWarp; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 2 * H; ++e) o[g][e] = 0.f;
  }
  const int g0 = rg * kRowsPerWarp;
  const int ng = warp_active ? min(kRowsPerWarp, G - g0) : 0;

  // inverse frequencies (in turns) of this lane's rotated pairs
  double inv_turns[H];
#pragma unroll
  for (int e = 0; e < H; ++e) inv_turns[e] = rope_inv_freq_turns(lane * H + e, D, a.log2_base);

  if (warp_active) {
    for (int v = v_lo + stream_id; v < v_hi; v += streams) {
      const int pos = first + v;
      const uint16_t* krow;
      const uint16_t* vrow;
      if (pos < len) {
        const size_t row = a.ring ? (size_t)(pos % a.capacity) : (size_t)pos;
        const size_t off = (((size_t)b * a.num_kv_heads + kvh) * a.capacity + row) * D;
        krow = a.k_cache + off;
        vrow = a.v_cache ? a.v_cache + off : krow;
      } else {
        const size_t off = (((size_t)b * a.n_q + (pos - len)) * a.num_kv_heads + kvh) * D;
        krow = a.new_k + off;
        vrow = a.new_v ? a.new_v + off : krow;
      }
      float kx[2 * H], vx[2 * H];
      if (lane < ACTIVE) {
        const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(krow);
        const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(vrow);
#pragma unroll
        for (int e = 0; e < H; ++e) {
          kx[e] = __bfloat162float(kb[lane * H + e]);
          kx[H + e] = __bfloat162float(kb[HALF + lane * H + e]);
          vx[e] = __bfloat162float(vb[lane * H + e]);
          vx[H + e] = __bfloat162float(vb[HALF + lane * H + e]);
        }
#pragma unroll
        for (int e = 0; e < H; ++e) {
          if (lane * H + e < a.r) {
            float c, s;
            rope_cos_sin((double)pos, inv_turns[e], &c, &s);
            const float x0 = kx[e], x1 = kx[H + e];
            kx[e] = x0 * c - x1 * s;
            kx[H + e] = x0 * s + x1 * c;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 2 * H; ++e) { kx[e] = 0.f; vx[e] = 0.f; }
      }
#pragma unroll
      for (int g = 0; g < kRowsPerWarp; ++g) {
        if (g >= ng) break;
        const int row = g0 + g;
        const int qpos = len + row / group;
        const float* qr = qs + (size_t)row * D;
        float dot = 0.f;
        if (lane < ACTIVE) {
#pragma unroll
          for (int e = 0; e < H; ++e) dot += qr[lane * H + e] * kx[e] + qr[HALF + lane * H + e] * kx[H + e];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const bool vis = pos <= qpos && (!a.is_local || pos > qpos - a.window);
        if (!vis) continue;
        const float mn = fmaxf(m[g], dot);
        const float alpha = exp2f(m[g] - mn);
        const float p = exp2f(dot - mn);
        l[g] = l[g] * alpha + p;
#pragma unroll
        for (int e = 0; e < 2 * H; ++e) o[g][e] = o[g][e] * alpha + p * vx[e];
        m[g] = mn;
      }
    }
  }

  // ---- merge the key streams of each row group in shared memory, write partials
  const int stride = D + 2;
  float* mine = red + (size_t)warp * kRowsPerWarp * stride;
  for (int g = 0; g < ng; ++g) {
    if (lane < ACTIVE) {
#pragma unroll
      for (int e = 0; e < H; ++e) {
        mine[g * stride + lane * H + e] = o[g][e];
        mine[g * stride + HALF + lane * H + e] = o[g][H + e];
      }
    }
    if (lane == 0) { mine[g * stride + D] = m[g]; mine[g * stride + D + 1] = l[g]; }
  }
  __syncthreads();
  const int rows_total = a.batch * a.n_q * a.num_q_heads;
  for (int idx = threadIdx.x; idx < G * D; idx += kDecThreads) {
    const int row = idx / D, c = idx % D;
    const int rgi = row / kRowsPerWarp, gi = row % kRowsPerWarp;
    float mm = -INFINITY;
    for (int s = 0; s < streams; ++s) {
      const float* st = red + (size_t)(s * nrg + rgi) * kRowsPerWarp * stride + gi * stride;
      mm = fmaxf(mm, st[D]);
    }
    float ll = 0.f, acc = 0.f;
    if (mm != -INFINITY) {
      for (int s = 0; s < streams; ++s) {
        const float* st = red + (size_t)(s * nrg + rgi) * kRowsPerWarp * stride + gi * stride;
        if (st[D] == -INFINITY) continue;
        const float w = exp2f(st[D] - mm);
        ll += w * st[D + 1];
        acc += w * st[c];
      }
    }
    const int i = row / group, hh = row % group;
    const size_t orow = ((size_t)b * a.n_q + i) * a.num_q_heads + kvh * group + hh;
    a.partial_o[((size_t)split * rows_total + orow) * D + c] = ll > 0.f ? acc / ll : 0.f;
    if (c == 0)
      a.partial_lse[(size_t)split * rows_total + orow] =
          ll > 0.f ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
  }
}

template <int D>
static cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t stream) {
  const int group = a.num_q_heads / a.num_kv_heads;
  const int G = group * a.n_q;
  const size_t smem = ((size_t)G * D + (size_t)kDecWarps * kRowsPerWarp * (D + 2)) * sizeof(float);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, a.num_kv_heads, a.batch);
  decode_kernel<D><<<grid, kDecThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int group = a.num_q_heads / a.num_kv_heads;
  if ((group * a.n_q + kRowsPerWarp - 1) / kRowsPerWarp > kDecWarps) return cudaErrorInvalidValue;
  switch (a.head_dim) {
    case 32: return launch_decode_d<32>(a, stream);
    case 64: return launch_decode_d<64>(a, stream);
    case 128: return launch_decode_d<128>(a, stream);
    case 256: return launch_decode_d<256>(a, stream);
    case 512: return launch_decode_d<512>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// Combine: one warp per output row.
// ---------------------------------------------------------------------------
__global__ void combine_kernel(CombineArgs a) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  float mm = -INFINITY;
  for (int s = lane; s < a.num_splits; s += 32) mm = fmaxf(mm, a.partial_lse[(size_t)s * a.rows + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
  float den = 0.f;
  for (int s = lane; s < a.num_splits; s += 32) {
    const float l = a.partial_lse[(size_t)s * a.rows + row];
    if (l != -INFINITY) den += __expf(l - mm);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  for (int c = lane; c < a.head_dim; c += 32) {
    float acc = 0.f;
    if (mm != -INFINITY) {
      for (int s = 0; s < a.num_splits; ++s) {
        const float l = a.partial_lse[(size_t)s * a.rows + row];
        if (l == -INFINITY) continue;
        acc += __expf(l - mm) * a.partial_o[((size_t)s * a.rows + row) * a.head_dim + c];
      }
      acc /= den;
    }
    if (a.out_f32)
      reinterpret_cast<float*>(a.out)[(size_t)row * a.head_dim + c] = acc;
    else
      reinterpret_cast<__nv_bfloat16*>(a.out)[(size_t)row * a.head_dim + c] = __float2bfloat16_rn(acc);
  }
  if (lane == 0 && a.lse != nullptr) a.lse[row] = (mm == -INFINITY) ? -INFINITY : mm + logf(den);
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const int warps = 8;
  combine_kernel<<<(a.rows + warps - 1) / warps, warps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gattn
