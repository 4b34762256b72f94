// decode.cu -- split-KV decode / speculative verify, and the log-sum-exp combine.
//
// n_q new query tokens per sequence attend to the sequence's cached keys plus the
// new tokens themselves. Local layers read a window-slot ring (token p in slot
// p mod W); global layers read a contiguous cache holding the single K=V tensor
// ("Visual guide to Gemma 4", sections "K=V technique" and "GQA": the KV cache is
// what GQA and K=V shrink). Keys are stored un-rotated; the copy used for scores is
// rotated after it lands in shared memory (p-RoPE: only the first r pairs), values
// are used as loaded.
//
// The visible keys of a sequence, in position order (cached tokens, then the new
// tokens), are cut into `num_splits` contiguous ranges. One CTA (4 warps) handles a
// (sequence, KV head, split) for every query head of that KV head and every new token
// -- the "rows". Per chunk of 64 keys:
//   1. cp.async brings the chunk's key (and, for local layers, value) rows into padded
//      shared memory, double-buffered so the next chunk streams in meanwhile;
//   2. the rotated copy for scores is formed (a per-thread angle recurrence over the
//      chunk's consecutive positions, re-anchored exactly every chunk);
//   3. S^T = K Q^T on tensor cores (mma.sync m16n8k16 bf16, keys on M, rows on N);
//   4. online softmax per row across the 4 warps;
//   5. O^T += V^T P^T on tensor cores, the warps splitting the head dim.
// The CTA writes an fp32 partial (O / l) and its log-sum-exp for the combine; with a
// single split and a final output given, it writes that output and log-sum-exp
// directly instead (the combine of one split is the identity).
#include "common.cuh"
#include "kernels.h"

namespace gattn {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = 4;
constexpr int kCK = 64;  // keys per chunk

constexpr size_t kMaxSmem = 227 * 1024;  // dynamic shared memory one CTA may hold
constexpr int kDecHeader = 128;  // bytes at the start of shared memory: two mbarriers, abort flag

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Result of one row element / one row: the split partial, or, in direct mode (one
// split, a.out set), the final output element in the caller's dtype.
__device__ __forceinline__ void put_o(const DecodeArgs& a, size_t i, float v) {
  if (a.out == nullptr)
    a.partial_o[i] = v;
  else if (a.out_f32)
    static_cast<float*>(a.out)[i] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[i] = __float2bfloat16_rn(v);
}
__device__ __forceinline__ void put_lse(const DecodeArgs& a, size_t i, float v) {
  if (a.out == nullptr)
    a.partial_lse[i] = v;
  else if (a.out_lse != nullptr)
    a.out_lse[i] = v;
}

// Shared-memory carve-up of the decode kernel (element counts are bf16 unless noted).
template <int D, int NT>
struct DecSmem {
  static constexpr int kRowPad = 8;                    // 16 bytes: conflict-free ldmatrix rows
  static constexpr int KST = D + kRowPad;              // key/value/query row stride
  static constexpr int RPAD = 8 * NT;                  // query rows, padded to n-tiles
  static constexpr int PST = kCK + kRowPad;            // P row stride
  static constexpr int NKS = D / 16;                   // k-steps of the head dim
};

}  // namespace

// Bytes of dynamic shared memory for decode_tc_kernel<D, NT> given the rotated k-step
// count nrk (0 when the keys are rotated in place).
template <int D, int NT>
__host__ __device__ constexpr size_t dec_smem_bytes(bool separate_v, int nrk) {
  using S = DecSmem<D, NT>;
  size_t b = kDecHeader;
  b += 2ull * kCK * S::KST * 2;                        // key buffers
  if (separate_v) b += 2ull * kCK * S::KST * 2;        // value buffers
  b += (size_t)kCK * (nrk * 16 + S::kRowPad) * 2;      // rotated copy (K=V layers)
  b += (size_t)S::RPAD * S::KST * 2;                   // rotated queries
  b += (size_t)S::RPAD * S::PST * 2;                   // P
  b += 2ull * kDecWarps * S::RPAD * 4;                 // per-warp row max / sum
  b += (size_t)S::NKS * 4;                             // k-step -> rotated slot
  return b;
}

template <int D, int NT>
__global__ void __launch_bounds__(kDecThreads)
decode_tc_kernel(DecodeArgs a) {
  using S = DecSmem<D, NT>;
  constexpr int HALF = D / 2;
  constexpr int KST = S::KST;
  constexpr int RPAD = S::RPAD;
  constexpr int PST = S::PST;
  constexpr int NKS = S::NKS;
  constexpr int MT_TOTAL = D / 16;                              // 16-dim m-tiles of O^T
  constexpr int PV_WARPS = MT_TOTAL < kDecWarps ? MT_TOTAL : kDecWarps;
  constexpr int MTW = MT_TOTAL / PV_WARPS;                      // m-tiles per PV warp

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int group = a.num_q_heads / a.num_kv_heads;
  const int R = group * a.n_q;
  const bool kv_same = a.v_cache == nullptr;
  const int len = a.cache_seqlens[b];
  const int first = a.is_local ? max(0, len - a.window + 1) : 0;  // oldest position any query sees
  const int nk = (len - first) + (a.new_keys ? a.n_q : 0);
  const int qoff = a.q_pos_offset ? a.q_pos_offset[b] : 0;  // queries after a key-range shard
  const int per = (nk + a.num_splits - 1) / a.num_splits;
  const int v_lo = min(nk, split * per);
  const int v_hi = min(nk, v_lo + per);
  const int r = a.r;
  // rotated k-steps (only for K=V layers, where the values must stay un-rotated)
  int nrk = 0;
  if (kv_same)
    for (int s = 0; s < NKS; ++s)
      if (s * 16 < r || (s * 16 < HALF + r && s * 16 + 16 > HALF)) ++nrk;
  const int RST = nrk * 16 + S::kRowPad;
  uint32_t rot_bits = 0;  // bit s: k-step s of the scores reads the rotated copy
  if (kv_same)
    for (int s = 0; s < NKS; ++s)
      if (s * 16 < r || (s * 16 < HALF + r && s * 16 + 16 > HALF)) rot_bits |= 1u << s;

  extern __shared__ __align__(128) uint8_t dsm[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(dsm);          // [2], one per chunk buffer
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + 16);
  uint16_t* kbuf = reinterpret_cast<uint16_t*>(dsm + kDecHeader);
  uint16_t* vbuf = kbuf + 2 * kCK * KST;
  uint16_t* rbuf = kv_same ? vbuf : vbuf + 2 * kCK * KST;
  uint16_t* qs = rbuf + kCK * RST;
  uint16_t* ps = qs + RPAD * KST;
  float* red_max = reinterpret_cast<float*>(ps + RPAD * PST);
  float* red_sum = red_max + kDecWarps * RPAD;
  int* ks_slot = reinterpret_cast<int*>(red_sum + kDecWarps * RPAD);

  if (tid == 0) {
    mbar_init(&full_bar[0], 1);
    mbar_init(&full_bar[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid < NKS) {
    int slot = -1;
    if (kv_same) {
      int c = 0;
      for (int s = 0; s <= tid; ++s) {
        const bool rot = s * 16 < r || (s * 16 < HALF + r && s * 16 + 16 > HALF);
        if (s == tid && rot) slot = c;
        if (rot) ++c;
      }
    }
    ks_slot[tid] = slot;
  }

  // ---- rotated queries (bf16) into shared memory; padding rows are zero
  for (int idx = tid; idx < RPAD * HALF; idx += kDecThreads) {
    const int row = idx / HALF, j = idx % HALF;
    float y0 = 0.f, y1 = 0.f;
    if (row < R) {
      const int i = row / group, hh = row % group;
      const uint16_t* qrow = a.q + (((size_t)b * a.n_q + i) * a.num_q_heads + kvh * group + hh) * D;
      const float x0 = bf2f(qrow[j]), x1 = bf2f(qrow[j + HALF]);
      y0 = x0; y1 = x1;
      if (j < r) {
        float c, s;
        rope_cos_sin((double)(len + i + qoff), rope_inv_freq_turns(j, D, a.log2_base), &c, &s);
        y0 = x0 * c - x1 * s;
        y1 = x0 * s + x1 * c;
      }
    }
    qs[row * KST + j] = f2bf(y0);
    qs[row * KST + j + HALF] = f2bf(y1);
  }

  // ---- rotation work assignment: thread -> pair j, walking keys ks0, ks0 + kstride, ...
  int rj = -1, rks0 = 0, rkstride = 1;
  if (r > 0) {
    if (r <= kDecThreads) {
      const int grp = kDecThreads / r;
      if (tid < grp * r) { rj = tid % r; rks0 = tid / r; rkstride = grp; }
    } else {
      rj = tid;  // r > 128: each thread takes pairs tid, tid + 128, ... (handled in the loop)
    }
  }
  // cos/sin of the per-thread key step (kstride * theta_j), exact
  float step_c = 1.f, step_s = 0.f;
  double inv_turns = 0.0;
  if (rj >= 0 && r <= kDecThreads) {
    inv_turns = rope_inv_freq_turns(rj, D, a.log2_base);
    rope_cos_sin((double)rkstride, inv_turns, &step_c, &step_s);
  }

  // ---- chunk loader: warp 0 issues one bulk copy per key (and value) row of the chunk
  // into the padded buffer rows; the copies complete on the buffer's mbarrier.
  auto issue_chunk = [&](int chunk, int buf) {
    const int v0 = v_lo + chunk * kCK;
    const int nvalid = min(kCK, v_hi - v0);
    uint16_t* kd = kbuf + buf * kCK * KST;
    uint16_t* vd = vbuf + buf * kCK * KST;
    fence_proxy_async_smem();  // earlier generic accesses to this buffer come first
    if (lane == 0) mbar_arrive_expect_tx(&full_bar[buf], (uint32_t)(nvalid * D * 2 * (kv_same ? 1 : 2)));
    __syncwarp();
    for (int row = lane; row < nvalid; row += 32) {
      const int pos = first + v0 + row;
      const uint16_t* ksrc;
      const uint16_t* vsrc;
      if (pos < len) {
        const size_t rr = a.ring ? (size_t)(pos % a.capacity) : (size_t)pos;
        const size_t off = (((size_t)b * a.num_kv_heads + kvh) * a.capacity + rr) * D;
        ksrc = a.k_cache + off;
        vsrc = kv_same ? nullptr : a.v_cache + off;
      } else {
        const size_t off = (((size_t)b * a.n_q + (pos - len)) * a.num_kv_heads + kvh) * D;
        ksrc = a.new_k + off;
        vsrc = kv_same ? nullptr : a.new_v + off;
      }
      bulk_load(kd + row * KST, ksrc, D * 2, &full_bar[buf]);
      if (!kv_same) bulk_load(vd + row * KST, vsrc, D * 2, &full_bar[buf]);
    }
  };

  const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) { m_run[nt][e] = -INFINITY; l_run[nt][e] = 0.f; }
  float oacc[MTW][NT][4];
#pragma unroll
  for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[mt][nt][e] = 0.f;

  const int nchunks = (v_hi - v_lo + kCK - 1) / kCK;
  __syncthreads();  // barrier init and the rotated queries are visible to every thread
  if (warp == 0 && nchunks > 0) issue_chunk(0, 0);
  int in_flight = nchunks > 0 ? 0 : -1;  // chunk whose copies are issued but not yet waited on

  for (int chunk = 0; chunk < nchunks; ++chunk) {
    const int buf = chunk & 1;
    if (warp == 0 && chunk + 1 < nchunks) issue_chunk(chunk + 1, buf ^ 1);
    const bool ok = mbar_wait(&full_bar[buf], (uint32_t)(chunk >> 1) & 1u, abort_flag);
    in_flight = chunk + 1 < nchunks ? chunk + 1 : -1;
    if (__syncthreads_or(!ok)) break;
    uint16_t* kd = kbuf + buf * kCK * KST;
    uint16_t* vdw = kv_same ? kd : vbuf + buf * kCK * KST;
    const uint16_t* vd = vdw;
    const int v0 = v_lo + chunk * kCK;
    const int pos0 = first + v0;
    const int nvalid = min(kCK, v_hi - v0);
    if (nvalid < kCK) {  // rows past the split end: zero, so that P = 0 meets finite values
      for (int idx = tid; idx < (kCK - nvalid) * (D / 8); idx += kDecThreads) {
        const int row = nvalid + idx / (D / 8), c8 = idx % (D / 8);
        *reinterpret_cast<uint4*>(kd + row * KST + c8 * 8) = make_uint4(0, 0, 0, 0);
        if (!kv_same) *reinterpret_cast<uint4*>(vdw + row * KST + c8 * 8) = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
    }

    // ---- rotated copy for scores (with pre-rotated cached keys only the new tokens' rows)
    if (r > 0 && (!a.keys_rotated || pos0 + kCK > len)) {
      if (kv_same) {
        // non-rotated dims that share a 16-dim k-step with rotated ones are copied first
        if (r % 16 != 0) {
          for (int idx = tid; idx < kCK * nrk * 16; idx += kDecThreads) {
            const int row = idx / (nrk * 16), col = idx % (nrk * 16);
            int s = 0;
            for (int q = 0, c = 0; q < NKS; ++q)
              if (ks_slot[q] >= 0) { if (c == col / 16) { s = q; break; } ++c; }
            rbuf[row * RST + col] = kd[row * KST + s * 16 + col % 16];
          }
          __syncthreads();
        }
      }
      for (int j = rj; j >= 0 && j < r; j += kDecThreads) {
        float ac, as;
        int ks0 = rks0, kstride = rkstride;
        float sc = step_c, ss = step_s;
        if (r > kDecThreads) {  // one pair per iteration over all keys
          ks0 = 0; kstride = 1;
          const double it = rope_inv_freq_turns(j, D, a.log2_base);
          rope_cos_sin(1.0, it, &sc, &ss);
          rope_cos_sin((double)pos0, it, &ac, &as);
        } else {
          rope_cos_sin((double)(pos0 + ks0), inv_turns, &ac, &as);
        }
        const int sj = ks_slot[j / 16], sp = ks_slot[(j + HALF) / 16];
#pragma unroll 4
        for (int u = ks0; u < kCK; u += kstride) {
          const float x0 = bf2f(kd[u * KST + j]), x1 = bf2f(kd[u * KST + j + HALF]);
          const uint16_t y0 = f2bf(x0 * ac - x1 * as), y1 = f2bf(x0 * as + x1 * ac);
          if (kv_same) {
            rbuf[u * RST + sj * 16 + (j % 16)] = y0;
            rbuf[u * RST + sp * 16 + ((j + HALF) % 16)] = y1;
          } else if (!a.keys_rotated || pos0 + u >= len) {
            kd[u * KST + j] = y0;
            kd[u * KST + j + HALF] = y1;
          }
          const float nc = ac * sc - as * ss;
          as = ac * ss + as * sc;
          ac = nc;
        }
        if (r <= kDecThreads) break;
      }
      __syncthreads();
    }

    // ---- S^T = K Q^T for this warp's 16 keys. Two accumulator sets (even / odd
    // k-steps) halve the dependent mma chain; the rotated-slot lookup uses a register
    // bitmask so no shared-memory load sits on the address path.
    float sacc[NT][4];
    {
      float sacc2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) { sacc[nt][e] = 0.f; sacc2[nt][e] = 0.f; }
      const int krow = warp * 16 + (lane & 15);
      const int kcol = (lane >> 4) * 8;
      const uint32_t kbase = smem_u32(kd + krow * KST + kcol);
      const uint32_t rbase = smem_u32(rbuf + krow * RST + kcol);
      const uint32_t qbase = smem_u32(qs + (lane & 7) * KST + ((lane >> 3) & 1) * 8);
#pragma unroll
      for (int s = 0; s < NKS; ++s) {
        const bool rot = (rot_bits >> s) & 1u;
        const int slot = __popc(rot_bits & ((1u << s) - 1u));
        const uint32_t aaddr = rot ? rbase + slot * 32 : kbase + s * 32;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(aaddr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t b0, b1;
          ldsm_x2(qbase + (nt * 8 * KST + s * 16) * 2, b0, b1);
          mma_16816((s & 1) ? sacc2[nt] : sacc[nt], a0, a1, a2, a3, b0, b1);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] += sacc2[nt][e];
    }

    // ---- mask, chunk max per row
    float cmax[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = nt * 8 + 2 * t + e;
        const int qpos = len + qoff + (row < R ? row / group : 0);
        float mx = -INFINITY;
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {
          const int key = warp * 16 + g + hk * 8;
          const int v = v0 + key;
          const int pos = first + v;
          const bool vis = row < R && v < v_hi && pos <= qpos && (!a.is_local || pos > qpos - a.window);
          float& sv = sacc[nt][hk * 2 + e];
          sv = vis ? sv * scale_log2 : -INFINITY;
          mx = fmaxf(mx, sv);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        cmax[nt][e] = mx;
      }
    }
    if (g == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) red_max[warp * RPAD + nt * 8 + 2 * t + e] = cmax[nt][e];
    }
    __syncthreads();

    // ---- probabilities, row sums, P to shared memory
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * t + e;
        float cm = red_max[col];
#pragma unroll
        for (int w = 1; w < kDecWarps; ++w) cm = fmaxf(cm, red_max[w * RPAD + col]);
        const float mn = fmaxf(m_run[nt][e], cm);
        alpha[nt][e] = (mn == -INFINITY) ? 1.f : exp2f(m_run[nt][e] - mn);
        const float msub = (mn == -INFINITY) ? 0.f : mn;
        m_run[nt][e] = mn;
        float sum = 0.f;
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {
          const float p = exp2f(sacc[nt][hk * 2 + e] - msub);
          const uint16_t pb = f2bf(p);
          sum += bf2f(pb);
          ps[col * PST + warp * 16 + g + hk * 8] = pb;
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        sum += __shfl_xor_sync(0xffffffffu, sum, 8);
        sum += __shfl_xor_sync(0xffffffffu, sum, 16);
        if (g == 0) red_sum[warp * RPAD + col] = sum;
      }
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * t + e;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) sum += red_sum[w * RPAD + col];
        l_run[nt][e] = l_run[nt][e] * alpha[nt][e] + sum;
      }

    // ---- O^T += V^T P^T over this warp's head-dim slice
    if (warp < PV_WARPS) {
#pragma unroll
      for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          oacc[mt][nt][0] *= alpha[nt][0];
          oacc[mt][nt][1] *= alpha[nt][1];
          oacc[mt][nt][2] *= alpha[nt][0];
          oacc[mt][nt][3] *= alpha[nt][1];
        }
#pragma unroll
      for (int ks = 0; ks < kCK / 16; ++ks) {
        uint32_t bfr[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int prow = nt * 8 + (lane & 7);
          const int pcol = ks * 16 + ((lane >> 3) & 1) * 8;
          ldsm_x2(smem_u32(ps + prow * PST + pcol), bfr[nt][0], bfr[nt][1]);
        }
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt) {
          const int d0 = (warp * MTW + mt) * 16;
          const int vrow = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int vcol = d0 + ((lane >> 3) & 1) * 8;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(smem_u32(vd + vrow * KST + vcol), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816(oacc[mt][nt], a0, a1, a2, a3, bfr[nt][0], bfr[nt][1]);
        }
      }
    }
    __syncthreads();  // buffers of this chunk are free for the load two chunks ahead
  }
  // Copies still in flight after an early exit land before the CTA leaves.
  if (in_flight >= 0 && tid == 0) {
    const uint32_t par = (uint32_t)(in_flight >> 1) & 1u;
    unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(&full_bar[in_flight & 1], par) && globaltimer_ns() - t0 < kWaitLimitNs) {}
  }

  // ---- partial O (normalised by this split's l) and log-sum-exp
  const int rows_total = a.batch * a.n_q * a.num_q_heads;
  if (warp < PV_WARPS) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = nt * 8 + 2 * t + e;
        if (row >= R) continue;
        const int i = row / group, hh = row % group;
        const size_t orow = ((size_t)b * a.n_q + i) * a.num_q_heads + kvh * group + hh;
        const float l = l_run[nt][e];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const size_t po = ((size_t)split * rows_total + orow) * D;
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt) {
          const int d0 = (warp * MTW + mt) * 16;
          put_o(a, po + d0 + g, oacc[mt][nt][e] * inv);
          put_o(a, po + d0 + g + 8, oacc[mt][nt][2 + e] * inv);
        }
        if (warp == 0 && g == 0)
          put_lse(a, (size_t)split * rows_total + orow,
                  l > 0.f ? (m_run[nt][e] + log2f(l)) * 0.6931471805599453f : -INFINITY);
      }
  }
}

template <int D, int NT>
static cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  const bool kv_same = a.v_cache == nullptr;
  int nrk = 0;
  if (kv_same)
    for (int s = 0; s < D / 16; ++s)
      if (s * 16 < a.r || (s * 16 < D / 2 + a.r && s * 16 + 16 > D / 2)) ++nrk;
  const size_t smem = dec_smem_bytes<D, NT>(!kv_same, nrk);
  if (smem > kMaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, a.num_kv_heads, a.batch);
  decode_tc_kernel<D, NT><<<grid, kDecThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Warp-independent decode for up to 8 query rows per (sequence, KV head): plain decode
// (n_q = 1) and short verify. Each of the NW warps (8, or 4 where 8 do not fit) streams its
// own 16-key blocks (blocks w, w + NW, ... of the split) through a private ring (one or two
// stages) of per-row bulk copies
// and runs the whole block itself:
//   1. the p-RoPE rotation of the block's keys: each lane takes two pairs, computes
//      the exact angle of the block's first key and steps it by theta_j per key;
//   2. S^T = K Q^T with mma.sync (keys on M, query rows on N);
//   3. mask and online softmax in registers, with the running maximum raised only when
//      a block's maximum exceeds it by more than 2^8;
//   4. P^T becomes the B operand of the value product by an 8x8 transpose (movmatrix)
//      of the packed score fragments, and O^T over the whole head dim accumulates in
//      registers.
// No barrier joins the warps until their partial states are merged at the end.
// ---------------------------------------------------------------------------
namespace {

constexpr int kWB = 16;        // keys per warp block
// header: mbarriers [warps][stages] at 0, abort flag at 128, value-stage mbarriers
// [warps][value stages] at 160 (split form), merge maxima [warps][8] at 256 and sums
// [warps][8] after them
constexpr int kWMgM = 256;
__host__ __device__ constexpr int wmg_l(int nw) { return kWMgM + nw * 32; }
__host__ __device__ constexpr int wheader(int nw) { return (wmg_l(nw) + nw * 32 + 127) / 128 * 128; }

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__host__ __device__ constexpr size_t align128(size_t x) { return (x + 127) / 128 * 128; }

// Shared-memory carve-up of decode_warp_kernel<D, NS, NW, NSV>; r is the rotated pair count
// and nrk the number of rotated 16-dim k-steps kept in the per-warp rotated copy (K=V
// layers). NS key stages per warp; separate-V layers add NSV value stages.
template <int D, int NS, int NW, int NSV>
struct DecWLayout {
  static constexpr int KST = D + 8;  // bf16 row stride of key / value / query rows
  static constexpr int RED = D + 4;  // fp32 row stride of the merge buffer
  size_t qs, stp, bstp, itf, regions, region, k_off, v_off, rot_off, ast_off, total;
  int rr2, rst;
  __host__ __device__ DecWLayout(bool kv_same, int r, int nrk) {
    // table length: even, past r, and covering every word the rotation pass visits
    rr2 = (r + 2) & ~1;
    if (kv_same && 16 * ((r + 15) / 16) > rr2) rr2 = 16 * ((r + 15) / 16);
    rst = nrk * 16 + 8;
    qs = wheader(NW);
    stp = qs + align128((size_t)8 * KST * 2);
    bstp = stp + align128((size_t)rr2 * 8);
    itf = bstp + align128((size_t)rr2 * 8);
    regions = itf + align128((size_t)rr2 * 8);
    k_off = 0;
    v_off = (size_t)NS * kWB * KST * 2;
    rot_off = kv_same ? v_off : v_off + (size_t)NSV * kWB * KST * 2;
    ast_off = rot_off + (kv_same ? (size_t)kWB * rst * 2 : 0);
    const int nwords = kv_same ? 8 * ((r + 15) / 16) : (r + 1) / 2;
    region = align128(ast_off + (size_t)(nwords > 0 ? nwords : 1) * 16);
    const size_t merge = (size_t)NW * 8 * RED * 4;  // the merge buffer reuses the regions
    total = regions + (NW * region > merge ? NW * region : merge);
  }
};

__host__ __device__ inline bool rotated_kstep(int s, int half, int r) {
  return s * 16 < r || (s * 16 < half + r && s * 16 + 16 > half);
}

}  // namespace

template <int D, int NS, int NW, int NSV>
__global__ void __launch_bounds__(NW * 32)
decode_warp_kernel(DecodeArgs a) {
  using L = DecWLayout<D, NS, NW, NSV>;
  constexpr int kWWarps = NW;
  constexpr int kWStages = NS;  // ring stages per warp
  // Split form (separate-V layers only): key rows and value rows stream through their
  // own stages with their own barriers, so the next block's keys are in flight while
  // this block's values are used and the next values while the next keys are rotated.
  constexpr bool kSplit = NSV < NS;
  constexpr int HALF = D / 2;
  constexpr int KST = L::KST;
  constexpr int NKS = D / 16;
  constexpr bool kQReg = D <= 256;  // query fragments held in registers
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int group = a.num_q_heads / a.num_kv_heads;
  const int R = group * a.n_q;  // <= 8
  const bool kv_same = a.v_cache == nullptr;
  const int len = a.cache_seqlens[b];
  const int first = a.is_local ? max(0, len - a.window + 1) : 0;  // oldest position any query sees
  const int nk = (len - first) + (a.new_keys ? a.n_q : 0);
  const int qoff = a.q_pos_offset ? a.q_pos_offset[b] : 0;  // queries after a key-range shard
  const int per = (nk + a.num_splits - 1) / a.num_splits;
  const int v_lo = min(nk, split * per);
  const int v_hi = min(nk, v_lo + per);
  const int r = a.r;
  const int c16 = (r + 15) / 16;  // rotated k-steps in each half of the head dim
  uint32_t rot_bits = 0;          // bit s: k-step s of the scores reads the rotated copy
  int nrk = 0;
  if (kv_same)
    for (int s = 0; s < NKS; ++s)
      if (rotated_kstep(s, HALF, r)) { rot_bits |= 1u << s; ++nrk; }
  const L lay(kv_same, r, nrk);
  const int RST = lay.rst;

  extern __shared__ __align__(128) uint8_t dsm[];
  static_assert(kWWarps * NS * 8 <= 128 && (!kSplit || kWWarps * NSV * 8 <= 96), "mbarriers overflow their header slots");
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm);  // [warps][stages]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + 128);
  float* mg_m = reinterpret_cast<float*>(dsm + kWMgM);  // [warps][8]
  float* mg_l = reinterpret_cast<float*>(dsm + wmg_l(NW));  // [warps][8]
  uint16_t* qs = reinterpret_cast<uint16_t*>(dsm + lay.qs);
  float2* stp = reinterpret_cast<float2*>(dsm + lay.stp);
  float2* bstp = reinterpret_cast<float2*>(dsm + lay.bstp);
  double* itf = reinterpret_cast<double*>(dsm + lay.itf);
  uint8_t* region = dsm + lay.regions + (size_t)warp * lay.region;
  uint16_t* kst = reinterpret_cast<uint16_t*>(region + lay.k_off);
  uint16_t* vst = reinterpret_cast<uint16_t*>(region + lay.v_off);
  uint16_t* rbuf = reinterpret_cast<uint16_t*>(region + lay.rot_off);
  float4* ast = reinterpret_cast<float4*>(region + lay.ast_off);  // this warp's block anchors
  uint64_t* wbar = bars + warp * kWStages;
  uint64_t* vbar = reinterpret_cast<uint64_t*>(dsm + 160) + warp * NSV;  // split form

  // blocks of this warp: warp, warp + NW, ... of the split's ceil((v_hi - v_lo) / 16)
  const int nblk = (v_hi - v_lo + kWB - 1) / kWB;
  const int my_n = nblk > warp ? (nblk - warp + kWWarps - 1) / kWWarps : 0;

  // Bulk copies of block `itx` of this warp into stage itx % 2: lanes 0..15 copy key
  // rows, lanes 16..31 value rows (separate-V layers); rows past the split are not read.
  auto issue = [&](int itx) {
    const int st = itx % kWStages;
    const int v0 = v_lo + (warp + kWWarps * itx) * kWB;
    const int nvalid = min(kWB, v_hi - v0);
    fence_proxy_async_smem();  // earlier generic accesses to this stage come first
    if (lane == 0) mbar_arrive_expect_tx(&wbar[st], (uint32_t)(nvalid * D * 2 * (kv_same ? 1 : 2)));
    __syncwarp();
    const int row = lane & 15;
    const bool is_v = lane >= 16;
    if (row < nvalid && (!is_v || !kv_same)) {
      const int pos = first + v0 + row;
      const uint16_t* src;
      if (pos < len) {
        const size_t slot = a.ring ? (size_t)(pos % a.capacity) : (size_t)pos;
        src = (is_v ? a.v_cache : a.k_cache) + (((size_t)b * a.num_kv_heads + kvh) * a.capacity + slot) * D;
      } else {
        src = (is_v ? a.new_v : a.new_k) + (((size_t)b * a.n_q + (pos - len)) * a.num_kv_heads + kvh) * D;
      }
      uint16_t* dst = (is_v ? vst : kst) + (st * kWB + row) * KST;
      bulk_load(dst, src, D * 2, &wbar[st]);
    }
  };
  // Split form: the key rows (kv = 0) or value rows (kv = 1) of block `itx`, lanes 0..15.
  auto issue_half = [&](int itx, int kv) {
    const int st = kv ? itx % NSV : itx % kWStages;
    uint64_t* bar = kv ? &vbar[st] : &wbar[st];
    const int v0 = v_lo + (warp + kWWarps * itx) * kWB;
    const int nvalid = min(kWB, v_hi - v0);
    fence_proxy_async_smem();
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nvalid * D * 2));
    __syncwarp();
    const int row = lane;
    if (row < nvalid) {
      const int pos = first + v0 + row;
      const uint16_t* src;
      if (pos < len) {
        const size_t slot = a.ring ? (size_t)(pos % a.capacity) : (size_t)pos;
        src = (kv ? a.v_cache : a.k_cache) + (((size_t)b * a.num_kv_heads + kvh) * a.capacity + slot) * D;
      } else {
        src = (kv ? a.new_v : a.new_k) + (((size_t)b * a.n_q + (pos - len)) * a.num_kv_heads + kvh) * D;
      }
      bulk_load((kv ? vst : kst) + (st * kWB + row) * KST, src, D * 2, bar);
    }
  };

  if (lane == 0) {
    for (int s = 0; s < kWStages; ++s) mbar_init(&wbar[s], 1);
    if constexpr (kSplit)
      for (int s = 0; s < NSV; ++s) mbar_init(&vbar[s], 1);
    fence_barrier_init();
  }
  if (tid == 0) *abort_flag = 0;

  // The query rows are loaded, and land, before this CTA issues any copy: queued behind
  // the copies of the GPU's other CTAs (tens of MB at the start), a query load would
  // hold up the start of the computation by microseconds.
  constexpr int QCH = D / 8;  // 16-byte chunks per query row
  constexpr int QV = (8 * QCH + NW * 32 - 1) / (NW * 32);
#pragma unroll
  for (int k = 0; k < QV; ++k) {
    const int idx = tid + k * NW * 32;
    const int row = idx / QCH;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (row < R) {
      const int i = row / group, hh = row % group;
      x = *reinterpret_cast<const uint4*>(a.q + (((size_t)b * a.n_q + i) * a.num_q_heads + kvh * group + hh) * D +
                                          (idx % QCH) * 8);
    }
    if (idx < 8 * QCH) *reinterpret_cast<uint4*>(qs + row * KST + (idx % QCH) * 8) = x;  // rows R..7 zero
  }
  __syncthreads();
  // Only the first block's key rows are copied now: a warp's issue of bulk copies stalls
  // while the SM's copy queue is full, so the rest of the ring is issued at the top of
  // the first iteration, behind the wait for these rows.
  if constexpr (kSplit) {
    if (my_n > 0) issue_half(0, 0);
  } else {
    if (my_n > 0) issue(0);
  }
  // the first r pairs of the query rows, rotated in place (bf16)
  for (int idx = tid; idx < R * r; idx += kWWarps * 32) {
    const int row = idx / r, j = idx % r;
    const int i = row / group;
    const float x0 = bf2f(qs[row * KST + j]), x1 = bf2f(qs[row * KST + j + HALF]);
    float c, s;
    rope_cos_sin((double)(len + i + qoff), rope_inv_freq_turns(j, D, a.log2_base), &c, &s);
    qs[row * KST + j] = f2bf(x0 * c - x1 * s);
    qs[row * KST + j + HALF] = f2bf(x0 * s + x1 * c);
  }
  // per-pair frequencies (turns per position), cos / sin of theta_j (one key) and of
  // 16 NW theta_j (one block step of a warp); pairs past r get the identity
  for (int j = tid; j < lay.rr2; j += kWWarps * 32) {
    const double f = j < r ? rope_inv_freq_turns(j, D, a.log2_base) : 0.0;
    float c, s;
    rope_cos_sin(1.0, f, &c, &s);
    itf[j] = f;
    stp[j] = make_float2(c, s);
    rope_cos_sin((double)(kWWarps * kWB), f, &c, &s);
    bstp[j] = make_float2(c, s);
  }
  __syncthreads();

  uint32_t qf[kQReg ? NKS : 1][2];
  const uint32_t qbase = smem_u32(qs + (lane & 7) * KST + ((lane >> 3) & 1) * 8);
  if constexpr (kQReg) {
#pragma unroll
    for (int s = 0; s < NKS; ++s) ldsm_x2(qbase + s * 32, qf[s][0], qf[s][1]);
  }

  // per-thread rows 2t and 2t + 1: validity and the query position they belong to
  bool row_ok[2];
  int qpos[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int row = 2 * t + e;
    row_ok[e] = row < R;
    qpos[e] = len + qoff + (row < R ? row / group : 0);
  }
  const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float oacc[NKS][4];
#pragma unroll
  for (int mt = 0; mt < NKS; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;

  // rotation work: words of two dims; K=V layers copy every word of the rotated
  // k-steps into the rotated buffer, separate-V layers rotate in place
  const int nwords = kv_same ? 8 * c16 : (r + 1) / 2;
  const uint32_t kfrag = (uint32_t)((lane & 15) * KST + (lane >> 4) * 8) * 2;
  const uint32_t rfrag = (uint32_t)((lane & 15) * RST + (lane >> 4) * 8) * 2;
  const uint32_t vfrag = (uint32_t)(((lane & 7) + ((lane >> 4) << 3)) * KST + ((lane >> 3) & 1) * 8) * 2;

  int it = 0;
  bool ok = true;
  for (; it < my_n; ++it) {
    const int st = it % kWStages;
    if (it == 0) {  // the rest of the ring: the first value rows, then further key stages
      if constexpr (kSplit) {
        for (int s = 0; s < NSV && s < my_n; ++s) issue_half(s, 1);
        for (int s = 1; s < kWStages && s < my_n; ++s) issue_half(s, 0);
      } else {
        for (int s = 1; s < kWStages && s < my_n; ++s) issue(s);
      }
    }
    ok = mbar_wait(&wbar[st], (uint32_t)(it / kWStages) & 1u, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    uint16_t* kd = kst + st * kWB * KST;
    uint16_t* vdw = kv_same ? kd : vst + (kSplit ? it % NSV : st) * kWB * KST;
    const int v0 = v_lo + (warp + kWWarps * it) * kWB;
    const int nvalid = min(kWB, v_hi - v0);
    const int pos0 = first + v0;
    if (!kSplit && nvalid < kWB) {  // value rows past the split end: zero, so that P = 0 meets finite values
      for (int idx = lane; idx < (kWB - nvalid) * (D / 8); idx += 32) {
        const int row = nvalid + idx / (D / 8), c8 = idx % (D / 8);
        *reinterpret_cast<uint4*>(vdw + row * KST + c8 * 8) = make_uint4(0, 0, 0, 0);
      }
    }

    // ---- 1. rotation: each lane owns words (pairs j, j + 1) and walks the block's 16
    // keys from the angle of the block's first key, stepping by theta_j per key. That
    // anchor angle is exact every 16th block and otherwise the previous block's anchor
    // advanced by 16 NW theta_j (the warp's stride); all loads come first.
    // With pre-rotated cached keys only a block holding new tokens is rotated (those rows
    // only), from an exact anchor since the recurrence skipped the blocks before it.
    if (r > 0 && (!a.keys_rotated || pos0 + kWB > len)) {
      uint16_t* dst0 = kv_same ? rbuf : kd;
      const int dst_hi = kv_same ? 16 * c16 : HALF;
      const int dst_st = kv_same ? RST : KST;
      const bool exact = (it & 15) == 0 || a.keys_rotated;
      for (int w = lane; w < nwords; w += 32) {
        const int j = 2 * w;
        uint32_t w0[kWB], w1[kWB];
#pragma unroll
        for (int u = 0; u < kWB; ++u) {
          w0[u] = *reinterpret_cast<const uint32_t*>(kd + u * KST + j);
          w1[u] = *reinterpret_cast<const uint32_t*>(kd + u * KST + HALF + j);
        }
        float4 an;
        if (exact) {
          rope_cos_sin((double)pos0, itf[j], &an.x, &an.y);
          rope_cos_sin((double)pos0, itf[j + 1], &an.z, &an.w);
        } else {
          const float4 pa = ast[w];
          const float4 bs = *reinterpret_cast<const float4*>(bstp + j);
          an = make_float4(pa.x * bs.x - pa.y * bs.y, pa.x * bs.y + pa.y * bs.x,
                           pa.z * bs.z - pa.w * bs.w, pa.z * bs.w + pa.w * bs.z);
        }
        ast[w] = an;
        const float4 st = *reinterpret_cast<const float4*>(stp + j);
        float ac[2] = {an.x, an.z}, as[2] = {an.y, an.w};
        const float sc[2] = {st.x, st.z}, ss[2] = {st.y, st.w};
#pragma unroll
        for (int u = 0; u < kWB; ++u) {
          const float x00 = __uint_as_float(w0[u] << 16), x01 = __uint_as_float(w0[u] & 0xFFFF0000u);
          const float x10 = __uint_as_float(w1[u] << 16), x11 = __uint_as_float(w1[u] & 0xFFFF0000u);
          const uint32_t o0 = pack_bf16x2(x00 * ac[0] - x10 * as[0], x01 * ac[1] - x11 * as[1]);
          const uint32_t o1 = pack_bf16x2(x00 * as[0] + x10 * ac[0], x01 * as[1] + x11 * ac[1]);
          if (!a.keys_rotated || pos0 + u >= len) {
            *reinterpret_cast<uint32_t*>(dst0 + u * dst_st + j) = o0;
            *reinterpret_cast<uint32_t*>(dst0 + u * dst_st + dst_hi + j) = o1;
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float nc = ac[e] * sc[e] - as[e] * ss[e];
            as[e] = ac[e] * ss[e] + as[e] * sc[e];
            ac[e] = nc;
          }
        }
      }
    }
    __syncwarp();

    // ---- 2. S^T = K Q^T for the block's 16 keys (four accumulator chains)
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      float sch[3][4] = {};
      const uint32_t kbase = smem_u32(kd) + kfrag;
      const uint32_t rbase = smem_u32(rbuf) + rfrag;
#pragma unroll
      for (int s = 0; s < NKS; ++s) {
        const bool rot = (rot_bits >> s) & 1u;
        const int slot = __popc(rot_bits & ((1u << s) - 1u));
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(rot ? rbase + slot * 32 : kbase + s * 32, a0, a1, a2, a3);
        if constexpr (kQReg) {
          b0 = qf[s][0];
          b1 = qf[s][1];
        } else {
          ldsm_x2(qbase + s * 32, b0, b1);
        }
        mma_16816((s & 3) ? sch[(s & 3) - 1] : sacc, a0, a1, a2, a3, b0, b1);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[e] += (sch[0][e] + sch[1][e]) + sch[2][e];
    }

    if constexpr (kSplit) {
      __syncwarp();  // every lane is done with this block's key rows
      if (it + kWStages < my_n) issue_half(it + kWStages, 0);
    }

    // ---- 3. mask and online softmax; fragment element e: key g + 8 * (e >> 1), row 2t + (e & 1)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int v = v0 + g + 8 * (e >> 1);
      const int pos = first + v;
      const int h = e & 1;
      const bool vis = row_ok[h] && v < v_hi && pos <= qpos[h] && (!a.is_local || pos > qpos[h] - a.window);
      sacc[e] = vis ? sacc[e] * scale_log2 : -INFINITY;
      mx[h] = fmaxf(mx[h], sacc[e]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
    }
    // the running maximum moves only when a row's block maximum passes it by more than
    // 8 (log2 units), so P stays below 2^8; the decision is warp-uniform
    if (__any_sync(0xffffffffu, mx[0] > m_run[0] + 8.f || mx[1] > m_run[1] + 8.f)) {
      float al[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float mn = fmaxf(m_run[h], mx[h]);
        al[h] = mn == -INFINITY ? 1.f : exp2f(m_run[h] - mn);
        m_run[h] = mn;
        l_run[h] *= al[h];
      }
#pragma unroll
      for (int mt = 0; mt < NKS; ++mt) {
        oacc[mt][0] *= al[0];
        oacc[mt][1] *= al[1];
        oacc[mt][2] *= al[0];
        oacc[mt][3] *= al[1];
      }
    }
    const float msub[2] = {m_run[0] == -INFINITY ? 0.f : m_run[0], m_run[1] == -INFINITY ? 0.f : m_run[1]};
    const uint32_t p01 = pack_bf16x2(exp2f(sacc[0] - msub[0]), exp2f(sacc[1] - msub[1]));  // key g
    const uint32_t p23 = pack_bf16x2(exp2f(sacc[2] - msub[0]), exp2f(sacc[3] - msub[1]));  // key g + 8
    l_run[0] += __uint_as_float(p01 << 16) + __uint_as_float(p23 << 16);
    l_run[1] += __uint_as_float(p01 & 0xFFFF0000u) + __uint_as_float(p23 & 0xFFFF0000u);
    // P^T B fragment: keys 2t, 2t + 1 (b0) and 2t + 8, 2t + 9 (b1) of query row g
    const uint32_t pb0 = movmatrix_trans(p01);
    const uint32_t pb1 = movmatrix_trans(p23);

    if constexpr (kSplit) {
      ok = mbar_wait(&vbar[it % NSV], (uint32_t)(it / NSV) & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (nvalid < kWB) {  // value rows past the split end: zero, so that P = 0 meets finite values
        for (int idx = lane; idx < (kWB - nvalid) * (D / 8); idx += 32) {
          const int row = nvalid + idx / (D / 8), c8 = idx % (D / 8);
          *reinterpret_cast<uint4*>(vdw + row * KST + c8 * 8) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
    }

    // ---- 4. O^T += V^T P^T over the whole head dim
    {
      const uint32_t vbase = smem_u32(vdw) + vfrag;
#pragma unroll
      for (int mt = 0; mt < NKS; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vbase + mt * 32, a0, a1, a2, a3);
        mma_16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();  // every lane is done with this stage and the rotated copy
    if constexpr (kSplit) {
      if (it + NSV < my_n) issue_half(it + NSV, 1);
    } else {
      if (it + kWStages < my_n) issue(it + kWStages);
    }
  }
  // Copies still in flight after an early exit land before the warp moves on.
  if (!ok && lane == 0) {
    // key (or combined) stages issued for blocks it .. it + NS - 1; in the split form the
    // keys may already be one block further (issued after this block's scores)
    for (int k = it; k < my_n && k < it + kWStages + (kSplit ? 1 : 0); ++k) {
      const uint32_t par = (uint32_t)(k / kWStages) & 1u;
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&wbar[k % kWStages], par) && globaltimer_ns() - t0 < kWaitLimitNs) {}
    }
    if constexpr (kSplit)
      for (int k = it; k < my_n && k < it + NSV; ++k) {
        const uint32_t par = (uint32_t)(k / NSV) & 1u;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&vbar[k % NSV], par) && globaltimer_ns() - t0 < kWaitLimitNs) {}
      }
  }

  // ---- merge the warps' (max, sum, O) and write this split's partial
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 4);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 8);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 16);
    if (g == 0) {
      mg_m[warp * 8 + 2 * t + h] = m_run[h];
      mg_l[warp * 8 + 2 * t + h] = l_run[h];
    }
  }
  __syncthreads();  // every warp has left its loop: the stage buffers are free
  auto merged = [&](int row, float& M, float& Lsum) {
    M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWWarps; ++w) M = fmaxf(M, mg_m[w * 8 + row]);
    Lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWWarps; ++w) {
      const float mw = mg_m[w * 8 + row];
      if (mw != -INFINITY) Lsum += mg_l[w * 8 + row] * exp2f(mw - M);
    }
  };
  float* red = reinterpret_cast<float*>(dsm + lay.regions);  // [warps][8][D + 4]
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float M, Lsum;
    merged(2 * t + h, M, Lsum);
    const float f = (Lsum > 0.f && m_run[h] != -INFINITY) ? exp2f(m_run[h] - M) / Lsum : 0.f;
    float* dst = red + (size_t)(warp * 8 + 2 * t + h) * L::RED + g;
#pragma unroll
    for (int mt = 0; mt < NKS; ++mt) {
      dst[mt * 16] = oacc[mt][h] * f;
      dst[mt * 16 + 8] = oacc[mt][2 + h] * f;
    }
  }
  __syncthreads();
  const int rows_total = a.batch * a.n_q * a.num_q_heads;
  for (int idx = tid; idx < R * D; idx += kWWarps * 32) {
    const int row = idx / D, d = idx % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWWarps; ++w) acc += red[(size_t)(w * 8 + row) * L::RED + d];
    const size_t orow = ((size_t)b * a.n_q + row / group) * a.num_q_heads + kvh * group + row % group;
    put_o(a, ((size_t)split * rows_total + orow) * D + d, acc);
  }
  if (tid < R) {
    float M, Lsum;
    merged(tid, M, Lsum);
    const size_t orow = ((size_t)b * a.n_q + tid / group) * a.num_q_heads + kvh * group + tid % group;
    put_lse(a, (size_t)split * rows_total + orow, Lsum > 0.f ? (M + log2f(Lsum)) * 0.6931471805599453f : -INFINITY);
  }
}

template <int D, int NS, int NW, int NSV>
static size_t decode_warp_smem(const DecodeArgs& a) {
  const bool kv_same = a.v_cache == nullptr;
  int nrk = 0;
  if (kv_same)
    for (int s = 0; s < D / 16; ++s)
      if (rotated_kstep(s, D / 2, a.r)) ++nrk;
  return DecWLayout<D, NS, NW, NSV>(kv_same, a.r, nrk).total;
}

template <int D, int NS, int NW, int NSV>
static cudaError_t launch_decode_warp(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = decode_warp_smem<D, NS, NW, NSV>(a);
  if (smem > kMaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_warp_kernel<D, NS, NW, NSV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, a.num_kv_heads, a.batch);
  decode_warp_kernel<D, NS, NW, NSV><<<grid, NW * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

// Largest supported query-row count per CTA (group * n_q) for a head dim.
int decode_max_rows(int head_dim) { return head_dim >= 512 ? 32 : 64; }

// Decode kernel variant for a shape: the warp-independent kernel for up to 8 rows (the
// first that fits of 8 warps x 2 ring stages, 8 warps x 2 key stages + 1 value stage
// (separate-V layers), 8 x 1, 4 x 1), the
// CTA-wide kernel with 16, 32 or 64 row slots above that; kDecNone when no variant fits
// in shared memory.
enum DecodeVariant { kDecNone = 0, kDecWarp8x2, kDecWarp8x2s, kDecWarp8x1, kDecWarp4x1, kDecTc2, kDecTc4, kDecTc8 };

template <int D>
static int decode_variant_d(const DecodeArgs& a) {
  const int R = (a.num_q_heads / a.num_kv_heads) * a.n_q;
  const bool kv_same = a.v_cache == nullptr;
  int nrk = 0;
  if (kv_same)
    for (int s = 0; s < D / 16; ++s)
      if (rotated_kstep(s, D / 2, a.r)) ++nrk;
  if (R <= 8) {
    if (decode_warp_smem<D, 2, 8, 2>(a) <= kMaxSmem) return kDecWarp8x2;
    if (!kv_same && decode_warp_smem<D, 2, 8, 1>(a) <= kMaxSmem) return kDecWarp8x2s;
    if (decode_warp_smem<D, 1, 8, 1>(a) <= kMaxSmem) return kDecWarp8x1;
    if (decode_warp_smem<D, 1, 4, 1>(a) <= kMaxSmem) return kDecWarp4x1;
    return kDecNone;
  }
  if (R <= 16) return dec_smem_bytes<D, 2>(!kv_same, nrk) <= kMaxSmem ? kDecTc2 : kDecNone;
  if (R <= 32) return dec_smem_bytes<D, 4>(!kv_same, nrk) <= kMaxSmem ? kDecTc4 : kDecNone;
  if (R <= 64 && D < 512) return dec_smem_bytes<D, 8>(!kv_same, nrk) <= kMaxSmem ? kDecTc8 : kDecNone;
  return kDecNone;
}

template <int D>
static cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t stream) {
  switch (decode_variant_d<D>(a)) {
    case kDecWarp8x2: return launch_decode_warp<D, 2, 8, 2>(a, stream);
    case kDecWarp8x2s: return launch_decode_warp<D, 2, 8, 1>(a, stream);
    case kDecWarp8x1: return launch_decode_warp<D, 1, 8, 1>(a, stream);
    case kDecWarp4x1: return launch_decode_warp<D, 1, 4, 1>(a, stream);
    case kDecTc2: return launch_decode_tc<D, 2>(a, stream);
    case kDecTc4: return launch_decode_tc<D, 4>(a, stream);
    case kDecTc8:
      if constexpr (D < 512) return launch_decode_tc<D, 8>(a, stream);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

bool decode_supported(const DecodeArgs& a) {
  switch (a.head_dim) {
    case 32: return decode_variant_d<32>(a) != kDecNone;
    case 64: return decode_variant_d<64>(a) != kDecNone;
    case 128: return decode_variant_d<128>(a) != kDecNone;
    case 256: return decode_variant_d<256>(a) != kDecNone;
    case 512: return decode_variant_d<512>(a) != kDecNone;
    default: return false;
  }
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (decode_umma_applies(a)) return launch_decode_umma_any(a, stream);
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
// One thread per output element (row, dim): the row's split weights exp(lse_s - max)
// are recomputed by every thread of the row (the split log-sum-exps stay in L1), and
// the partial reads are coalesced across the threads of a row.
__global__ void combine_kernel(CombineArgs a) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.rows * a.head_dim) return;
  const int row = (int)(idx / a.head_dim), c = (int)(idx % a.head_dim);
  float mm = -INFINITY;
  for (int s = 0; s < a.num_splits; ++s) mm = fmaxf(mm, a.partial_lse[(size_t)s * a.rows + row]);
  float den = 0.f, acc = 0.f;
  if (mm != -INFINITY) {
    for (int s = 0; s < a.num_splits; ++s) {
      const float l = a.partial_lse[(size_t)s * a.rows + row];
      if (l == -INFINITY) continue;
      const float w = __expf(l - mm);
      den += w;
      acc += w * a.partial_o[((size_t)s * a.rows + row) * a.head_dim + c];
    }
    acc /= den;
  }
  if (a.out_f32)
    reinterpret_cast<float*>(a.out)[idx] = acc;
  else
    reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(acc);
  if (c == 0 && a.lse != nullptr) a.lse[row] = (mm == -INFINITY) ? -INFINITY : mm + logf(den);
}

// The same merge with 16-byte accesses: a warp takes 128 columns of one row, four per lane.
// Each lane forms the maximum and the weight sum over the splits in split order and
// accumulates its columns in split order, exactly as the per-element kernel does, so the
// two give identical results; the lse values a warp reads are one broadcast load each, and
// the partial rows arrive as whole 512-byte segments.
__global__ void __launch_bounds__(256) combine_vec_kernel(CombineArgs a) {
  const int chunks = (a.head_dim + 127) / 128;
  const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= (long long)a.rows * chunks) return;
  const int lane = threadIdx.x & 31;
  const int row = (int)(wid / chunks);
  const int c0 = (int)(wid % chunks) * 128 + lane * 4;
  const bool mine = c0 < a.head_dim;
  float mm = -INFINITY;
  for (int s = 0; s < a.num_splits; ++s) mm = fmaxf(mm, a.partial_lse[(size_t)s * a.rows + row]);
  float den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mm != -INFINITY) {
#pragma unroll 4
    for (int s = 0; s < a.num_splits; ++s) {
      const float l = a.partial_lse[(size_t)s * a.rows + row];
      if (l == -INFINITY) continue;
      const float w = __expf(l - mm);
      den += w;
      if (mine) {
        const float4 v = *reinterpret_cast<const float4*>(a.partial_o + ((size_t)s * a.rows + row) * a.head_dim + c0);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
    }
    acc.x /= den;
    acc.y /= den;
    acc.z /= den;
    acc.w /= den;
  }
  if (mine) {
    const size_t o = (size_t)row * a.head_dim + c0;
    if (a.out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) = acc;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&lo);
      u.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) = u;
    }
  }
  if (c0 == 0 && a.lse != nullptr) a.lse[row] = (mm == -INFINITY) ? -INFINITY : mm + logf(den);
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  const long long total = (long long)a.rows * a.head_dim;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  // The warp-per-128-columns form needs 16-byte aligned rows and enough warps to hide its
  // loads' latency (measured: 2048 rows x 512 columns, 8192 warps, 14 us against 31 us per
  // element; 256 rows x 512, 1024 warps, 12 us against 10 us): below about two full
  // residencies of 256-thread blocks the per-element form, with four times the warps, wins.
  const uintptr_t out_mask = a.out_f32 ? 15u : 7u;
  const long long warps = (long long)a.rows * ((a.head_dim + 127) / 128);
  const bool vec = a.head_dim % 4 == 0 && (reinterpret_cast<uintptr_t>(a.partial_o) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(a.out) & out_mask) == 0 && warps >= 2048;
  if (vec) {
    combine_vec_kernel<<<(unsigned)((warps + 7) / 8), threads, 0, stream>>>(a);
  } else {
    combine_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace gattn
