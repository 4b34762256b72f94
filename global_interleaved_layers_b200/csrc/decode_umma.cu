// decode_umma.cu -- split-KV decode / speculative verify of global (K=V) layers on the
// tcgen05 tensor cores, for 9 to 32 query rows per KV head at head dim 256 or 512: the
// 4-token verify of a draft model's tokens with 8 query heads per KV head is 32 rows.
//
// One CTA handles a work item, a (sequence, KV head, split): every query row of the KV
// head (the group's heads x the new tokens) against a contiguous range of 128-key tiles of
// the sequence's visible keys (the cached tokens, then the new tokens themselves). Items
// cover equal tile counts, so a long sequence takes more splits than a short one. Keys sit on
// the MMA's M dimension, rows on N = 32:
//   S^T = K Q^T     M = 128 keys, N = 32 rows, K = head dim (64-dim chunks)
//   O^T += V^T P^T  M = 128 head dims per block (head_dim / 128 blocks), N = 32, K = 128 keys
// The single stored K=V tensor is the score operand (read K-major) and the value operand
// (read MN-major) ("Visual guide to Gemma 4", section "K=V technique"). It streams through
// two rings of 16 KB chunk slots: the key ring feeds the scores and the value ring the
// value product. Both read the same rows; the value ring's copy is normally still in L2,
// so HBM sees every row once. The two chunks holding rotated dims ([0, 64) and
// [d/2, d/2 + 64): p-RoPE with at most 64 rotated pairs, section "p-RoPE") are rotated in
// place in the key ring; the value ring keeps them as stored.
//
// Roles (512 threads):
//   warp 0      key-ring producer: TMA loads, chunk by chunk (the rotated chunks last)
//   warp 1      TMEM owner and issuer of the score MMAs, which run ahead into the next
//               tile (its scores overlap this tile's softmax)
//   warp 2      value-ring producer
//   warp 3      issuer of the value-product MMAs
//   warps 4-7   rotation of the key ring's two rotated chunks, in place
//   warps 8-15  softmax: two warps per TMEM lane quadrant (32 keys of the tile each), one
//               taking rows 0-15 and the other rows 16-31; row maxima and sums reduced
//               across the lanes and the four warps of a row half; P^T into shared memory
//               (double-buffered); output rescale; epilogue O / l and log-sum-exp
// The last tile of a sequence (cached rows, then the new tokens, then zeros) is loaded by
// TMA like any other and then patched by the producer warp: the rows past the cache end
// hold no data the kernel may use, so they are overwritten in shared memory with the new
// tokens' rows and zeros before the chunk is released to its consumers. Every wait is
// bounded: one that runs out records a timeout and the CTA unwinds.
#include "common.cuh"
#include "kernels.h"

namespace gattn {

namespace {

constexpr int kUThreads = 512;
constexpr int kUKeys = 128;             // keys per tile (the MMA's M)
constexpr int kUN = 32;                 // query rows (padded): the MMA's N
constexpr int kUChunkBytes = 16384;     // 128 keys x 64 dims bf16
constexpr int kUKSlots = 6;             // key ring
constexpr int kUVSlots = 4;             // value ring (chunk pairs stay adjacent)
constexpr int kUHeaderBytes = 4096;     // mbarriers, TMEM base, flags, reductions, angle tables
constexpr int kURankMax = 2048;         // sequences ranked by length in the P^T buffers (16 KB)
constexpr int kUStartTiles = 3;         // a CTA's start-up cost, in 128-key tiles

__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of (row, byte column) inside a 128-byte-swizzled block whose rows are 128
// bytes (groups of 8 rows, 1024 bytes each; 16-byte units XOR-ed with the row mod 8).
__device__ __forceinline__ uint32_t sw128(int row, int colb) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((colb >> 4) ^ (row & 7)) << 4) | (colb & 15)));
}

struct __align__(8) UmmaHeader {
  uint64_t k_full[kUKSlots], k_empty[kUKSlots];
  uint64_t v_full[kUVSlots], v_empty[kUVSlots];
  uint64_t k_tail[kUKSlots], v_tail[kUVSlots];  // a tail chunk's TMA landed (before the patch)
  uint64_t q_ready;     // softmax warps: the query rows are in shared memory
  uint64_t rot_ready[2];  // rotation warps: tile t's rotated chunks are in place (barrier t & 1)
  uint64_t s_full[2];   // S^T(t) complete (buffer t & 1)
  uint64_t p_full[2];   // softmax warps: P^T(t) written, O rescaled
  uint64_t pv_done[2];  // O^T += V^T P^T (t) complete
  uint64_t hmeet[2];    // the four softmax warps of a row half meet
  uint64_t mma_done[2];  // each MMA issuer's last operations complete
  uint32_t tmem_base;
  int abort_flag;
  int seq;              // the sequence this CTA serves (-1: no work item)
  int split, tile_per, seq_splits;  // its split, tiles per split, splits the sequence uses
  int tile_floor, max_tiles, search;  // tile-count choice: 4-wave floor, longest sequence, on/off
  long long cand_cost[16];  // estimated duration of each candidate tile count (one per warp)
  int cand_tiles[16];
  float red[2][2][4][16];  // [meeting parity][row half][quadrant][row]
  double itf[64];       // theta_j / (2 pi) of rotary pair j (0 past the rotated pairs)
  float2 stp[64];       // cos / sin of theta_j (identity past the rotated pairs)
};
static_assert(sizeof(UmmaHeader) <= kUHeaderBytes, "header");

// Chunk order of a key tile in the key ring: the chunks without rotated dims first, the two
// rotated ones (0 and d/128) last, so the ring keeps streaming while they are turned.
template <int D>
__device__ __forceinline__ int key_chunk(int i) {
  constexpr int kCh = D / 64, R = D / 128;
  if (i == kCh - 2) return 0;
  if (i == kCh - 1) return R;
  return i + 1 + (i + 1 >= R ? 1 : 0);
}

}  // namespace

template <int D>
constexpr size_t umma_smem_bytes() {
  return 1024 /*align*/ + kUHeaderBytes + (size_t)(D / 64) * kUN * 128 /*Q*/ + 2 * (size_t)kUN * 256 /*P x2*/ +
         (size_t)(kUKSlots + kUVSlots) * kUChunkBytes;
}

template <int D>
__global__ void __launch_bounds__(kUThreads, 1)
decode_umma_kernel(const __grid_constant__ CUtensorMap cache_map, DecodeArgs a, int num_sms) {
  constexpr int kCh = D / 64;        // chunks per key tile
  constexpr int kBlocks = D / 128;   // 128-dim blocks of O^T
  static_assert(kCh * kUN * 128 >= kURankMax * 4 && 2 * kUN * 256 >= kURankMax * 8, "ranking tables");
  static_assert(2 * kUN * 256 >= kUN * 64 * 8, "query angle table");
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  UmmaHeader* hd = reinterpret_cast<UmmaHeader*>(base);
  uint8_t* q_s = base + kUHeaderBytes;                 // chunk c at c * N * 128
  uint8_t* p_s = q_s + (size_t)kCh * kUN * 128;        // [2 buffers][2 key chunks][N rows x 128 B]
  uint8_t* kring = p_s + 2 * (size_t)kUN * 256;
  uint8_t* vring = kring + (size_t)kUKSlots * kUChunkBytes;

  const int kvh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work items. Every split of every sequence covers the same number of key tiles T, at
  // least max(the longest sequence's tiles / num_splits, all tiles / (4 waves of CTAs)), so
  // the items are near-equal in work; a sequence uses ceil(tiles / T) of the num_splits
  // splits. T is the candidate ceil(longest / s), s <= num_splits, with the fewest rounds
  // times tiles per round (below).
  // Items are numbered longest sequence first (ties by index), then by split, and CTA i of
  // the KV head (blockIdx.x + num_splits * blockIdx.z) takes item i, so the longest work
  // starts first and the short items fill the tail. CTAs past the last item leave at once;
  // the last split of a sequence writes -inf log-sum-exps for the splits it leaves unused.
  // (The lengths are staged in the Q^T buffer and the ranking table lives in the P^T
  // buffers, both free until the query rows are loaded: one global load per length, not one
  // dependent load per comparison.)
  {
    int* sl = reinterpret_cast<int*>(q_s);
    int* rk_tiles = reinterpret_cast<int*>(p_s);
    int* rk_seq = rk_tiles + kURankMax;
    const int extra = a.new_keys ? a.n_q : 0;
    if (a.batch <= kURankMax)
      for (int i = threadIdx.x; i < a.batch; i += kUThreads) sl[i] = a.cache_seqlens[i];
    __syncthreads();
    if (a.batch <= kURankMax) {
      for (int me = threadIdx.x; me < a.batch; me += kUThreads) {
        const int lme = sl[me];
        int rank = 0;
        for (int o = 0; o < a.batch; ++o) {
          const int lo = sl[o];
          rank += (lo > lme || (lo == lme && o < me)) ? 1 : 0;
        }
        rk_tiles[rank] = (lme + extra + kUKeys - 1) / kUKeys;
        rk_seq[rank] = me;
      }
    }
    __syncthreads();
    const bool ranked = a.batch <= kURankMax;
    const int sms = num_sms > 0 ? num_sms : 148;
    if (threadIdx.x == 0) {
      long long total = 0;
      int mx = 0;
      for (int r = 0; r < a.batch; ++r) {
        const int tl = ranked ? rk_tiles[r] : (a.cache_seqlens[r] + extra + kUKeys - 1) / kUKeys;
        total += tl;
        mx = max(mx, tl);
      }
      total *= a.num_kv_heads;
      const long long ctas = 4LL * sms;
      const int floor4 = max(1, (int)((total + ctas - 1) / ctas));
      hd->tile_floor = floor4;
      hd->max_tiles = mx;
      hd->tile_per = max(floor4, (mx + a.num_splits - 1) / a.num_splits);
      hd->search = ranked && a.num_splits > 1;
    }
    __syncthreads();
    if (hd->search) {
      // Candidates T = ceil(longest / s) for s = num_splits, num_splits - 1, ... (one per
      // warp). A launch runs its items in rounds of one CTA per SM, and a round lasts about as
      // long as its longest item, so a candidate costs (T + start-up) x ceil(items / SMs).
      // Just more items than SMs makes a second round of long items; the fewest rounds of the
      // shortest items win (ties to the larger T: fewer partials to combine).
      const int w = threadIdx.x >> 5, ln = threadIdx.x & 31;
      const int s_c = a.num_splits - w;
      if (w < 16) {
        long long cost = -1;
        int Tc = 0;
        if (s_c >= 1) {
          Tc = max(hd->tile_floor, (hd->max_tiles + s_c - 1) / s_c);
          int n = 0;
          for (int r = ln; r < a.batch; r += 32) n += max(1, (rk_tiles[r] + Tc - 1) / Tc);
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
          const long long items = (long long)n * a.num_kv_heads;
          cost = (long long)(Tc + kUStartTiles) * ((items + sms - 1) / sms);
        }
        if (ln == 0) {
          hd->cand_cost[w] = cost;
          hd->cand_tiles[w] = Tc;
        }
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        long long best = -1;
        for (int c = 0; c < 16; ++c)
          if (hd->cand_cost[c] >= 0 && (best < 0 || hd->cand_cost[c] <= best)) {
            best = hd->cand_cost[c];
            hd->tile_per = hd->cand_tiles[c];
          }
      }
    }
    if (threadIdx.x == 0) {
      const int T = hd->tile_per;
      const int item = (int)blockIdx.x + a.num_splits * (int)blockIdx.z;
      int acc = 0;
      hd->seq = -1;
      for (int r = 0; r < a.batch; ++r) {
        const int tl = ranked ? rk_tiles[r] : (a.cache_seqlens[r] + extra + kUKeys - 1) / kUKeys;
        const int sr = max(1, (tl + T - 1) / T);
        if (item < acc + sr) {
          hd->seq = ranked ? rk_seq[r] : r;
          hd->split = item - acc;
          hd->seq_splits = sr;
          break;
        }
        acc += sr;
      }
    }
    __syncthreads();
  }
  if (hd->seq < 0) return;  // no work item: nothing allocated or armed yet
  const int b = hd->seq;
  const int split = hd->split;
  const int group = a.num_q_heads / a.num_kv_heads;
  const int R = group * a.n_q;
  const int len = a.cache_seqlens[b];
  const int nk = len + (a.new_keys ? a.n_q : 0);           // visible keys: the cache, then the new tokens
  const int qoff = a.q_pos_offset ? a.q_pos_offset[b] : 0;  // queries after a key-range shard
  const int ntiles = (nk + kUKeys - 1) / kUKeys;
  const int per = hd->tile_per;
  const int t0 = min(ntiles, split * per);
  const int nt = min(ntiles, t0 + per) - t0;
  const int rows_total = a.batch * a.n_q * a.num_q_heads;
  const int r = a.r;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kUKSlots; ++s) { mbar_init(&hd->k_full[s], 1); mbar_init(&hd->k_empty[s], 1); }
    for (int s = 0; s < kUVSlots; ++s) { mbar_init(&hd->v_full[s], 1); mbar_init(&hd->v_empty[s], 1); }
    for (int s = 0; s < kUKSlots; ++s) mbar_init(&hd->k_tail[s], 1);
    for (int s = 0; s < kUVSlots; ++s) mbar_init(&hd->v_tail[s], 1);
    mbar_init(&hd->q_ready, 8);
    mbar_init(&hd->rot_ready[0], 4);
    mbar_init(&hd->rot_ready[1], 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&hd->s_full[i], 1);
      mbar_init(&hd->p_full[i], 8);
      mbar_init(&hd->pv_done[i], 1);
      mbar_init(&hd->hmeet[i], 4);
    }
    mbar_init(&hd->mma_done[0], 1);
    mbar_init(&hd->mma_done[1], 1);
    hd->abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    const int j = threadIdx.x;
    const double f = j < r ? rope_inv_freq_turns(j, D, a.log2_base) : 0.0;
    float c = 1.f, sn = 0.f;
    rope_cos_sin(1.0, f, &c, &sn);
    hd->itf[j] = f;
    hd->stp[j] = make_float2(c, sn);
  }
  if (warp == 1) {
    tmem_alloc(&hd->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hd->tmem_base;
  // S^T buffers at columns 0 and 32; O^T block m at 64 + 32 m
  const uint32_t col_o = 64;
  volatile int* abort_flag = &hd->abort_flag;

  // A tile that reaches past the cache end (the sequence's last one or two) is patched by
  // the whole producer warp once its TMA load (if any) has landed: rows from the cache end
  // on take the new tokens' rows, then zeros (finite values: the value product multiplies
  // them by zero weights).
  auto patch_tail_chunk = [&](uint8_t* dst, int c, int key0) {
    const int u0 = len - key0 > 0 ? len - key0 : 0;  // first row past the cache
    for (int idx = u0 * 8 + lane; idx < kUKeys * 8; idx += 32) {
      const int u = idx >> 3, k16 = idx & 7;
      const int v = key0 + u;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (v < nk)
        val = *reinterpret_cast<const uint4*>(a.new_k + (((size_t)b * a.n_q + (v - len)) * a.num_kv_heads + kvh) * D +
                                               c * 64 + k16 * 8);
      *reinterpret_cast<uint4*>(dst + sw128(u, k16 * 16)) = val;
    }
    fence_proxy_async_smem();
    __syncwarp();
  };

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers (key ring, value ring)
    const bool is_k = warp == 0;
    const int nslots = is_k ? kUKSlots : kUVSlots;
    uint64_t* full = is_k ? hd->k_full : hd->v_full;
    uint64_t* empty = is_k ? hd->k_empty : hd->v_empty;
    uint64_t* tailb = is_k ? hd->k_tail : hd->v_tail;
    uint8_t* ring = is_k ? kring : vring;
    if (lane == 0 && nt > 0) prefetch_tensormap(&cache_map);
    const int plane = b * a.num_kv_heads + kvh;
    bool ok = true;
    int seq = 0;
    // A tail chunk whose cache rows are on their way: it is patched and released one
    // chunk later, so its load overlaps the next chunk's (slot s, parity bit per slot).
    int pend_s = -1, pend_c = 0, pend_key0 = 0;
    uint32_t tail_par = 0u;
    auto finish_pending = [&]() -> bool {
      if (pend_s < 0) return true;
      const int s = pend_s;
      if (!__all_sync(0xffffffffu, mbar_wait(&tailb[s], (tail_par >> s) & 1u, abort_flag))) return false;
      pend_s = -1;
      tail_par ^= 1u << s;
      patch_tail_chunk(ring + s * kUChunkBytes, pend_c, pend_key0);
      if (lane == 0) mbar_arrive(&full[s]);
      return true;
    };
    for (int lt = 0; lt < nt && ok; ++lt) {
      const int key0 = (t0 + lt) * kUKeys;
      const bool tail = key0 + kUKeys > len;
      for (int i = 0; i < kCh && ok; ++i, ++seq) {
        const int c = is_k ? key_chunk<D>(i) : i;
        const int s = seq % nslots;
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ((uint32_t)(seq / nslots) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        uint8_t* dst = ring + s * kUChunkBytes;
        if (!tail) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], kUChunkBytes);
            tma_load_3d(dst, &cache_map, &full[s], c * 64, key0, plane);
          }
        } else if (key0 < len) {  // cache rows by TMA (rows past the capacity read as zeros)
          if (lane == 0) {
            mbar_arrive_expect_tx(&tailb[s], kUChunkBytes);
            tma_load_3d(dst, &cache_map, &tailb[s], c * 64, key0, plane);
          }
        }
        // the previous chunk, if it was a tail chunk in flight: its slot was taken before
        // this one, so the consumers see the chunks in order
        ok = finish_pending();
        if (!ok) break;
        if (tail) {
          if (key0 < len) {
            pend_s = s; pend_c = c; pend_key0 = key0;
          } else {  // no cached rows in this tile: new tokens and zeros only
            patch_tail_chunk(dst, c, key0);
            if (lane == 0) mbar_arrive(&full[s]);
          }
        }
      }
    }
    if (ok) ok = finish_pending();
    if (pend_s >= 0 && lane == 0) {
      // an abort left a tail chunk's load in flight: it lands before the CTA can exit, and
      // its slot is released so the drain below finds every fill complete
      const uint32_t par = (tail_par >> pend_s) & 1u;
      const unsigned long long ts = globaltimer_ns();
      while (!mbar_try_wait(&tailb[pend_s], par) && globaltimer_ns() - ts < kWaitLimitNs) {}
      mbar_arrive(&full[pend_s]);
    }
    // the last loads land before the CTA can exit (one per slot at most is outstanding)
    if (lane == 0) {
      for (int back = 1; back <= nslots && back <= seq; ++back) {
        const int sq = seq - back;
        const uint32_t par = (uint32_t)(sq / nslots) & 1u;
        if (!mbar_try_wait(&full[sq % nslots], par)) {
          const unsigned long long ts = globaltimer_ns();
          while (!mbar_try_wait(&full[sq % nslots], par) && globaltimer_ns() - ts < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers: warp 1 the scores,
    // warp 3 the value products (each waits only on its own inputs; commits track the
    // issuing thread's MMAs)
    if (lane == 0 && nt > 0) {
      bool ok = mbar_wait(&hd->q_ready, 0, abort_flag);
      if (warp == 1) {
        const uint32_t idesc_s = umma_idesc_bf16(kUKeys, kUN, 0, 0);
        int kseq = 0;
        for (int lt = 0; lt < nt && ok; ++lt) {
          const uint32_t sb = (uint32_t)(lt & 1) * kUN;
          // S^T(t) overwrites the buffer softmax(t-2) read: P(t-2) arrived before PV(t-2), which
          // the value issuer issued only after that softmax had finished reading
          if (lt >= 2) ok = mbar_wait(&hd->p_full[lt & 1], (uint32_t)((lt - 2) >> 1) & 1u, abort_flag);
          for (int i = 0; i < kCh && ok; ++i, ++kseq) {
            const int c = key_chunk<D>(i);
            const int s = kseq % kUKSlots;
            ok = mbar_wait(&hd->k_full[s], (uint32_t)(kseq / kUKSlots) & 1u, abort_flag);
            if (ok && i == kCh - 2) ok = mbar_wait(&hd->rot_ready[lt & 1], (uint32_t)(lt >> 1) & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint64_t kd = sdesc_sw128(smem_u32(kring + s * kUChunkBytes), 16, 1024);
            const uint64_t qd = sdesc_sw128(smem_u32(q_s + (size_t)c * kUN * 128), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) umma_ss(tmem + sb, kd + 2 * kk, qd + 2 * kk, idesc_s, (i | kk) != 0);
            umma_commit(&hd->k_empty[s]);
          }
          if (ok) umma_commit(&hd->s_full[lt & 1]);
        }
      } else {
        const uint32_t idesc_o = umma_idesc_bf16(128, kUN, 1, 0);
        int vseq = 0;
        for (int lt = 0; lt < nt && ok; ++lt) {
          ok = mbar_wait(&hd->p_full[lt & 1], (uint32_t)(lt >> 1) & 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint8_t* pb = p_s + (size_t)(lt & 1) * kUN * 256;
          for (int m = 0; m < kBlocks && ok; ++m, vseq += 2) {
            const int s0 = vseq % kUVSlots;
            const uint32_t par = (uint32_t)(vseq / kUVSlots) & 1u;
            ok = mbar_wait(&hd->v_full[s0], par, abort_flag);
            if (ok) ok = mbar_wait(&hd->v_full[s0 + 1], par, abort_flag);
            if (!ok) break;
            tc_fence_after();
            // V^T: two adjacent 64-dim chunks (MN-major, 16 KB apart); P^T: K-major, keys in two
            // 64-key chunks of N rows
            const uint64_t vd = sdesc_sw128(smem_u32(vring + s0 * kUChunkBytes), kUChunkBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < kUKeys / 16; ++kk) {
              const uint64_t pd = sdesc_sw128(smem_u32(pb + (size_t)(kk >> 2) * kUN * 128), 16, 1024) + 2 * (kk & 3);
              umma_ss(tmem + col_o + (uint32_t)(m * kUN), vd + 128 * kk, pd, idesc_o, lt != 0 || kk != 0);
            }
            umma_commit(&hd->v_empty[s0]);
            umma_commit(&hd->v_empty[s0 + 1]);
          }
          if (ok) umma_commit(&hd->pv_done[lt & 1]);
        }
      }
      // every MMA this thread issued is complete before the CTA frees tensor memory
      umma_commit(&hd->mma_done[warp == 1 ? 0 : 1]);
      const unsigned long long ts = globaltimer_ns();
      while (!mbar_try_wait(&hd->mma_done[warp == 1 ? 0 : 1], 0) && globaltimer_ns() - ts < kWaitLimitNs) {}
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ rotation of the key ring's rotated chunks
    // thread (k, g): the 8 pairs of 16-byte unit k (pairs 8k .. 8k + 7: dims j and d/2 + j)
    // for keys 8g .. 8g + 7, from the exact angle of key 8g, stepping by theta_j per key;
    // pairs past r keep the identity (the tables hold cos 1, sin 0 for them)
    const int tid = threadIdx.x - 128;  // 0..127
    const int k = tid & 7, g = tid >> 3;
    // this thread's pairs' frequencies and one-key steps, held in registers: read from
    // shared memory inside the loop they would be reloaded after every store to the ring
    // (and the lanes' stride of 8 pairs puts four lanes on each bank)
    double itfv[8];
    float2 stv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      itfv[e] = hd->itf[8 * k + e];
      stv[e] = hd->stp[8 * k + e];
    }
    bool ok = true;
    for (int lt = 0; lt < nt && ok; ++lt) {
      const int key0 = (t0 + lt) * kUKeys;
      const int sq0 = lt * kCh + kCh - 2;  // key-ring sequence index of the tile's chunk 0; chunk d/128 follows
      const int s0 = sq0 % kUKSlots, s1 = (sq0 + 1) % kUKSlots;
      // the anchors need no data: they are computed while the chunks are on their way
      float ac[8], as[8];
      {
        const double pos0 = (double)(key0 + 8 * g);
#pragma unroll
        for (int e = 0; e < 8; ++e) rope_cos_sin(pos0, itfv[e], &ac[e], &as[e]);
      }
      // A parity wait is exact only while the slot's previous fill has completed and the next
      // cannot have: the next needs this rotation. Fills of tile t-1 have completed once
      // S^T(t-1) is done; a previous fill within this tile (sequence index minus the slot
      // count) has once the score MMA released it (its release cannot advance again before
      // this rotation either).
      if (lt >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&hd->s_full[(lt - 1) & 1], (uint32_t)((lt - 1) >> 1) & 1u, abort_flag));
        if (!ok) break;
      }
#pragma unroll
      for (int e = 0; e < 2 && ok; ++e) {
        const int sq = sq0 + e;
        if (sq - kUKSlots >= lt * kCh)
          ok = __all_sync(0xffffffffu, mbar_wait(&hd->k_empty[(sq - kUKSlots) % kUKSlots],
                                                 (uint32_t)((sq - kUKSlots) / kUKSlots) & 1u, abort_flag));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&hd->k_full[sq % kUKSlots], (uint32_t)(sq / kUKSlots) & 1u, abort_flag));
      }
      if (!ok) break;
      uint8_t* c0 = kring + s0 * kUChunkBytes;
      uint8_t* c1 = kring + s1 * kUChunkBytes;
#pragma unroll 2
      for (int i = 0; i < 8; ++i) {
        const uint32_t off = sw128(8 * g + i, 16 * k);
        const uint4 w0 = *reinterpret_cast<const uint4*>(c0 + off);
        const uint4 w1 = *reinterpret_cast<const uint4*>(c1 + off);
        const uint32_t x0w[4] = {w0.x, w0.y, w0.z, w0.w}, x1w[4] = {w1.x, w1.y, w1.z, w1.w};
        uint32_t y0w[4], y1w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float y0[2], y1[2];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int e = 2 * h + e2;
            const float x0 = __uint_as_float(e2 ? (x0w[h] & 0xFFFF0000u) : (x0w[h] << 16));
            const float x1 = __uint_as_float(e2 ? (x1w[h] & 0xFFFF0000u) : (x1w[h] << 16));
            y0[e2] = x0 * ac[e] - x1 * as[e];
            y1[e2] = x0 * as[e] + x1 * ac[e];
            const float2 st = stv[e];
            const float nc = ac[e] * st.x - as[e] * st.y;
            as[e] = ac[e] * st.y + as[e] * st.x;
            ac[e] = nc;
          }
          y0w[h] = pack_bf16x2(y0[0], y0[1]);
          y1w[h] = pack_bf16x2(y1[0], y1[1]);
        }
        *reinterpret_cast<uint4*>(c0 + off) = make_uint4(y0w[0], y0w[1], y0w[2], y0w[3]);
        *reinterpret_cast<uint4*>(c1 + off) = make_uint4(y1w[0], y1w[1], y1w[2], y1w[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hd->rot_ready[lt & 1]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ softmax warps
    const int sw = warp - 8;            // 0..7
    const int quad = warp & 3;          // TMEM lane quadrant: keys quad*32 .. +31 (and those O^T dims)
    const int half = sw >> 2;           // rows 16 half .. 16 half + 15
    const int tid = threadIdx.x - 256;  // 0..255
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
    constexpr int H = 16;               // rows per thread

    // ---- query rows, rotated for their positions, into the swizzled K-major layout: item
    // (row, unit ku) holds dims 8ku .. 8ku + 7 and their partners d/2 + 8ku ..; every thread
    // issues all of its 16-byte loads before it computes. The angles depend only on the
    // token and the pair: each is computed once into a table (in the P^T buffers, free
    // until the first tile; n_q <= 32 tokens x r <= 64 pairs of cos / sin fill 16 KB at most).
    {
      float2* qcs = reinterpret_cast<float2*>(p_s);
      constexpr int kU = D / 16;                  // 16-byte units in each half of a row
      constexpr int kItems = kUN * kU / 256;      // items per thread
      uint4 x0[kItems], x1[kItems];
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int idx = tid + 256 * it, row = idx / kU, ku = idx % kU;
        x0[it] = x1[it] = make_uint4(0u, 0u, 0u, 0u);
        if (row < R) {
          const uint16_t* qrow = a.q + (((size_t)b * a.n_q + row / group) * a.num_q_heads + kvh * group + row % group) * D;
          x0[it] = *reinterpret_cast<const uint4*>(qrow + 8 * ku);
          x1[it] = *reinterpret_cast<const uint4*>(qrow + D / 2 + 8 * ku);
        }
      }
      for (int idx = tid; idx < a.n_q * r; idx += 256) {
        const int tok = idx / r, j = idx % r;
        float cs, sn;
        rope_cos_sin((double)(len + tok + qoff), hd->itf[j], &cs, &sn);
        qcs[idx] = make_float2(cs, sn);
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");  // the softmax warps' table is complete
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int idx = tid + 256 * it, row = idx / kU, ku = idx % kU;
        const uint32_t w0[4] = {x0[it].x, x0[it].y, x0[it].z, x0[it].w};
        const uint32_t w1[4] = {x1[it].x, x1[it].y, x1[it].z, x1[it].w};
        uint32_t y0w[4], y1w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float y0[2], y1[2];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int j = 8 * ku + 2 * h + e2;
            const float a0 = __uint_as_float(e2 ? (w0[h] & 0xFFFF0000u) : (w0[h] << 16));
            const float a1 = __uint_as_float(e2 ? (w1[h] & 0xFFFF0000u) : (w1[h] << 16));
            y0[e2] = a0;
            y1[e2] = a1;
            if (row < R && j < r) {
              const float2 t = qcs[(row / group) * r + j];
              y0[e2] = a0 * t.x - a1 * t.y;
              y1[e2] = a0 * t.y + a1 * t.x;
            }
          }
          y0w[h] = pack_bf16x2(y0[0], y0[1]);
          y1w[h] = pack_bf16x2(y1[0], y1[1]);
        }
        const int c0 = ku / 8, c1 = (D / 2) / 64 + ku / 8;  // chunks of the two halves
        *reinterpret_cast<uint4*>(q_s + (size_t)c0 * kUN * 128 + sw128(row, (ku % 8) * 16)) =
            make_uint4(y0w[0], y0w[1], y0w[2], y0w[3]);
        *reinterpret_cast<uint4*>(q_s + (size_t)c1 * kUN * 128 + sw128(row, (ku % 8) * 16)) =
            make_uint4(y1w[0], y1w[1], y1w[2], y1w[3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&hd->q_ready);

    // The four softmax warps of a row half meet through one mbarrier; each makes the same
    // meetings in the same order, so the meeting count gives the phase.
    uint32_t meets = 0;
    bool ok = nt > 0;
    // Row reduction over the tile's 128 keys: reduce-scatter over the warp's lanes (each
    // even lane ends with one row), then over the half's four warps through shared memory;
    // every lane gets every row of its half back.
    auto rows_reduce = [&](float (&x)[H], bool sum) {
#pragma unroll
      for (int w = 16; w >= 2; w >>= 1) {
        const int cnt = w >> 1;  // values kept after this step
#pragma unroll
        for (int q = 0; q < cnt; ++q) {
          const bool hi = (lane & w) != 0;
          const float send = hi ? x[q] : x[q + cnt];
          const float keep = hi ? x[q + cnt] : x[q];
          const float got = __shfl_xor_sync(0xffffffffu, send, w);
          x[q] = sum ? keep + got : fmaxf(keep, got);
        }
      }
      {
        const float got = __shfl_xor_sync(0xffffffffu, x[0], 1);
        x[0] = sum ? x[0] + got : fmaxf(x[0], got);
      }
      // each halving kept rows q + cnt where the lane bit was set: lane bit 4 chose +8,
      // bit 3 +4, bit 2 +2, bit 1 +1
      if ((lane & 1) == 0)
        hd->red[meets & 1u][half][quad][((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                                        ((lane >> 1) & 1)] = x[0];
      __syncwarp();
      if (lane == 0) mbar_arrive(&hd->hmeet[half]);
      ok = __all_sync(0xffffffffu, mbar_wait(&hd->hmeet[half], meets & 1u, abort_flag));
      ++meets;
      const float* rr = hd->red[(meets - 1) & 1u][half][0];
      const int row = lane & 15;
      const float mine = sum ? (rr[row] + rr[16 + row]) + (rr[32 + row] + rr[48 + row])
                             : fmaxf(fmaxf(rr[row], rr[16 + row]), fmaxf(rr[32 + row], rr[48 + row]));
#pragma unroll
      for (int q = 0; q < H; ++q) x[q] = __shfl_sync(0xffffffffu, mine, q);
    };

    float m_used[H], l_acc[H];
#pragma unroll
    for (int q = 0; q < H; ++q) { m_used[q] = -INFINITY; l_acc[q] = 0.f; }
    const int u = quad * 32 + lane;  // this thread's key in a tile (its TMEM lane)

    for (int lt = 0; lt < nt && ok; ++lt) {
      const int bb = lt & 1;
      const int key0 = (t0 + lt) * kUKeys;
      ok = __all_sync(0xffffffffu, mbar_wait(&hd->s_full[bb], (uint32_t)(lt >> 1) & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float sv[H];
      tmem_ld_x16(tmem + lane_off + (uint32_t)(bb * kUN + half * H), reinterpret_cast<uint32_t*>(sv));
      tmem_ld_wait();
      const int v = key0 + u;  // the key's index among the visible keys (= its position)
#pragma unroll
      for (int q = 0; q < H; ++q) {
        const int row = half * H + q;
        const bool vis = row < R && v < nk && (v < len || v - len <= row / group);
        sv[q] = vis ? sv[q] * scale_log2 : -INFINITY;
      }
      // ---- the tile's row maxima; a running max moves only past 2^8 (as in prefill), and
      // mt[q] becomes row q's rescale factor (the same in the half's four warps)
      float mt[H];
#pragma unroll
      for (int q = 0; q < H; ++q) mt[q] = sv[q];
      rows_reduce(mt, false);
      if (!ok) break;
      bool rescale = false;
#pragma unroll
      for (int q = 0; q < H; ++q) {
        float alpha = 1.f;
        if (mt[q] > m_used[q] + 8.f || (m_used[q] == -INFINITY && mt[q] > -INFINITY)) {
          if (m_used[q] != -INFINITY) {
            alpha = ex2_sfu(m_used[q] - mt[q]);
            rescale = true;
          }
          m_used[q] = mt[q];
        }
        l_acc[q] *= alpha;
        mt[q] = alpha;
      }
      // ---- P^T buffer bb was read by PV(t-2); O^T may only be rescaled once PV(t-1) is done
      if (lt >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&hd->pv_done[bb], (uint32_t)((lt - 2) >> 1) & 1u, abort_flag));
        if (!ok) break;
      }
      if (rescale && lt >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&hd->pv_done[bb ^ 1], (uint32_t)((lt - 1) >> 1) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int m = 0; m < kBlocks; ++m) {
          uint32_t o[H];
          const uint32_t ta = tmem + lane_off + col_o + (uint32_t)(m * kUN + half * H);
          tmem_ld_x16(ta, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < H; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * mt[i]);
          tmem_st_x16(ta, o);
        }
        tmem_st_wait();
      }
      // ---- P^T: row q's probability of this key, bf16, into the K-major operand (keys
      // 0-63 in the first 64-key chunk, 64-127 in the second); the row sums take the rounded values
      uint8_t* pc = p_s + (size_t)bb * kUN * 256 + (size_t)(u >> 6) * kUN * 128;
#pragma unroll
      for (int q = 0; q < H; ++q) {
        const float msub = m_used[q] == -INFINITY ? 0.f : m_used[q];
        const __nv_bfloat16 pbv = __float2bfloat16_rn(ex2_sfu(sv[q] - msub));
        l_acc[q] += __bfloat162float(pbv);
        *reinterpret_cast<__nv_bfloat16*>(pc + sw128(half * H + q, (u & 63) * 2)) = pbv;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hd->p_full[bb]);
    }

    // ---- epilogue: row sums, then O / l for this split (or the final output with one split)
    if (ok && nt > 0) {
      rows_reduce(l_acc, true);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&hd->pv_done[(nt - 1) & 1], (uint32_t)((nt - 1) >> 1) & 1u, abort_flag));
      if (ok) tc_fence_after();
    }
    if (ok || nt == 0) {
      // an empty split writes only its log-sum-exp (-inf): the combine never reads its output
#pragma unroll 1
      for (int m = 0; m < (nt > 0 ? kBlocks : 0); ++m) {
        const int dim = m * 128 + quad * 32 + lane;
        uint32_t o[H];
        if (nt > 0) {
          tmem_ld_x16(tmem + lane_off + col_o + (uint32_t)(m * kUN + half * H), o);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const int q = half * H + i;
          if (q >= R) continue;
          const float val = (nt > 0 && l_acc[i] > 0.f) ? __uint_as_float(o[i]) / l_acc[i] : 0.f;
          const size_t orow = ((size_t)b * a.n_q + q / group) * a.num_q_heads + kvh * group + q % group;
          const size_t oi = ((size_t)split * rows_total + orow) * D + dim;
          if (a.out == nullptr) a.partial_o[oi] = val;
          else if (a.out_f32) static_cast<float*>(a.out)[oi] = val;
          else static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(val);
        }
      }
      if (quad == 0 && lane < H) {
        const int q = half * H + lane;
        float lq = 0.f, mq = -INFINITY;
#pragma unroll
        for (int i = 0; i < H; ++i)
          if (i == lane) { lq = l_acc[i]; mq = m_used[i]; }
        if (q < R) {
          const size_t orow = ((size_t)b * a.n_q + q / group) * a.num_q_heads + kvh * group + q % group;
          const float lse = (nt > 0 && lq > 0.f) ? (mq + log2f(lq)) * 0.6931471805599453f : -INFINITY;
          if (a.out == nullptr) {
            a.partial_lse[(size_t)split * rows_total + orow] = lse;
            const int seq_splits = hd->seq_splits;
            if (split == seq_splits - 1)  // the sequence's splits past its last are empty
              for (int sp = seq_splits; sp < a.num_splits; ++sp) a.partial_lse[(size_t)sp * rows_total + orow] = -INFINITY;
          } else if (a.out_lse != nullptr) {
            a.out_lse[orow] = lse;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
cudaError_t launch_decode_umma(const DecodeArgs& a, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const size_t smem = umma_smem_bytes<D>();
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_umma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap map;
  if (!encode_cache_map(&map, a.k_cache, D, a.capacity, a.batch * a.num_kv_heads)) return cudaErrorInvalidValue;
  static int sms_cached[64] = {0};
  if (sms_cached[dev] == 0 && cudaDeviceGetAttribute(&sms_cached[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms_cached[dev] = 0;
  dim3 grid(a.num_splits, a.num_kv_heads, a.batch);
  decode_umma_kernel<D><<<grid, kUThreads, smem, stream>>>(map, a, sms_cached[dev]);
  return cudaGetLastError();
}

bool decode_umma_applies(const DecodeArgs& a) {
  const int R = (a.num_q_heads / a.num_kv_heads) * a.n_q;
  const char* e = getenv("GEMMA_ATTN_DECODE_MMA_SYNC");
  if (e && e[0] == '1') return false;
  return a.v_cache == nullptr && !a.ring && !a.keys_rotated && (a.head_dim == 256 || a.head_dim == 512) && R > 8 &&
         R <= kUN && a.r <= 64 && (reinterpret_cast<uintptr_t>(a.k_cache) & 15u) == 0;
}

bool decode_umma_shape(const gemma_attn_params* p, int n_q) {
  const char* e = getenv("GEMMA_ATTN_DECODE_MMA_SYNC");
  if (e && e[0] == '1') return false;
  if (p->kind != GEMMA_ATTN_GLOBAL || p->num_kv_heads < 1) return false;
  const int R = (p->num_q_heads / p->num_kv_heads) * n_q;
  return (p->head_dim == 256 || p->head_dim == 512) && R > 8 && R <= kUN &&
         rotated_pairs(p->rope_p, p->head_dim) <= 64;
}

cudaError_t launch_decode_umma_any(const DecodeArgs& a, cudaStream_t stream) {
  return a.head_dim == 512 ? launch_decode_umma<512>(a, stream) : launch_decode_umma<256>(a, stream);
}

}  // namespace gattn
