// prefill.cu -- flash-style attention for Gemma-4-style local (sliding window, causal)
// and global (causal, K=V, p-RoPE) layers, and the vision encoder's bidirectional
// layers, on sm_100a.
//
// A work unit is a 128-row query tile of one query head against the key tiles its
// rows can see (global: all earlier keys; local: the last W keys; "Visual guide to
// Gemma 4", section "Interleaving Layers"; bidirectional: every key of the sequence,
// section "Vision encoder"). Fully masked key tiles are never loaded; only tiles that
// straddle the diagonal, the window edge or a sequence end are masked.
//
// Roles (320 threads per CTA):
//   warp 0     TMA producer: the Q tile once per unit, then stages of K and V (16 KB, or
//              32 KB for the paired form at head dims >= 256) through a ring (128-byte
//              swizzle).
//   warp 1     TMEM owner and MMA issuer: S = Q K^T into one of two TMEM score buffers
//              (tcgen05.mma, both operands in shared memory), then O += P V with P read
//              from TMEM and V from the ring.
//   warps 2-9  softmax: two warps per TMEM lane quadrant, each taking one query row per
//              lane and half of the score tile's columns; online softmax in fp32 with the
//              running max only raised when it grows by more than 2^8 (the halves agree
//              on the tile maximum through shared memory), P written back to TMEM as
//              bf16 over the scores, epilogue O / l.
// The MMA order is S(j), PV(j-1), S(j+1), PV(j), ... so the tensor core works on
// S(j+1) while the softmax warps turn S(j) into P(j). The kernel is persistent: each
// CTA (pair) stays resident and walks a list of work units, so barrier setup, TMEM
// allocation and teardown happen once, and the next unit's Q load and first score tiles
// overlap the current unit's last value product and epilogue.
//
// Paired form (PAIR): the two query heads of a GQA pair share every K and V tile. Two
// CTAs on two SMs form a cluster; the even CTA issues 256-row MMAs (tcgen05 cta_group::2)
// whose rows 0-127 are its head and rows 128-255 the odd CTA's head. Each CTA loads only
// half of every K tile (64 of the 128 keys) and half of every V stage's columns, so the
// bytes each SM pulls from L2 per FLOP are halved; the loads of both CTAs complete on the
// even CTA's barriers, and the paired MMA commits signal both CTAs.
//
// Global layers: the single K=V tensor feeds both operands. Key chunks that hold rotated
// dimensions come from a rotated side copy (workspace); every other key chunk and every
// value chunk are read from the un-rotated tensor ("Visual guide to Gemma 4", sections
// "K=V technique" and "p-RoPE"). With head_dim 512 the 128 x 512 fp32 output tile would
// fill all of TMEM, so two work units each own one 256-column half of the output and both
// compute the full score tile.
#include "common.cuh"
#include "kernels.h"
#include "tile_plan.h"

namespace gattn {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kChunk = 64;                   // dims per TMA box / swizzle row
constexpr int kChunkBytes = 16384;           // 128 rows x 64 dims of bf16: a Q chunk or a V chunk
constexpr int kMaxStages = 16;
constexpr int kBarrierBytes = 2048;           // mbarriers, TMEM base, softmax exchange
constexpr int kThreads = 320;           // producer, MMA issuer, 8 softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

template <int D, bool PAIR>
struct PrefillCfg {
  static constexpr int kDv = D > 256 ? 256 : D;             // output columns per work unit
  static constexpr int kSplit = D / kDv;                      // work units per (tile, head)
  static constexpr int kQChunks = D / kChunk;
  static constexpr int kVChunks = kDv / kChunk;
  static constexpr int kQBytes = kQChunks * kChunkBytes;
  // Ring stages. Single CTA: 16 KB, a K stage is one 64-dim chunk of 128 keys and a V
  // stage one 64-column chunk. Pair with d >= 256: 32 KB, a K stage is four 64-dim chunks
  // of this CTA's 64 keys and a V stage two 64-column chunks of 128 keys (the pair's CTAs
  // hold adjacent column pairs, so one PV MMA is N = 256). Pair with d = 128: 16 KB, two
  // K chunks or one V chunk. Fewer, larger stages mean fewer barrier round trips per tile.
  static constexpr int kStageBytes = (PAIR && D >= 256) ? 2 * kChunkBytes : kChunkBytes;
  static constexpr int kKChunkBytes = PAIR ? kChunkBytes / 2 : kChunkBytes;
  static constexpr int kKPerStage = kStageBytes / kKChunkBytes;
  static constexpr int kVPerStage = kStageBytes / kChunkBytes;
  static constexpr int kKStages = kQChunks / kKPerStage;
  static constexpr int kVStages = (PAIR ? kVChunks / 2 : kVChunks) / kVPerStage;
  static constexpr int kPvN = (PAIR ? 2 : 1) * kVPerStage * kChunk;  // output columns per V stage
  static constexpr int kRingBudget = 232448 - 1024 /*align*/ - kBarrierBytes - kQBytes;
  static constexpr int kStages = kRingBudget / kStageBytes < kMaxStages ? kRingBudget / kStageBytes : kMaxStages;
  static constexpr int kSmemData = kQBytes + kStages * kStageBytes;
  static constexpr int kSmemBytes = kSmemData + 1024 /*align*/ + kBarrierBytes;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(!PAIR || D >= 128, "paired form needs at least two 64-dim chunks");
  static_assert(kKStages >= 1 && kVStages >= 1 && kStages >= 2, "ring shape");
  static_assert(kPvN <= 256, "PV MMA width");
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];  // by tile parity: PV(t) completes phase t >> 1 of pv_done[t & 1]
  uint64_t q_empty;  // per unit: its last score MMA finished, Q may be replaced
  uint64_t o_ready;  // per unit: its last value MMA finished
  uint64_t o_empty;  // per unit: the softmax warps have read O out
  uint64_t mma_done;
  uint64_t ring_full[kMaxStages];
  uint64_t ring_empty[kMaxStages];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t xfull[4];   // per TMEM lane quadrant: both halves wrote their exchange values
  uint64_t xfree[4];   // per quadrant: both halves read them (the slots may be rewritten)
  float xch[2 * 128];  // softmax half-row exchange: [half][row] tile maxima, then row sums
};
static_assert(sizeof(Barriers) <= kBarrierBytes, "barrier block");

// 2^x on the SFU (ex2.approx, flush-to-zero): P is rounded to bf16 and the row sums
// carry far more error than the approximation's few ulp.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Waits that may be satisfied by the other CTA of a pair use cluster-scope acquire.
template <bool PAIR>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if constexpr (PAIR) return mbar_wait_cluster(bar, parity, abort);
  else return mbar_wait(bar, parity, abort);
}

}  // namespace

// Persistent form: the grid holds as many CTAs (or CTA pairs) as can be resident, and
// each walks a fixed list of work units. Unit u (0 .. U-1, heaviest query tiles first)
// goes to cluster u mod C in forward order on even rounds and reverse order on odd
// rounds (C = number of clusters), which balances the causal tile counts. Every role
// of a CTA walks the same list; barrier phases continue across units:
//   ring stages          continuous (st, ph) in the producer and the MMA issuer
//   s_full / p_full /    tile counter g over all tiles this CTA has processed; each is
//   pv_done              a pair of barriers indexed by tile parity, so that a waiter's
//                        phase is never two behind (after a unit's last PV the next
//                        unit's first S waits for the PV before it)
//   q_full / q_empty /   one phase per unit: Q landed / the unit's last score MMA
//   o_ready / o_empty    finished (Q may be replaced) / the unit's last value MMA
//                        finished / the softmax warps have read O out (the next
//                        unit's first value MMA may overwrite it)
// The next unit's Q load and its first two score tiles overlap the current unit's
// last value product and epilogue.
template <int D, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap qs_map,
               const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap ks_map,
               const __grid_constant__ CUtensorMap v_map, const __grid_constant__ CUtensorMap k64_map,
               const __grid_constant__ CUtensorMap ks64_map, PrefillArgs args) {
  using Cfg = PrefillCfg<D, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* ring = smem + Cfg::kQBytes;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + Cfg::kSmemData);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int is_local = args.is_local;

  // ---- the unit schedule ----
  const int units_x = (PAIR ? args.num_q_heads / 2 : args.num_q_heads) * Cfg::kSplit;
  const int num_units = units_x * args.num_seqs * args.max_qtiles;
  const int nclusters = (int)gridDim.x / (PAIR ? 2 : 1);
  const int cid = (int)blockIdx.x / (PAIR ? 2 : 1);
  struct Unit {
    int head, vpart, qt, tok0, len, row0, kvh, kt_lo, ntiles;
  };
  // Unit of round r for this cluster; false when the round has none or the unit is empty
  // (a query tile past its sequence's end).
  auto unit_of_round = [&](int r, Unit& w) -> bool {
    const int u = r * nclusters + ((r & 1) ? nclusters - 1 - cid : cid);
    if (u >= num_units) return false;
    const int slot = u / units_x, ux = u % units_x;
    const int seq = slot % args.num_seqs;
    w.qt = args.max_qtiles - 1 - slot / args.num_seqs;
    w.vpart = ux % Cfg::kSplit;
    w.head = PAIR ? (ux / Cfg::kSplit) * 2 + (int)rank : ux / Cfg::kSplit;
    w.tok0 = args.cu_seqlens[seq];
    w.len = args.cu_seqlens[seq + 1] - w.tok0;
    if (w.qt * kBM >= w.len) return false;
    w.row0 = w.qt * kBM;
    w.kvh = w.head / args.group;
    int hi;
    kv_tile_range(is_local, args.window, w.len, w.qt, kBM, kBN, &w.kt_lo, &hi, args.bidir);
    w.ntiles = hi - w.kt_lo;
    return true;
  };
  const int nrounds = (num_units + nclusters - 1) / nclusters;

  if (threadIdx.x == 0) {
    // sequence-length check, once per sequence, by the CTA that owns round 0 of cluster 0
    if (cid == 0 && leader)
      for (int sq = 0; sq < args.num_seqs; ++sq) {
        const int n = args.cu_seqlens[sq + 1] - args.cu_seqlens[sq];
        if (n > args.max_seqlen || n < 1) atomicOr(&g_status, kStatusSeqlen);
      }
    const uint32_t load_arrivals = PAIR ? 2u : 1u;  // pair: both producers register their bytes
    mbar_init(&bars->q_full, load_arrivals);
    mbar_init(&bars->q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], PAIR ? 16 : 8);  // one arrival per softmax warp (of both CTAs)
    }
    mbar_init(&bars->pv_done[0], 1);
    mbar_init(&bars->pv_done[1], 1);
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->o_empty, PAIR ? 16 : 8);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bars->xfull[q], 2);
      mbar_init(&bars->xfree[q], 2);
    }
    mbar_init(&bars->mma_done, 1);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&bars->ring_full[s], load_arrivals);
      mbar_init(&bars->ring_empty[s], 1);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(&bars->tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&bars->tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {  // the peer's barriers are initialised before any remote arrival
    __syncwarp();
    cluster_sync_all();
  }
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&q_map); prefetch_tensormap(&v_map);
      if (PAIR) prefetch_tensormap(&k64_map); else prefetch_tensormap(&k_map);
      if (args.rot_mask) { prefetch_tensormap(&qs_map); prefetch_tensormap(PAIR ? &ks64_map : &ks_map); }
      // Register `bytes` on the load barrier that counts them: this CTA's own barrier, or
      // in the paired form the even CTA's (the odd CTA arrives remotely).
      auto expect = [&](uint64_t* bar, uint32_t bytes) {
        if (!PAIR || leader) mbar_arrive_expect_tx(bar, bytes);
        else mbar_arrive_expect_tx_cluster(smem_u32(bar) & kPeerBitMask, bytes);
      };
      auto load = [&](void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
        if constexpr (PAIR) tma_load_3d_pair(dst, map, bar, c0, c1, c2);
        else tma_load_3d(dst, map, bar, c0, c1, c2);
      };
      auto rot_idx = [&](int c) { return __popc(args.rot_mask & ((1u << c) - 1)); };

      int st = 0; uint32_t ph = 0;
      auto next = [&]() { if (++st == Cfg::kStages) { st = 0; ph ^= 1u; } };
      bool ok = true;
      int unit_iter = 0, q_issued = 0;
      for (int r = 0; r < nrounds && ok; ++r) {
        Unit w;
        if (!unit_of_round(r, w)) continue;
        // Q of this unit replaces the previous unit's once its last score MMA finished
        if (unit_iter > 0) {
          ok = mbar_wait(&bars->q_empty, (uint32_t)(unit_iter - 1) & 1u, abort_flag);
          if (!ok) break;
        }
        expect(&bars->q_full, Cfg::kQBytes);
        for (int c = 0; c < Cfg::kQChunks; ++c) {
          if ((args.rot_mask >> c) & 1)
            load(q_smem + c * kChunkBytes, &qs_map, &bars->q_full, rot_idx(c) * kChunk, w.head, w.tok0 + w.row0);
          else
            load(q_smem + c * kChunkBytes, &q_map, &bars->q_full, c * kChunk, w.head, w.tok0 + w.row0);
        }
        ++q_issued;
        for (int jj = 0; jj <= w.ntiles && ok; ++jj) {
          if (jj < w.ntiles) {  // K stages of tile jj
            const int key0 = w.tok0 + (w.kt_lo + jj) * kBN;
            for (int s = 0; s < Cfg::kKStages && ok; ++s) {
              ok = mbar_wait(&bars->ring_empty[st], ph ^ 1u, abort_flag);
              if (!ok) break;
              expect(&bars->ring_full[st], Cfg::kStageBytes);
              uint8_t* dst = ring + st * Cfg::kStageBytes;
              if constexpr (PAIR) {
                // chunks kKPerStage * s + sub of this CTA's 64 keys
                for (int sub = 0; sub < Cfg::kKPerStage; ++sub) {
                  const int c = Cfg::kKPerStage * s + sub;
                  if ((args.rot_mask >> c) & 1)
                    load(dst + sub * Cfg::kKChunkBytes, &ks64_map, &bars->ring_full[st], rot_idx(c) * kChunk, w.kvh,
                         key0 + 64 * (int)rank);
                  else
                    load(dst + sub * Cfg::kKChunkBytes, &k64_map, &bars->ring_full[st], c * kChunk, w.kvh,
                         key0 + 64 * (int)rank);
                }
              } else {
                const int c = s;
                if ((args.rot_mask >> c) & 1) load(dst, &ks_map, &bars->ring_full[st], rot_idx(c) * kChunk, w.kvh, key0);
                else load(dst, &k_map, &bars->ring_full[st], c * kChunk, w.kvh, key0);
              }
              next();
            }
          }
          if (jj >= 1) {  // V stages of tile jj-1 (this unit's output columns)
            const int key0 = w.tok0 + (w.kt_lo + jj - 1) * kBN;
            for (int s = 0; s < Cfg::kVStages && ok; ++s) {
              ok = mbar_wait(&bars->ring_empty[st], ph ^ 1u, abort_flag);
              if (!ok) break;
              expect(&bars->ring_full[st], Cfg::kStageBytes);
              // this CTA's column chunks of V stage s: the pair's two CTAs hold adjacent groups
              for (int sub = 0; sub < Cfg::kVPerStage; ++sub) {
                const int c = ((PAIR ? 2 * s + (int)rank : s) * Cfg::kVPerStage) + sub;
                load(ring + st * Cfg::kStageBytes + sub * kChunkBytes, &v_map, &bars->ring_full[st],
                     w.vpart * Cfg::kDv + c * kChunk, w.kvh, key0);
              }
              next();
            }
          }
        }
        ++unit_iter;
      }
      // Let the copies counted on this CTA's barriers land before the CTA can exit: the
      // last kStages ring loads and the last Q load are the only ones that may still be
      // in flight. (st, ph) is the next slot to fill; each slot's most recent fill
      // completed the phase of parity ph ^ 1 (the wrap inside next() flips ph for the
      // slots filled this round). In the paired form the odd CTA's copies complete on the
      // even CTA's barriers, whose MMA consumes every one of them before the final
      // cluster barrier.
      if (!PAIR || leader) {
        for (int s = 0; s < Cfg::kStages; ++s) {
          if (!mbar_try_wait(&bars->ring_full[st], ph ^ 1u)) {
            unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars->ring_full[st], ph ^ 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {}
          }
          next();
          (void)s;
        }
        if (q_issued > 0 && !mbar_try_wait(&bars->q_full, (uint32_t)(q_issued - 1) & 1u)) {
          unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&bars->q_full, (uint32_t)(q_issued - 1) & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      constexpr int M = PAIR ? 2 * kBM : kBM;
      constexpr int PV_N = Cfg::kPvN;
      const uint32_t idesc_qk = umma_idesc_bf16(M, kBN, 0, 0);
      const uint32_t idesc_pv = umma_idesc_bf16(M, PV_N, 0, 1);
      // descriptors of stage 0 / Q chunk 0; other stages and k-steps are offsets of
      // (bytes >> 4) in the low start-address field
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(q_smem), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(ring), 16, 1024);
      // V is MN-major: 64-column chunks of a stage are kChunkBytes apart (leading offset)
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(ring), kChunkBytes, 1024);
      auto commit_both = [&](uint64_t* bar) {
        if constexpr (PAIR) umma_commit_pair_both(bar);
        else umma_commit(bar);
      };
      int st = 0; uint32_t ph = 0;
      auto next = [&]() { if (++st == Cfg::kStages) { st = 0; ph ^= 1u; } };
      bool ok = true;
      int g = 0;  // tiles of earlier units
      int unit_iter = 0;
      for (int r = 0; r < nrounds && ok; ++r) {
        Unit w;
        if (!unit_of_round(r, w)) continue;
        ok = wait_bar<PAIR>(&bars->q_full, (uint32_t)unit_iter & 1u, abort_flag);
        for (int jj = 0; jj <= w.ntiles && ok; ++jj) {
          if (jj < w.ntiles) {
            const int t = g + jj;
            const int b = t & 1;
            const uint32_t s_col = b ? kColS1 : kColS0;
            // S(t) overwrites the buffer whose P fed PV(t-2)
            if (t >= 2) ok = wait_bar<PAIR>(&bars->pv_done[t & 1], (uint32_t)((t - 2) >> 1) & 1u, abort_flag);
            tc_fence_after();
            for (int s = 0; s < Cfg::kKStages && ok; ++s) {
              ok = wait_bar<PAIR>(&bars->ring_full[st], ph, abort_flag);
              if (!ok) break;
              tc_fence_after();
              const uint64_t kd = k_desc0 + (uint64_t)((st * Cfg::kStageBytes) >> 4);
#pragma unroll
              for (int sub = 0; sub < Cfg::kKPerStage; ++sub) {
                const int c = Cfg::kKPerStage * s + sub;
                const uint64_t qd = q_desc0 + (uint64_t)((c * kChunkBytes) >> 4);
                const uint64_t kds = kd + (uint64_t)((sub * Cfg::kKChunkBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk) {
                  if constexpr (PAIR) umma_ss_pair(tmem + s_col, qd + 2 * kk, kds + 2 * kk, idesc_qk, (c | kk) != 0);
                  else umma_ss(tmem + s_col, qd + 2 * kk, kds + 2 * kk, idesc_qk, (c | kk) != 0);
                }
              }
              commit_both(&bars->ring_empty[st]);
              next();
            }
            if (!ok) break;
            commit_both(&bars->s_full[b]);
            if (jj == w.ntiles - 1) commit_both(&bars->q_empty);  // the unit's last read of Q
          }
          if (jj >= 1) {
            const int pt = g + jj - 1;
            const int pb = pt & 1;
            const uint32_t p_col = pb ? kColS1 : kColS0;
            ok = wait_bar<PAIR>(&bars->p_full[pb], (uint32_t)(pt >> 1) & 1u, abort_flag);
            if (!ok) break;
            // the unit's first value MMA overwrites O: the previous unit's epilogue has read it
            if (jj == 1 && unit_iter > 0) {
              ok = wait_bar<PAIR>(&bars->o_empty, (uint32_t)(unit_iter - 1) & 1u, abort_flag);
              if (!ok) break;
            }
            tc_fence_after();
            for (int s = 0; s < Cfg::kVStages && ok; ++s) {
              ok = wait_bar<PAIR>(&bars->ring_full[st], ph, abort_flag);
              if (!ok) break;
              tc_fence_after();
              const uint64_t vd = v_desc0 + (uint64_t)((st * Cfg::kStageBytes) >> 4);
              const uint32_t o_col = kColO + s * PV_N;
#pragma unroll
              for (int kk = 0; kk < kBN / 16; ++kk) {
                const bool acc = (jj - 1) != 0 || kk != 0;
                if constexpr (PAIR) umma_ts_pair(tmem + o_col, tmem + p_col + kk * 8, vd + 128 * kk, idesc_pv, acc);
                else umma_ts(tmem + o_col, tmem + p_col + kk * 8, vd + 128 * kk, idesc_pv, acc);
              }
              commit_both(&bars->ring_empty[st]);
              next();
            }
            if (!ok) break;
            commit_both(&bars->pv_done[pt & 1]);
          }
        }
        if (!ok) break;
        // O of the unit is final once every value MMA issued so far has finished
        commit_both(&bars->o_ready);
        g += w.ntiles;
        ++unit_iter;
      }
      // All MMAs issued by this thread are complete once mma_done fires.
      if constexpr (PAIR) umma_commit_pair_local(&bars->mma_done);
      else umma_commit(&bars->mma_done);
      unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&bars->mma_done, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Eight warps: warps w and w + 4 share the TMEM lane quadrant w % 4 (rows quad*32 ..
    // +31, one row per lane) and split each score tile's 128 columns, half h taking
    // columns 64h .. 64h + 63 (and O columns h*kDv/2 ..). The two halves of a row agree on
    // the tile maximum through a shared-memory slot per row and half, handed over with two
    // bounded mbarriers per quadrant (written / read); row sums are combined once, at the
    // epilogue. Both halves run the same exchanges in the same order, so the exchange
    // count x gives both barriers' phase.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float scale_log2 = args.softmax_scale * 1.4426950408889634f;
    constexpr int kHC = kBN / 2;               // score columns per half
    constexpr int kHO = Cfg::kDv / 2;          // output columns per half
    float* xch = bars->xch;                    // [2 halves][128 rows]
    uint32_t xk = 0;                           // exchanges so far (both halves alike)
    // Publish v for this row and return the partner half's value (ok = false on abort).
    auto exchange = [&](float v, bool& okx) -> float {
      xch[half * kBM + row] = v;
      tc_fence_before();  // this half's score loads are ordered before the arrival
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xfull[quad]);
      okx = __all_sync(0xffffffffu, mbar_wait(&bars->xfull[quad], xk & 1u, abort_flag));
      tc_fence_after();
      const float other = okx ? xch[(1 - half) * kBM + row] : v;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xfree[quad]);
      if (okx) okx = __all_sync(0xffffffffu, mbar_wait(&bars->xfree[quad], xk & 1u, abort_flag));
      ++xk;
      return other;
    };
    bool ok = true;
    int g = 0;
    int unit_iter = 0;
    for (int r = 0; r < nrounds && ok; ++r) {
      Unit w;
      if (!unit_of_round(r, w)) continue;
      float m_used = -INFINITY;
      float l_part = 0.f;
      const int grow = w.row0 + row;  // in-sequence offset of this thread's query row
      for (int jj = 0; jj < w.ntiles && ok; ++jj) {
        const int t = g + jj;
        const int b = t & 1;
        const uint32_t s_col = (b ? kColS1 : kColS0) + half * kHC;
        ok = __all_sync(0xffffffffu, wait_bar<PAIR>(&bars->s_full[b], (uint32_t)(t >> 1) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        float sv[kHC];
        uint32_t* tr = reinterpret_cast<uint32_t*>(sv);
#pragma unroll
        for (int c = 0; c < kHC / 32; ++c) tmem_ld_x32(tmem + lane_off + s_col + c * 32, tr + c * 32);
        tmem_ld_wait();
        const int kt = w.kt_lo + jj;
        // A key tile that runs past the end of the sequence holds the next sequence's
        // tokens (or padding) and is masked even when its in-sequence pairs are all visible.
        const bool partial = (kt + 1) * kBN > w.len ||
                             kv_tile_class(is_local, args.window, w.len, w.qt, kt, kBM, kBN, args.bidir) != kTileFull;
        // Scores stay unscaled: the scale is folded into the exponent's FFMA (scale > 0, so
        // the max commutes with it). In a masked tile the keys a row sees are one run of
        // the half's columns, [c_lo, c_hi] (causal: key <= row; local: key > row - window;
        // past the row's sequence end nothing, since row < len; bidirectional: every key
        // before the sequence end); the rest become -inf.
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
        if (partial) {
          const int k0 = kt * kBN + half * kHC;
          const int c_hi = (args.bidir ? w.len - 1 : grow) - k0;
          const int c_lo = is_local ? grow - args.window + 1 - k0 : 0;
#pragma unroll
          for (int c = 0; c < kHC; ++c) {
            sv[c] = (c >= c_lo && c <= c_hi) ? sv[c] : -INFINITY;
            mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kHC; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
        }
        const float coef = scale_log2;
        const float m_half = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
        // the row's tile maximum: both halves take the max of the same two values (this
        // also orders both halves' score loads before either writes its P below)
        const float m_tile = fmaxf(m_half, exchange(m_half, ok));
        if (!ok) break;
        // Raise the running max only when it grows by more than 2^8 (or was empty); P
        // may then exceed 1 by up to 2^8, which fp32 sums and bf16 P absorb.
        float alpha = 1.f;
        bool rescale_o = false;
        if (m_tile > m_used + kRescaleThreshold || (m_used == -INFINITY && m_tile > -INFINITY)) {
          if (m_used != -INFINITY) {
            alpha = fast_exp2(m_used - m_tile);
            l_part *= alpha;
            rescale_o = true;
          }
          m_used = m_tile;
        }
        // P(t) goes over S(t) right away: that buffer's previous P (tile t-2) was consumed
        // by PV(t-2), which finished before S(t) was computed.
        const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
        uint32_t p[kHC / 2];
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kHC / 2; ++c) {
          const float p0 = fast_exp2(fmaf(sv[2 * c], coef, -m_sub));
          const float p1 = fast_exp2(fmaf(sv[2 * c + 1], coef, -m_sub));
          rs4[c & 3] += p0 + p1;
          p[c] = pack_bf16x2(p0, p1);
        }
        l_part += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
        // this half's P: TMEM columns (tile base) + 32 half .. + 31 (two bf16 per column)
        tmem_st_x32(tmem + lane_off + (b ? kColS1 : kColS0) + half * (kHC / 2), p);
        // tcgen05.ld/st are warp-collective: the warp rescales its half of the O rows together
        // when any lane needs it, each lane with its own factor (1 for lanes that do not). O
        // may only be touched once PV(t-1) has finished; without a rescale the warp does not
        // wait, since PV(t) is issued after PV(t-1) and the tensor core runs them in order.
        // The parity wait is exact: PV(t-3) finished before S(t-1) was issued, and PV(t+1)
        // needs this warp's p_full(t+1) arrival, so PV(t-1) is the only phase of its barrier
        // that can still be pending. A unit's first tile never rescales (m_used starts empty).
        const bool rescale_warp = __any_sync(0xffffffffu, rescale_o);
        if (rescale_warp && jj >= 1) {
          ok = __all_sync(0xffffffffu, wait_bar<PAIR>(&bars->pv_done[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u, abort_flag));
          if (!ok) {
            tmem_st_wait();  // the P stores land before the teardown frees TMEM
            break;
          }
          tc_fence_after();
        }
        if (rescale_warp) {
#pragma unroll 1
          for (int c = 0; c < kHO / 32; ++c) {
            uint32_t o[32];
            tmem_ld_x32(tmem + lane_off + kColO + half * kHO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_x32(tmem + lane_off + kColO + half * kHO + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();  // every lane's P and O stores precede the warp's single arrival
        if (lane == 0) {
          if (!PAIR || leader) mbar_arrive(&bars->p_full[b]);
          else mbar_arrive_cluster(smem_u32(&bars->p_full[b]) & kPeerBitMask);
        }
      }
      if (!ok) break;
      // the row sum: this half's part plus the partner half's
      const float l_sum = l_part + exchange(l_part, ok);
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar<PAIR>(&bars->o_ready, (uint32_t)unit_iter & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const bool valid = grow < w.len;
      const int tok = w.tok0 + grow;
      const size_t obase = ((size_t)tok * args.num_q_heads + w.head) * args.head_dim + w.vpart * Cfg::kDv;
      // O leaves TMEM two 32-column chunks per wait; once the last chunks are in
      // registers the warp signals o_empty, before its stores.
      constexpr int kOC = kHO / 32;               // 32-column chunks of this half
      constexpr int kOG = kOC >= 2 ? 2 : 1;       // chunks per TMEM wait
#pragma unroll 1
      for (int cg = 0; cg < kOC; cg += kOG) {
        uint32_t ohg[kOG][32];
#pragma unroll
        for (int k = 0; k < kOG; ++k) tmem_ld_x32(tmem + lane_off + kColO + half * kHO + (cg + k) * 32, ohg[k]);
        tmem_ld_wait();
        if (cg + kOG >= kOC) {
          // O has been read out: the next unit's first value MMA may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (!PAIR || leader) mbar_arrive(&bars->o_empty);
            else mbar_arrive_cluster(smem_u32(&bars->o_empty) & kPeerBitMask);
          }
        }
#pragma unroll
      for (int k = 0; k < kOG; ++k) {
        const uint32_t* oh = ohg[k];
        const int col = half * kHO + (cg + k) * 32;
        if (valid && w.vpart * Cfg::kDv + col < args.head_dim) {
          // a row segment of 32 columns: 128 bytes (f32) or 64 bytes (bf16), written with
          // 32-byte stores where the output is 32-byte aligned (half the store
          // instructions of 16-byte ones), else 16-byte stores
          uint32_t wd[32];
          int nw;
          if (args.out_f32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) wd[i] = __float_as_uint(__uint_as_float(oh[i]) * inv_l);
            nw = 32;
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              wd[i] = pack_bf16x2(__uint_as_float(oh[2 * i]) * inv_l, __uint_as_float(oh[2 * i + 1]) * inv_l);
            nw = 16;
          }
          uint8_t* dst = reinterpret_cast<uint8_t*>(args.out) + (obase + col) * (args.out_f32 ? 4 : 2);
          if (args.out_align32) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (8 * i < nw)
                st_global_32B(dst + 32 * i, make_uint4(wd[8 * i], wd[8 * i + 1], wd[8 * i + 2], wd[8 * i + 3]),
                              make_uint4(wd[8 * i + 4], wd[8 * i + 5], wd[8 * i + 6], wd[8 * i + 7]));
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (4 * i < nw)
                *reinterpret_cast<uint4*>(dst + 16 * i) = make_uint4(wd[4 * i], wd[4 * i + 1], wd[4 * i + 2], wd[4 * i + 3]);
          }
        }
      }
      }
      if (half == 0 && valid && w.vpart == 0 && args.lse != nullptr)
        args.lse[(size_t)w.head * args.total_tokens + tok] = (m_used + log2f(l_sum)) * 0.6931471805599453f;
      g += w.ntiles;
      ++unit_iter;
    }
  }

  tc_fence_before();
  __syncthreads();
  // A pair leaves together: no remote arrival or copy may target a CTA that has exited.
  if constexpr (PAIR) {
    __syncwarp();
    cluster_sync_all();
  }
  if (warp == 1) {
    // tcgen05.dealloc is warp-collective: lane 0 ran the MMA loop alone, so the warp
    // reconverges explicitly before the whole warp frees the columns.
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool PAIR>
constexpr int Cfg_smem() { return PrefillCfg<D, PAIR>::kSmemBytes; }

// Clusters (pairs) or CTAs of prefill_kernel<D, PAIR> that fit on the device at once,
// computed once per device.
template <int D, bool PAIR>
static int resident_clusters(const cudaLaunchConfig_t& cfg) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  int n = 0;
  if constexpr (PAIR) {
    cudaLaunchConfig_t c = cfg;
    c.gridDim = dim3(2, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&n, prefill_kernel<D, PAIR>, &c) != cudaSuccess) n = 0;
  } else {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_kernel<D, PAIR>, kThreads,
                                                      Cfg_smem<D, PAIR>()) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      n = per_sm * sms;
  }
  cached[dev] = n;
  return n;
}

template <int D, bool PAIR>
cudaError_t launch_prefill_t(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream) {
  using Cfg = PrefillCfg<D, PAIR>;
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  // Persistent grid: as many CTAs (pairs) as can be resident at once, at most one per unit.
  const long long units = (long long)(PAIR ? args.num_q_heads / 2 : args.num_q_heads) * Cfg::kSplit *
                          args.num_seqs * args.max_qtiles;
  if (units == 0) return cudaSuccess;
  const int resident = resident_clusters<D, PAIR>(cfg);
  if (resident < 1) return cudaErrorInvalidConfiguration;
  const long long clusters = units < resident ? units : resident;
  cfg.gridDim = dim3((unsigned)(clusters * (PAIR ? 2 : 1)), 1, 1);
  return cudaLaunchKernelEx(&cfg, prefill_kernel<D, PAIR>, maps.q, maps.qs, maps.k, maps.ks, maps.v, maps.k64,
                            maps.ks64, args);
}

// The paired form runs when a pair of query heads shares a KV head (even GQA group)
// and the head dim has at least two 64-dim chunks.
template <int D>
cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream) {
  if constexpr (D >= 128) {
    if (args.group % 2 == 0 && args.pair_allowed) return launch_prefill_t<D, true>(maps, args, stream);
  }
  return launch_prefill_t<D, false>(maps, args, stream);
}

template cudaError_t launch_prefill<64>(const PrefillMaps&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill<128>(const PrefillMaps&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill<256>(const PrefillMaps&, const PrefillArgs&, cudaStream_t);
template cudaError_t launch_prefill<512>(const PrefillMaps&, const PrefillArgs&, cudaStream_t);

}  // namespace gattn
