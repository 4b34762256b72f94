// tile_plan.h -- which key tiles a query tile visits, and whether each needs a mask.
//
// A sliding-window layer lets a query at in-sequence offset i see keys
// i - W < j <= i; a global layer sees j <= i ("Visual guide to Gemma 4", section
// "Interleaving Layers": local layers see only a fixed range of recent tokens, which
// is what cuts their cost); the vision encoder's bidirectional layer sees every key of
// its image (section "Vision encoder"). Tiles are bm query rows by bn keys, aligned to
// each sequence's first token. Tiles with no visible pair are never visited, so a local
// layer touches O(len * W) pairs.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define GATTN_HD __host__ __device__ __forceinline__
#else
#define GATTN_HD inline
#endif

namespace gattn {

enum : int { kTilePartial = 1, kTileFull = 2 };

// Key tiles [*lo, *hi) visited by query tile qt of a sequence of `len` tokens.
// is_local != 0 selects the sliding window of `window` keys; bidir != 0 every key.
GATTN_HD void kv_tile_range(int is_local, int window, int len, int qt, int bm, int bn, int* lo, int* hi,
                            int bidir = 0) {
  if (bidir) {
    *lo = 0;
    *hi = (len + bn - 1) / bn;
    return;
  }
  int r0 = qt * bm;
  int r1 = r0 + bm - 1;
  if (r1 > len - 1) r1 = len - 1;
  *hi = r1 / bn + 1;
  if (is_local) {
    int first = r0 - window + 1;  // oldest key visible to the first row
    *lo = first > 0 ? first / bn : 0;
  } else {
    *lo = 0;
  }
}

// Class of key tile kt for query tile qt: kTileFull when every (row, key) pair inside
// the sequence is visible, else kTilePartial (callers only ask about visited tiles).
GATTN_HD int kv_tile_class(int is_local, int window, int len, int qt, int kt, int bm, int bn, int bidir = 0) {
  if (bidir) return kTileFull;  // every pair inside the sequence is visible
  int r0 = qt * bm;
  int r1 = r0 + bm - 1;
  if (r1 > len - 1) r1 = len - 1;
  int k0 = kt * bn;
  int k1 = k0 + bn - 1;
  if (k1 > len - 1) k1 = len - 1;
  bool causal_ok = k1 <= r0;                          // every key at or before every row
  bool window_ok = !is_local || (k0 > r1 - window);   // every key inside every row's window
  return (causal_ok && window_ok) ? kTileFull : kTilePartial;
}

}  // namespace gattn
