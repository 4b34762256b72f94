/*
 * attn_oracle.c -- plain, slow, fp64 reference for Gemma-4-style interleaved
 * attention layers. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the bench's CPU-baseline leg may call it; the product path never does.
 * It shares no code, header or table with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *   - sliding-window ("local") vs full causal ("global") attention:
 *       "Visual guide to Gemma 4", section "Interleaving Layers" (local layers
 *       see only a fixed range of recent tokens; global layers see the whole
 *       sequence); DeepMind talk summary, section "Optimised attention"
 *       (global layers always see the whole preceding sequence).
 *   - grouped-query attention (8 query heads per KV head on global layers,
 *       2 per KV head on local layers): guide, section "GQA"; talk summary,
 *       section "Optimised attention".
 *   - K = V on global layers (one tensor serves as keys and values): guide,
 *       section "K=V technique".
 *   - p-RoPE (only the top p fraction of rotary pairs rotated, the
 *       low-frequency remainder passed through): guide, section "p-RoPE".
 *   - 2D RoPE of the vision encoder's patches (the embedding split in two
 *       parts, one encoding the horizontal position w, the other the vertical
 *       position h): guide, section "Vision encoder"; the encoder's attention
 *       over an image's patches is bidirectional (a ViT sees every patch).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   window = keys with  pos_q - W < pos_k <= pos_q  (W keys including self);
 *   global = keys with  pos_k <= pos_q;
 *   query head h uses KV head  h / (Hq / Hkv);
 *   r = floor(p * d / 2) rotated pairs, pairs (j, j + d/2), j = 0 .. r-1,
 *   theta_j = base^(-2j/d), counter-clockwise rotation by pos * theta_j,
 *   applied to q and to the key copy used for scores; values are the
 *   un-rotated tensor (for K=V this is the single stored tensor).
 *   2D RoPE: dims [0, d/2) rotated for w and dims [d/2, d) for h, each half
 *   by the 1D rule above with d/2 in place of d (pairs (j, j + d/4),
 *   theta_j = base^(-2j/(d/2))); bidirectional = every key of the sequence.
 *
 * Every computation widens the bf16 inputs exactly to double and works in
 * double; angles, cosines and sines are double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_LOCAL 0
#define ORACLE_GLOBAL 1
#define ORACLE_BIDIR 2

static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Number of rotated pairs: floor(p * d / 2). */
int oracle_rotated_pairs(double rope_p, int head_dim) {
  return (int)floor(rope_p * (double)head_dim / 2.0);
}

/* cos and sin of the rotation angle pos * base^(-2j/d) for pair j. */
static void rope_angle(double pos, int j, int d, double rope_base, double* c, double* s) {
  double theta = pow(rope_base, -2.0 * (double)j / (double)d);
  double a = pos * theta;
  *c = cos(a);
  *s = sin(a);
}

/* Rotate x (length d) given cos/sin of each rotated pair: pairs (j, j + d/2), j < r,
 * counter-clockwise. The other coordinates are copied unchanged. */
static void rope_apply(const double* x, double* y, int d, int r, const double* cs) {
  int half = d / 2;
  for (int i = 0; i < d; ++i) y[i] = x[i];
  for (int j = 0; j < r; ++j) {
    double c = cs[2 * j], s = cs[2 * j + 1];
    double x0 = x[j], x1 = x[j + half];
    y[j] = x0 * c - x1 * s;
    y[j + half] = x0 * s + x1 * c;
  }
}

/* Rotate x (length d) for position pos. */
void oracle_rope(const double* x, double* y, int d, double rope_p, double rope_base, double pos) {
  int r = oracle_rotated_pairs(rope_p, d);
  double* cs = (double*)malloc(sizeof(double) * 2 * (r > 0 ? r : 1));
  for (int j = 0; j < r; ++j) rope_angle(pos, j, d, rope_base, &cs[2 * j], &cs[2 * j + 1]);
  rope_apply(x, y, d, r, cs);
  free(cs);
}

/* 2D rotation of x (length d, d divisible by 4): the first half of the dims for the
 * horizontal position w, the second half for the vertical position h, each half by the
 * 1D rotation of a d/2-dim vector (every pair rotated). */
void oracle_rope2d(const double* x, double* y, int d, double rope_base, double pos_h, double pos_w) {
  const int half = d / 2, pairs = d / 4;
  double* cs = (double*)malloc(sizeof(double) * 2 * (pairs > 0 ? pairs : 1));
  for (int j = 0; j < pairs; ++j) rope_angle(pos_w, j, half, rope_base, &cs[2 * j], &cs[2 * j + 1]);
  rope_apply(x, y, half, pairs, cs);
  for (int j = 0; j < pairs; ++j) rope_angle(pos_h, j, half, rope_base, &cs[2 * j], &cs[2 * j + 1]);
  rope_apply(x + half, y + half, half, pairs, cs);
  free(cs);
}

static int seq_of_token(const int32_t* cu_seqlens, int num_seqs, int t) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (cu_seqlens[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

static int key_visible(int kind, int window, int32_t pos_q, int32_t pos_k) {
  if (kind == ORACLE_BIDIR) return 1;  /* every key of the sequence */
  if (pos_k > pos_q) return 0;
  if (kind == ORACLE_LOCAL && !(pos_q - window < pos_k)) return 0;
  return 1;
}

/*
 * Attention for selected query tokens.
 *   q [T, Hq, d], k [T, Hkv, d], v [T, Hkv, d] as bf16 bits; v == NULL means K=V (v = k).
 *   positions [T]; cu_seqlens [num_seqs + 1]; tokens of sequence s are
 *   cu_seqlens[s] .. cu_seqlens[s+1]-1 and never see other sequences.
 *   rows: n_rows token indices to evaluate (NULL: all T tokens, n_rows = T).
 *   key_lo/key_hi: if key_hi > key_lo, only keys whose in-sequence index lies
 *   in [key_lo, key_hi) take part (a split of the keys; empty -> lse = -inf, out = 0).
 *   out [n_rows, Hq, d] double; lse [n_rows, Hq] double (natural log; may be NULL).
 */
int oracle_attention(int kind, int window, double rope_p, double rope_base, double scale,
                     int Hq, int Hkv, int d,
                     const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const int32_t* positions, const int32_t* cu_seqlens, int num_seqs,
                     const int32_t* rows, int n_rows, int key_lo, int key_hi,
                     double* out, double* lse) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || d % 2 != 0 || num_seqs <= 0) return -1;
  const int group = Hq / Hkv;
  const uint16_t* vv = v ? v : k;
  int T = cu_seqlens[num_seqs];
  if (!rows) n_rows = T;
  const int r = oracle_rotated_pairs(rope_p, d);

  /* cos/sin of every (position, pair) that occurs, computed once: the same values
   * rope_angle would return at each use. */
  int pmin = 0, pmax = 0;
  for (int t = 0; t < T; ++t) {
    if (t == 0 || positions[t] < pmin) pmin = positions[t];
    if (t == 0 || positions[t] > pmax) pmax = positions[t];
  }
  const long long npos = (long long)pmax - pmin + 1;
  const int rr = r > 0 ? r : 1;
  double* table = (double*)malloc(sizeof(double) * 2 * (size_t)rr * (size_t)npos);
  if (!table) return -2;
#pragma omp parallel for schedule(static)
  for (long long pi = 0; pi < npos; ++pi)
    for (int j = 0; j < r; ++j)
      rope_angle((double)(pmin + pi), j, d, rope_base, &table[(pi * rr + j) * 2], &table[(pi * rr + j) * 2 + 1]);

  long long jobs = (long long)n_rows * Hq;
#pragma omp parallel
  {
    double* qv = (double*)malloc(sizeof(double) * d);
    double* qr = (double*)malloc(sizeof(double) * d);
    double* kv = (double*)malloc(sizeof(double) * d);
    double* kr = (double*)malloc(sizeof(double) * d);
    double* acc = (double*)malloc(sizeof(double) * d);
    int cap = 0;
    double* z = NULL;
#pragma omp for schedule(dynamic, 4)
    for (long long job = 0; job < jobs; ++job) {
      int ri = (int)(job / Hq), h = (int)(job % Hq);
      int t = rows ? rows[ri] : ri;
      int s = seq_of_token(cu_seqlens, num_seqs, t);
      int beg = cu_seqlens[s], end = cu_seqlens[s + 1];
      int g = h / group;
      if (end - beg > cap) { cap = end - beg; z = (double*)realloc(z, sizeof(double) * cap); }
      for (int i = 0; i < d; ++i) qv[i] = bf16_to_double(q[((size_t)t * Hq + h) * d + i]);
      rope_apply(qv, qr, d, r, &table[(size_t)(positions[t] - pmin) * rr * 2]);
      /* scores of visible keys */
      double zmax = -INFINITY;
      int any = 0;
      for (int u = beg; u < end; ++u) {
        int idx = u - beg;
        z[idx] = -INFINITY;
        if (key_hi > key_lo && (idx < key_lo || idx >= key_hi)) continue;
        if (!key_visible(kind, window, positions[t], positions[u])) continue;
        for (int i = 0; i < d; ++i) kv[i] = bf16_to_double(k[((size_t)u * Hkv + g) * d + i]);
        rope_apply(kv, kr, d, r, &table[(size_t)(positions[u] - pmin) * rr * 2]);
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qr[i] * kr[i];
        z[idx] = scale * dot;
        if (z[idx] > zmax) zmax = z[idx];
        any = 1;
      }
      double* o = out + ((size_t)ri * Hq + h) * d;
      if (!any) {
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (lse) lse[(size_t)ri * Hq + h] = -INFINITY;
        continue;
      }
      double denom = 0.0;
      for (int i = 0; i < d; ++i) acc[i] = 0.0;
      for (int u = beg; u < end; ++u) {
        double zz = z[u - beg];
        if (zz == -INFINITY) continue;
        double w = exp(zz - zmax);
        denom += w;
        const uint16_t* vrow = vv + ((size_t)u * Hkv + g) * d; /* values are never rotated */
        for (int i = 0; i < d; ++i) acc[i] += w * bf16_to_double(vrow[i]);
      }
      for (int i = 0; i < d; ++i) o[i] = acc[i] / denom;
      if (lse) lse[(size_t)ri * Hq + h] = zmax + log(denom);
    }
    free(qv); free(qr); free(kv); free(kr); free(acc); free(z);
  }
  free(table);
  return 0;
}

/*
 * Bidirectional attention with 2D RoPE (the vision encoder's patches).
 *   q [T, Hq, d], k [T, Hkv, d], v [T, Hkv, d] as bf16 bits; v == NULL means K=V.
 *   positions_hw [T, 2]: (h, w) of each token; cu_seqlens [num_seqs + 1]: each image's
 *   patches, which see every patch of their own image and nothing else.
 *   rows / n_rows, out [n_rows, Hq, d], lse [n_rows, Hq] (may be NULL) as in
 *   oracle_attention. Scores use the rotated q and k, values the un-rotated tensor.
 */
int oracle_attention_2d(double rope_base, double scale, int Hq, int Hkv, int d,
                        const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* positions_hw, const int32_t* cu_seqlens, int num_seqs,
                        const int32_t* rows, int n_rows, double* out, double* lse) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || d % 4 != 0 || num_seqs <= 0) return -1;
  const int group = Hq / Hkv;
  const uint16_t* vv = v ? v : k;
  int T = cu_seqlens[num_seqs];
  if (!rows) n_rows = T;
  long long jobs = (long long)n_rows * Hq;
#pragma omp parallel
  {
    double* qv = (double*)malloc(sizeof(double) * d);
    double* qr = (double*)malloc(sizeof(double) * d);
    double* kv = (double*)malloc(sizeof(double) * d);
    double* kr = (double*)malloc(sizeof(double) * d);
    double* acc = (double*)malloc(sizeof(double) * d);
    int cap = 0;
    double* z = NULL;
#pragma omp for schedule(dynamic, 4)
    for (long long job = 0; job < jobs; ++job) {
      int ri = (int)(job / Hq), h = (int)(job % Hq);
      int t = rows ? rows[ri] : ri;
      int s = seq_of_token(cu_seqlens, num_seqs, t);
      int beg = cu_seqlens[s], end = cu_seqlens[s + 1];
      int g = h / group;
      if (end - beg > cap) { cap = end - beg; z = (double*)realloc(z, sizeof(double) * cap); }
      for (int i = 0; i < d; ++i) qv[i] = bf16_to_double(q[((size_t)t * Hq + h) * d + i]);
      oracle_rope2d(qv, qr, d, rope_base, positions_hw[2 * t], positions_hw[2 * t + 1]);
      double zmax = -INFINITY;
      for (int u = beg; u < end; ++u) {
        for (int i = 0; i < d; ++i) kv[i] = bf16_to_double(k[((size_t)u * Hkv + g) * d + i]);
        oracle_rope2d(kv, kr, d, rope_base, positions_hw[2 * u], positions_hw[2 * u + 1]);
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qr[i] * kr[i];
        z[u - beg] = scale * dot;
        if (z[u - beg] > zmax) zmax = z[u - beg];
      }
      double* o = out + ((size_t)ri * Hq + h) * d;
      double denom = 0.0;
      for (int i = 0; i < d; ++i) acc[i] = 0.0;
      for (int u = beg; u < end; ++u) {
        double w = exp(z[u - beg] - zmax);
        denom += w;
        const uint16_t* vrow = vv + ((size_t)u * Hkv + g) * d;
        for (int i = 0; i < d; ++i) acc[i] += w * bf16_to_double(vrow[i]);
      }
      for (int i = 0; i < d; ++i) o[i] = acc[i] / denom;
      if (lse) lse[(size_t)ri * Hq + h] = zmax + log(denom);
    }
    free(qv); free(qr); free(kv); free(kr); free(acc); free(z);
  }
  return 0;
}

/*
 * Merge split results: out = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),
 * M = max_s lse_s, lse = M + log(sum_s exp(lse_s - M)).
 * partial_o [splits, rows, d], partial_lse [splits, rows]; empty splits carry -inf.
 */
int oracle_combine(const double* partial_o, const double* partial_lse, int splits, long long rows, int d,
                   double* out, double* lse) {
  if (splits <= 0 || rows < 0 || d <= 0) return -1;
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r) {
    double m = -INFINITY;
    for (int s = 0; s < splits; ++s) {
      double l = partial_lse[(size_t)s * rows + r];
      if (l > m) m = l;
    }
    double* o = out + (size_t)r * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    if (m == -INFINITY) { if (lse) lse[r] = -INFINITY; continue; }
    double den = 0.0;
    for (int s = 0; s < splits; ++s) {
      double l = partial_lse[(size_t)s * rows + r];
      if (l == -INFINITY) continue;
      double w = exp(l - m);
      den += w;
      const double* po = partial_o + ((size_t)s * rows + r) * d;
      for (int i = 0; i < d; ++i) o[i] += w * po[i];
    }
    for (int i = 0; i < d; ++i) o[i] /= den;
    if (lse) lse[r] = m + log(den);
  }
  return 0;
}

/*
 * Tile classification by brute force over every (query, key) pair of a tile.
 * Tiles are bm query rows x bn keys, aligned to the start of each sequence.
 * Emits, for every tile with at least one visible pair, the 4-tuple
 *   (sequence, q_tile, kv_tile, class) with class 1 = partial, 2 = full,
 * in order of sequence, then q_tile, then kv_tile. Fully masked tiles are skipped.
 * Returns the number of tuples; writes at most cap tuples into out.
 */
long long oracle_tile_plan(int kind, int window, const int32_t* positions, const int32_t* cu_seqlens,
                           int num_seqs, int bm, int bn, int32_t* out, long long cap) {
  long long n = 0;
  for (int s = 0; s < num_seqs; ++s) {
    int beg = cu_seqlens[s], len = cu_seqlens[s + 1] - beg;
    int nqt = (len + bm - 1) / bm, nkt = (len + bn - 1) / bn;
    for (int qt = 0; qt < nqt; ++qt) {
      for (int kt = 0; kt < nkt; ++kt) {
        long long vis = 0, tot = 0;
        for (int i = qt * bm; i < len && i < (qt + 1) * bm; ++i)
          for (int j = kt * bn; j < len && j < (kt + 1) * bn; ++j) {
            ++tot;
            vis += key_visible(kind, window, positions[beg + i], positions[beg + j]);
          }
        if (vis == 0) continue;
        if (n < cap && out) {
          out[4 * n + 0] = s;
          out[4 * n + 1] = qt;
          out[4 * n + 2] = kt;
          out[4 * n + 3] = (vis == tot) ? 2 : 1;
        }
        ++n;
      }
    }
  }
  return n;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
