// api.cu -- the extern "C" entry points declared in include/gemma_attn.h: argument
// validation, workspace carving, tensor-map encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "../../include/gemma_attn.h"
#include "common.cuh"
#include "kernels.h"
#include "tile_plan.h"

namespace gattn {

cudaError_t launch_umma_selftest(const CUtensorMap& a, const CUtensorMap& b, const uint16_t* p, float* d,
                                 int mode, cudaStream_t stream);

namespace {

thread_local int t_launches = 0;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 map over [tokens][heads][inner] with a {64, 1, rows} box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int inner, int heads, int tokens, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)heads, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * heads * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The two-CTA paired prefill kernel is the default; GEMMA_ATTN_NO_PAIR=1 in the
// environment selects the single-CTA kernel (used by the tests to cover both forms).
bool pair_kernel_enabled() {
  const char* e = getenv("GEMMA_ATTN_NO_PAIR");
  return !(e && e[0] == '1');
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_params(const gemma_attn_params* p) {
  if (!p) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (p->kind != GEMMA_ATTN_LOCAL && p->kind != GEMMA_ATTN_GLOBAL && p->kind != GEMMA_ATTN_BIDIR)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads != 0)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  const int d = p->head_dim;
  if (d != 32 && d != 64 && d != 128 && d != 256 && d != 512) return GEMMA_ATTN_ERR_UNSUPPORTED;
  // the 2D rotation turns every pair of both halves: p = 1, whole 64-dim chunks
  if (p->kind == GEMMA_ATTN_BIDIR && p->rope_p != 1.f) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (p->kind == GEMMA_ATTN_BIDIR && d < 64) return GEMMA_ATTN_ERR_UNSUPPORTED;
  if (p->kind == GEMMA_ATTN_LOCAL && p->window < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (!(p->rope_p >= 0.f && p->rope_p <= 1.f)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (!(p->rope_base > 0.f) || !(p->softmax_scale > 0.f)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (p->out_dtype != GEMMA_ATTN_OUT_BF16 && p->out_dtype != GEMMA_ATTN_OUT_F32) return GEMMA_ATTN_ERR_INVALID_ARG;
  return GEMMA_ATTN_OK;
}

// Chunks (64 dims) of the kernel head dim that come from the rotated side copy.
uint32_t rotated_chunk_mask(int d, int r) {
  if (d < 64) return 1u;  // padded operand: the whole (single) chunk comes from the copy
  uint32_t mask = 0;
  const int half = d / 2;
  for (int c = 0; c < d / 64; ++c) {
    const int lo = c * 64, hi = lo + 64;
    const bool first_half = lo < r;
    const bool second_half = lo < half + r && hi > half;
    if (r > 0 && (first_half || second_half)) mask |= 1u << c;
  }
  return mask;
}

struct PrefillLayout {
  int kd;           // kernel head dim (>= 64)
  int r;
  uint32_t mask;
  int n_out;        // columns in each side copy
  size_t q_off, k_off, v_off, total;
};

PrefillLayout prefill_layout(const gemma_attn_params* p, int64_t T) {
  PrefillLayout L;
  L.kd = p->head_dim < 64 ? 64 : p->head_dim;
  L.r = rotated_pairs(p->rope_p, p->head_dim);
  L.mask = rotated_chunk_mask(p->head_dim, L.r);
  L.n_out = __builtin_popcount(L.mask) * 64;
  const size_t qb = (size_t)T * p->num_q_heads * L.n_out * 2;
  const size_t kb = (size_t)T * p->num_kv_heads * L.n_out * 2;
  const size_t vb = p->head_dim < 64 ? (size_t)T * p->num_kv_heads * 64 * 2 : 0;
  L.q_off = 0;
  L.k_off = round_up(qb, 256);
  L.v_off = L.k_off + round_up(kb, 256);
  L.total = L.v_off + round_up(vb, 256);
  return L;
}

}  // namespace

void set_launch_count(int n) { t_launches = n; }

bool encode_cache_map(CUtensorMap* m, const void* base, int d, int capacity, int planes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)capacity, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * capacity * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int decode_prepare(const gemma_attn_params* params, const void* q, const void* new_k, const void* new_v,
                   const void* k_cache, const void* v_cache, int32_t cache_layout, int32_t cache_capacity,
                   const int32_t* cache_seqlens, int32_t batch, int32_t n_q, int32_t max_cache_len,
                   int32_t num_splits, DecodeArgs* a) {
  int rc = check_params(params);
  if (rc != GEMMA_ATTN_OK) return rc;
  if (params->kind == GEMMA_ATTN_BIDIR) return GEMMA_ATTN_ERR_UNSUPPORTED;  // prefill only
  const bool global = params->kind == GEMMA_ATTN_GLOBAL;
  if (!q || !new_k || !k_cache || !cache_seqlens) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (global != (new_v == nullptr) || global != (v_cache == nullptr)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (batch < 1 || n_q < 1 || num_splits < 1 || max_cache_len < 0) return GEMMA_ATTN_ERR_INVALID_ARG;
  const bool keys_rotated = (cache_layout & GEMMA_ATTN_CACHE_KEYS_ROTATED) != 0;
  if (keys_rotated && global) return GEMMA_ATTN_ERR_INVALID_ARG;  // the K=V tensor is also the values
  cache_layout &= ~GEMMA_ATTN_CACHE_KEYS_ROTATED;
  if (cache_layout != GEMMA_ATTN_CACHE_CONTIGUOUS && cache_layout != GEMMA_ATTN_CACHE_RING)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_layout == GEMMA_ATTN_CACHE_RING && (global || cache_capacity != params->window))
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_layout == GEMMA_ATTN_CACHE_CONTIGUOUS && cache_capacity < max_cache_len)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_capacity < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  const int group = params->num_q_heads / params->num_kv_heads;
  if (group * n_q > decode_max_rows(params->head_dim)) return GEMMA_ATTN_ERR_UNSUPPORTED;
  if (((uintptr_t)q | (uintptr_t)new_k | (uintptr_t)new_v | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15u)
    return GEMMA_ATTN_ERR_MISALIGNED;
  *a = DecodeArgs{};
  a->q = static_cast<const uint16_t*>(q);
  a->new_k = static_cast<const uint16_t*>(new_k);
  a->new_v = static_cast<const uint16_t*>(new_v);
  a->k_cache = static_cast<const uint16_t*>(k_cache);
  a->v_cache = static_cast<const uint16_t*>(v_cache);
  a->cache_seqlens = cache_seqlens;
  a->batch = batch; a->n_q = n_q; a->num_q_heads = params->num_q_heads; a->num_kv_heads = params->num_kv_heads;
  a->head_dim = params->head_dim; a->is_local = global ? 0 : 1; a->window = global ? 0 : params->window;
  a->ring = cache_layout == GEMMA_ATTN_CACHE_RING; a->capacity = cache_capacity; a->num_splits = num_splits;
  a->keys_rotated = keys_rotated ? 1 : 0;
  a->r = rotated_pairs(params->rope_p, params->head_dim);
  a->log2_base = log2((double)params->rope_base);
  a->softmax_scale = params->softmax_scale;
  a->q_pos_offset = nullptr;
  a->new_keys = 1;
  if (!decode_supported(*a)) return GEMMA_ATTN_ERR_UNSUPPORTED;
  return GEMMA_ATTN_OK;
}

}  // namespace gattn

using namespace gattn;

extern "C" {

const char* gemma_attn_error_string(int status) {
  switch (status) {
    case GEMMA_ATTN_OK: return "ok";
    case GEMMA_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case GEMMA_ATTN_ERR_UNSUPPORTED: return "unsupported shape (head_dim must be 32, 64, 128, 256 or 512)";
    case GEMMA_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case GEMMA_ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case GEMMA_ATTN_ERR_LAUNCH: return "kernel launch failed";
    case GEMMA_ATTN_ERR_TIMEOUT: return "a device-side wait ran out of time";
    case GEMMA_ATTN_ERR_DEVICE: return "CUDA error";
    case GEMMA_ATTN_ERR_SEQLEN: return "a sequence length is < 1 or exceeds max_seqlen";
    default: return "unknown status";
  }
}

int gemma_attn_last_launch_count(void) { return t_launches; }

int gemma_attn_prefill_workspace_size(const gemma_attn_params* params, int32_t total_tokens, size_t* bytes) {
  int rc = check_params(params);
  if (rc != GEMMA_ATTN_OK) return rc;
  if (total_tokens < 0 || !bytes) return GEMMA_ATTN_ERR_INVALID_ARG;
  *bytes = prefill_layout(params, total_tokens).total;
  return GEMMA_ATTN_OK;
}

}  // extern "C"

namespace {
enum : int { kPhaseRotate = 1, kPhaseAttend = 2 };

// Prefill in two phases: the rotated side copies into the workspace, then the attention
// kernel that reads them. gemma_attn_prefill runs both; the split entry points run one.
int prefill_phases(const gemma_attn_params* params, const void* q, const void* k, const void* v, void* out,
                   float* lse, const int32_t* positions, const int32_t* cu_seqlens, int32_t num_seqs,
                   int32_t total_tokens, int32_t max_seqlen, void* workspace, size_t workspace_bytes,
                   void* stream_, int phases) {
  t_launches = 0;
  int rc = check_params(params);
  if (rc != GEMMA_ATTN_OK) return rc;
  const bool global = params->kind == GEMMA_ATTN_GLOBAL;
  const bool bidir = params->kind == GEMMA_ATTN_BIDIR;
  if (!q || !k || !out || !positions || !cu_seqlens) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (global != (v == nullptr)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (num_seqs < 1 || total_tokens < 1 || max_seqlen < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (v && !aligned16(v)) || !aligned16(out))
    return GEMMA_ATTN_ERR_MISALIGNED;
  const PrefillLayout L = prefill_layout(params, total_tokens);
  if (L.total > 0 && (!workspace || workspace_bytes < L.total)) return GEMMA_ATTN_ERR_WORKSPACE;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GEMMA_ATTN_ERR_MISALIGNED;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const int d = params->head_dim;
  const int Hq = params->num_q_heads, Hkv = params->num_kv_heads;
  const bool pad = d < 64;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* qside = reinterpret_cast<uint16_t*>(ws + L.q_off);
  uint16_t* kside = reinterpret_cast<uint16_t*>(ws + L.k_off);
  uint16_t* vpad = reinterpret_cast<uint16_t*>(ws + L.v_off);
  const double log2_base = log2((double)params->rope_base);

  if (bidir && (phases & kPhaseRotate)) {
    // whole rows rotated (positions are (h, w) pairs), queries and keys in one launch
    Rope2dArgs ra;
    ra.src = static_cast<const uint16_t*>(q); ra.dst = qside; ra.heads = Hq;
    ra.src2 = static_cast<const uint16_t*>(k); ra.dst2 = kside; ra.heads2 = Hkv;
    ra.positions_hw = positions; ra.tokens = total_tokens; ra.d = d; ra.log2_base = log2_base;
    if (launch_rope2d_side(ra, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
    ++t_launches;
  } else if (L.mask && (phases & kPhaseRotate)) {
    RopeArgs ra;
    ra.positions = positions; ra.tokens = total_tokens; ra.d = d; ra.r = L.r; ra.chunk_mask = L.mask;
    ra.n_out = L.n_out; ra.log2_base = log2_base;
    // groups of 8 pairs (j, j + d/2) with a dim in a copied chunk: a prefix of the d/16 groups
    ra.groups_active = 0;
    for (int g = 0; g < d / 16; ++g) {
      const int c0 = (8 * g) / 64, c1 = (8 * g + d / 2) / 64;
      if (((L.mask >> c0) & 1u) || ((L.mask >> c1) & 1u)) ra.groups_active = g + 1;
    }
    // queries and keys in one launch (the angles of a token serve both)
    ra.src = static_cast<const uint16_t*>(q); ra.dst = qside; ra.heads = Hq;
    ra.src2 = static_cast<const uint16_t*>(k); ra.dst2 = kside; ra.heads2 = Hkv;
    if (launch_rope_side(ra, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
    ++t_launches;
    if (pad) {
      ra.heads2 = 0; ra.src2 = nullptr; ra.dst2 = nullptr;
      ra.src = static_cast<const uint16_t*>(global ? k : v); ra.dst = vpad; ra.heads = Hkv; ra.r = 0;
      if (launch_rope_side(ra, stream) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
      ++t_launches;
    }
  }

  if (!(phases & kPhaseAttend)) return GEMMA_ATTN_OK;

  PrefillMaps maps;
  bool ok = true;
  if (pad) {
    ok &= make_map(&maps.qs, qside, L.n_out, Hq, total_tokens, 128);
    ok &= make_map(&maps.ks, kside, L.n_out, Hkv, total_tokens, 128);
    maps.q = maps.qs;
    maps.k = maps.ks;
    ok &= make_map(&maps.v, vpad, 64, Hkv, total_tokens, 128);
    maps.k64 = maps.k;
    maps.ks64 = maps.ks;
  } else {
    ok &= make_map(&maps.q, q, d, Hq, total_tokens, 128);
    ok &= make_map(&maps.k, k, d, Hkv, total_tokens, 128);
    ok &= make_map(&maps.v, global ? k : v, d, Hkv, total_tokens, 128);
    ok &= make_map(&maps.k64, k, d, Hkv, total_tokens, 64);
    if (L.mask) {
      ok &= make_map(&maps.qs, qside, L.n_out, Hq, total_tokens, 128);
      ok &= make_map(&maps.ks, kside, L.n_out, Hkv, total_tokens, 128);
      ok &= make_map(&maps.ks64, kside, L.n_out, Hkv, total_tokens, 64);
    } else {
      maps.qs = maps.q;
      maps.ks = maps.k;
      maps.ks64 = maps.k64;
    }
  }
  if (!ok) return GEMMA_ATTN_ERR_LAUNCH;

  PrefillArgs a;
  a.cu_seqlens = cu_seqlens; a.out = out; a.lse = lse; a.num_seqs = num_seqs;
  a.max_qtiles = (max_seqlen + 127) / 128; a.max_seqlen = max_seqlen; a.total_tokens = total_tokens;
  a.num_q_heads = Hq; a.group = Hq / Hkv; a.head_dim = d;
  a.is_local = params->kind == GEMMA_ATTN_LOCAL ? 1 : 0;
  a.bidir = bidir ? 1 : 0;
  a.window = a.is_local ? params->window : 0; a.softmax_scale = params->softmax_scale; a.rot_mask = L.mask;
  a.out_f32 = params->out_dtype == GEMMA_ATTN_OUT_F32;
  a.pair_allowed = pair_kernel_enabled();
  // 32-byte stores need the base and the row stride (head_dim elements) 32-byte aligned
  a.out_align32 = ((reinterpret_cast<uintptr_t>(out) & 31u) == 0 &&
                   (d * (a.out_f32 ? 4 : 2)) % 32 == 0) ? 1 : 0;
  cudaError_t e;
  switch (L.kd) {
    case 64: e = launch_prefill<64>(maps, a, stream); break;
    case 128: e = launch_prefill<128>(maps, a, stream); break;
    case 256: e = launch_prefill<256>(maps, a, stream); break;
    case 512: e = launch_prefill<512>(maps, a, stream); break;
    default: return GEMMA_ATTN_ERR_UNSUPPORTED;
  }
  if (e != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  ++t_launches;
  return GEMMA_ATTN_OK;
}
}  // namespace

extern "C" {

int gemma_attn_prefill(const gemma_attn_params* params, const void* q, const void* k, const void* v, void* out,
                       float* lse, const int32_t* positions, const int32_t* cu_seqlens, int32_t num_seqs,
                       int32_t total_tokens, int32_t max_seqlen, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return prefill_phases(params, q, k, v, out, lse, positions, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                        workspace, workspace_bytes, stream, kPhaseRotate | kPhaseAttend);
}

int gemma_attn_prefill_rotate(const gemma_attn_params* params, const void* q, const void* k, const void* v,
                              void* out, float* lse, const int32_t* positions, const int32_t* cu_seqlens,
                              int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return prefill_phases(params, q, k, v, out, lse, positions, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                        workspace, workspace_bytes, stream, kPhaseRotate);
}

int gemma_attn_prefill_attend(const gemma_attn_params* params, const void* q, const void* k, const void* v,
                              void* out, float* lse, const int32_t* positions, const int32_t* cu_seqlens,
                              int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return prefill_phases(params, q, k, v, out, lse, positions, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                        workspace, workspace_bytes, stream, kPhaseAttend);
}

int gemma_attn_decode_num_splits(const gemma_attn_params* params, int32_t batch, int32_t n_q,
                                 int32_t max_cache_len, int32_t* num_splits) {
  int rc = check_params(params);
  if (rc != GEMMA_ATTN_OK) return rc;
  if (params->kind == GEMMA_ATTN_BIDIR) return GEMMA_ATTN_ERR_UNSUPPORTED;  // prefill only
  if (batch < 1 || n_q < 1 || max_cache_len < 0 || !num_splits) return GEMMA_ATTN_ERR_INVALID_ARG;
  int keys = params->kind == GEMMA_ATTN_LOCAL ? std::min(max_cache_len, params->window) : max_cache_len;
  keys += n_q;
  // One decode CTA per SM at a time. Splits run in waves of 148 CTAs, and each CTA
  // pays a fixed cost (angle tables, the first copies' latency, the merge) worth about
  // kSplitOverheadKeys keys of streaming: take the split count with the least
  // waves * (keys per split + that overhead), at least 256 keys per split.
  constexpr int kSplitOverheadKeys = 512;
  const int sms = 148;
  const long long units = (long long)batch * params->num_kv_heads;
  const int s_cap = std::max(1, std::min(keys / 256, 4096));
  int best = 1;
  double best_cost = 0.0;
  for (int s = 1; s <= s_cap; ++s) {
    const long long waves = (units * s + sms - 1) / sms;
    const double cost = (double)waves * ((double)((keys + s - 1) / s) + kSplitOverheadKeys);
    if (s == 1 || cost < best_cost * (1.0 - 1e-9)) { best_cost = cost; best = s; }
  }
  // The verify kernel picks its own tiles per split from the lengths it sees, among
  // ceil(longest / s) for s up to the split count: twice the uniform choice leaves it room
  // for ragged batches (no more than one split per 128-key tile).
  if (decode_umma_shape(params, n_q)) best = std::max(1, std::min(2 * best, (keys + 127) / 128));
  *num_splits = best;
  return GEMMA_ATTN_OK;
}

int gemma_attn_decode(const gemma_attn_params* params, const void* q, const void* new_k, const void* new_v,
                      const void* k_cache, const void* v_cache, int32_t cache_layout, int32_t cache_capacity,
                      const int32_t* cache_seqlens, int32_t batch, int32_t n_q, int32_t max_cache_len,
                      float* partial_o, float* partial_lse, int32_t num_splits, void* stream_) {
  t_launches = 0;
  if (!partial_o || !partial_lse) return GEMMA_ATTN_ERR_INVALID_ARG;
  DecodeArgs a{};  // out == nullptr: the kernel writes the split partials
  const int rc = decode_prepare(params, q, new_k, new_v, k_cache, v_cache, cache_layout, cache_capacity,
                                cache_seqlens, batch, n_q, max_cache_len, num_splits, &a);
  if (rc != GEMMA_ATTN_OK) return rc;
  a.partial_o = partial_o; a.partial_lse = partial_lse;
  if (launch_decode(a, static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = 1;
  return GEMMA_ATTN_OK;
}

int gemma_attn_decode_shard(const gemma_attn_params* params, const void* q, const void* new_k, const void* k_cache,
                            int32_t cache_capacity, const int32_t* shard_seqlens, const int32_t* q_pos_offset,
                            int32_t include_new, int32_t batch, int32_t n_q, int32_t max_shard_len,
                            float* partial_o, float* partial_lse, int32_t num_splits, void* stream_) {
  t_launches = 0;
  if (!params || params->kind != GEMMA_ATTN_GLOBAL) return GEMMA_ATTN_ERR_INVALID_ARG;  // K=V caches only
  if (include_new != 0 && include_new != 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (!partial_o || !partial_lse || !q_pos_offset) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (include_new && !new_k) return GEMMA_ATTN_ERR_INVALID_ARG;
  DecodeArgs a{};
  // without new keys the kernels never read new_k: q stands in for the pointer checks
  const int rc = decode_prepare(params, q, include_new ? new_k : q, nullptr, k_cache, nullptr,
                                GEMMA_ATTN_CACHE_CONTIGUOUS, cache_capacity, shard_seqlens, batch, n_q,
                                max_shard_len, num_splits, &a);
  if (rc != GEMMA_ATTN_OK) return rc;
  if (reinterpret_cast<uintptr_t>(q_pos_offset) & 3u) return GEMMA_ATTN_ERR_MISALIGNED;
  a.q_pos_offset = q_pos_offset;
  a.new_keys = include_new;
  if (!include_new) a.new_k = nullptr;
  a.partial_o = partial_o; a.partial_lse = partial_lse;
  if (launch_decode(a, static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = 1;
  return GEMMA_ATTN_OK;
}

int gemma_attn_cache_append(const gemma_attn_params* params, const void* new_k, const void* new_v, void* k_cache,
                            void* v_cache, int32_t cache_layout, int32_t cache_capacity,
                            const int32_t* cache_seqlens, int32_t batch, int32_t n_q, void* stream_) {
  t_launches = 0;
  int rc = check_params(params);
  if (rc != GEMMA_ATTN_OK) return rc;
  if (params->kind == GEMMA_ATTN_BIDIR) return GEMMA_ATTN_ERR_UNSUPPORTED;  // prefill only
  const bool global = params->kind == GEMMA_ATTN_GLOBAL;
  if (!new_k || !k_cache || !cache_seqlens) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (global != (new_v == nullptr) || global != (v_cache == nullptr)) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (batch < 1 || n_q < 1 || cache_capacity < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  const bool keys_rotated = (cache_layout & GEMMA_ATTN_CACHE_KEYS_ROTATED) != 0;
  if (keys_rotated && global) return GEMMA_ATTN_ERR_INVALID_ARG;  // the K=V tensor is also the values
  cache_layout &= ~GEMMA_ATTN_CACHE_KEYS_ROTATED;
  if (cache_layout != GEMMA_ATTN_CACHE_CONTIGUOUS && cache_layout != GEMMA_ATTN_CACHE_RING)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (cache_layout == GEMMA_ATTN_CACHE_RING && (global || cache_capacity != params->window))
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (((uintptr_t)new_k | (uintptr_t)new_v | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15u)
    return GEMMA_ATTN_ERR_MISALIGNED;
  AppendArgs a{};
  a.new_k = static_cast<const uint16_t*>(new_k);
  a.new_v = static_cast<const uint16_t*>(new_v);
  a.k_cache = static_cast<uint16_t*>(k_cache);
  a.v_cache = static_cast<uint16_t*>(v_cache);
  a.cache_seqlens = cache_seqlens;
  a.batch = batch; a.n_q = n_q; a.num_kv_heads = params->num_kv_heads; a.head_dim = params->head_dim;
  a.capacity = cache_capacity;
  a.ring = cache_layout == GEMMA_ATTN_CACHE_RING;
  a.keys_rotated = keys_rotated ? 1 : 0;
  a.r = rotated_pairs(params->rope_p, params->head_dim);
  a.log2_base = log2((double)params->rope_base);
  if (launch_cache_append(a, static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = 1;
  return GEMMA_ATTN_OK;
}

int gemma_attn_combine(const float* partial_o, const float* partial_lse, int32_t num_splits, int32_t rows,
                       int32_t head_dim, int32_t out_dtype, void* out, float* lse, void* stream_) {
  t_launches = 0;
  if (!partial_o || !partial_lse || !out || num_splits < 1 || rows < 0 || head_dim < 1)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (out_dtype != GEMMA_ATTN_OUT_BF16 && out_dtype != GEMMA_ATTN_OUT_F32) return GEMMA_ATTN_ERR_INVALID_ARG;
  CombineArgs a;
  a.partial_o = partial_o; a.partial_lse = partial_lse; a.out = out; a.lse = lse;
  a.num_splits = num_splits; a.rows = rows; a.head_dim = head_dim;
  a.out_f32 = out_dtype == GEMMA_ATTN_OUT_F32;
  if (launch_combine(a, static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = rows > 0 ? 1 : 0;
  return GEMMA_ATTN_OK;
}

int gemma_attn_tile_plan(int32_t kind, int32_t window, const int32_t* cu_seqlens_host, int32_t num_seqs,
                         int32_t bm, int32_t bn, int32_t* out, int64_t cap, int64_t* count) {
  if (!cu_seqlens_host || num_seqs < 1 || bm < 1 || bn < 1 || !count) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (kind != GEMMA_ATTN_LOCAL && kind != GEMMA_ATTN_GLOBAL && kind != GEMMA_ATTN_BIDIR)
    return GEMMA_ATTN_ERR_INVALID_ARG;
  if (kind == GEMMA_ATTN_LOCAL && window < 1) return GEMMA_ATTN_ERR_INVALID_ARG;
  const int is_local = kind == GEMMA_ATTN_LOCAL;
  const int bidir = kind == GEMMA_ATTN_BIDIR;
  int64_t n = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int len = cu_seqlens_host[s + 1] - cu_seqlens_host[s];
    if (len < 0) return GEMMA_ATTN_ERR_INVALID_ARG;
    const int nqt = (len + bm - 1) / bm;
    for (int qt = 0; qt < nqt; ++qt) {
      int lo, hi;
      kv_tile_range(is_local, window, len, qt, bm, bn, &lo, &hi, bidir);
      for (int kt = lo; kt < hi; ++kt) {
        if (out && n < cap) {
          out[4 * n + 0] = s;
          out[4 * n + 1] = qt;
          out[4 * n + 2] = kt;
          out[4 * n + 3] = kv_tile_class(is_local, window, len, qt, kt, bm, bn, bidir);
        }
        ++n;
      }
    }
  }
  *count = n;
  return GEMMA_ATTN_OK;
}

int gemma_attn_check(void* stream_) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_DEVICE;
  int status = 0;
  if (cudaMemcpyFromSymbol(&status, g_status, sizeof(int)) != cudaSuccess) return GEMMA_ATTN_ERR_DEVICE;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return GEMMA_ATTN_ERR_DEVICE;
  if (status & kStatusTimeout) return GEMMA_ATTN_ERR_TIMEOUT;
  if (status & kStatusSeqlen) return GEMMA_ATTN_ERR_SEQLEN;
  return GEMMA_ATTN_OK;
}

int gemma_attn_selftest_timeout(int32_t* gave_up, void* stream_) {
  t_launches = 0;
  if (!gave_up) return GEMMA_ATTN_ERR_INVALID_ARG;
  if (launch_timeout_selftest(gave_up, static_cast<cudaStream_t>(stream_)) != cudaSuccess) return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = 1;
  return GEMMA_ATTN_OK;
}

int gemma_attn_selftest_umma(int32_t mode, const void* a, const void* b, const void* p, float* d, void* stream_) {
  t_launches = 0;
  if (mode < 0 || mode > 2 || !b || !d || (mode == 0 && !a) || (mode != 0 && !p))
    return GEMMA_ATTN_ERR_INVALID_ARG;
  CUtensorMap am, bm;
  bool ok = true;
  if (mode == 0) {
    ok &= make_map(&am, a, 128, 1, 128, 128);
    ok &= make_map(&bm, b, 128, 1, 128, 128);
  } else {
    ok &= make_map(&bm, b, mode == 1 ? 64 : 128, 1, 128, 128);
    am = bm;
  }
  if (!ok) return GEMMA_ATTN_ERR_LAUNCH;
  if (launch_umma_selftest(am, bm, static_cast<const uint16_t*>(p), d, mode, static_cast<cudaStream_t>(stream_)) !=
      cudaSuccess)
    return GEMMA_ATTN_ERR_LAUNCH;
  t_launches = 1;
  return GEMMA_ATTN_OK;
}

}  // extern "C"
