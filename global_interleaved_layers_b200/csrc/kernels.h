// kernels.h -- launch interfaces between the host entry points and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gattn {

struct PrefillArgs {
  const int32_t* cu_seqlens;
  void* out;
  float* lse;
  int num_seqs;
  int max_qtiles;     // ceil(max_seqlen / 128)
  int max_seqlen;
  int total_tokens;
  int num_q_heads;
  int group;          // query heads per KV head
  int head_dim;       // real head dim (row stride of out); the kernel dim may be padded to 64
  int is_local;
  int bidir;          // bidirectional (every key of the sequence); is_local is then 0
  int window;
  float softmax_scale;
  int out_f32;        // 1: write fp32 output, 0: bf16
  int pair_allowed;   // 1: use the two-CTA paired kernel where the shape permits
  int out_align32;    // 1: every output row segment is 32-byte aligned (256-bit stores)
  uint32_t rot_mask;  // bit c set: key/query chunk c (64 dims) is read from the rotated side copy
};

struct PrefillMaps {
  CUtensorMap q, qs, k, ks, v;   // 128-row boxes
  CUtensorMap k64, ks64;         // 64-row boxes: one CTA's half of a key tile (paired form)
};

template <int D>
cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream);

// Rotated (or zero-padded) side copy of selected 64-dim chunks.
struct RopeArgs {
  const uint16_t* src;      // [T, H, d] bf16
  uint16_t* dst;            // [T, H, n_out] bf16, n_out = popcount(chunk_mask) * 64
  const uint16_t* src2;     // optional second tensor [T, H2, d] (the keys), same rotation
  uint16_t* dst2;           // [T, H2, n_out]
  int heads2;               // 0: no second tensor
  const int32_t* positions; // [T]
  int tokens;
  int heads;
  int d;                    // real head dim
  int r;                    // rotated pairs (0: copy only)
  uint32_t chunk_mask;      // chunks of the (padded) head dim that are copied
  int n_out;
  int groups_active;        // leading groups of 8 pairs with any dim in the copy (the rest: none)
  double log2_base;
};
cudaError_t launch_rope_side(const RopeArgs& a, cudaStream_t stream);

// Rotated copies of whole rows for the 2D rotation: dims [0, d/2) rotated for w and
// [d/2, d) for h (each half: pairs (j, j + d/4), theta_j = base^(-2j/(d/2))).
struct Rope2dArgs {
  const uint16_t* src;       // [T, H, d] bf16
  uint16_t* dst;             // [T, H, d] bf16
  const uint16_t* src2;      // optional second tensor [T, H2, d] (the keys)
  uint16_t* dst2;
  int heads, heads2;
  const int32_t* positions_hw;  // [T, 2]: (h, w)
  int tokens, d;
  double log2_base;
};
cudaError_t launch_rope2d_side(const Rope2dArgs& a, cudaStream_t stream);

struct DecodeArgs {
  const uint16_t* q;        // [B, n_q, Hq, d]
  const uint16_t* new_k;    // [B, n_q, Hkv, d]
  const uint16_t* new_v;    // [B, n_q, Hkv, d] or null (K=V)
  const uint16_t* k_cache;
  const uint16_t* v_cache;  // null for K=V
  const int32_t* cache_seqlens;
  float* partial_o;         // [splits, rows, d]
  float* partial_lse;       // [splits, rows]
  void* out;                // null: write the partials; else (num_splits == 1) the final [rows, d] output
  float* out_lse;           // with out: final log-sum-exp [rows] or null
  int out_f32;              // with out: 1 fp32, 0 bf16
  int batch, n_q, num_q_heads, num_kv_heads, head_dim;
  int is_local, window, ring, capacity, num_splits;
  int keys_rotated;         // cached keys are stored rotated: only new tokens' keys are rotated here
  int r;
  double log2_base;
  float softmax_scale;
  // A key-range shard of a longer history (global layers): the queries sit q_pos_offset[b]
  // positions later than the shard's own end, and new_keys = 0 leaves the n_q new tokens out
  // of the keys (another shard holds them). Defaults: no offset, new_keys = 1.
  const int32_t* q_pos_offset;
  int new_keys;
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
// Global (K=V, contiguous cache) layers with 9-32 query rows per KV head at head dim 256 or
// 512 and at most 64 rotated pairs: the tcgen05 verify kernel (decode_umma.cu).
bool decode_umma_applies(const DecodeArgs& a);
// The shape test of decode_umma_applies (a global layer's cache is contiguous and un-rotated).
bool decode_umma_shape(const gemma_attn_params* p, int n_q);
cudaError_t launch_decode_umma_any(const DecodeArgs& a, cudaStream_t stream);
// 3-D bf16 tensor map over a decode cache [planes][capacity][d] with {64, 128, 1} boxes,
// 128-byte swizzle.
bool encode_cache_map(CUtensorMap* m, const void* base, int d, int capacity, int planes);
int decode_max_rows(int head_dim);  // largest group * n_q one decode CTA handles
bool decode_supported(const DecodeArgs& a);  // a kernel variant fits this shape

struct CombineArgs {
  const float* partial_o;
  const float* partial_lse;
  void* out;
  float* lse;
  int num_splits, rows, head_dim;
  int out_f32;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);
cudaError_t launch_timeout_selftest(int* gave_up, cudaStream_t stream);

// New tokens' rows into a decode cache (ring slot p mod capacity, or row p).
struct AppendArgs {
  const uint16_t* new_k;    // [B, n_q, Hkv, d]
  const uint16_t* new_v;    // [B, n_q, Hkv, d] or null (K=V)
  uint16_t* k_cache;        // [B, Hkv, capacity, d]
  uint16_t* v_cache;        // same, or null (K=V)
  const int32_t* cache_seqlens;
  int batch, n_q, num_kv_heads, head_dim, capacity;
  int ring;
  int keys_rotated;         // store the key rotated for its position (first r pairs)
  int r;
  double log2_base;
};
cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream);

}  // namespace gattn

struct gemma_attn_params;

namespace gattn {

// Argument checks and DecodeArgs set-up shared by the decode entry points: fills every
// field except the partial / final output pointers; returns a GEMMA_ATTN_* status.
int decode_prepare(const gemma_attn_params* params, const void* q, const void* new_k, const void* new_v,
                   const void* k_cache, const void* v_cache, int32_t cache_layout, int32_t cache_capacity,
                   const int32_t* cache_seqlens, int32_t batch, int32_t n_q, int32_t max_cache_len,
                   int32_t num_splits, DecodeArgs* a);
// The count gemma_attn_last_launch_count reports for this host thread.
void set_launch_count(int n);

}  // namespace gattn
