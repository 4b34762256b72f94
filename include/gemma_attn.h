/*
 * gemma_attn.h -- C ABI of the B200 (sm_100a) attention kernels for
 * Gemma-4-style interleaved layers.
 *
 * Two layer kinds, as described in "Visual guide to Gemma 4":
 *   LOCAL  -- sliding-window causal attention (section "Interleaving Layers":
 *             a local layer looks only at tokens within a fixed range), with
 *             grouped-query attention (2 query heads per KV head on local
 *             layers per the DeepMind talk summary, section "Optimised
 *             attention: local and global layers"), separate K and V.
 *   GLOBAL -- full causal attention (same sections: a global layer sees the whole
 *             preceding sequence) with GQA (8 query heads per KV head, guide
 *             section "GQA"), K = V (guide section "K=V technique": one stored
 *             tensor per KV head serves as keys and values) and p-RoPE (guide
 *             section "p-RoPE": only the highest-frequency fraction p of the
 *             rotary pairs is rotated; the rest pass through).
 *
 * Conventions shared by every entry point:
 *   - bf16 tensors are passed as device pointers to raw bfloat16 storage; LSE and
 *     split partials are float32; positions and lengths are int32.
 *   - Head layout of q/k/v/out is row-major [tokens, heads, head_dim].
 *   - Visible keys of a query at position i: pos_k <= i (GLOBAL) and additionally
 *     pos_k > i - window (LOCAL): exactly `window` keys including the query itself.
 *   - Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *   - Rotary embedding: r = floor(rope_p * head_dim / 2) pairs (j, j + head_dim/2),
 *     j = 0 .. r-1, rotated counter-clockwise by pos * rope_base^(-2j/head_dim).
 *     q and the key copy used for scores are rotated; values never are (for
 *     GLOBAL the single K=V tensor is stored un-rotated).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream). The caller owns every buffer, including
 *     workspaces; the library allocates no device memory.
 *   - Return value: GEMMA_ATTN_OK (0) or a negative status. On an argument error
 *     nothing is launched. Device-side failures (a bounded wait that ran out, a
 *     sequence longer than the stated maximum) are recorded in a device status
 *     word that gemma_attn_check() reads and clears.
 *   - Pointers to bf16 tensors read by the tensor-memory-accelerator loads must be
 *     16-byte aligned; head_dim * 2 bytes must be a multiple of 16.
 */
#ifndef GEMMA_ATTN_H_
#define GEMMA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  GEMMA_ATTN_LOCAL = 0,
  GEMMA_ATTN_GLOBAL = 1,
  /* The vision encoder's attention over an image's patches ("Visual guide to Gemma 4",
   * section "Vision encoder"): bidirectional (every patch of the sequence visible),
   * 2D RoPE (dims [0, d/2) rotated for the horizontal position w, dims [d/2, d) for the
   * vertical position h, each half as a d/2-dim rotation: pairs (j, j + d/4),
   * theta_j = rope_base^(-2j/(d/2))). Prefill only; rope_p must be 1, head_dim >= 64,
   * v given (separate values), window ignored. */
  GEMMA_ATTN_BIDIR = 2
};

enum {
  GEMMA_ATTN_CACHE_CONTIGUOUS = 0, /* [batch, kv_heads, capacity, head_dim]; token p at row p */
  GEMMA_ATTN_CACHE_RING = 1,       /* [batch, kv_heads, window, head_dim]; token p at slot p mod window */
  /* Flag OR-ed into cache_layout, LOCAL layers only (separate value tensor): the cached
   * keys are stored already rotated for their positions, as they were when written
   * (token p's key rotated by p-RoPE at position p); the call then rotates only the new
   * tokens' keys. Without it the cache holds un-rotated keys. A GLOBAL layer's single K=V
   * tensor serves as the values too, so its cache stays un-rotated. */
  GEMMA_ATTN_CACHE_KEYS_ROTATED = 0x100
};

enum {
  GEMMA_ATTN_OK = 0,
  GEMMA_ATTN_ERR_INVALID_ARG = -1,
  GEMMA_ATTN_ERR_UNSUPPORTED = -2,
  GEMMA_ATTN_ERR_WORKSPACE = -3,
  GEMMA_ATTN_ERR_MISALIGNED = -4,
  GEMMA_ATTN_ERR_LAUNCH = -5,
  GEMMA_ATTN_ERR_TIMEOUT = -6,
  GEMMA_ATTN_ERR_DEVICE = -7,
  GEMMA_ATTN_ERR_SEQLEN = -8
};

enum {
  GEMMA_ATTN_OUT_BF16 = 0, /* outputs rounded to bfloat16 (round to nearest even) */
  GEMMA_ATTN_OUT_F32 = 1   /* outputs left in the fp32 accumulator precision */
};

/* Layer description. head_dim in {32, 64, 128, 256, 512}; num_q_heads a multiple of
 * num_kv_heads; window >= 1 for LOCAL (ignored for GLOBAL); 0 <= rope_p <= 1;
 * rope_base > 0; softmax_scale > 0 (typically 1/sqrt(head_dim)); out_dtype selects
 * the element type of `out` (GEMMA_ATTN_OUT_BF16 or GEMMA_ATTN_OUT_F32). */
typedef struct gemma_attn_params {
  int32_t kind;
  int32_t window;
  float rope_p;
  float rope_base;
  float softmax_scale;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t out_dtype;
} gemma_attn_params;

/* Bytes of device workspace gemma_attn_prefill needs for `total_tokens` tokens
 * (a rotated copy of the key columns that p-RoPE touches, and of small heads'
 * operands padded to 64 dims). Written to *bytes. */
int gemma_attn_prefill_workspace_size(const gemma_attn_params* params, int32_t total_tokens,
                                      size_t* bytes);

/*
 * Prefill: attention of every token of a ragged batch against the earlier tokens
 * of its own sequence (flash-style; fully masked key tiles are never visited, so a
 * LOCAL layer costs O(tokens * window)); for GEMMA_ATTN_BIDIR against every token of
 * its own sequence (an image's patches).
 *   q         [total_tokens, num_q_heads, head_dim] bf16, device.
 *   k         [total_tokens, num_kv_heads, head_dim] bf16, device (GLOBAL: the K=V tensor).
 *   v         same shape as k for LOCAL; must be NULL for GLOBAL (values = k, un-rotated).
 *   out       [total_tokens, num_q_heads, head_dim] bf16 or f32 (params->out_dtype), device, written.
 *   lse       [num_q_heads, total_tokens] float32 natural-log sum-exp of the scaled
 *             scores, device, written; may be NULL.
  *   positions [total_tokens] int32, device: rotary position of each token. Within a
 *             sequence the positions must be consecutive (p, p+1, ...): the masks are
 *             evaluated on in-sequence offsets, which equals the position rule then.
 *             GEMMA_ATTN_BIDIR: [total_tokens, 2] int32, the (h, w) patch coordinates of
 *             each token, in any order (no mask depends on them).
 *   cu_seqlens [num_seqs + 1] int32, device: sequence s is tokens cu[s] .. cu[s+1]-1.
 *             Lengths must be >= 1 and <= max_seqlen (violations are reported through
 *             gemma_attn_check as GEMMA_ATTN_ERR_SEQLEN).
 *   workspace  device buffer of at least gemma_attn_prefill_workspace_size() bytes,
 *             256-byte aligned; contents are scratch.
 */
int gemma_attn_prefill(const gemma_attn_params* params, const void* q, const void* k, const void* v,
                       void* out, float* lse, const int32_t* positions, const int32_t* cu_seqlens,
                       int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * The two phases of gemma_attn_prefill, for callers that schedule or time them apart:
 * _rotate writes the rotated side copies of q and k (and, for head_dim < 64, the padded
 * copies) into the workspace; _attend runs the attention kernel, which reads them, so it
 * must follow a _rotate of the same q, k, v, positions and workspace on the same stream
 * (or be otherwise ordered after it). Arguments, validation and errors are those of
 * gemma_attn_prefill; _rotate ignores out, lse, cu_seqlens' contents and max_seqlen
 * beyond validation. ("Visual guide to Gemma 4", section "p-RoPE": the rotation; the rest
 * as gemma_attn_prefill.)
 */
int gemma_attn_prefill_rotate(const gemma_attn_params* params, const void* q, const void* k,
                              const void* v, void* out, float* lse, const int32_t* positions,
                              const int32_t* cu_seqlens, int32_t num_seqs, int32_t total_tokens,
                              int32_t max_seqlen, void* workspace, size_t workspace_bytes, void* stream);
int gemma_attn_prefill_attend(const gemma_attn_params* params, const void* q, const void* k,
                              const void* v, void* out, float* lse, const int32_t* positions,
                              const int32_t* cu_seqlens, int32_t num_seqs, int32_t total_tokens,
                              int32_t max_seqlen, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode / speculative verify, split-KV stage: n_q new query tokens per sequence
 * attend to that sequence's cache plus the new tokens themselves.
 *   q          [batch, n_q, num_q_heads, head_dim] bf16; query i of sequence b sits at
 *              position cache_seqlens[b] + i.
 *   new_k      [batch, n_q, num_kv_heads, head_dim] bf16: keys of the new tokens
 *              (GLOBAL: their K=V rows). Required (n_q >= 1).
 *   new_v      same shape for LOCAL; NULL for GLOBAL.
 *   k_cache    GEMMA_ATTN_CACHE_CONTIGUOUS: [batch, num_kv_heads, cache_capacity, head_dim],
 *              token p of sequence b at row p (p < cache_seqlens[b] <= cache_capacity).
 *              GEMMA_ATTN_CACHE_RING (LOCAL only): [batch, num_kv_heads, window, head_dim],
 *              token p at slot p mod window, holding the last min(len, window) tokens;
 *              cache_capacity must equal window.
 *              Caches hold un-rotated keys (GLOBAL: the K=V tensor), or for LOCAL with
 *              GEMMA_ATTN_CACHE_KEYS_ROTATED in cache_layout, keys rotated for their
 *              positions (new_k is always un-rotated).
 *   v_cache    same layout as k_cache for LOCAL; NULL for GLOBAL.
 *   cache_seqlens [batch] int32 device: tokens already cached (>= 0).
 *   max_cache_len  upper bound on cache_seqlens (sizes the launch).
 *   partial_o  [num_splits, batch * n_q * num_q_heads, head_dim] float32, written.
 *   partial_lse [num_splits, batch * n_q * num_q_heads] float32, written (-inf for an
 *              empty split). Row index = (b * n_q + i) * num_q_heads + h.
 *   The visible keys of each sequence are cut into at most num_splits contiguous ranges,
 *   in split order; a split with no keys (for a short sequence, the splits past its last)
 *   has lse -inf and its partial_o row is not written (the combine does not read it).
 *   Limits: (num_q_heads / num_kv_heads) * n_q <= 64 (<= 32 for head_dim 512), else
 *   GEMMA_ATTN_ERR_UNSUPPORTED; q, new_k, new_v and the caches 16-byte aligned.
 */
int gemma_attn_decode(const gemma_attn_params* params, const void* q, const void* new_k,
                      const void* new_v, const void* k_cache, const void* v_cache,
                      int32_t cache_layout, int32_t cache_capacity, const int32_t* cache_seqlens,
                      int32_t batch, int32_t n_q, int32_t max_cache_len,
                      float* partial_o, float* partial_lse, int32_t num_splits, void* stream);

/*
 * Decode + combine in one call that allocates nothing. The pages have no counterpart
 * to this entry point: it serves callers of this library that cannot allocate device
 * memory -- an op inside a framework that owns every device allocation and offers it
 * no scratch allocator, or a caller capturing a CUDA graph, where cudaMalloc is not
 * allowed -- so they cannot provide the split partials that gemma_attn_decode writes.
 * Here the partials live in a static array of GEMMA_ATTN_NOALLOC_SCRATCH_BYTES inside
 * the library; every GPU that loads the library holds it until the process exits.
 *   Arguments: as gemma_attn_decode (q, new_k, new_v, caches, layout, capacity,
 *   cache_seqlens, batch, n_q, max_cache_len, num_splits), then out [batch, n_q,
 *   num_q_heads, head_dim] (bf16 or f32 per params->out_dtype) and lse [batch * n_q *
 *   num_q_heads] f32 or NULL, as gemma_attn_combine writes them. The caller passes and
 *   owns every input and output buffer.
 *   Limit: num_splits * batch * n_q * num_q_heads * (head_dim + 1) * 4 bytes (each of
 *   the two partial arrays rounded up to 256 bytes) must not exceed
 *   GEMMA_ATTN_NOALLOC_SCRATCH_BYTES; a larger request returns GEMMA_ATTN_ERR_WORKSPACE
 *   and launches nothing (use fewer splits).
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any
 *   stream capture. All calls share the array and it keeps the last call's contents;
 *   each call rewrites every partial it reads, so nothing is cleared between calls.
 *   Calls that overlap on the GPU (concurrent streams, or threads whose streams are
 *   not ordered) race on the array and corrupt each other's results.
 *   num_splits == 1: the decode kernel writes out and lse itself (one launch); the
 *   static array is neither used nor size-checked, and such calls do not race.
 */
#define GEMMA_ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
int gemma_attn_decode_noalloc(const gemma_attn_params* params, const void* q, const void* new_k,
                              const void* new_v, const void* k_cache, const void* v_cache,
                              int32_t cache_layout, int32_t cache_capacity,
                              const int32_t* cache_seqlens, int32_t batch, int32_t n_q,
                              int32_t max_cache_len, int32_t num_splits, void* out, float* lse,
                              void* stream);

/*
 * KV-cache append: the rows of the new tokens join the cache ("Visual guide to Gemma 4",
 * sections "K=V technique" and "GQA": one stored KV tensor per KV head; section "p-RoPE":
 * which pairs a stored key has rotated). Token i of sequence b, at position
 * p = cache_seqlens[b] + i, is written to slot p mod window (GEMMA_ATTN_CACHE_RING) or to
 * row p (GEMMA_ATTN_CACHE_CONTIGUOUS) of k_cache (and v_cache for LOCAL). With
 * GEMMA_ATTN_CACHE_KEYS_ROTATED (LOCAL only) the key is stored rotated for p (pairs
 * (j, j + d/2), j < r = floor(rope_p * d / 2), angle p * rope_base^(-2j/d), fp32 math from
 * the bf16 inputs, bf16 result), the form gemma_attn_decode reads from such a cache;
 * values and GLOBAL K=V rows are copied unchanged.
 *   Arguments: new_k / new_v [batch, n_q, num_kv_heads, head_dim] bf16 (new_v NULL for
 *   GLOBAL), k_cache / v_cache and cache_layout / cache_capacity as gemma_attn_decode
 *   (v_cache NULL for GLOBAL), cache_seqlens [batch] int32 device: the tokens cached
 *   before these (not modified: the caller advances it by n_q). All device pointers,
 *   16-byte aligned; the caller owns every buffer.
 *   Order: call it after the decode / verify step that read these tokens from new_k /
 *   new_v. In a W-slot ring the new rows overwrite the slots of positions p - W, which
 *   that step's earlier queries still see (p - W > position - W for a query before p).
 *   A ring holds the newest window positions: when n_q > cache_capacity, only the last
 *   cache_capacity new tokens of a sequence are written (an earlier token's slot belongs
 *   to a later one), so the result does not depend on the order the rows are written in.
 *   Errors: GEMMA_ATTN_ERR_INVALID_ARG / _MISALIGNED as gemma_attn_decode, before any
 *   launch. A contiguous-cache position p >= cache_capacity (or a negative length) writes
 *   nothing for that row and records GEMMA_ATTN_ERR_SEQLEN in the device status word,
 *   read by gemma_attn_check.
 */
int gemma_attn_cache_append(const gemma_attn_params* params, const void* new_k, const void* new_v,
                            void* k_cache, void* v_cache, int32_t cache_layout, int32_t cache_capacity,
                            const int32_t* cache_seqlens, int32_t batch, int32_t n_q, void* stream);

/*
 * Decode / verify over one key-range shard of a long K=V history (GLOBAL layers only), for
 * a history spread over several GPUs: each GPU holds a contiguous range of every sequence's
 * tokens and runs this on its range; the fp32 partials of all GPUs, stacked as splits
 * (GPU-major), go through gemma_attn_combine (in-memory on one GPU, or after an all-gather
 * between GPUs) to give the attention over the whole history. The medium models' 256K
 * context is what makes one GPU's cache too small ("Visão geral do modelo Gemma 4", section
 * "Recursos": the context window); the scores are those of the whole history because a rotation depends only
 * on the distance between the query and the key ("Visual guide to Gemma 4", section
 * "p-RoPE").
 *   Arguments: q, new_k as gemma_attn_decode (new_k may be NULL when include_new is 0);
 *   k_cache [batch, num_kv_heads, cache_capacity, head_dim] bf16 holding the shard's tokens
 *   at rows 0 .. shard_seqlens[b] - 1 (device int32 [batch]); q_pos_offset (device int32
 *   [batch], 4-byte aligned): how many tokens of sequence b come after the shard and before
 *   the new tokens, i.e. the queries sit at shard-local positions shard_seqlens[b] +
 *   q_pos_offset[b] + i; include_new: 1 for the shard that ends the history (its offset
 *   must be 0), whose keys then also include the n_q new tokens (causally), 0 for the
 *   others; max_shard_len >= every shard_seqlens[b]; partial_o / partial_lse / num_splits as
 *   gemma_attn_decode (an empty shard writes lse = -inf, which the combine skips).
 *   Errors: GEMMA_ATTN_ERR_INVALID_ARG for a LOCAL or BIDIR kind or a bad flag, otherwise
 *   as gemma_attn_decode.
 */
int gemma_attn_decode_shard(const gemma_attn_params* params, const void* q, const void* new_k,
                            const void* k_cache, int32_t cache_capacity, const int32_t* shard_seqlens,
                            const int32_t* q_pos_offset, int32_t include_new, int32_t batch, int32_t n_q,
                            int32_t max_shard_len, float* partial_o, float* partial_lse,
                            int32_t num_splits, void* stream);

/* A split count for gemma_attn_decode that fills the GPU for this shape. For the shapes
 * of the tcgen05 verify kernel (a GLOBAL layer, head dim 256 or 512, 9..32 query rows per
 * KV head) it is twice the uniform-length choice, at most one split per 128 keys: that
 * kernel sizes its work items from the actual lengths and uses at most this many splits
 * per sequence. */
int gemma_attn_decode_num_splits(const gemma_attn_params* params, int32_t batch, int32_t n_q,
                                 int32_t max_cache_len, int32_t* num_splits);

/*
 * Combine split partials: out = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M) with
 * M = max_s lse_s; lse = M + log(sum_s exp(lse_s - M)).
 *   partial_o [num_splits, rows, head_dim] f32, partial_lse [num_splits, rows] f32 (device).
 *   out [rows, head_dim] (device, written): bf16 or f32 per out_dtype; lse [rows] f32 or NULL.
 */
int gemma_attn_combine(const float* partial_o, const float* partial_lse, int32_t num_splits,
                       int32_t rows, int32_t head_dim, int32_t out_dtype, void* out, float* lse,
                       void* stream);

/*
 * Host-side tile plan (the same rule the prefill kernels apply): for every sequence,
 * query tile of bm rows and key tile of bn keys with at least one visible pair, one
 * 4-tuple (sequence, q_tile, kv_tile, class) with class 1 = partially masked,
 * 2 = fully visible, ordered by sequence, q_tile, kv_tile. cu_seqlens is HOST memory.
 * Writes min(cap, count) tuples to out (may be NULL) and the count to *count.
 */
int gemma_attn_tile_plan(int32_t kind, int32_t window, const int32_t* cu_seqlens_host,
                         int32_t num_seqs, int32_t bm, int32_t bn, int32_t* out, int64_t cap,
                         int64_t* count);

/* Synchronise `stream`, return (and clear) the device status word: GEMMA_ATTN_OK,
 * GEMMA_ATTN_ERR_TIMEOUT or GEMMA_ATTN_ERR_SEQLEN; GEMMA_ATTN_ERR_DEVICE on a CUDA error. */
int gemma_attn_check(void* stream);

/* Static description of a status code. */
const char* gemma_attn_error_string(int status);

/* Number of kernel launches the last successful call on this host thread issued. */
int gemma_attn_last_launch_count(void);

/*
 * Diagnostic: one 128-row tile through each tensor-core operand form the prefill
 * kernel uses, for tests that recompute the product on the host. Device pointers:
 *   mode 0: a [128][128] bf16, b [128][128] bf16 (both K-major in shared memory);
 *           d [128][128] f32 = a * b^T.
 *   mode 1: p [128][128] bf16 staged through tensor memory, b [128][64] bf16 read
 *           MN-major; d [128][64] f32 = p * b.
 *   mode 2: as mode 1 with b [128][128] (two 64-column MN-major chunks, N = 128);
 *           d [128][128] f32 = p * b.
 * a must be NULL-or-ignored in modes 1 and 2, and p in mode 0.
 */
int gemma_attn_selftest_umma(int32_t mode, const void* a, const void* b, const void* p, float* d,
                             void* stream);

/*
 * Diagnostic of the failure path: launches one CTA that waits on an mbarrier nothing
 * arrives at. Every wait in the kernels is bounded (about 2 s of the GPU's global timer);
 * this one runs out, records a timeout in the device status word (the next
 * gemma_attn_check returns GEMMA_ATTN_ERR_TIMEOUT and clears it) and writes 1 to the
 * device int *gave_up. The context stays usable. The pages have no counterpart to it.
 */
int gemma_attn_selftest_timeout(int32_t* gave_up, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GEMMA_ATTN_H_ */
