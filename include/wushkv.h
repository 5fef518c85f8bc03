/*
 * wushkv.h - C ABI of the WUSH-KV runtime hot path on one NVIDIA B200 (sm_100a).
 *
 * The method: WUSH-KV (preprint "WUSH-KV: KV Cache Quantization with
 * Data-Adaptive Transforms").  Its only published description here is a set of
 * summary pages; the passages each call follows are named below as
 *   [ai4s N]  ai4snews summary "WUSH-KV cuts 2-bit KV-cache perplexity from
 *             OSCAR's 13.74 to 10.51 ...", paragraph N (1-6),
 *   [blog]    cere-bro page "WUSH-KV: 2-bit KV-Cache Quantization with
 *             Data-Adaptive Transforms" (TL;DR, flowchart, Gaps),
 *   [abs]     the arXiv abstract as listed by readsearch.ai and searcharxiv.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless a parameter says otherwise.  All
 *     buffers are owned by the caller; the library never allocates, frees or
 *     synchronizes.  Every call enqueues work on `stream` (a cudaStream_t, or
 *     NULL for the legacy default stream) and returns immediately.
 *   - head_dim is 128 and one quantization group is one (token, KV head) row of
 *     128 values.
 *   - Return value: WUSHKV_OK, or a negative wushkv_error.  Argument errors are
 *     detected on the host before anything is enqueued.  Problems only visible
 *     on the device (see WUSHKV_STATUS_*) are OR-ed into the optional `status`
 *     int32 (device memory, caller clears it); no kernel ever traps.
 *   - Calls keep no state between them and are safe to issue from several
 *     host threads on different streams (except wushkv_decode_attention_noalloc,
 *     whose fixed scratch array is shared; see its declaration).
 */
#ifndef WUSHKV_H_
#define WUSHKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WUSHKV_API __attribute__((visibility("default")))
#else
#define WUSHKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define WUSHKV_HEAD_DIM 128

typedef enum {
  WUSHKV_OK = 0,
  WUSHKV_ERR_INVALID = -1,      /* null pointer, non-positive size, bad rank pair, ... */
  WUSHKV_ERR_UNSUPPORTED = -2,  /* bits not in {2,3,4}, unknown kind/dtype, head_dim != 128 */
  WUSHKV_ERR_MISALIGNED = -3,   /* a pointer is not 16-byte aligned */
  WUSHKV_ERR_WORKSPACE = -4,    /* workspace smaller than wushkv_decode_workspace_bytes() */
  WUSHKV_ERR_CUDA = -5          /* a CUDA runtime call or kernel launch failed */
} wushkv_error;

/* Device-side conditions, OR-ed into *status (never a trap). */
#define WUSHKV_STATUS_CAPACITY 1       /* start_pos[b] + t >= capacity: that row was not written */
#define WUSHKV_STATUS_NONFINITE 2      /* a group had a NaN/Inf input: its codes are unspecified */
#define WUSHKV_STATUS_META_OVERFLOW 4  /* a step/scale/zero overflowed fp16 (stored as Inf) */
#define WUSHKV_STATUS_CTX_OVERFLOW 8   /* ctx_len[b] > capacity: clamped to capacity */
#define WUSHKV_STATUS_TIMEOUT 16       /* an internal pipeline wait gave up; output unspecified */
#define WUSHKV_STATUS_BAD_PAGE 32      /* a block-table entry outside [0, num_pages): that row was
                                          not written (append) or was left out (decode) */

/* Quantizer family [ai4s 3-5], [abs]:
 *  QUEST_INT  - QuEST-INT-style symmetric RMS-clipped grid (the quantizer of the
 *               pages' theory and perplexity runs).  Per group:
 *               Delta = fp16(clip_alpha * RMS * 2^(1-bits)), RMS = sqrt(sum x^2 / 128);
 *               code = clamp(floor(x / Delta) + 2^(bits-1), 0, 2^bits - 1);
 *               x_hat = (code - 2^(bits-1) + 1/2) * Delta.  One fp16 meta value (Delta).
 *  PCT_AFFINE - OSCAR-style percentile-clipped affine grid (the quantizer of the
 *               SGLang runs).  lo, hi = elements of 0-based ascending rank
 *               rank_lo, rank_hi; scale = fp16((hi - lo) / (2^bits - 1));
 *               zero = fp16(lo); code = clamp(round_half_even((x - zero) / scale),
 *               0, 2^bits - 1); x_hat = zero + code * scale.  Two fp16 meta values
 *               (scale, zero), in that order.
 * fp16 conversions round to nearest even once; codes are decided by exact
 * comparisons with the grid's thresholds.  Delta == 0 gives code 2^(bits-1);
 * scale == 0 gives code 0. */
typedef enum { WUSHKV_QUEST_INT = 0, WUSHKV_PCT_AFFINE = 1 } wushkv_quant_kind;

typedef enum { WUSHKV_BF16 = 0, WUSHKV_FP32 = 1 } wushkv_dtype;

typedef struct {
  int32_t kind;        /* wushkv_quant_kind */
  int32_t bits;        /* 2, 3 or 4 */
  double clip_alpha;   /* QUEST_INT clip multiplier (e.g. 1.99 / 2.34 / 2.68 for 2 / 3 / 4 bits); > 0 */
  int32_t rank_lo;     /* PCT_AFFINE ranks; supported: 0 <= rank_lo <= 2, 125 <= rank_hi <= 127 */
  int32_t rank_hi;
} wushkv_quant_params;

/* The packed KV cache of one layer (host struct describing caller-owned device memory).
 *   k_codes, v_codes: uint8 [batch][num_kv_heads][capacity][16*bits].  Row
 *       (b, h, t) is the LSB-first bit string of the group's 128 codes: code i at
 *       bits [bits*i, bits*i + bits), bit n is bit (n mod 8) of byte n / 8.
 *   k_meta, v_meta: fp16 bit patterns [batch][num_kv_heads][capacity][m], m = 1
 *       (Delta) for QUEST_INT, m = 2 (scale, zero) for PCT_AFFINE.
 *   Keys are stored in the transformed basis x = T_k k [ai4s 5]; values are stored
 *   as given, since their transform is folded into the model weights [ai4s 5],
 *   [blog flowchart].  Code pointers must be 16-byte aligned, meta pointers
 *   4-byte aligned.
 * Paged layout (an addition of this library for serving engines that allocate the
 * cache in pages; the pages do not describe one): with block_table != NULL the four
 * buffers are pools of num_pages pages, codes [num_pages][num_kv_heads][page_size]
 * [16*bits] and meta [num_pages][num_kv_heads][page_size][m]; position t of sequence b
 * is row t % page_size of page block_table[b * pages_per_seq + t / page_size].
 * page_size is a power of two in [16, 4096] and capacity = pages_per_seq * page_size.
 * block_table is int32 device memory, caller-owned and never modified; entries
 * outside [0, num_pages) are skipped with WUSHKV_STATUS_BAD_PAGE.  With block_table ==
 * NULL the three paging fields are ignored. */
typedef struct {
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint16_t* k_meta;
  uint16_t* v_meta;
  int32_t batch;
  int32_t num_kv_heads;
  int32_t capacity;    /* T_max, tokens per sequence */
  int32_t head_dim;    /* must be 128 */
  wushkv_quant_params qp;
  const int32_t* block_table;   /* NULL: contiguous layout; else [batch][pages_per_seq] */
  int32_t pages_per_seq;
  int32_t page_size;
  int32_t num_pages;
} wushkv_cache;

/* Key transform + clipped quantization + bit-packing + append.
 * [ai4s 1]: one key transform per KV head; [ai4s 5], [blog TL;DR], [abs]: it is
 * applied to post-RoPE keys online; keys and values are then quantized per token
 * with a clipped quantizer and written to the cache.
 *   k_new, v_new : [batch][n_new][num_kv_heads][128], dtype in_dtype, contiguous,
 *                  16-byte aligned.  k_new must already be post-RoPE.
 *   n_new        : tokens per sequence in this call (>= 1).
 *   start_pos    : int32 [batch] (device); row t of sequence b goes to position
 *                  start_pos[b] + t.  Positions >= capacity are skipped
 *                  (WUSHKV_STATUS_CAPACITY).  Not modified.
 *   Tk           : fp32 [num_kv_heads][128][128] row-major, x_i = sum_j Tk[h][i][j] k_j;
 *                  NULL means identity (the keys are taken as already transformed,
 *                  which is how the quantizer is tested on exact fp32 inputs).
 *   status       : optional int32 (device).
 * Routing: bf16 calls of at most 64 token rows (batch * n_new) take a latency
 * kernel (FFMA transform, one warp per 128-value group); larger bf16 calls run the
 * transform on the tensor cores with Tk split exactly into three bf16 parts
 * (products exact, fp32 accumulation); fp32 inputs take an FFMA kernel.  In every
 * case the quantizer works on the fp32 transform result and values never pass
 * through the transform. */
WUSHKV_API int wushkv_quantize_append(const wushkv_cache* cache, const void* k_new, const void* v_new,
                           int32_t in_dtype, int32_t n_new, const int32_t* start_pos,
                           const float* Tk, int32_t* status, void* stream);

/* wushkv_quantize_append with RoPE fused in front of the key transform ([ai4s 5]: the
 * transform is applied to keys after RoPE).  k_new holds the keys BEFORE RoPE; the key
 * of position p = start_pos[b] + t is rotated in rotate-half pairs (c, c + 64), c < 64:
 *   (x, y) -> (x cos_c - y sin_c, y cos_c + x sin_c),
 * with cos_c = rope_table[p][c] and sin_c = rope_table[p][64 + c], in fp32 and without
 * rounding the rotated key, then transformed, quantized and appended as
 * wushkv_quantize_append does.  Values are not rotated.
 *   rope_table : fp32 [rope_rows][128] (device, caller-owned, 16-byte aligned), the
 *                serving engine's cos/sin cache; rope_rows >= capacity.
 * Built for decode-step appends: bf16 inputs and batch * n_new <= 64 token rows;
 * other calls return WUSHKV_ERR_UNSUPPORTED (rotate first, then call
 * wushkv_quantize_append).  Other arguments, errors and status bits as
 * wushkv_quantize_append. */
WUSHKV_API int wushkv_quantize_append_rope(const wushkv_cache* cache, const void* k_new, const void* v_new,
                                int32_t in_dtype, int32_t n_new, const int32_t* start_pos, const float* Tk,
                                const float* rope_table, int32_t rope_rows, int32_t* status, void* stream);

/* Key transform families ([ai4s 6]: cheaper structured transforms are the authors'
 * future work; Hadamard is a baseline), all invertible T_k applied as x = T_k k:
 *   DENSE         - data fp32 [Hkv][128][128] row-major (as Tk above);
 *   BLOCK_DIAG    - data fp32 [Hkv][128/b][b][b]: block j (row-major) acts on channels
 *                   [j b, (j+1) b), b = 16, 32 or 64;
 *   HADAMARD_DIAG - data fp32 s [Hkv][128]: T_k = H diag(s) / sqrt(128), H the
 *                   Sylvester Hadamard matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]);
 *                   its query map is the same family with 1/s. */
typedef enum {
  WUSHKV_TRANSFORM_DENSE = 1,
  WUSHKV_TRANSFORM_BLOCK_DIAG = 2,
  WUSHKV_TRANSFORM_HADAMARD_DIAG = 3
} wushkv_transform_kind;

/* wushkv_quantize_append with a structured key transform.  kind is a
 * wushkv_transform_kind; block is b for BLOCK_DIAG (ignored otherwise); data is device
 * fp32, 16-byte aligned, laid out as above.  DENSE takes every call
 * wushkv_quantize_append takes.  The structured kinds take bf16 inputs: decode-step
 * appends (batch * n_new <= 64 token rows) cost b instead of 128 multiply-adds per
 * channel (block-diagonal) or a scale and a seven-stage butterfly (Hadamard-diagonal);
 * larger appends expand the transform into the tensor-core kernel's exact bf16 parts
 * of T_k and cost the same as a dense one.  fp32 inputs return WUSHKV_ERR_UNSUPPORTED.
 * Results equal wushkv_quantize_append given the expanded dense T_k up to the fp32
 * rounding of the transform; for BLOCK_DIAG they are identical to the dense path of the
 * same size given the expanded matrix.  Other arguments, errors and status bits as
 * wushkv_quantize_append. */
WUSHKV_API int wushkv_quantize_append_structured(const wushkv_cache* cache, const void* k_new, const void* v_new,
                                      int32_t in_dtype, int32_t n_new, const int32_t* start_pos, int32_t kind,
                                      int32_t block, const float* data, int32_t* status, void* stream);

/* Decode-query map q' = T_k^{-T} q, with T_k of the query head's KV head h / g,
 * g = num_q_heads / num_kv_heads.  Needed because keys are cached as T_k k, and
 * (T_k^{-T} q) . (T_k k) = q . k keeps the attention scores unchanged (implied by
 * [ai4s 5]: keys are transformed online after RoPE while attention stays exact).
 *   q       : [batch][num_q_heads][128], dtype q_dtype, contiguous, 16-byte aligned.
 *   Tk_invT : fp32 [num_kv_heads][128][128] row-major (the caller computes the
 *             inverse-transpose once per layer, off the hot path).
 *   q_out   : fp32 [batch][num_q_heads][128]; may not alias q. */
WUSHKV_API int wushkv_transform_query(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                           int32_t num_kv_heads, const float* Tk_invT, float* q_out, void* stream);

/* wushkv_transform_query for the structured key transforms above: the query is mapped
 * by T_k^{-T} of the head's KV head ([ai4s 6]: cheaper structured transforms), given as
 *   DENSE         - data = T_k^{-T}, fp32 [Hkv][128][128] (exactly wushkv_transform_query);
 *   BLOCK_DIAG    - data = the blocks of T_k^{-T}, fp32 [Hkv][128/b][b][b] (block j of T_k
 *                   inverted and transposed, computed once per layer by the caller), b = block;
 *   HADAMARD_DIAG - data = s, fp32 [Hkv][128], the same scales as the key transform
 *                   (T_k^{-T} = H diag(1/s) / sqrt(128), since H / sqrt(128) is symmetric
 *                   and orthogonal); every s must be nonzero.
 * kind is a wushkv_transform_kind; block is 16, 32 or 64 for BLOCK_DIAG and ignored
 * otherwise; data is device memory, 16-byte aligned.  Other arguments and errors as
 * wushkv_transform_query. */
WUSHKV_API int wushkv_transform_query_structured(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t kind, int32_t block, const float* data,
                                      float* q_out, void* stream);

/* Bytes of decode workspace needed for wushkv_decode_attention with the same
 * cache shape, num_q_heads and num_splits (0 = the automatic split count, else
 * 1 .. 4096).  Returns 0 for invalid arguments.  Host only: it enqueues nothing (the
 * automatic split count reads the current device's SM count). */
WUSHKV_API size_t wushkv_decode_workspace_bytes(const wushkv_cache* cache, int32_t num_q_heads,
                                     int32_t num_splits);

/* Split-K GQA decode attention directly over the packed cache ([ai4s 5]: serving
 * with grouped-query attention over a 2-bit cache; long contexts [ai4s 4]).
 * For each sequence b and query head h (KV head h / g):
 *   s_t = softmax_scale * q_t[b][h] . k_hat_t,  t < ctx_len[b]
 *   out[b][h] = sum_t softmax(s)_t * v_hat_t   (in the transformed value basis).
 *   q_t        : fp32 [batch][num_q_heads][128] from wushkv_transform_query.
 *   ctx_len    : int32 [batch] (device), cached tokens per sequence; 0 gives a zero
 *                row; values > capacity are clamped (WUSHKV_STATUS_CTX_OVERFLOW).
 *   out        : fp32 [batch][num_q_heads][128].
 *   workspace  : scratch of at least wushkv_decode_workspace_bytes() bytes,
 *                16-byte aligned; contents on entry are ignored.
 *   num_splits : splits of each sequence's context (0 = automatic). */
WUSHKV_API int wushkv_decode_attention(const wushkv_cache* cache, const float* q_t, int32_t num_q_heads,
                            const int32_t* ctx_len, float softmax_scale, float* out,
                            void* workspace, size_t workspace_bytes, int32_t num_splits,
                            int32_t* status, void* stream);

/* Size of the fixed decode scratch array used by wushkv_decode_attention_noalloc:
 * 8 MiB of device memory per device, enough for the automatic split count of e.g.
 * batch 32 x 64 query heads at 8K context or batch 16 x 32 heads at 32K. */
#define WUSHKV_DECODE_STATIC_SCRATCH_BYTES (8u << 20)

/* wushkv_decode_attention without a workspace argument (an addition of this
 * library; the method on the pages has no counterpart).  The split partials go to
 * a fixed array of WUSHKV_DECODE_STATIC_SCRATCH_BYTES in the library's own device
 * memory, so the call allocates nothing.  It is meant for callers that cannot give
 * the library scratch memory: a plugin in a host runtime that owns every device
 * allocation and offers extensions no allocator, or a serving loop that forbids
 * allocation after start-up to keep its device-memory footprint fixed.
 *   Arguments, results and errors are those of wushkv_decode_attention, except:
 *   - WUSHKV_ERR_WORKSPACE when wushkv_decode_workspace_bytes(cache, num_q_heads,
 *     num_splits) exceeds WUSHKV_DECODE_STATIC_SCRATCH_BYTES (pass a smaller
 *     num_splits, or use wushkv_decode_attention with a workspace);
 *   - the first call on each device looks up the array's device address in the
 *     device's current CUDA context (a CUDA runtime call, no allocation by this
 *     library) and keeps it for later calls in that context; a call in a new context
 *     on the device (for instance after cudaDeviceReset) looks it up again.  Make the
 *     first call on a device, and the first after a reset, before any stream capture
 *     on that device;
 *   - every call on a device shares the one array and leaves its partials there;
 *     nothing in it needs clearing between calls (each call writes every partial it
 *     reads), but calls that may overlap in time on one device (different streams,
 *     unordered host threads) race on it and must be serialised by the caller. */
WUSHKV_API int wushkv_decode_attention_noalloc(const wushkv_cache* cache, const float* q_t,
                                    int32_t num_q_heads, const int32_t* ctx_len, float softmax_scale,
                                    float* out, int32_t num_splits, int32_t* status, void* stream);

/* Largest number of queries per sequence that wushkv_chunk_attention takes. */
#define WUSHKV_MAX_CHUNK 16

/* Bytes of workspace needed for wushkv_chunk_attention with the same cache shape,
 * num_q_heads, n_q and num_splits.  Returns 0 for invalid arguments.  Host only. */
WUSHKV_API size_t wushkv_chunk_workspace_bytes(const wushkv_cache* cache, int32_t num_q_heads, int32_t n_q,
                                    int32_t num_splits);

/* Causal attention of a chunk of n_q queries per sequence over the packed cache
 * ([ai4s 3]: perplexity runs feed each sequence in 16-token forward chunks).  The
 * chunk's tokens must already be appended (wushkv_quantize_append), so every key and
 * value is read in packed form.  With ctx = min(ctx_len[b], capacity), query i of
 * sequence b sits at position ctx - n_q + i and attends positions 0 .. ctx - n_q + i:
 *   s_t = softmax_scale * q_t[b][i][h] . k_hat_t,
 *   out[b][i][h] = sum_t softmax(s)_t * v_hat_t   (KV head h / g).
 * A query whose position is negative (ctx < n_q - i) gives a zero row.
 *   q_t        : fp32 [batch][n_q][num_q_heads][128], each query mapped by
 *                wushkv_transform_query (batch * n_q rows); 16-byte aligned.
 *   n_q        : 1 .. WUSHKV_MAX_CHUNK.
 *   ctx_len    : int32 [batch] (device), cached tokens including the chunk; values
 *                > capacity are clamped (WUSHKV_STATUS_CTX_OVERFLOW).
 *   out        : fp32 [batch][n_q][num_q_heads][128]; may not alias q_t.
 *   workspace  : at least wushkv_chunk_workspace_bytes() bytes, 16-byte aligned.
 *   num_splits : splits of the cached positions (1 .. 4096); 0 = automatic.
 * The chunk's queries are folded into the head group (row i * g + h) and run on the
 * tensor cores 128 rows at a time, so the cache is read once per (sequence, KV head)
 * and block of 128 rows; the workspace holds one fp32 partial (m, l, o) per row and
 * split, merged by a second launch.  Results do not depend on num_splits beyond fp32
 * rounding.  Errors as wushkv_decode_attention. */
WUSHKV_API int wushkv_chunk_attention(const wushkv_cache* cache, const float* q_t, int32_t n_q,
                           int32_t num_q_heads, const int32_t* ctx_len, float softmax_scale, float* out,
                           void* workspace, size_t workspace_bytes, int32_t num_splits, int32_t* status,
                           void* stream);

/* Static text for a wushkv_error code, or the last CUDA error text for WUSHKV_ERR_CUDA
 * on the calling thread. */
WUSHKV_API const char* wushkv_strerror(int code);

/* Library version string. */
WUSHKV_API const char* wushkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WUSHKV_H_ */
