// C ABI of the WUSH-KV hot path: argument checks on the host, then kernel launches
// on the caller's stream.  No allocation, no synchronization, no global state
// besides the per-thread text of the last CUDA error.  (The allocation-free decode
// entry, with its fixed scratch array, is in decode_noalloc.cu.)
#include <cmath>
#include <cstdio>
#include <cstring>

#include "wushkv_launch.h"

namespace wushkv {
cudaError_t launch_quantize_append_tc(const wushkv_cache& c, const void* k_new, const void* v_new, int n_new,
                                      const int32_t* start_pos, const float* Tk, int tkind, int tblock,
                                      int32_t* status, cudaStream_t stream);
cudaError_t launch_quantize_append_simt(const wushkv_cache& c, const void* k_new, const void* v_new,
                                        int in_dtype, int n_new, const int32_t* start_pos,
                                        const float* Tk, int32_t* status, cudaStream_t stream);
cudaError_t launch_quantize_append_small(const wushkv_cache& c, const void* k_new, const void* v_new, int n_new,
                                         const int32_t* start_pos, const float* Tk, int tkind, int tblock,
                                         const float* rope, int rope_rows, int32_t* status, cudaStream_t stream);
}

namespace {
thread_local char g_cuda_msg[256];
}  // namespace

namespace wushkv {
int record_cuda_error(cudaError_t e) {
  std::snprintf(g_cuda_msg, sizeof(g_cuda_msg), "CUDA error %d: %s", (int)e, cudaGetErrorString(e));
  return WUSHKV_ERR_CUDA;
}
}  // namespace wushkv

namespace {

int cuda_fail(cudaError_t e) { return wushkv::record_cuda_error(e); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape, quantizer and pointer checks shared by every call that takes a cache.  The
// clip multiplier only matters when quantizing (append), not when reading the cache.
int check_cache(const wushkv_cache* c, bool quantizing) {
  if (c == nullptr) return WUSHKV_ERR_INVALID;
  if (c->head_dim != WUSHKV_HEAD_DIM) return WUSHKV_ERR_UNSUPPORTED;
  if (c->qp.bits < 2 || c->qp.bits > 4) return WUSHKV_ERR_UNSUPPORTED;
  if (c->qp.kind != WUSHKV_QUEST_INT && c->qp.kind != WUSHKV_PCT_AFFINE) return WUSHKV_ERR_UNSUPPORTED;
  if (c->batch <= 0 || c->num_kv_heads <= 0 || c->capacity <= 0) return WUSHKV_ERR_INVALID;
  if ((int64_t)c->batch * c->num_kv_heads * c->capacity > (int64_t)1 << 40) return WUSHKV_ERR_INVALID;
  if (c->qp.kind == WUSHKV_QUEST_INT) {
    if (quantizing && (!(c->qp.clip_alpha > 0.0) || !std::isfinite(c->qp.clip_alpha))) return WUSHKV_ERR_INVALID;
  } else {
    if (c->qp.rank_lo < 0 || c->qp.rank_hi > WUSHKV_HEAD_DIM - 1) return WUSHKV_ERR_INVALID;
    if (c->qp.rank_lo >= c->qp.rank_hi) return WUSHKV_ERR_INVALID;
    if (c->qp.rank_lo > 2 || c->qp.rank_hi < WUSHKV_HEAD_DIM - 3) return WUSHKV_ERR_UNSUPPORTED;
  }
  if (c->block_table != nullptr) {      // paged pools: see wushkv_cache
    const int p = c->page_size;
    if (p < 16 || p > 4096 || (p & (p - 1)) != 0) return WUSHKV_ERR_INVALID;
    if (c->pages_per_seq <= 0 || c->num_pages <= 0) return WUSHKV_ERR_INVALID;
    if ((int64_t)c->pages_per_seq * p != c->capacity) return WUSHKV_ERR_INVALID;
    if ((int64_t)c->num_pages * c->num_kv_heads * p > (int64_t)1 << 40) return WUSHKV_ERR_INVALID;
    if (!aligned(c->block_table, 4)) return WUSHKV_ERR_MISALIGNED;
  }
  if (!c->k_codes || !c->v_codes || !c->k_meta || !c->v_meta) return WUSHKV_ERR_INVALID;
  if (!aligned(c->k_codes, 16) || !aligned(c->v_codes, 16)) return WUSHKV_ERR_MISALIGNED;
  if (!aligned(c->k_meta, 4) || !aligned(c->v_meta, 4)) return WUSHKV_ERR_MISALIGNED;
  return WUSHKV_OK;
}

int check_heads(int num_q_heads, int num_kv_heads) {
  if (num_q_heads <= 0 || num_kv_heads <= 0) return WUSHKV_ERR_INVALID;
  if (num_q_heads % num_kv_heads != 0) return WUSHKV_ERR_INVALID;
  const int g = num_q_heads / num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16) return WUSHKV_ERR_UNSUPPORTED;
  return WUSHKV_OK;
}

}  // namespace

extern "C" {

int wushkv_quantize_append(const wushkv_cache* cache, const void* k_new, const void* v_new,
                           int32_t in_dtype, int32_t n_new, const int32_t* start_pos,
                           const float* Tk, int32_t* status, void* stream) {
  int rc = check_cache(cache, true);
  if (rc != WUSHKV_OK) return rc;
  if (in_dtype != WUSHKV_BF16 && in_dtype != WUSHKV_FP32) return WUSHKV_ERR_UNSUPPORTED;
  if (n_new <= 0 || !k_new || !v_new || !start_pos) return WUSHKV_ERR_INVALID;
  if ((int64_t)cache->batch * n_new > (int64_t)1 << 30) return WUSHKV_ERR_INVALID;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(start_pos, 4)) return WUSHKV_ERR_MISALIGNED;
  if (Tk != nullptr && !aligned(Tk, 16)) return WUSHKV_ERR_MISALIGNED;
  if (status != nullptr && !aligned(status, 4)) return WUSHKV_ERR_MISALIGNED;
  // bf16 rows (the serving path) go through TMA + tcgen05, except a decode step's few
  // rows, which a latency-oriented kernel (one warp per group) takes; fp32 rows (exact
  // pre-transformed values, used to test the quantizer alone) go through the per-row
  // kernel.  All decide every code exactly for the fp32 value they quantize.
  constexpr int64_t kSmallAppendRows = 64;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (in_dtype == WUSHKV_BF16 && (int64_t)cache->batch * n_new <= kSmallAppendRows)
    e = wushkv::launch_quantize_append_small(*cache, k_new, v_new, n_new, start_pos, Tk, WUSHKV_TRANSFORM_DENSE, 0,
                                             nullptr, 0, status, st);
  else if (in_dtype == WUSHKV_BF16)
    e = wushkv::launch_quantize_append_tc(*cache, k_new, v_new, n_new, start_pos, Tk, WUSHKV_TRANSFORM_DENSE, 0,
                                          status, st);
  else
    e = wushkv::launch_quantize_append_simt(*cache, k_new, v_new, in_dtype, n_new, start_pos, Tk, status, st);
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

int wushkv_quantize_append_rope(const wushkv_cache* cache, const void* k_new, const void* v_new,
                                int32_t in_dtype, int32_t n_new, const int32_t* start_pos, const float* Tk,
                                const float* rope_table, int32_t rope_rows, int32_t* status, void* stream) {
  int rc = check_cache(cache, true);
  if (rc != WUSHKV_OK) return rc;
  if (in_dtype != WUSHKV_BF16 && in_dtype != WUSHKV_FP32) return WUSHKV_ERR_UNSUPPORTED;
  if (n_new <= 0 || !k_new || !v_new || !start_pos || !rope_table) return WUSHKV_ERR_INVALID;
  if (rope_rows < cache->capacity) return WUSHKV_ERR_INVALID;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(start_pos, 4) || !aligned(rope_table, 16))
    return WUSHKV_ERR_MISALIGNED;
  if (Tk != nullptr && !aligned(Tk, 16)) return WUSHKV_ERR_MISALIGNED;
  if (status != nullptr && !aligned(status, 4)) return WUSHKV_ERR_MISALIGNED;
  // fused RoPE is built for decode-step appends (bf16, at most 64 token rows per call)
  if (in_dtype != WUSHKV_BF16 || (int64_t)cache->batch * n_new > 64) return WUSHKV_ERR_UNSUPPORTED;
  cudaError_t e = wushkv::launch_quantize_append_small(*cache, k_new, v_new, n_new, start_pos, Tk,
                                                       WUSHKV_TRANSFORM_DENSE, 0, rope_table, rope_rows, status,
                                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

int wushkv_quantize_append_structured(const wushkv_cache* cache, const void* k_new, const void* v_new,
                                      int32_t in_dtype, int32_t n_new, const int32_t* start_pos, int32_t kind,
                                      int32_t block, const float* data, int32_t* status, void* stream) {
  if (kind == WUSHKV_TRANSFORM_DENSE) {
    if (data == nullptr) return WUSHKV_ERR_INVALID;
    return wushkv_quantize_append(cache, k_new, v_new, in_dtype, n_new, start_pos, data, status, stream);
  }
  if (kind != WUSHKV_TRANSFORM_BLOCK_DIAG && kind != WUSHKV_TRANSFORM_HADAMARD_DIAG) return WUSHKV_ERR_UNSUPPORTED;
  if (kind == WUSHKV_TRANSFORM_BLOCK_DIAG && block != 16 && block != 32 && block != 64) return WUSHKV_ERR_UNSUPPORTED;
  int rc = check_cache(cache, true);
  if (rc != WUSHKV_OK) return rc;
  if (in_dtype != WUSHKV_BF16 && in_dtype != WUSHKV_FP32) return WUSHKV_ERR_UNSUPPORTED;
  if (n_new <= 0 || !k_new || !v_new || !start_pos || !data) return WUSHKV_ERR_INVALID;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(start_pos, 4) || !aligned(data, 16))
    return WUSHKV_ERR_MISALIGNED;
  if (status != nullptr && !aligned(status, 4)) return WUSHKV_ERR_MISALIGNED;
  if (in_dtype != WUSHKV_BF16) return WUSHKV_ERR_UNSUPPORTED;
  if ((int64_t)cache->batch * n_new > (int64_t)1 << 30) return WUSHKV_ERR_INVALID;
  const int tblock = kind == WUSHKV_TRANSFORM_BLOCK_DIAG ? block : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = (int64_t)cache->batch * n_new <= 64
                      ? wushkv::launch_quantize_append_small(*cache, k_new, v_new, n_new, start_pos, data, kind,
                                                             tblock, nullptr, 0, status, st)
                      : wushkv::launch_quantize_append_tc(*cache, k_new, v_new, n_new, start_pos, data, kind, tblock,
                                                          status, st);
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

int wushkv_transform_query_structured(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t kind, int32_t block, const float* data,
                                      float* q_out, void* stream) {
  if (kind == WUSHKV_TRANSFORM_DENSE)
    return wushkv_transform_query(q, q_dtype, batch, num_q_heads, num_kv_heads, data, q_out, stream);
  if (kind != WUSHKV_TRANSFORM_BLOCK_DIAG && kind != WUSHKV_TRANSFORM_HADAMARD_DIAG) return WUSHKV_ERR_UNSUPPORTED;
  if (kind == WUSHKV_TRANSFORM_BLOCK_DIAG && block != 16 && block != 32 && block != 64) return WUSHKV_ERR_UNSUPPORTED;
  if (q_dtype != WUSHKV_BF16 && q_dtype != WUSHKV_FP32) return WUSHKV_ERR_UNSUPPORTED;
  int rc = check_heads(num_q_heads, num_kv_heads);
  if (rc != WUSHKV_OK) return rc;
  if (batch <= 0 || !q || !data || !q_out) return WUSHKV_ERR_INVALID;
  if (batch > 65535) return WUSHKV_ERR_INVALID;
  if ((const void*)q == (const void*)q_out) return WUSHKV_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(data, 16) || !aligned(q_out, 16)) return WUSHKV_ERR_MISALIGNED;
  cudaError_t e = wushkv::launch_transform_query_structured(q, q_dtype, batch, num_q_heads, num_kv_heads, kind,
                                                            kind == WUSHKV_TRANSFORM_BLOCK_DIAG ? block : 0, data,
                                                            q_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

int wushkv_transform_query(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                           int32_t num_kv_heads, const float* Tk_invT, float* q_out, void* stream) {
  if (q_dtype != WUSHKV_BF16 && q_dtype != WUSHKV_FP32) return WUSHKV_ERR_UNSUPPORTED;
  int rc = check_heads(num_q_heads, num_kv_heads);
  if (rc != WUSHKV_OK) return rc;
  if (batch <= 0 || !q || !Tk_invT || !q_out) return WUSHKV_ERR_INVALID;
  if ((const void*)q == (const void*)q_out) return WUSHKV_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(Tk_invT, 16) || !aligned(q_out, 16)) return WUSHKV_ERR_MISALIGNED;
  cudaError_t e = wushkv::launch_transform_query(q, q_dtype, batch, num_q_heads, num_kv_heads, Tk_invT,
                                                 q_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

size_t wushkv_chunk_workspace_bytes(const wushkv_cache* cache, int32_t num_q_heads, int32_t n_q,
                                    int32_t num_splits) {
  if (check_cache(cache, false) != WUSHKV_OK) return 0;
  if (check_heads(num_q_heads, cache->num_kv_heads) != WUSHKV_OK) return 0;
  if (n_q < 1 || n_q > WUSHKV_MAX_CHUNK || num_splits < 0 || num_splits > 4096) return 0;
  return wushkv::chunk_workspace_bytes(*cache, num_q_heads, n_q, num_splits);
}

int wushkv_chunk_attention(const wushkv_cache* cache, const float* q_t, int32_t n_q, int32_t num_q_heads,
                           const int32_t* ctx_len, float softmax_scale, float* out, void* workspace,
                           size_t workspace_bytes, int32_t num_splits, int32_t* status, void* stream) {
  int rc = check_cache(cache, false);
  if (rc != WUSHKV_OK) return rc;
  rc = check_heads(num_q_heads, cache->num_kv_heads);
  if (rc != WUSHKV_OK) return rc;
  if (n_q < 1 || n_q > WUSHKV_MAX_CHUNK) return WUSHKV_ERR_INVALID;
  if (!q_t || !ctx_len || !out || !workspace) return WUSHKV_ERR_INVALID;
  if ((const void*)q_t == (const void*)out) return WUSHKV_ERR_INVALID;
  if (num_splits < 0 || num_splits > 4096) return WUSHKV_ERR_INVALID;
  if (!std::isfinite(softmax_scale)) return WUSHKV_ERR_INVALID;
  if (!aligned(q_t, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(ctx_len, 4))
    return WUSHKV_ERR_MISALIGNED;
  if (status != nullptr && !aligned(status, 4)) return WUSHKV_ERR_MISALIGNED;
  if (workspace_bytes < wushkv::chunk_workspace_bytes(*cache, num_q_heads, n_q, num_splits))
    return WUSHKV_ERR_WORKSPACE;
  cudaError_t e = wushkv::launch_chunk_attention(*cache, q_t, n_q, num_q_heads, ctx_len, softmax_scale, out,
                                                 workspace, num_splits, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

size_t wushkv_decode_workspace_bytes(const wushkv_cache* cache, int32_t num_q_heads, int32_t num_splits) {
  if (check_cache(cache, false) != WUSHKV_OK) return 0;
  if (check_heads(num_q_heads, cache->num_kv_heads) != WUSHKV_OK) return 0;
  if (num_splits < 0 || num_splits > 4096) return 0;
  return wushkv::decode_workspace_bytes(*cache, num_q_heads, num_splits);
}

int wushkv_decode_attention(const wushkv_cache* cache, const float* q_t, int32_t num_q_heads,
                            const int32_t* ctx_len, float softmax_scale, float* out,
                            void* workspace, size_t workspace_bytes, int32_t num_splits,
                            int32_t* status, void* stream) {
  int rc = check_cache(cache, false);
  if (rc != WUSHKV_OK) return rc;
  rc = check_heads(num_q_heads, cache->num_kv_heads);
  if (rc != WUSHKV_OK) return rc;
  if (!q_t || !ctx_len || !out || !workspace) return WUSHKV_ERR_INVALID;
  if (num_splits < 0 || num_splits > 4096) return WUSHKV_ERR_INVALID;
  if (!std::isfinite(softmax_scale)) return WUSHKV_ERR_INVALID;
  if (!aligned(q_t, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(ctx_len, 4))
    return WUSHKV_ERR_MISALIGNED;
  if (status != nullptr && !aligned(status, 4)) return WUSHKV_ERR_MISALIGNED;
  if (workspace_bytes < wushkv::decode_workspace_bytes(*cache, num_q_heads, num_splits))
    return WUSHKV_ERR_WORKSPACE;
  cudaError_t e = wushkv::launch_decode_attention(*cache, q_t, num_q_heads, ctx_len, softmax_scale, out,
                                                  workspace, num_splits, status,
                                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : cuda_fail(e);
}

const char* wushkv_strerror(int code) {
  switch (code) {
    case WUSHKV_OK: return "ok";
    case WUSHKV_ERR_INVALID: return "invalid argument";
    case WUSHKV_ERR_UNSUPPORTED: return "unsupported configuration (bits, kind, dtype, head_dim or group size)";
    case WUSHKV_ERR_MISALIGNED: return "misaligned pointer";
    case WUSHKV_ERR_WORKSPACE: return "workspace too small";
    case WUSHKV_ERR_CUDA: return g_cuda_msg[0] ? g_cuda_msg : "CUDA error";
    default: return "unknown error code";
  }
}

const char* wushkv_version(void) { return "wushkv 0.1.0 (sm_100a)"; }

}  // extern "C"
