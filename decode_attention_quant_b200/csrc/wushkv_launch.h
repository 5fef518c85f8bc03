// Internal launcher interface between the C ABI (abi.cu) and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/wushkv.h"

namespace wushkv {

// Stores the text of a CUDA error for wushkv_strerror on this thread; returns WUSHKV_ERR_CUDA.
int record_cuda_error(cudaError_t e);

cudaError_t launch_quantize_append(const wushkv_cache& c, const void* k_new, const void* v_new,
                                   int in_dtype, int n_new, const int32_t* start_pos,
                                   const float* Tk, int32_t* status, cudaStream_t stream);

cudaError_t launch_transform_query(const void* q, int q_dtype, int batch, int num_q_heads,
                                   int num_kv_heads, const float* Tk_invT, float* q_out,
                                   cudaStream_t stream);

// Query map by a structured transform's inverse-transpose (kind: wushkv_transform_kind).
cudaError_t launch_transform_query_structured(const void* q, int q_dtype, int batch, int num_q_heads,
                                              int num_kv_heads, int kind, int block, const float* data,
                                              float* q_out, cudaStream_t stream);

// Split count used when the caller passes num_splits = 0.
int auto_num_splits(const wushkv_cache& c, int num_q_heads);
size_t decode_workspace_bytes(const wushkv_cache& c, int num_q_heads, int num_splits);

cudaError_t launch_decode_attention(const wushkv_cache& c, const float* q_t, int num_q_heads,
                                    const int32_t* ctx_len, float softmax_scale, float* out,
                                    void* workspace, int num_splits, int32_t* status,
                                    cudaStream_t stream);

// Combine of log2-domain split partials (m, l, pad, pad, o[128] per row and split) into
// fp32 rows of 128: out[r] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
cudaError_t launch_combine_partials(const float* ws, int rows, int num_splits, float* out, cudaStream_t stream);

// Chunk attention (chunk_fa.cu): workspace bytes and the call.
size_t chunk_workspace_bytes(const wushkv_cache& c, int num_q_heads, int n_q, int num_splits);
cudaError_t launch_chunk_attention(const wushkv_cache& c, const float* q_t, int n_q, int num_q_heads,
                                   const int32_t* ctx_len, float softmax_scale, float* out, void* workspace,
                                   int num_splits, int32_t* status, cudaStream_t stream);

}  // namespace wushkv
