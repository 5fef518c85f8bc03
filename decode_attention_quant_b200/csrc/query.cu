// Decode-query map q' = T_k^{-T} q per query head, with T_k of the head's KV group.
//
// Keys are cached in the transformed basis x = T_k k (WUSH-KV: the key transform is
// applied online after RoPE, ai4snews summary paragraph 5), so scores are kept
// exact by mapping the query with the inverse-transpose: (T^{-T} q) . (T k) = q . k.
// One CTA = one KV head of one sequence (its g query heads); thread i owns output
// channel i, keeps row i of T_k^{-T} in registers and sums each product in four
// interleaved chains, so the short launch is not one long dependent FMA chain.
#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

constexpr int kBatchPerCta = 1;

template <bool BF16_IN>
__global__ void __launch_bounds__(kHeadDim) transform_query_kernel(
    const void* __restrict__ q, int batch, int hq, int hkv, const float* __restrict__ m,
    float* __restrict__ out) {
  extern __shared__ __align__(16) float qs[];   // [kBatchPerCta * g][128]
  const int kv = blockIdx.x, b0 = blockIdx.y * kBatchPerCta, i = threadIdx.x;
  const int g = hq / hkv;
  const int nb = min(kBatchPerCta, batch - b0);
  for (int e = i; e < nb * g * kHeadDim; e += kHeadDim) {
    const int r = e / kHeadDim, c = e % kHeadDim;
    const int b = b0 + r / g, h = kv * g + r % g;
    const size_t off = ((size_t)b * hq + h) * kHeadDim + c;
    qs[e] = BF16_IN ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                    : static_cast<const float*>(q)[off];
  }
  float mr[kHeadDim];
  const float4* mrow = reinterpret_cast<const float4*>(m + ((size_t)kv * kHeadDim + i) * kHeadDim);
#pragma unroll
  for (int j = 0; j < kHeadDim / 4; ++j) {
    const float4 v = __ldg(mrow + j);
    mr[4 * j] = v.x; mr[4 * j + 1] = v.y; mr[4 * j + 2] = v.z; mr[4 * j + 3] = v.w;
  }
  __syncthreads();
#pragma unroll 1
  for (int r = 0; r < nb * g; ++r) {
    const float4* qr = reinterpret_cast<const float4*>(qs + r * kHeadDim);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j) {
      const float4 v = qr[j];
      a0 = fmaf(mr[4 * j], v.x, a0);
      a1 = fmaf(mr[4 * j + 1], v.y, a1);
      a2 = fmaf(mr[4 * j + 2], v.z, a2);
      a3 = fmaf(mr[4 * j + 3], v.w, a3);
    }
    const int b = b0 + r / g, h = kv * g + r % g;
    out[((size_t)b * hq + h) * kHeadDim + i] = (a0 + a1) + (a2 + a3);
  }
}

// Structured maps (the inverse-transposes of the structured key transforms):
//   block-diagonal: q'_i = sum_j B[i / b][i % b][j] q_{(i / b) b + j}, with B the blocks of
//                   T_k^{-T} (block j of T_k inverted and transposed by the caller);
//   Hadamard-diagonal: T_k = H diag(s) / sqrt(128) gives T_k^{-T} = H diag(1/s) / sqrt(128)
//                   (H / sqrt(128) is symmetric and orthogonal), so q' is the seven-stage
//                   butterfly of the Sylvester Hadamard transform applied to q / s, times
//                   1 / sqrt(128).
// One CTA = one KV head of one sequence; thread i owns channel i.
template <bool BF16_IN, int TF>
__global__ void __launch_bounds__(kHeadDim) transform_query_structured_kernel(
    const void* __restrict__ q, int batch, int hq, int hkv, int block, const float* __restrict__ data,
    float* __restrict__ out) {
  __shared__ __align__(16) float qs[kHeadDim];
  const int kv = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
  const int g = hq / hkv;
  float coef = 0.f;
  if (TF == WUSHKV_TRANSFORM_HADAMARD_DIAG) coef = __ldg(data + (size_t)kv * kHeadDim + i);
#pragma unroll 1
  for (int hh = 0; hh < g; ++hh) {
    const int h = kv * g + hh;
    const size_t off = ((size_t)b * hq + h) * kHeadDim;
    const float qv = BF16_IN ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off + i])
                             : static_cast<const float*>(q)[off + i];
    float r;
    if (TF == WUSHKV_TRANSFORM_BLOCK_DIAG) {
      qs[i] = qv;
      __syncthreads();
      const int blk = i / block, ii = i % block;
      const float* brow = data + (((size_t)kv * (kHeadDim / block) + blk) * block + ii) * block;
      const float* qb = qs + blk * block;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int j = 0; j < block; j += 4) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(brow + j));
        a0 = fmaf(t.x, qb[j], a0);
        a1 = fmaf(t.y, qb[j + 1], a1);
        a2 = fmaf(t.z, qb[j + 2], a2);
        a3 = fmaf(t.w, qb[j + 3], a3);
      }
      r = (a0 + a1) + (a2 + a3);
    } else {
      qs[i] = __fdiv_rn(qv, coef);
      __syncthreads();
      // stage `half` pairs channels base and base + half; thread i owns one side of a pair
      for (int half = kHeadDim / 2; half >= 1; half >>= 1) {
        const int partner = i ^ half;
        const float u = qs[i], w = qs[partner];
        __syncthreads();
        qs[i] = (i & half) ? (w - u) : (u + w);
        __syncthreads();
      }
      r = qs[i] * 0.08838834764831845f;
    }
    out[off + i] = r;
    __syncthreads();                       // qs is rewritten for the next head
  }
}

}  // namespace

cudaError_t launch_transform_query_structured(const void* q, int q_dtype, int batch, int num_q_heads,
                                              int num_kv_heads, int kind, int block, const float* data,
                                              float* q_out, cudaStream_t stream) {
  if (kind == WUSHKV_TRANSFORM_DENSE)
    return launch_transform_query(q, q_dtype, batch, num_q_heads, num_kv_heads, data, q_out, stream);
  dim3 grid(num_kv_heads, batch);
  const bool bf = q_dtype == WUSHKV_BF16;
  if (kind == WUSHKV_TRANSFORM_BLOCK_DIAG) {
    if (bf) transform_query_structured_kernel<true, WUSHKV_TRANSFORM_BLOCK_DIAG><<<grid, kHeadDim, 0, stream>>>(
        q, batch, num_q_heads, num_kv_heads, block, data, q_out);
    else transform_query_structured_kernel<false, WUSHKV_TRANSFORM_BLOCK_DIAG><<<grid, kHeadDim, 0, stream>>>(
        q, batch, num_q_heads, num_kv_heads, block, data, q_out);
  } else {
    if (bf) transform_query_structured_kernel<true, WUSHKV_TRANSFORM_HADAMARD_DIAG><<<grid, kHeadDim, 0, stream>>>(
        q, batch, num_q_heads, num_kv_heads, block, data, q_out);
    else transform_query_structured_kernel<false, WUSHKV_TRANSFORM_HADAMARD_DIAG><<<grid, kHeadDim, 0, stream>>>(
        q, batch, num_q_heads, num_kv_heads, block, data, q_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_transform_query(const void* q, int q_dtype, int batch, int num_q_heads,
                                   int num_kv_heads, const float* Tk_invT, float* q_out,
                                   cudaStream_t stream) {
  const int g = num_q_heads / num_kv_heads;
  const int smem = kBatchPerCta * g * kHeadDim * (int)sizeof(float);
  dim3 grid(num_kv_heads, (batch + kBatchPerCta - 1) / kBatchPerCta);
  if (q_dtype == WUSHKV_BF16) {
    cudaError_t e = cudaFuncSetAttribute(transform_query_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    transform_query_kernel<true><<<grid, kHeadDim, smem, stream>>>(q, batch, num_q_heads,
                                                                   num_kv_heads, Tk_invT, q_out);
  } else {
    cudaError_t e = cudaFuncSetAttribute(transform_query_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    transform_query_kernel<false><<<grid, kHeadDim, smem, stream>>>(q, batch, num_q_heads,
                                                                    num_kv_heads, Tk_invT, q_out);
  }
  return cudaGetLastError();
}

}  // namespace wushkv
