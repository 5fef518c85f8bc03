// Split-K GQA decode attention over the packed cache, CUDA-core version, and the
// log-sum-exp combine of the split partials.
//
// WUSH-KV targets serving with grouped-query attention over a 2-bit KV cache
// (ai4snews summary, paragraph 5) at long contexts (paragraph 4).  One CTA = one
// (sequence, KV head, split); it walks its token range in 128-token tiles with an
// online softmax for all g query heads of the group, dequantizing codes in
// registers.  Partials (m, l, o[128]) go to the workspace; the combine kernel merges
// them.  Scores: s_t = tau * q' . k_hat_t, with
//   QuEST  k_hat = (c - 2^(b-1) + 1/2) Delta  ->  s = tau * Delta * sum q'_i (c_i - 2^(b-1) + 1/2)
//   affine k_hat = zero + c scale            ->  s = tau * (scale * sum q'_i c_i + zero * sum q'_i)
#include <math_constants.h>

#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kPartialStride = 132;   // m, l, pad, pad, o[128]

struct DecArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint16_t* k_meta;
  const uint16_t* v_meta;
  int hkv, hq, capacity, num_splits;
  const float* q;        // [B][Hq][128]
  const int32_t* ctx_len;
  float scale;
  float* ws;             // [B][Hq][S][132]
  int32_t* status;
};

template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t* w, int i) {
  const int o = BITS * i, wi = o >> 5, sh = o & 31;
  uint32_t c = w[wi] >> sh;
  if (sh + BITS > 32) c |= w[wi + 1] << (32 - sh);
  return c & ((1u << BITS) - 1u);
}

template <int KIND>
__device__ __forceinline__ void meta_of(const uint16_t* meta, size_t row, float& s, float& z) {
  if (KIND == WUSHKV_QUEST_INT) {
    s = f16_bits_to_f32(meta[row]);
    z = 0.f;
  } else {
    const uint32_t u = reinterpret_cast<const uint32_t*>(meta)[row];
    s = f16_bits_to_f32((uint16_t)(u & 0xffffu));
    z = f16_bits_to_f32((uint16_t)(u >> 16));
  }
}

template <int BITS, int KIND, int G>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(DecArgs a) {
  constexpr int kWords = 4 * BITS;
  constexpr float kOff = (float)(1 << (BITS - 1)) - 0.5f;
  constexpr int kHpt = G >= 2 ? G / 2 : 1;   // heads per thread
  __shared__ __align__(16) float qs[G][kHeadDim];
  __shared__ float qsum[G];
  __shared__ float sc[kTile][G];
  __shared__ __align__(16) uint32_t vt[kTile][kWords];
  __shared__ float vs[kTile], vz[kTile];
  __shared__ float m_run[G], l_run[G], corr[G];

  const int s_idx = blockIdx.x, kv = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  int L = __ldg(a.ctx_len + b);
  if (L > a.capacity) {
    if (s_idx == 0 && kv == 0 && tid == 0) report(a.status, WUSHKV_STATUS_CTX_OVERFLOW);
    L = a.capacity;
  }
  if (L < 0) L = 0;
  const int per = (L + a.num_splits - 1) / a.num_splits;
  const int chunk = (per + kTile - 1) / kTile * kTile;
  const int t0 = s_idx * chunk;
  const int t1 = min(L, t0 + chunk);

  for (int e = tid; e < G * kHeadDim; e += kThreads) {
    const int h = e / kHeadDim, c = e % kHeadDim;
    qs[h][c] = a.q[((size_t)b * a.hq + kv * G + h) * kHeadDim + c];
  }
  if (tid < G) { m_run[tid] = -CUDART_INF_F; l_run[tid] = 0.f; }
  __syncthreads();
  if (tid < G) {
    float acc = 0.f;
    for (int c = 0; c < kHeadDim; ++c) acc += qs[tid][c];
    qsum[tid] = acc;
  }
  __syncthreads();

  const int ch = tid & (kHeadDim - 1), hh = tid >> 7;   // output channel, head half
  float o[kHpt];
#pragma unroll
  for (int k = 0; k < kHpt; ++k) o[k] = 0.f;

  const size_t pair = (size_t)b * a.hkv + kv;
  for (int tb = t0; tb < t1; tb += kTile) {
    const int nt = min(kTile, t1 - tb);
    // stage V codes and meta of the tile (coalesced)
    for (int e = tid; e < nt * kWords; e += kThreads) {
      const int r = e / kWords, q = e % kWords;
      vt[r][q] = reinterpret_cast<const uint32_t*>(a.v_codes + (pair * a.capacity + tb + r) * (16 * BITS))[q];
    }
    for (int r = tid; r < nt; r += kThreads) meta_of<KIND>(a.v_meta, pair * a.capacity + tb + r, vs[r], vz[r]);
    // scores: thread (token r, head half hh)
    {
      const int r = tid & (kTile - 1);
      if (r < nt && (G >= 2 || hh == 0)) {
        const size_t row = pair * a.capacity + tb + r;
        uint32_t w[kWords];
        const uint4* src = reinterpret_cast<const uint4*>(a.k_codes + row * (16 * BITS));
#pragma unroll
        for (int q = 0; q < BITS; ++q) {
          const uint4 u = __ldg(src + q);
          w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
        }
        float ks, kz;
        meta_of<KIND>(a.k_meta, row, ks, kz);
        float acc[kHpt];
#pragma unroll
        for (int k = 0; k < kHpt; ++k) acc[k] = 0.f;
#pragma unroll
        for (int i = 0; i < kHeadDim; ++i) {
          const float cv = (float)code_at<BITS>(w, i) - (KIND == WUSHKV_QUEST_INT ? kOff : 0.f);
#pragma unroll
          for (int k = 0; k < kHpt; ++k) acc[k] = fmaf(qs[hh * kHpt + k][i], cv, acc[k]);
        }
#pragma unroll
        for (int k = 0; k < kHpt; ++k) {
          const int h = hh * kHpt + k;
          const float s = KIND == WUSHKV_QUEST_INT ? acc[k] * ks : fmaf(ks, acc[k], kz * qsum[h]);
          sc[r][h] = a.scale * s;
        }
      }
    }
    __syncthreads();
    // tile max, correction, probabilities and running sums: warp h handles head h
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < G; h += kThreads / 32) {
      float mx = -CUDART_INF_F;
      for (int r = lane; r < nt; r += 32) mx = fmaxf(mx, sc[r][h]);
#pragma unroll
      for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_run[h];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int r = lane; r < nt; r += 32) {
        const float p = expf(sc[r][h] - m_new);
        sc[r][h] = p;
        sum += p;
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      __syncwarp();
      if (lane == 0) {
        const float cf = expf(m_old - m_new);   // 0 on the first tile (m_old = -inf)
        corr[h] = cf;
        l_run[h] = l_run[h] * cf + sum;
        m_run[h] = m_new;
      }
    }
    __syncthreads();
    // o[h][ch] = o * corr + sum_t p_t v_hat_t[ch]
    if (G >= 2 || hh == 0) {
#pragma unroll
      for (int k = 0; k < kHpt; ++k) o[k] *= corr[hh * kHpt + k];
      for (int r = 0; r < nt; ++r) {
        const float cv = (float)code_at<BITS>(vt[r], ch);
        const float v = KIND == WUSHKV_QUEST_INT ? (cv - kOff) * vs[r] : fmaf(cv, vs[r], vz[r]);
#pragma unroll
        for (int k = 0; k < kHpt; ++k) o[k] = fmaf(sc[r][hh * kHpt + k], v, o[k]);
      }
    }
    __syncthreads();
  }

  if (G >= 2 || hh == 0) {
#pragma unroll
    for (int k = 0; k < kHpt; ++k) {
      const int h = hh * kHpt + k;
      float* dst = a.ws + (((size_t)b * a.hq + kv * G + h) * a.num_splits + s_idx) * kPartialStride;
      if (ch == 0) { dst[0] = m_run[h]; dst[1] = l_run[h]; }
      dst[4 + ch] = o[k];
    }
  }
}

__global__ void __launch_bounds__(kHeadDim) combine_kernel(const float* __restrict__ ws, int num_splits,
                                                          float* __restrict__ out) {
  const size_t bh = blockIdx.x;
  const int c = threadIdx.x;
  const float* p = ws + bh * num_splits * kPartialStride;
  float mx = -CUDART_INF_F;
  for (int s = 0; s < num_splits; ++s) mx = fmaxf(mx, p[s * kPartialStride]);
  float l = 0.f, o = 0.f;
  if (mx > -CUDART_INF_F) {
    for (int s = 0; s < num_splits; ++s) {
      const float ms = p[s * kPartialStride];
      if (ms == -CUDART_INF_F) continue;
      const float w = expf(ms - mx);
      l = fmaf(w, p[s * kPartialStride + 1], l);
      o = fmaf(w, p[s * kPartialStride + 4 + c], o);
    }
  }
  out[bh * kHeadDim + c] = l > 0.f ? o / l : 0.f;
}

template <int BITS, int KIND, int G>
cudaError_t launch_g(const DecArgs& a, int batch, float* out, cudaStream_t stream) {
  dim3 grid(a.num_splits, a.hkv, batch);
  decode_split_kernel<BITS, KIND, G><<<grid, kThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<<<batch * a.hq, kHeadDim, 0, stream>>>(a.ws, a.num_splits, out);
  return cudaGetLastError();
}

template <int BITS, int KIND>
cudaError_t launch_kind(const DecArgs& a, int batch, float* out, cudaStream_t stream) {
  switch (a.hq / a.hkv) {
    case 1: return launch_g<BITS, KIND, 1>(a, batch, out, stream);
    case 2: return launch_g<BITS, KIND, 2>(a, batch, out, stream);
    case 4: return launch_g<BITS, KIND, 4>(a, batch, out, stream);
    case 8: return launch_g<BITS, KIND, 8>(a, batch, out, stream);
    default: return launch_g<BITS, KIND, 16>(a, batch, out, stream);
  }
}

template <int BITS>
cudaError_t launch_bits(const DecArgs& a, int kind, int batch, float* out, cudaStream_t stream) {
  if (kind == WUSHKV_QUEST_INT) return launch_kind<BITS, WUSHKV_QUEST_INT>(a, batch, out, stream);
  return launch_kind<BITS, WUSHKV_PCT_AFFINE>(a, batch, out, stream);
}

}  // namespace

int auto_num_splits(const wushkv_cache& c, int num_q_heads) {
  (void)num_q_heads;
  const int pairs = c.batch * c.num_kv_heads;
  const int max_splits = (c.capacity + 511) / 512;
  int s = (2 * 148 + pairs - 1) / pairs;
  if (s > max_splits) s = max_splits;
  return s < 1 ? 1 : s;
}

size_t decode_workspace_bytes(const wushkv_cache& c, int num_q_heads, int num_splits) {
  const int s = num_splits > 0 ? num_splits : auto_num_splits(c, num_q_heads);
  return (size_t)c.batch * num_q_heads * s * kPartialStride * sizeof(float);
}

cudaError_t launch_decode_attention(const wushkv_cache& c, const float* q_t, int num_q_heads,
                                    const int32_t* ctx_len, float softmax_scale, float* out,
                                    void* workspace, int num_splits, int32_t* status,
                                    cudaStream_t stream) {
  DecArgs a{};
  a.k_codes = c.k_codes;
  a.v_codes = c.v_codes;
  a.k_meta = c.k_meta;
  a.v_meta = c.v_meta;
  a.hkv = c.num_kv_heads;
  a.hq = num_q_heads;
  a.capacity = c.capacity;
  a.num_splits = num_splits > 0 ? num_splits : auto_num_splits(c, num_q_heads);
  a.q = q_t;
  a.ctx_len = ctx_len;
  a.scale = softmax_scale;
  a.ws = static_cast<float*>(workspace);
  a.status = status;
  switch (c.qp.bits) {
    case 2: return launch_bits<2>(a, c.qp.kind, c.batch, out, stream);
    case 3: return launch_bits<3>(a, c.qp.kind, c.batch, out, stream);
    default: return launch_bits<4>(a, c.qp.kind, c.batch, out, stream);
  }
}

}  // namespace wushkv
