// Causal attention of a chunk of n_q <= 16 queries per sequence over the packed cache.
//
// WUSH-KV runs its perplexity evaluation with every sequence fed in 16-token forward
// chunks (ai4snews summary, paragraph 3).  The chunk's tokens are appended to the
// cache first, so every key and value is read in its packed form: query i of sequence
// b sits at position p_i = ctx - n_q + i (ctx = min(ctx_len[b], capacity)) and attends
// positions 0 .. p_i of its KV head.
//
// The positions before the chunk, [0, ctx - n_q), are seen by every query of the
// chunk.  They go through the split-K decode kernel with the chunk folded into the GQA
// group: row f = i * g + h of a KV head's n_q * g rows is query i of head h, and the
// rows run in passes of at most 16, so the cache is read once per pass rather than once
// per query.  The chunk's own positions need the causal mask.  A small kernel (eight
// rows of one (sequence, KV head) per CTA) dequantizes them, scores every row against
// them, and merges that with the prefix partials (log2-domain m, l, o per split) that
// the decode kernel left in the workspace.
#include <math_constants.h>

#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

constexpr int kMaxChunk = 16;
constexpr int kPassRows = 16;                                 // rows per KV head in one decode pass
constexpr int kMaxPasses = kMaxChunk * 16 / kPassRows;      // n_q * g <= 256
constexpr int kPartialStride = 132;                           // m (log2 domain), l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;

// Workspace layout (offsets in floats from its base, each a multiple of 64):
//   ctx_off      int32 [batch]: context length of the prefix, max(ctx - n_q, 0)
//   scratch_off  fp32 [batch][Hkv * 16][128]: the decode call's own output (unused)
//   q_off[p]     fp32 [batch][Hkv][g_fold[p]][128]: the folded queries of pass p
//   part_off[p]  fp32 [batch][Hkv * g_fold[p]][splits[p]][132]: pass p's split partials
struct ChunkPlan {
  int passes;
  int g_fold[kMaxPasses];
  int splits[kMaxPasses];
  long long q_off[kMaxPasses];
  long long part_off[kMaxPasses];
  long long ctx_off, scratch_off;
  long long floats;
};

long long round64(long long n) { return (n + 63) / 64 * 64; }

ChunkPlan make_plan(const wushkv_cache& c, int num_q_heads, int n_q, int num_splits) {
  ChunkPlan pl{};
  const int g = num_q_heads / c.num_kv_heads;
  const int rows = n_q * g;
  const long long bh = (long long)c.batch * c.num_kv_heads;
  pl.passes = (rows + kPassRows - 1) / kPassRows;
  long long off = 0;
  pl.ctx_off = off;
  off += round64(c.batch);
  pl.scratch_off = off;
  off += round64(bh * kPassRows * kHeadDim);
  for (int p = 0; p < pl.passes; ++p) {
    const int left = rows - p * kPassRows;
    int gf = 1;
    while (gf < left && gf < kPassRows) gf *= 2;
    pl.g_fold[p] = gf;
    pl.splits[p] = num_splits > 0 ? num_splits : auto_num_splits(c, c.num_kv_heads * gf);
    pl.q_off[p] = off;
    off += round64(bh * gf * kHeadDim);
  }
  for (int p = 0; p < pl.passes; ++p) {
    pl.part_off[p] = off;
    off += round64(bh * pl.g_fold[p] * pl.splits[p] * kPartialStride);
  }
  pl.floats = off;
  return pl;
}

struct PassDev {
  int g_fold[kMaxPasses];
  int splits[kMaxPasses];
  long long q_off[kMaxPasses];
  long long part_off[kMaxPasses];
};

PassDev pass_dev(const ChunkPlan& pl) {
  PassDev d{};
  for (int p = 0; p < pl.passes; ++p) {
    d.g_fold[p] = pl.g_fold[p];
    d.splits[p] = pl.splits[p];
    d.q_off[p] = pl.q_off[p];
    d.part_off[p] = pl.part_off[p];
  }
  return d;
}

__device__ __forceinline__ int clamp_ctx(const int32_t* ctx_len, int b, int capacity) {
  return min(max(__ldg(ctx_len + b), 0), capacity);
}

// Folded queries of every pass and the prefix lengths.  grid (ceil(padded rows / 4),
// Hkv, batch), 4 warps: warp w copies folded row f = 4 * blockIdx.x + w (zeros for the
// padding rows of the last pass), lane l channels 4l .. 4l + 3.
constexpr int kPrepRows = 4;
__global__ void __launch_bounds__(32 * kPrepRows) chunk_prep_kernel(const float* __restrict__ q, int n_q, int hq,
                                                                    int hkv, int capacity, int padded,
                                                                    const int32_t* __restrict__ ctx_len,
                                                                    float* __restrict__ ws, long long ctx_off,
                                                                    PassDev pd, int32_t* status) {
  const int kv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * kPrepRows + warp;
  const int g = hq / hkv;
  if (f < padded) {
    const int p = f / kPassRows, j = f % kPassRows;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (f < n_q * g) {
      const int i = f / g, h = kv * g + f % g;
      val = __ldg(reinterpret_cast<const float4*>(q + (((size_t)b * n_q + i) * hq + h) * kHeadDim) + lane);
    }
    reinterpret_cast<float4*>(ws + pd.q_off[p] + (((size_t)b * hkv + kv) * pd.g_fold[p] + j) * kHeadDim)[lane] = val;
  }
  if (blockIdx.x == 0 && kv == 0 && threadIdx.x == 0) {
    const int raw = __ldg(ctx_len + b);
    if (raw > capacity) report(status, WUSHKV_STATUS_CTX_OVERFLOW);
    const int ctx = min(max(raw, 0), capacity);
    reinterpret_cast<int32_t*>(ws + ctx_off)[b] = max(ctx - n_q, 0);
  }
}

// Code of channel c in an LSB-first packed row of 16 * BITS bytes.
template <int BITS>
__device__ __forceinline__ int code_at(const uint8_t* row, int c) {
  const int bit = BITS * c, byte = bit >> 3;
  unsigned w = __ldg(row + byte);
  if (byte + 1 < 16 * BITS) w |= (unsigned)__ldg(row + byte + 1) << 8;
  return (int)((w >> (bit & 7)) & ((1u << BITS) - 1u));
}

template <int BITS, int KIND>
__device__ __forceinline__ float dequant_at(const uint8_t* codes, const uint16_t* meta, long long row, int c) {
  const int code = code_at<BITS>(codes + row * (16 * BITS), c);
  if (KIND == WUSHKV_QUEST_INT) {
    const float delta = f16_bits_to_f32(__ldg(meta + row));
    return ((float)(code - (1 << (BITS - 1))) + 0.5f) * delta;
  }
  const float scale = f16_bits_to_f32(__ldg(meta + 2 * row));
  const float zero = f16_bits_to_f32(__ldg(meta + 2 * row + 1));
  return fmaf((float)code, scale, zero);
}

struct MergeArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint16_t* k_meta;
  const uint16_t* v_meta;
  CacheRows rows;
  const float* q;          // [B][n_q][Hq][128]
  const int32_t* ctx_len;
  const float* ws;
  float* out;              // [B][n_q][Hq][128]
  int32_t* status;
  int n_q, hq, hkv, capacity;
  float scale_log2;
};

// Sum over the warp of 16 per-lane partial values by recursive halving: at each step a
// lane keeps the half of its values that its lane bit selects and adds the partner's
// copy of that half.  Lane l returns the full sum of value (l >> 1) & 15.
__device__ __forceinline__ float reduce_scatter16(const float (&v)[16], int lane) {
  float a8[8], a4[4], a2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    a8[k] = (b4 ? v[k + 8] : v[k]) + __shfl_xor_sync(0xffffffffu, b4 ? v[k] : v[k + 8], 16);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    a4[k] = (b3 ? a8[k + 4] : a8[k]) + __shfl_xor_sync(0xffffffffu, b3 ? a8[k] : a8[k + 4], 8);
#pragma unroll
  for (int k = 0; k < 2; ++k)
    a2[k] = (b2 ? a4[k + 2] : a4[k]) + __shfl_xor_sync(0xffffffffu, b2 ? a4[k] : a4[k + 2], 4);
  const float a1 = (b1 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? a2[0] : a2[1], 2);
  return a1 + __shfl_xor_sync(0xffffffffu, a1, 1);
}

__device__ __forceinline__ float warp_max_f(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Causal tail + merge with the prefix partials.  grid (ceil(n_q * g / 8), Hkv, batch),
// 8 warps; warp w takes folded row f = 8 * blockIdx.x + w, lane l channels 4l .. 4l + 3.
// Every CTA of a (sequence, KV head) dequantizes the chunk's own positions itself.
constexpr int kMergeWarps = 8;
template <int BITS, int KIND>
__global__ void __launch_bounds__(32 * kMergeWarps) chunk_merge_kernel(MergeArgs a, PassDev pd) {
  __shared__ __align__(16) float kh[kMaxChunk][kHeadDim];
  __shared__ __align__(16) float vh[kMaxChunk][kHeadDim];
  __shared__ int row_ok[kMaxChunk];
  const int kv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ctx = clamp_ctx(a.ctx_len, b, a.capacity);
  const int tail0 = max(ctx - a.n_q, 0);
  const int nt = ctx - tail0;

  // dequantize positions tail0 .. ctx - 1, element e = (row r, channel c)
  for (int e = threadIdx.x; e < nt * kHeadDim; e += 32 * kMergeWarps) {
    const int r = e / kHeadDim, c = e % kHeadDim;
    const long long row = a.rows.row(b, kv, tail0 + r);
    if (c == 0) {
      row_ok[r] = row >= 0;
      if (row < 0 && blockIdx.x == 0) report(a.status, WUSHKV_STATUS_BAD_PAGE);
    }
    if (row < 0) continue;
    kh[r][c] = dequant_at<BITS, KIND>(a.k_codes, a.k_meta, row, c);
    vh[r][c] = dequant_at<BITS, KIND>(a.v_codes, a.v_meta, row, c);
  }
  __syncthreads();

  const int g = a.hq / a.hkv;
  const int f = blockIdx.x * kMergeWarps + warp;
  if (f >= a.n_q * g) return;
  const int i = f / g, h = kv * g + f % g;
  const size_t qrow = ((size_t)b * a.n_q + i) * a.hq + h;
  const float4 q4 = __ldg(reinterpret_cast<const float4*>(a.q + qrow * kHeadDim) + lane);
  const int last = ctx - a.n_q + i - tail0;            // last visible tail row (may be < 0)

  // prefix partials of this row (pass p = f / 16, row j = f % 16 of the pass)
  const int p = f / kPassRows, j = f % kPassRows;
  const int gf = pd.g_fold[p], ns = pd.splits[p];
  const float* part = a.ws + pd.part_off[p] + (((size_t)b * a.hkv + kv) * gf + j) * ns * kPartialStride;
  float mp = -CUDART_INF_F;
  for (int s = lane; s < ns; s += 32) mp = fmaxf(mp, __ldg(part + (size_t)s * kPartialStride));

  // tail scores, log2 domain: lane l holds key (l >> 1) & 15
  float d[kMaxChunk];
#pragma unroll
  for (int r = 0; r < kMaxChunk; ++r) {
    d[r] = 0.f;
    if (r < nt) {
      const float4 k4 = reinterpret_cast<const float4*>(kh[r])[lane];
      d[r] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, q4.w * k4.w)));
    }
  }
  const float dk = reduce_scatter16(d, lane);
  const int kk = (lane >> 1) & 15;
  const float s2 = (kk < nt && kk <= last && row_ok[kk]) ? dk * a.scale_log2 : -CUDART_INF_F;
  const float mx = warp_max_f(fmaxf(mp, s2));

  float l = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -CUDART_INF_F) {
    float lp = 0.f;
    for (int s0 = 0; s0 < ns; s0 += 32) {
      const int s = s0 + lane;
      const float ms = s < ns ? __ldg(part + (size_t)s * kPartialStride) : -CUDART_INF_F;
      const float wsp = ms == -CUDART_INF_F ? 0.f : exp2f(ms - mx);
      if (s < ns) lp = fmaf(wsp, __ldg(part + (size_t)s * kPartialStride + 1), lp);
      const int cnt = min(32, ns - s0);
      for (int t = 0; t < cnt; ++t) {
        const float w = __shfl_sync(0xffffffffu, wsp, t);
        if (w == 0.f) continue;                        // empty split (same on every lane)
        const float4 os = __ldg(reinterpret_cast<const float4*>(part + (size_t)(s0 + t) * kPartialStride + 4) + lane);
        o.x = fmaf(w, os.x, o.x);
        o.y = fmaf(w, os.y, o.y);
        o.z = fmaf(w, os.z, o.z);
        o.w = fmaf(w, os.w, o.w);
      }
    }
    l = warp_sum_f(lp);
    const float wt = s2 == -CUDART_INF_F ? 0.f : exp2f(s2 - mx);
#pragma unroll
    for (int r = 0; r < kMaxChunk; ++r) {
      const float w = __shfl_sync(0xffffffffu, wt, 2 * r);
      if (w == 0.f) continue;                          // masked or past the tail
      const float4 v4 = reinterpret_cast<const float4*>(vh[r])[lane];
      l += w;
      o.x = fmaf(w, v4.x, o.x);
      o.y = fmaf(w, v4.y, o.y);
      o.z = fmaf(w, v4.z, o.z);
      o.w = fmaf(w, v4.w, o.w);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  reinterpret_cast<float4*>(a.out + qrow * kHeadDim)[lane] = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
}

template <int BITS>
cudaError_t launch_merge_bits(const MergeArgs& a, int kind, int batch, const PassDev& pd, cudaStream_t st) {
  const int rows = a.n_q * (a.hq / a.hkv);
  const dim3 grid((rows + kMergeWarps - 1) / kMergeWarps, a.hkv, batch);
  if (kind == WUSHKV_QUEST_INT)
    chunk_merge_kernel<BITS, WUSHKV_QUEST_INT><<<grid, 32 * kMergeWarps, 0, st>>>(a, pd);
  else
    chunk_merge_kernel<BITS, WUSHKV_PCT_AFFINE><<<grid, 32 * kMergeWarps, 0, st>>>(a, pd);
  return cudaGetLastError();
}

}  // namespace

size_t chunk_workspace_bytes(const wushkv_cache& c, int num_q_heads, int n_q, int num_splits) {
  return (size_t)make_plan(c, num_q_heads, n_q, num_splits).floats * sizeof(float);
}

cudaError_t launch_chunk_attention(const wushkv_cache& c, const float* q_t, int n_q, int num_q_heads,
                                   const int32_t* ctx_len, float softmax_scale, float* out, void* workspace,
                                   int num_splits, int32_t* status, cudaStream_t stream) {
  const ChunkPlan pl = make_plan(c, num_q_heads, n_q, num_splits);
  const PassDev pd = pass_dev(pl);
  float* ws = static_cast<float*>(workspace);
  const int padded = (pl.passes - 1) * kPassRows + pl.g_fold[pl.passes - 1];
  chunk_prep_kernel<<<dim3((padded + kPrepRows - 1) / kPrepRows, c.num_kv_heads, c.batch), 32 * kPrepRows, 0,
                      stream>>>(q_t, n_q, num_q_heads, c.num_kv_heads, c.capacity, padded, ctx_len, ws, pl.ctx_off,
                                pd, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int32_t* ctx_prefix = reinterpret_cast<const int32_t*>(ws + pl.ctx_off);
  for (int p = 0; p < pl.passes; ++p) {
    e = launch_decode_attention(c, ws + pl.q_off[p], c.num_kv_heads * pl.g_fold[p], ctx_prefix, softmax_scale,
                                ws + pl.scratch_off, ws + pl.part_off[p], pl.splits[p], status, stream);
    if (e != cudaSuccess) return e;
  }
  MergeArgs a{};
  a.k_codes = c.k_codes;
  a.v_codes = c.v_codes;
  a.k_meta = c.k_meta;
  a.v_meta = c.v_meta;
  a.rows = CacheRows::of(c);
  a.q = q_t;
  a.ctx_len = ctx_len;
  a.ws = ws;
  a.out = out;
  a.status = status;
  a.n_q = n_q;
  a.hq = num_q_heads;
  a.hkv = c.num_kv_heads;
  a.capacity = c.capacity;
  a.scale_log2 = softmax_scale * kLog2e;
  switch (c.qp.bits) {
    case 2: return launch_merge_bits<2>(a, c.qp.kind, c.batch, pd, stream);
    case 3: return launch_merge_bits<3>(a, c.qp.kind, c.batch, pd, stream);
    default: return launch_merge_bits<4>(a, c.qp.kind, c.batch, pd, stream);
  }
}

}  // namespace wushkv
