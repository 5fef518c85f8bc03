// Quantize-append for a few token rows (a decode step appends one token per
// sequence): latency matters, not throughput.  One CTA = kRows token rows of one KV
// head (one: the most CTAs, the shortest dependent chain per CTA).  The key transform is a dot product per output channel (thread i owns
// channel i and reads row i of T_k), then each 128-value group (key or value of one
// row) is quantized by one warp, four values per lane, with every code decided by
// exact threshold comparisons.  Optionally the keys arrive before RoPE and are rotated
// here with the caller's cos/sin table, in front of the transform.
//
// WUSH-KV (ai4snews summary, paragraphs 1 and 5; cere-bro page, flowchart): one key
// transform per KV head applied online to post-RoPE keys; values already in the
// transformed basis; both quantized per token with a clipped quantizer and packed.
// The grids (QuEST-INT-style RMS step, percentile-clipped affine) are those of the
// bulk append kernels; results differ from theirs only through the fp32 rounding of
// the transform.
#include <math_constants.h>

#include "sm100.cuh"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kRows = 1;            // token rows per CTA (1 measured fastest: 5.6 against 7.4 us at 4 for a decode step)
constexpr int kThreads = 128;       // 4 warps: one group (key or value of a row) each at a time

struct SmallArgs {
  const __nv_bfloat16* k;           // [B*n_new][Hkv][128]
  const __nv_bfloat16* v;
  int num_kv_heads, total_rows, n_new, capacity;
  CacheRows rows;                   // (sequence, head, position) -> row, contiguous or paged
  const int32_t* start_pos;
  const float* tk;                  // dense [Hkv][128][128], blocks [Hkv][128/b][b][b], scales [Hkv][128], or nullptr
  int tkind, tblock;                // transform variant (kTf*), block size of the block-diagonal one
  const float* rope;                // [rope_rows][128] (cos | sin per position) or nullptr
  int rope_rows;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint16_t* k_meta;
  uint16_t* v_meta;
  double alpha;
  int rank_lo, rank_hi;
  int32_t* status;
};

__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// The value of ascending rank `rank` (0-based) among the warp's 128 values, four
// ascending per lane; `up` = false gives descending rank instead.
__device__ __forceinline__ float warp_rank(const float (&s)[4], int rank, bool up) {
  int ptr = up ? 0 : 3;
  float m = 0.f;
  for (int r = 0; r <= rank; ++r) {
    const bool has = up ? ptr < 4 : ptr >= 0;
    const float cand = has ? (ptr == 0 ? s[0] : ptr == 1 ? s[1] : ptr == 2 ? s[2] : s[3])
                           : (up ? CUDART_INF_F : -CUDART_INF_F);
    m = up ? warp_min(cand) : warp_max(cand);
    const unsigned who = __ballot_sync(0xffffffffu, has && cand == m);
    if (who != 0u && (int)(threadIdx.x & 31) == __ffs(who) - 1) ptr += up ? 1 : -1;
  }
  return m;
}

// Packed codes of lane l (codes of elements 4l .. 4l+3, BITS bits each) into the
// group's LSB-first bit string at dst.
template <int BITS>
__device__ __forceinline__ void store_lane_codes(uint8_t* dst, uint32_t c4) {
  const int lane = threadIdx.x & 31;
  if (BITS == 2) {
    dst[lane] = (uint8_t)c4;                                   // 8 bits per lane
  } else if (BITS == 4) {
    reinterpret_cast<uint16_t*>(dst)[lane] = (uint16_t)c4;     // 16 bits per lane
  } else {                                                     // 12 bits per lane: pairs form 3 bytes
    const uint32_t other = __shfl_down_sync(0xffffffffu, c4, 1);
    if ((lane & 1) == 0) {
      const uint32_t w = c4 | (other << 12);
      uint8_t* p = dst + 3 * (lane >> 1);
      p[0] = (uint8_t)w;
      p[1] = (uint8_t)(w >> 8);
      p[2] = (uint8_t)(w >> 16);
    }
  }
}

// Quantize the group x[0..127] (shared memory, this lane's four values at 4 lane) and
// write codes and meta to cache row `row` (or only report, when store is false).
template <int BITS, int KIND>
__device__ void quantize_group_warp(const float* x, const SmallArgs& a, bool store, size_t row, uint8_t* codes,
                                    uint16_t* meta, int32_t& flags) {
  constexpr int kHalfCode = 1 << (BITS - 1);
  constexpr int kMaxCode = (1 << BITS) - 1;
  const int lane = threadIdx.x & 31;
  const float4 x4 = reinterpret_cast<const float4*>(x)[lane];
  const float v[4] = {x4.x, x4.y, x4.z, x4.w};
  const bool finite = isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3]);
  if (__any_sync(0xffffffffu, !finite)) flags |= WUSHKV_STATUS_NONFINITE;
  uint32_t c4 = 0;
  uint32_t meta_word = 0;
  if (KIND == WUSHKV_QUEST_INT) {
    // sum of the exact squares in fp64; alpha * RMS * 2^(1-b), one rounding to fp16
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) s = fma((double)v[e], (double)v[e], s);
    s = warp_sum(s);
    const double pre = a.alpha * sqrt(s * (1.0 / 128.0)) * ldexp(1.0, 1 - BITS);
    const uint16_t hb = f64_to_f16_bits(pre);
    const float delta = f16_bits_to_f32(hb);
    if (isinf(delta)) flags |= WUSHKV_STATUS_META_OVERFLOW;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t code = 0;                     // thresholds j * Delta are exact in fp32
#pragma unroll
      for (int j = -(kHalfCode - 1); j < kHalfCode; ++j) code += v[e] >= (float)j * delta ? 1u : 0u;
      if (delta == 0.f || isinf(delta)) code = kHalfCode;
      c4 |= code << (BITS * e);
    }
    meta_word = hb;
  } else {
    // lo, hi = values of ascending rank rank_lo and rank_hi
    float s[4] = {v[0], v[1], v[2], v[3]};
#define WUSHKV_CSWAP(i, j) { const float lo_ = fminf(s[i], s[j]); s[j] = fmaxf(s[i], s[j]); s[i] = lo_; }
    WUSHKV_CSWAP(0, 1) WUSHKV_CSWAP(2, 3) WUSHKV_CSWAP(0, 2) WUSHKV_CSWAP(1, 3) WUSHKV_CSWAP(1, 2)
#undef WUSHKV_CSWAP
    const float lo = warp_rank(s, a.rank_lo, true);
    const float hi = warp_rank(s, kHeadDim - 1 - a.rank_hi, false);
    const uint16_t sb = f64_to_f16_bits(((double)hi - (double)lo) / (double)kMaxCode);
    const uint16_t zb = f32_to_f16_bits(lo);
    const float sc = f16_bits_to_f32(sb), z = f16_bits_to_f32(zb);
    if (isinf(sc) || isinf(z)) flags |= WUSHKV_STATUS_META_OVERFLOW;
    const double zd = (double)z, sd = (double)sc;   // thresholds zero + (j + 1/2) scale: exact in fp64
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double xd = (double)v[e];
      uint32_t code = 0;
#pragma unroll
      for (int j = 0; j < kMaxCode; ++j) {
        const double t = zd + ((double)j + 0.5) * sd;
        code += (xd > t || (xd == t && (j & 1))) ? 1u : 0u;
      }
      if (sc == 0.f || isinf(sc)) code = 0;
      c4 |= code << (BITS * e);
    }
    meta_word = (uint32_t)sb | ((uint32_t)zb << 16);
  }
  if (store) {
    store_lane_codes<BITS>(codes + row * (16 * BITS), c4);
    if (lane == 0) {
      if (KIND == WUSHKV_QUEST_INT) meta[row] = (uint16_t)meta_word;
      else reinterpret_cast<uint32_t*>(meta)[row] = meta_word;
    }
  }
}

// Key transform variants: none (keys given transformed), dense T_k, block-diagonal T_k
// (blocks of tblock x tblock on the diagonal), and T_k = H diag(s) / sqrt(128).
enum { kTfNone = 0, kTfDense = 1, kTfBlock = 2, kTfHadamard = 3 };
static_assert((int)kTfDense == (int)WUSHKV_TRANSFORM_DENSE && (int)kTfBlock == (int)WUSHKV_TRANSFORM_BLOCK_DIAG &&
                  (int)kTfHadamard == (int)WUSHKV_TRANSFORM_HADAMARD_DIAG,
              "transform kinds follow the C ABI");

template <int BITS, int KIND, int TF, bool ROPE>
__global__ void __launch_bounds__(kThreads) append_small_kernel(SmallArgs a) {
  __shared__ __align__(16) float xk[kRows][kHeadDim];   // keys (transformed)
  __shared__ __align__(16) float xv[kRows][kHeadDim];   // values
  __shared__ __align__(16) float kr[kRows][kHeadDim];   // raw keys (RoPE / transform input)
  const int h = blockIdx.x, f0 = blockIdx.y * kRows, tid = threadIdx.x;
  const int nrows = min(kRows, a.total_rows - f0);
  for (int e = tid; e < nrows * kHeadDim; e += kThreads) {
    const int r = e / kHeadDim, c = e % kHeadDim;
    const size_t off = ((size_t)(f0 + r) * a.num_kv_heads + h) * kHeadDim + c;
    xv[r][c] = __bfloat162float(a.v[off]);
    const float kv = __bfloat162float(a.k[off]);
    if (TF != kTfNone || ROPE) kr[r][c] = kv;
    else xk[r][c] = kv;
  }
  __syncthreads();
  if (ROPE) {
    // rotate-half RoPE of each key row with the table row of its position: pair
    // (c, c + 64) -> (x cos - y sin, y cos + x sin); a thread owns whole pairs, so the
    // rotation can stay in place when the transform follows
    for (int e = tid; e < nrows * (kHeadDim / 2); e += kThreads) {
      const int r = e / (kHeadDim / 2), c = e % (kHeadDim / 2);
      const int f = f0 + r;
      const int b = f / a.n_new, t = f - b * a.n_new;
      const int pos = __ldg(a.start_pos + b) + t;
      const float x = kr[r][c], y = kr[r][c + kHeadDim / 2];
      float rx = x, ry = y;
      if (pos >= 0 && pos < a.rope_rows) {         // other positions are not stored
        const float cs = __ldg(a.rope + (size_t)pos * kHeadDim + c);
        const float sn = __ldg(a.rope + (size_t)pos * kHeadDim + kHeadDim / 2 + c);
        rx = fmaf(x, cs, -(y * sn));
        ry = fmaf(y, cs, x * sn);
      }
      float* dst = TF != kTfNone ? kr[r] : xk[r];
      dst[c] = rx;
      dst[c + kHeadDim / 2] = ry;
    }
    __syncthreads();
  }
  if (TF == kTfDense) {
    // x[r][i] = sum_j T[i][j] k[r][j]: thread i reads row i of T once for every row r
    const float4* trow = reinterpret_cast<const float4*>(a.tk + ((size_t)h * kHeadDim + tid) * kHeadDim);
    float acc[kRows][4];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
#pragma unroll 8
    for (int j = 0; j < kHeadDim / 4; ++j) {
      const float4 t = __ldg(trow + j);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const float4 k4 = reinterpret_cast<const float4*>(kr[r])[j];
        acc[r][0] = fmaf(t.x, k4.x, acc[r][0]);
        acc[r][1] = fmaf(t.y, k4.y, acc[r][1]);
        acc[r][2] = fmaf(t.z, k4.z, acc[r][2]);
        acc[r][3] = fmaf(t.w, k4.w, acc[r][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nrows) xk[r][tid] = (acc[r][0] + acc[r][1]) + (acc[r][2] + acc[r][3]);
    __syncthreads();
  }
  if (TF == kTfBlock) {
    // x[r][i] = sum_j B[i / b][i % b][j] k[r][(i / b) b + j]: the dense loop restricted to
    // the block, in the same four chains (the dense product of the expanded matrix adds
    // only exact zeros besides these terms)
    const int bs = a.tblock, blk = tid / bs, ii = tid % bs;
    const float4* brow =
        reinterpret_cast<const float4*>(a.tk + (((size_t)h * (kHeadDim / bs) + blk) * bs + ii) * bs);
    float acc[kRows][4];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    for (int j = 0; j < bs / 4; ++j) {
      const float4 t = __ldg(brow + j);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const float4 k4 = reinterpret_cast<const float4*>(kr[r] + blk * bs)[j];
        acc[r][0] = fmaf(t.x, k4.x, acc[r][0]);
        acc[r][1] = fmaf(t.y, k4.y, acc[r][1]);
        acc[r][2] = fmaf(t.z, k4.z, acc[r][2]);
        acc[r][3] = fmaf(t.w, k4.w, acc[r][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nrows) xk[r][tid] = (acc[r][0] + acc[r][1]) + (acc[r][2] + acc[r][3]);
    __syncthreads();
  }
  if (TF == kTfHadamard) {
    // x = H (s * k) / sqrt(128): scale, then the seven butterfly stages of the Sylvester
    // Hadamard transform in place (stage `half` pairs channels base and base + half)
    const float sc = __ldg(a.tk + (size_t)h * kHeadDim + tid);
    for (int r = 0; r < nrows; ++r) kr[r][tid] *= sc;
    __syncthreads();
    for (int half = kHeadDim / 2; half >= 1; half >>= 1) {
      for (int e = tid; e < nrows * (kHeadDim / 2); e += kThreads) {
        const int r = e / (kHeadDim / 2), p = e % (kHeadDim / 2);
        const int base = (p / half) * (2 * half) + p % half;
        const float u = kr[r][base], v = kr[r][base + half];
        kr[r][base] = u + v;
        kr[r][base + half] = u - v;
      }
      __syncthreads();
    }
    for (int r = 0; r < nrows; ++r) xk[r][tid] = kr[r][tid] * 0.08838834764831845f;   // 1 / sqrt(128)
    __syncthreads();
  }
  const int warp = tid >> 5;
  int32_t flags = 0;
  for (int gi = warp; gi < 2 * nrows; gi += kThreads / 32) {
    const int r = gi >> 1, side = gi & 1;
    const int f = f0 + r;
    const int b = f / a.n_new, t = f - b * a.n_new;
    const int pos = __ldg(a.start_pos + b) + t;
    const bool in_cap = pos >= 0 && pos < a.capacity;
    const long long rr = in_cap ? a.rows.row(b, h, pos) : 0;
    const bool store = in_cap && rr >= 0;
    if (!in_cap) flags |= WUSHKV_STATUS_CAPACITY;
    else if (!store) flags |= WUSHKV_STATUS_BAD_PAGE;
    const size_t row = store ? (size_t)rr : 0;
    if (side == 0) quantize_group_warp<BITS, KIND>(xk[r], a, store, row, a.k_codes, a.k_meta, flags);
    else quantize_group_warp<BITS, KIND>(xv[r], a, store, row, a.v_codes, a.v_meta, flags);
  }
  if (flags && (tid & 31) == 0) report(a.status, flags);
}

template <int BITS, int KIND>
cudaError_t launch_kind(const SmallArgs& a, cudaStream_t stream) {
  dim3 grid(a.num_kv_heads, (a.total_rows + kRows - 1) / kRows);
  const bool rope = a.rope != nullptr;
  switch (a.tk == nullptr ? (int)kTfNone : a.tkind) {
    case kTfDense:
      if (rope) append_small_kernel<BITS, KIND, kTfDense, true><<<grid, kThreads, 0, stream>>>(a);
      else append_small_kernel<BITS, KIND, kTfDense, false><<<grid, kThreads, 0, stream>>>(a);
      break;
    case kTfBlock:
      append_small_kernel<BITS, KIND, kTfBlock, false><<<grid, kThreads, 0, stream>>>(a);
      break;
    case kTfHadamard:
      append_small_kernel<BITS, KIND, kTfHadamard, false><<<grid, kThreads, 0, stream>>>(a);
      break;
    default:
      if (rope) append_small_kernel<BITS, KIND, kTfNone, true><<<grid, kThreads, 0, stream>>>(a);
      else append_small_kernel<BITS, KIND, kTfNone, false><<<grid, kThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

template <int KIND>
cudaError_t launch_bits(const SmallArgs& a, int bits, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_kind<2, KIND>(a, stream);
    case 3: return launch_kind<3, KIND>(a, stream);
    default: return launch_kind<4, KIND>(a, stream);
  }
}

}  // namespace

cudaError_t launch_quantize_append_small(const wushkv_cache& c, const void* k_new, const void* v_new, int n_new,
                                         const int32_t* start_pos, const float* Tk, int tkind, int tblock,
                                         const float* rope, int rope_rows, int32_t* status, cudaStream_t stream) {
  SmallArgs a{};
  a.k = static_cast<const __nv_bfloat16*>(k_new);
  a.v = static_cast<const __nv_bfloat16*>(v_new);
  a.num_kv_heads = c.num_kv_heads;
  a.total_rows = c.batch * n_new;
  a.n_new = n_new;
  a.capacity = c.capacity;
  a.rows = CacheRows::of(c);
  a.start_pos = start_pos;
  a.tk = Tk;
  a.tkind = tkind;
  a.tblock = tblock;
  a.rope = rope;
  a.rope_rows = rope_rows;
  a.k_codes = c.k_codes;
  a.v_codes = c.v_codes;
  a.k_meta = c.k_meta;
  a.v_meta = c.v_meta;
  a.alpha = c.qp.clip_alpha;
  a.rank_lo = c.qp.rank_lo;
  a.rank_hi = c.qp.rank_hi;
  a.status = status;
  if (c.qp.kind == WUSHKV_QUEST_INT) return launch_bits<WUSHKV_QUEST_INT>(a, c.qp.bits, stream);
  return launch_bits<WUSHKV_PCT_AFFINE>(a, c.qp.bits, stream);
}

}  // namespace wushkv
