// Quantize-append, CUDA-core version: key transform by FFMA, then the clipped
// quantizer and the packed store.  One CTA = 128 consecutive (sequence, token)
// rows of one KV head; one thread = one 128-value group.
//
// WUSH-KV (ai4snews summary, paragraphs 1 and 5): each KV head has its own key
// transform, applied to post-RoPE keys online; keys and values are quantized per
// token with a clipped quantizer.  Values are quantized untransformed (their
// transform is folded into the weights).
#include "wushkv_common.cuh"
#include "wushkv_launch.h"
#include "wushkv_quant.cuh"

namespace wushkv {
namespace {

constexpr int kRows = 128;
constexpr int kPad = kHeadDim + 1;  // padded fp32 row stride: row-per-thread reads hit distinct banks

struct RowArgs {
  const void* in;          // [B*n_new][Hkv][128]
  int num_kv_heads;
  int total_rows;          // B * n_new
  int n_new;
  const int32_t* start_pos;
  const float* tk;         // [Hkv][128][128] or nullptr
  uint8_t* codes;          // [B][Hkv][T][16 bits]
  uint16_t* meta;          // [B][Hkv][T][m]
  int capacity;
  CacheRows rows;          // (sequence, head, position) -> row, contiguous or paged
  double alpha;
  int rank_lo, rank_hi;
  int32_t* status;
};

template <bool BF16_IN>
__device__ __forceinline__ void load_tile(const RowArgs& a, int tile, int h, float* dst, int stride) {
  constexpr int kEpc = BF16_IN ? 8 : 4;            // elements per 16-byte chunk
  constexpr int kCpr = kHeadDim / kEpc;            // chunks per row
  for (int c = threadIdx.x; c < kRows * kCpr; c += blockDim.x) {
    const int r = c / kCpr, cc = c % kCpr;
    const int f = tile * kRows + r;
    float v[kEpc];
    if (f < a.total_rows) {
      const size_t off = ((size_t)f * a.num_kv_heads + h) * kHeadDim + cc * kEpc;
      if (BF16_IN) {
        const uint4 u = ld_global_nc_v4(static_cast<const __nv_bfloat16*>(a.in) + off);
        v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
        v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
      } else {
        const uint4 u = ld_global_nc_v4(static_cast<const float*>(a.in) + off);
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kEpc; ++e) v[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < kEpc; ++e) dst[r * stride + cc * kEpc + e] = v[e];
  }
}

template <int BITS, int KIND, bool BF16_IN, bool TRANSFORM>
__global__ void __launch_bounds__(kRows) append_rows_kernel(RowArgs a) {
  extern __shared__ __align__(16) float smem[];
  float* xs = smem;                              // [128][129] group values
  float* ks = smem + kRows * kPad;               // [128][128] raw keys (transform only)
  const int tile = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;

  if (TRANSFORM) {
    load_tile<BF16_IN>(a, tile, h, ks, kHeadDim);
    // thread i owns output channel i: x[t][i] = sum_j T[i][j] k[t][j]
    float tr[kHeadDim];
    const float4* trow = reinterpret_cast<const float4*>(a.tk + ((size_t)h * kHeadDim + tid) * kHeadDim);
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j) {
      const float4 t4 = __ldg(trow + j);
      tr[4 * j] = t4.x; tr[4 * j + 1] = t4.y; tr[4 * j + 2] = t4.z; tr[4 * j + 3] = t4.w;
    }
    __syncthreads();
#pragma unroll 1
    for (int t = 0; t < kRows; ++t) {
      const float4* kr = reinterpret_cast<const float4*>(ks + t * kHeadDim);
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < kHeadDim / 4; ++j) {
        const float4 k4 = kr[j];
        acc = fmaf(tr[4 * j], k4.x, acc);
        acc = fmaf(tr[4 * j + 1], k4.y, acc);
        acc = fmaf(tr[4 * j + 2], k4.z, acc);
        acc = fmaf(tr[4 * j + 3], k4.w, acc);
      }
      xs[t * kPad + tid] = acc;
    }
  } else {
    load_tile<BF16_IN>(a, tile, h, xs, kPad);
  }
  __syncthreads();

  const int f = tile * kRows + tid;
  if (f >= a.total_rows) return;
  SmemRowLoader ld{xs + tid * kPad};

  const int b = f / a.n_new, t = f - b * a.n_new;
  const int pos = __ldg(a.start_pos + b) + t;
  const bool in_cap = pos >= 0 && pos < a.capacity;
  const long long rr = in_cap ? a.rows.row(b, h, pos) : 0;
  const bool store = in_cap && rr >= 0;
  const size_t row = store ? (size_t)rr : 0;
  uint8_t* dst = store ? a.codes + row * (16 * BITS) : nullptr;
  uint16_t m0 = 0, m1 = 0;
  int32_t flags = !in_cap ? WUSHKV_STATUS_CAPACITY : store ? 0 : WUSHKV_STATUS_BAD_PAGE;
  if (KIND == WUSHKV_QUEST_INT) {
    quest_quantize<BITS>(ld, a.alpha, dst, m0, flags);
  } else {
    affine_quantize<BITS, 3>(ld, a.rank_lo, a.rank_hi, dst, m0, m1, flags);
  }
  if (store) {
    if (KIND == WUSHKV_QUEST_INT) {
      a.meta[row] = m0;
    } else {
      reinterpret_cast<uint32_t*>(a.meta)[row] = (uint32_t)m0 | ((uint32_t)m1 << 16);
    }
  }
  if (flags) report(a.status, flags);
}

template <int BITS, int KIND, bool BF16_IN, bool TRANSFORM>
cudaError_t launch_rows(const RowArgs& a, cudaStream_t stream) {
  auto kern = append_rows_kernel<BITS, KIND, BF16_IN, TRANSFORM>;
  const int smem = (kRows * kPad + (TRANSFORM ? kRows * kHeadDim : 0)) * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.total_rows + kRows - 1) / kRows, a.num_kv_heads);
  kern<<<grid, kRows, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int BITS, int KIND, bool BF16_IN>
cudaError_t launch_side(const RowArgs& a, cudaStream_t stream) {
  if (a.tk != nullptr) return launch_rows<BITS, KIND, BF16_IN, true>(a, stream);
  return launch_rows<BITS, KIND, BF16_IN, false>(a, stream);
}

template <int BITS, int KIND>
cudaError_t launch_dtype(const RowArgs& a, int in_dtype, cudaStream_t stream) {
  if (in_dtype == WUSHKV_BF16) return launch_side<BITS, KIND, true>(a, stream);
  return launch_side<BITS, KIND, false>(a, stream);
}

template <int KIND>
cudaError_t launch_bits(const RowArgs& a, int bits, int in_dtype, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_dtype<2, KIND>(a, in_dtype, stream);
    case 3: return launch_dtype<3, KIND>(a, in_dtype, stream);
    default: return launch_dtype<4, KIND>(a, in_dtype, stream);
  }
}

}  // namespace

cudaError_t launch_quantize_append_simt(const wushkv_cache& c, const void* k_new, const void* v_new,
                                        int in_dtype, int n_new, const int32_t* start_pos,
                                        const float* Tk, int32_t* status, cudaStream_t stream) {
  RowArgs a{};
  a.num_kv_heads = c.num_kv_heads;
  a.total_rows = c.batch * n_new;
  a.n_new = n_new;
  a.start_pos = start_pos;
  a.capacity = c.capacity;
  a.rows = CacheRows::of(c);
  a.alpha = c.qp.clip_alpha;
  a.rank_lo = c.qp.rank_lo;
  a.rank_hi = c.qp.rank_hi;
  a.status = status;
  for (int side = 0; side < 2; ++side) {
    a.in = side == 0 ? k_new : v_new;
    a.tk = side == 0 ? Tk : nullptr;
    a.codes = side == 0 ? c.k_codes : c.v_codes;
    a.meta = side == 0 ? c.k_meta : c.v_meta;
    cudaError_t e = c.qp.kind == WUSHKV_QUEST_INT
                        ? launch_bits<WUSHKV_QUEST_INT>(a, c.qp.bits, in_dtype, stream)
                        : launch_bits<WUSHKV_PCT_AFFINE>(a, c.qp.bits, in_dtype, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wushkv
