// Quantize-append on the tensor cores (sm_100a): the per-KV-head key transform
// x = T_k k runs as a 128x128x128 tcgen05 MMA per tile of 128 token rows, with T_k
// split exactly into three bf16 planes (T = P1 + P2 + P3; bf16 x bf16 products are
// exact, accumulation is fp32 in tensor memory).  K and V tiles arrive by TMA in the
// 128-byte-swizzled layout the MMA reads directly.
//
// WUSH-KV (ai4snews summary, paragraphs 1 and 5; cere-bro page, flowchart): one key
// transform per KV head, applied online to post-RoPE keys; values are already in
// the transformed basis (their transform is folded into the weights); both are then
// quantized per token with a clipped quantizer and packed into the cache.
//
// One persistent CTA per SM, pinned to one KV head (its T_k planes stay in shared
// memory), walks tiles j, j + C, j + 2C, ... of that head.  Warp roles:
//   warp 0       TMA producer (K and V tiles, 2-stage rings)
//   warp 1       TMEM allocation + MMA issue (one thread)
//   warps 2-9    key epilogue: TMEM -> registers (thread = token row) -> quantize -> store;
//                warps 2-5 take the even tiles (accumulator 0), warps 6-9 the odd ones
//   warps 10-17  value epilogue: shared memory -> registers -> quantize -> store; warps
//                10-13 take the even tiles (stage 0), 14-17 the odd ones
// Two tiles are quantized at once, so every scheduler has four epilogue warps to
// interleave (the quantizer is a long dependent chain per group).
// Without T_k (identity) the key tiles take the value path and no MMA runs.
#include "sm100.cuh"
#include "tmap.h"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"
#include "wushkv_quant.cuh"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kRowsPerTile = 128;
constexpr int kStages = 2;
constexpr int kBoxBytes = 128 * 128;                 // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;            // 128 rows x 128 bf16
constexpr int kPlaneBytes = kTileBytes;              // one bf16 plane of T_k
constexpr int kThreads = 576;                       // 18 warps
constexpr int kAccCols = 128;                        // fp32 accumulator columns per buffer

// dynamic shared memory layout (offsets from a 1024-byte aligned base)
constexpr int kOffPlanes = 0;
constexpr int kOffK = kOffPlanes + 3 * kPlaneBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffBar = kOffV + kStages * kTileBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;     // + barriers, TMEM address, alignment slack

struct TcArgs {
  int num_kv_heads, total_rows, n_new, capacity;
  CacheRows rows;          // (sequence, head, position) -> row, contiguous or paged
  int tiles_per_head, ctas_per_head;
  const int32_t* start_pos;
  const float* tk;          // dense [Hkv][128][128], blocks [Hkv][128/b][b][b] or scales [Hkv][128]
  int tkind, tblock;        // wushkv_transform_kind of tk, block size b of the block-diagonal kind
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint16_t* k_meta;
  uint16_t* v_meta;
  double alpha;
  int rank_lo, rank_hi;
  int32_t* status;
};

struct Bars {
  uint64_t full_k[kStages], empty_k[kStages], full_v[kStages], empty_v[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

// Row r of a 128-row tile held as two 128B-swizzled boxes of 64 bf16: chunk c of 32
// values lives in box c / 2, 16-byte pieces 4 (c & 1) .. 4 (c & 1) + 3, swizzled by r & 7.
struct Sw128RowLoader {
  static constexpr bool kBf16Exact = true;    // every value is a bf16 input
  const uint8_t* tile;
  int r;
  __device__ __forceinline__ void operator()(int c, float (&v)[kChunk]) const {
    static_assert(kChunk == 32, "loader reads 32 values per chunk");
    const uint8_t* row = tile + (c >> 1) * kBoxBytes + r * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int piece = 4 * (c & 1) + q;
      const uint4 u = *reinterpret_cast<const uint4*>(row + ((piece ^ (r & 7)) << 4));
      float* d = v + 8 * q;
      d[0] = bf16lo(u.x); d[1] = bf16hi(u.x); d[2] = bf16lo(u.y); d[3] = bf16hi(u.y);
      d[4] = bf16lo(u.z); d[5] = bf16hi(u.z); d[6] = bf16lo(u.w); d[7] = bf16hi(u.w);
    }
  }
};

// The fp32 accumulator row of this thread's TMEM lane: chunk c = columns 32c .. 32c+31.
struct TmemRowLoader {
  static constexpr bool kBf16Exact = false;   // fp32 transform results
  uint32_t taddr;
  __device__ __forceinline__ void operator()(int c, float (&v)[kChunk]) const {
    static_assert(kChunk == 32, "loader reads 32 values per chunk");
    uint32_t r[32];
    tmem_ld32(taddr + 32 * c, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
};

// Quantize one group (row f of the input, or f < 0 for a row past the end that only
// joins the warp-collective loads) and write its codes and meta at start_pos[b] + t.
template <int BITS, int KIND, class Loader>
__device__ __forceinline__ void quantize_store(Loader& ld, const TcArgs& a, int h, int f, uint8_t* codes,
                                               uint16_t* meta) {
  int32_t flags = 0;
  size_t row = 0;
  bool store = false;
  if (f >= 0) {
    const int b = f / a.n_new, t = f - b * a.n_new;
    const int pos = __ldg(a.start_pos + b) + t;
    const bool in_cap = pos >= 0 && pos < a.capacity;
    const long long rr = in_cap ? a.rows.row(b, h, pos) : 0;
    store = in_cap && rr >= 0;
    if (!in_cap) flags |= WUSHKV_STATUS_CAPACITY;
    else if (!store) flags |= WUSHKV_STATUS_BAD_PAGE;
    row = store ? (size_t)rr : 0;
  }
  uint8_t* dst = store ? codes + row * (16 * BITS) : nullptr;
  uint16_t m0 = 0, m1 = 0;
  if (KIND == WUSHKV_QUEST_INT) {
    quest_quantize<BITS>(ld, a.alpha, dst, m0, flags);
  } else {
    affine_quantize<BITS, 3>(ld, a.rank_lo, a.rank_hi, dst, m0, m1, flags);
  }
  if (store) {
    if (KIND == WUSHKV_QUEST_INT) {
      meta[row] = m0;
    } else {
      reinterpret_cast<uint32_t*>(meta)[row] = (uint32_t)m0 | ((uint32_t)m1 << 16);
    }
  }
  if (flags && f >= 0) report(a.status, flags);
}

// Entries T[i][j .. j+3] of KV head h's key transform as fp32: the dense matrix, the
// expanded block-diagonal one (zero off the diagonal blocks) or H diag(s) / sqrt(128)
// (H_ij = (-1)^popcount(i & j), the Sylvester Hadamard matrix).
__device__ __forceinline__ float4 transform_entries(const TcArgs& a, int h, int i, int j) {
  if (a.tkind == WUSHKV_TRANSFORM_BLOCK_DIAG) {
    const int bs = a.tblock, blk = i / bs;
    if (j / bs != blk) return make_float4(0.f, 0.f, 0.f, 0.f);   // b >= 16: j .. j+3 share a block
    return __ldg(reinterpret_cast<const float4*>(
        a.tk + (((size_t)h * (kHeadDim / bs) + blk) * bs + i % bs) * bs + j % bs));
  }
  if (a.tkind == WUSHKV_TRANSFORM_HADAMARD_DIAG) {
    const float4 sv = __ldg(reinterpret_cast<const float4*>(a.tk + (size_t)h * kHeadDim + j));
    const float c = 0.08838834764831845f;                           // 1 / sqrt(128)
    auto sgn = [&](int jj, float x) { return (__popc(i & jj) & 1) ? -(x * c) : x * c; };
    return make_float4(sgn(j, sv.x), sgn(j + 1, sv.y), sgn(j + 2, sv.z), sgn(j + 3, sv.w));
  }
  return __ldg(reinterpret_cast<const float4*>(a.tk + ((size_t)h * kHeadDim + i) * kHeadDim + j));
}

// T_k[h] (fp32, row-major [i][j]) -> three bf16 planes, each laid out as the MMA's B
// operand: K-major (j contiguous), two 64-column halves of 128 rows x 128 B, 16-byte
// chunks swizzled by (row & 7).  P1 = bf16(T), P2 = bf16(T - P1), P3 = T - P1 - P2
// (exact: the remainders of a 24-bit significand split into 8 + 8 + 8 bits).
__device__ __forceinline__ void split_transform(const TcArgs& a, int h, uint8_t* planes, int tid, int nthreads) {
  // all of this thread's loads first (independent, so their latencies overlap)
  constexpr int kMaxPer = kHeadDim * kHeadDim / 4 / (kThreads - 64);
  float4 t4[kMaxPer];
#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    const int q = tid + k * nthreads;
    if (q < kHeadDim * kHeadDim / 4) t4[k] = transform_entries(a, h, q >> 5, (q & 31) * 4);
  }
#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    const int q = tid + k * nthreads;
    if (q >= kHeadDim * kHeadDim / 4) break;
    const int i = q >> 5, j = (q & 31) * 4;
    const float tv[4] = {t4[k].x, t4[k].y, t4[k].z, t4[k].w};
    uint16_t p[3][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat16 b1 = __float2bfloat16_rn(tv[e]);
      const float r1 = tv[e] - __bfloat162float(b1);
      const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(b2);
      const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
      p[0][e] = __bfloat16_as_ushort(b1);
      p[1][e] = __bfloat16_as_ushort(b2);
      p[2][e] = __bfloat16_as_ushort(b3);
    }
    const int off = (j >> 6) * kBoxBytes + i * 128 + ((((j & 63) >> 3) ^ (i & 7)) << 4) + (j & 7) * 2;
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
      uint2 v;
      v.x = (uint32_t)p[pl][0] | ((uint32_t)p[pl][1] << 16);
      v.y = (uint32_t)p[pl][2] | ((uint32_t)p[pl][3] << 16);
      *reinterpret_cast<uint2*>(planes + pl * kPlaneBytes + off) = v;
    }
  }
}

template <int BITS, int KIND, bool HAS_T>
__global__ void __launch_bounds__(kThreads, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* planes = smem + kOffPlanes;
  uint8_t* kst = smem + kOffK;
  uint8_t* vst = smem + kOffV;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x / a.ctas_per_head;
  const int j0 = blockIdx.x % a.ctas_per_head;
  const int n_loc = (a.tiles_per_head - j0 + a.ctas_per_head - 1) / a.ctas_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full_k[s], 1);
      mbar_init(&bars->empty_k[s], HAS_T ? 1 : 4);
      mbar_init(&bars->full_v[s], 1);
      mbar_init(&bars->empty_v[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);
    }
    bars->abort = 0;
    fence_mbar_init();
    // the first fill of both rings goes out now, so it overlaps the transform split
    tma_prefetch(&kmap);
    tma_prefetch(&vmap);
    for (int li = 0; li < n_loc && li < kStages; ++li) {
      const int tile = j0 + li * a.ctas_per_head;
      mbar_arrive_expect_tx(&bars->full_k[li], kTileBytes);
      tma_load_3d(kst + li * kTileBytes, &kmap, &bars->full_k[li], 0, h, tile * kRowsPerTile);
      tma_load_3d(kst + li * kTileBytes + kBoxBytes, &kmap, &bars->full_k[li], 64, h, tile * kRowsPerTile);
      mbar_arrive_expect_tx(&bars->full_v[li], kTileBytes);
      tma_load_3d(vst + li * kTileBytes, &vmap, &bars->full_v[li], 0, h, tile * kRowsPerTile);
      tma_load_3d(vst + li * kTileBytes + kBoxBytes, &vmap, &bars->full_v[li], 64, h, tile * kRowsPerTile);
    }
  }
  if (HAS_T) {
    if (warp == 1) {
      tmem_alloc(&bars->tmem_base, 2 * kAccCols);
      tmem_relinquish();
    }
    if (warp >= 2) {
      split_transform(a, h, planes, threadIdx.x - 64, kThreads - 64);
      fence_proxy_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int first = n_loc < kStages ? n_loc : kStages;   // issued before the split
      int issued_k = first, issued_v = first;
      for (int li = first; li < n_loc; ++li) {
        const int tile = j0 + li * a.ctas_per_head;
        const int s = li % kStages;
        const uint32_t ph = (li / kStages) & 1;
        if (!mbar_wait(&bars->empty_k[s], ph ^ 1, abort)) break;
        mbar_arrive_expect_tx(&bars->full_k[s], kTileBytes);
        tma_load_3d(kst + s * kTileBytes, &kmap, &bars->full_k[s], 0, h, tile * kRowsPerTile);
        tma_load_3d(kst + s * kTileBytes + kBoxBytes, &kmap, &bars->full_k[s], 64, h, tile * kRowsPerTile);
        ++issued_k;
        if (!mbar_wait(&bars->empty_v[s], ph ^ 1, abort)) break;
        mbar_arrive_expect_tx(&bars->full_v[s], kTileBytes);
        tma_load_3d(vst + s * kTileBytes, &vmap, &bars->full_v[s], 0, h, tile * kRowsPerTile);
        tma_load_3d(vst + s * kTileBytes + kBoxBytes, &vmap, &bars->full_v[s], 64, h, tile * kRowsPerTile);
        ++issued_v;
      }
      // every load issued must land before the CTA may exit (matters only after an abort)
      volatile int no_abort = 0;
      for (int li = (issued_k > kStages ? issued_k - kStages : 0); li < issued_k; ++li)
        mbar_wait(&bars->full_k[li % kStages], (li / kStages) & 1, &no_abort);
      for (int li = (issued_v > kStages ? issued_v - kStages : 0); li < issued_v; ++li)
        mbar_wait(&bars->full_v[li % kStages], (li / kStages) & 1, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    if (HAS_T && lane == 0) {
      constexpr uint32_t kIdesc = idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 128, 128);
      const uint32_t pl_addr = smem_u32(planes);
      for (int li = 0; li < n_loc; ++li) {
        const int s = li % kStages;
        const uint32_t ph = (li / kStages) & 1;
        const int ab = li & 1;
        const uint32_t aph = (li >> 1) & 1;
        if (!mbar_wait(&bars->full_k[s], ph, abort)) break;
        if (!mbar_wait(&bars->acc_empty[ab], aph ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t d = bars->tmem_base + ab * kAccCols;
        const uint32_t k_addr = smem_u32(kst + s * kTileBytes);
#pragma unroll
        for (int p = 0; p < 3; ++p) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;
            mma_f16_ss(d, desc_kmajor_sw128(k_addr + off), desc_kmajor_sw128(pl_addr + p * kPlaneBytes + off),
                       kIdesc, (p | ks) != 0);
          }
        }
        mma_commit(&bars->empty_k[s]);
        mma_commit(&bars->acc_full[ab]);
      }
    }
  } else if (warp < 10) {
    // --------------------------------------------------------------- key epilogue
    const int g = (warp - 2) >> 2;            // tile parity this warp group handles
    const int r = 32 * (warp & 3) + lane;     // TMEM lane quarter of this warp
    for (int li = g; li < n_loc; li += 2) {
      const int tile = j0 + li * a.ctas_per_head;
      const int f = tile * kRowsPerTile + r;
      const uint32_t ph = (li >> 1) & 1;
      if (HAS_T) {
        if (!mbar_wait(&bars->acc_full[g], ph, abort)) break;
        tc_fence_after();
        TmemRowLoader ld{bars->tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + g * kAccCols};
        // tcgen05.ld is warp-collective: every lane takes part, rows past the end included
        quantize_store<BITS, KIND>(ld, a, h, f < a.total_rows ? f : -1, a.k_codes, a.k_meta);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[g]);
      } else {
        if (!mbar_wait(&bars->full_k[g], ph, abort)) break;
        Sw128RowLoader ld{kst + g * kTileBytes, r};
        if (f < a.total_rows) quantize_store<BITS, KIND>(ld, a, h, f, a.k_codes, a.k_meta);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty_k[g]);
      }
    }
  } else {
    // ------------------------------------------------------------- value epilogue
    const int g = (warp - 10) >> 2;
    const int r = 32 * ((warp - 10) & 3) + lane;
    for (int li = g; li < n_loc; li += 2) {
      const int tile = j0 + li * a.ctas_per_head;
      const uint32_t ph = (li >> 1) & 1;
      if (!mbar_wait(&bars->full_v[g], ph, abort)) break;
      const int f = tile * kRowsPerTile + r;
      Sw128RowLoader ld{vst + g * kTileBytes, r};
      if (f < a.total_rows) quantize_store<BITS, KIND>(ld, a, h, f, a.v_codes, a.v_meta);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty_v[g]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort) report(a.status, WUSHKV_STATUS_TIMEOUT);
  if (HAS_T && warp == 1) {
    tc_fence_after();
    tmem_dealloc(bars->tmem_base, 2 * kAccCols);
  }
}

template <int BITS, int KIND, bool HAS_T>
cudaError_t launch_tc(const CUtensorMap& km, const CUtensorMap& vm, const TcArgs& a, cudaStream_t stream) {
  auto kern = append_tc_kernel<BITS, KIND, HAS_T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<a.num_kv_heads * a.ctas_per_head, kThreads, kSmemBytes, stream>>>(km, vm, a);
  return cudaGetLastError();
}

template <int BITS, int KIND>
cudaError_t launch_t(const CUtensorMap& km, const CUtensorMap& vm, const TcArgs& a, cudaStream_t stream) {
  if (a.tk != nullptr) return launch_tc<BITS, KIND, true>(km, vm, a, stream);
  return launch_tc<BITS, KIND, false>(km, vm, a, stream);
}

template <int KIND>
cudaError_t launch_b(int bits, const CUtensorMap& km, const CUtensorMap& vm, const TcArgs& a, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_t<2, KIND>(km, vm, a, st);
    case 3: return launch_t<3, KIND>(km, vm, a, st);
    default: return launch_t<4, KIND>(km, vm, a, st);
  }
}

bool input_map(CUtensorMap* m, const void* base, int hkv, int rows) {
  const uint64_t dims[3] = {(uint64_t)kHeadDim, (uint64_t)hkv, (uint64_t)rows};
  const uint64_t strides[2] = {(uint64_t)kHeadDim * 2, (uint64_t)hkv * kHeadDim * 2};
  const uint32_t box[3] = {64, 1, kRowsPerTile};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_quantize_append_tc(const wushkv_cache& c, const void* k_new, const void* v_new, int n_new,
                                      const int32_t* start_pos, const float* Tk, int tkind, int tblock,
                                      int32_t* status, cudaStream_t stream) {
  TcArgs a{};
  a.num_kv_heads = c.num_kv_heads;
  a.total_rows = c.batch * n_new;
  a.n_new = n_new;
  a.capacity = c.capacity;
  a.rows = CacheRows::of(c);
  a.tiles_per_head = (a.total_rows + kRowsPerTile - 1) / kRowsPerTile;
  cudaError_t e = cudaSuccess;
  const int sms = num_sms(&e);
  if (e != cudaSuccess) return e;
  int cph = sms / c.num_kv_heads;
  if (cph < 1) cph = 1;
  if (cph > a.tiles_per_head) cph = a.tiles_per_head;
  a.ctas_per_head = cph;
  a.start_pos = start_pos;
  a.tk = Tk;
  a.tkind = tkind;
  a.tblock = tblock;
  a.k_codes = c.k_codes;
  a.v_codes = c.v_codes;
  a.k_meta = c.k_meta;
  a.v_meta = c.v_meta;
  a.alpha = c.qp.clip_alpha;
  a.rank_lo = c.qp.rank_lo;
  a.rank_hi = c.qp.rank_hi;
  a.status = status;
  CUtensorMap km, vm;
  if (!input_map(&km, k_new, c.num_kv_heads, a.total_rows) || !input_map(&vm, v_new, c.num_kv_heads, a.total_rows))
    return cudaErrorInvalidValue;
  if (c.qp.kind == WUSHKV_QUEST_INT) return launch_b<WUSHKV_QUEST_INT>(c.qp.bits, km, vm, a, stream);
  return launch_b<WUSHKV_PCT_AFFINE>(c.qp.bits, km, vm, a, stream);
}

}  // namespace wushkv
