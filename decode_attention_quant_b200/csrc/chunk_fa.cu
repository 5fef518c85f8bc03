// Causal attention of a chunk of n_q <= 16 queries per sequence over the packed cache,
// on the tensor cores with the chunk's rows on the MMA's M side.
//
// WUSH-KV runs its perplexity evaluation with every sequence fed in 16-token forward
// chunks (ai4snews summary, paragraph 3).  The chunk's tokens are appended first, so
// every key and value is read in packed form: query i of sequence b sits at position
// p_i = ctx - n_q + i (ctx = min(ctx_len[b], capacity)) and attends positions 0 .. p_i.
//
// One CTA = (split of the positions, KV head, block of 128 folded rows, sequence); row
// f = i * g + h is query i of head h.  Per 128-position tile:
//   converters (warps 0-3, thread = position): packed K and V codes -> exact fp16 codes in
//     the 128-byte-swizzled layout both MMAs read, plus the tile's fp16 meta as fp32;
//   MMA issuer (warp 12): S = Q' K^T as two fp16 MMAs (q' split into fp16 hi + lo, so the
//     products carry 22 bits of q'; codes are exact), fp32 accumulation in tensor memory;
//     then O += P V with P' = p * scale split the same way (P in tensor memory);
//   softmax (warps 4-11, thread = row and half of the tile's positions): scores
//     s = tau log2e (scale_t q'.c + zero_t sum q') in the log2 domain, causal mask, the
//     tile maximum, e = 2^(s - m) against a running reference m that moves only when the
//     maximum passes it by 8 (then O, l and z are rescaled), sums l = sum e and
//     z = sum e * zero, and P' = e * scale in fp16 hi + lo.
// The split partial (m, l, o + z) goes to the workspace; a combine pass merges splits.
// 2- and 4-bit codes are converted in pairs straight from their packed words, which
// orders the channels of each 16 (8) channel group as (k, k + 8) ((k, k + 4)) pairs; the
// query and the output use the same order.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "sm100.cuh"
#include "tmap.h"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kN = 128;                         // cached positions per tile
constexpr int kRows = 128;                      // folded rows per CTA = TMEM lanes
constexpr int kConvWarps = 4;
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = kConvWarps + kSoftWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);   // 416
constexpr int kPartialStride = 132;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;                   // log2 headroom of the running reference
constexpr int kHalfBytes = 16384;               // [128 rows][64 x 16-bit], 128-byte swizzled

constexpr int kColS = 0;                        // 2 x 128 columns: double-buffered scores
constexpr int kColP = 256;                      // P' hi (64 columns) then P' lo (64)
constexpr int kColO = 384;                      // 128 columns
constexpr int kCols = 512;

struct FaBars {
  uint64_t full, cfree;            // code stage: filled by TMA / read by the converters
  uint64_t conv[2], kvfree[2];     // operand buffers: written / released by their MMAs
  uint64_t sfull[2], sfree[2];     // score buffers: computed / read by the softmax warps
  uint64_t pfull, pvdone;          // P' written (and O rescaled) / PV MMA done
  uint32_t tmem_base;
  int abort;
};

template <int BITS>
struct FaCfg {
  static constexpr int kCode = 16 * BITS;
  static constexpr int kStage = 2 * kN * kCode;              // K then V codes of one tile
  static constexpr int kOffQh = 0;                            // A of S: q' hi [2 halves][128 rows][128 B]
  static constexpr int kOffQl = kOffQh + 2 * kHalfBytes;      // q' lo
  static constexpr int kOffKb = kOffQl + 2 * kHalfBytes;      // B of S: 2 buffers [2 halves][128 pos][128 B]
  static constexpr int kOffVb = kOffKb + 4 * kHalfBytes;      // B of PV: 2 buffers, same layout (MN-major)
  static constexpr int kOffStage = kOffVb + 4 * kHalfBytes;
  static constexpr int kOffMeta = kOffStage + kStage;         // 2 buffers of {ks, kz, vs, vz}[128] + 4 mask words
  static constexpr int kMetaBytes = 4 * kN * 4 + 16;
  static constexpr int kOffRow = kOffMeta + 2 * kMetaBytes;   // row exchange [2][2][128] + [2][128] x 2
  static constexpr int kOffBar = kOffRow + 8 * kRows * 4;
  static constexpr int kSmem = kOffBar + (int)sizeof(FaBars) + 1024;
  static_assert(kOffStage % 1024 == 0, "TMA boxes need 1 KB alignment");
  static_assert(kSmem <= 227 * 1024, "one CTA per SM");
};

struct FaArgs {
  const uint16_t* k_meta;
  const uint16_t* v_meta;
  CacheRows rows;
  const float* q;              // [B][n_q][Hq][128]
  const int32_t* ctx_len;
  float* ws;                   // partials [(b, i, h)][splits][132]
  int32_t* status;
  int n_q, hq, hkv, capacity, num_splits, row_blocks, box_rows;
  float scale_log2;            // softmax scale * log2 e
};

// Channel held by slot s of a converted 128-value row (see the header).
template <int BITS>
__host__ __device__ __forceinline__ int slot_channel(int s) {
  if (BITS == 2) return (s & ~15) | ((s >> 1) & 7) | ((s & 1) << 3);
  if (BITS == 4) return (s & ~7) | ((s >> 1) & 3) | ((s & 1) << 2);
  return s;
}

// TMA swizzle of a stage's code rows (as the decode kernel's tensor maps lay them out).
template <int BITS>
__device__ __forceinline__ int stage_swizzle(int row) {
  return BITS == 2 ? ((row >> 2) & 1) : BITS == 4 ? ((row >> 1) & 3) : 0;
}

template <int BITS>
__device__ __forceinline__ void load_code_row(const uint8_t* tile, int row, uint32_t (&w)[4 * BITS]) {
  const uint8_t* p = tile + row * (16 * BITS);
  const int sw = stage_swizzle<BITS>(row);
#pragma unroll
  for (int q = 0; q < BITS; ++q) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + 16 * (q ^ sw));
    w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
  }
}

// fp16 pair (1024 + a, 1024 + b) -> (a, b), exact for small integers
__device__ __forceinline__ uint32_t unbias2(uint32_t x) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&x), __halves2half2(__ushort_as_half(0x6400),
                                                                                    __ushort_as_half(0x6400)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Word j (slots 2j, 2j + 1) of a packed row's 128 codes as an fp16 pair, slot order.
template <int BITS>
__device__ __forceinline__ uint32_t code_pair_f16(const uint32_t (&w)[4 * BITS], int j) {
  if (BITS == 2) return unbias2(((w[j >> 3] >> (2 * (j & 7))) & 0x00030003u) | 0x64006400u);
  if (BITS == 4) return unbias2(((w[j >> 2] >> (4 * (j & 3))) & 0x000F000Fu) | 0x64006400u);
  const int bit = 6 * j, wi = bit >> 5, sh = bit & 31;   // channels 2j, 2j + 1 at bits 6j .. 6j + 5
  const uint32_t hi = (wi + 1 < 4 * BITS) ? w[wi + 1] : 0u;
  const uint32_t f = __funnelshift_r(w[wi], hi, sh);
  return unbias2(((f & 7u) | ((f & 0x38u) << 13)) | 0x64006400u);
}

// A packed row's codes as exact fp16 in slot order, stored as row r of a [2 halves][128
// rows][128 B] 128-byte-swizzled operand, one 16-byte chunk at a time.
template <int BITS>
__device__ __forceinline__ void store_code_row(uint8_t* base, int r, const uint32_t (&w)[4 * BITS]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t x0 = code_pair_f16<BITS>(w, 4 * c), x1 = code_pair_f16<BITS>(w, 4 * c + 1);
    const uint32_t x2 = code_pair_f16<BITS>(w, 4 * c + 2), x3 = code_pair_f16<BITS>(w, 4 * c + 3);
    *reinterpret_cast<uint4*>(base + (c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
        make_uint4(x0, x1, x2, x3);
  }
}

template <int KIND>
__device__ __forceinline__ void meta_of(uint32_t raw, int bits, float& scale, float& zero) {
  if (KIND == WUSHKV_QUEST_INT) {
    scale = f16_bits_to_f32((uint16_t)raw);
    zero = -((float)(1 << (bits - 1)) - 0.5f) * scale;
  } else {
    scale = f16_bits_to_f32((uint16_t)(raw & 0xffffu));
    zero = f16_bits_to_f32((uint16_t)(raw >> 16));
  }
}

template <int BITS, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_fa_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, FaArgs a) {
  using C = FaCfg<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qh = smem + C::kOffQh;
  uint8_t* ql = smem + C::kOffQl;
  uint8_t* kb = smem + C::kOffKb;
  uint8_t* vb = smem + C::kOffVb;
  uint8_t* stage = smem + C::kOffStage;
  uint8_t* meta = smem + C::kOffMeta;
  float* rowx = reinterpret_cast<float*>(smem + C::kOffRow);
  FaBars* bars = reinterpret_cast<FaBars*>(smem + C::kOffBar);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, kv = blockIdx.y / a.row_blocks, rb = blockIdx.y % a.row_blocks, b = blockIdx.z;
  const int g = a.hq / a.hkv, R = a.n_q * g;
  int ctx = __ldg(a.ctx_len + b);
  if (ctx > a.capacity) {
    if (split == 0 && blockIdx.y == 0 && threadIdx.x == 0) report(a.status, WUSHKV_STATUS_CTX_OVERFLOW);
    ctx = a.capacity;
  }
  if (ctx < 0) ctx = 0;
  const int tiles_all = (ctx + kN - 1) / kN;
  const int per = (tiles_all + a.num_splits - 1) / a.num_splits;
  const int tile0 = split * per;
  const int n = max(0, min(per, tiles_all - tile0));
  const int pair = b * a.hkv + kv;
  const bool paged = a.rows.block_table != nullptr;

  if (threadIdx.x == 0) {
    mbar_init(&bars->full, 1);
    mbar_init(&bars->cfree, kConvWarps);
    for (int j = 0; j < 2; ++j) {
      mbar_init(&bars->conv[j], kConvWarps);
      mbar_init(&bars->kvfree[j], 1);
      mbar_init(&bars->sfull[j], 1);
      mbar_init(&bars->sfree[j], kSoftWarps);
    }
    mbar_init(&bars->pfull, kSoftWarps);
    mbar_init(&bars->pvdone, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kCols);
    tmem_relinquish();
  }

  // Warp 12: the copies of tile i's K and V code rows into the stage (one 3-D box per
  // side, or one per page the tile touches; rows past the capacity arrive as zeros).
  int issued = 0;
  auto issue_load = [&](int i) {
    ++issued;
    const int t0 = (tile0 + i) * kN;
    uint8_t* kdst = stage;
    uint8_t* vdst = stage + kN * C::kCode;
    if (lane == 0) mbar_arrive_expect_tx(&bars->full, C::kStage);
    __syncwarp();
    if (!paged) {
      if (lane == 0) {
        tma_load_3d(kdst, &kmap, &bars->full, 0, t0, pair);
        tma_load_3d(vdst, &vmap, &bars->full, 0, t0, pair);
      }
    } else if (lane < kN / a.box_rows) {
      const int t = t0 + lane * a.box_rows;
      const int page = t < a.capacity
                           ? __ldg(a.rows.block_table + (size_t)b * a.rows.pages_per_seq + (t >> a.rows.page_shift))
                           : -1;
      const bool in = page >= 0 && page < a.rows.num_pages;
      const int c1 = in ? (t & ((1 << a.rows.page_shift) - 1)) : 0;
      const int c2 = in ? page * a.hkv + kv : a.rows.num_pages * a.hkv;
      const int off = lane * a.box_rows * C::kCode;
      tma_load_3d(kdst + off, &kmap, &bars->full, 0, c1, c2);
      tma_load_3d(vdst + off, &vmap, &bars->full, 0, c1, c2);
    }
  };
  if (warp == kMmaWarp) {
    __syncwarp();
    tma_prefetch(&kmap);
    tma_prefetch(&vmap);
    if (n > 0) issue_load(0);
  }

  // Softmax warps: row r of this block, half hf of each tile's positions (and of the
  // query's slots while preparing the query operand).
  const int sw = warp - kConvWarps;
  const int r = 32 * (warp & 3) + lane;
  const int hf = sw >> 2;
  const int f = rb * kRows + r;
  const bool row_ok = f < R;
  const int qi = row_ok ? f / g : 0;
  const int qh_idx = row_ok ? kv * g + f % g : 0;
  const int p_last = ctx - a.n_q + qi;                 // last visible position of this row
  float rowc = 0.f, qs = 0.f;                            // per row: tau log2e / sigma, tau log2e sum q'
  const uint32_t bar_pair = 2 + (warp & 3);              // the two softmax warps of a lane quarter
  if (warp >= kConvWarps && warp < kMmaWarp) {
    // q' row (fp32) -> sigma q' in fp16 hi + lo, slots 64 hf .. 64 hf + 63
    const float* qrow = a.q + (((size_t)b * a.n_q + qi) * a.hq + qh_idx) * kHeadDim;
    float v[64];
    float mx = 0.f, sm = 0.f;
#pragma unroll
    for (int s = 0; s < 64; ++s) {
      v[s] = row_ok ? __ldg(qrow + slot_channel<BITS>(64 * hf + s)) : 0.f;
      mx = fmaxf(mx, fabsf(v[s]));
      sm += v[s];
    }
    rowx[hf * kRows + r] = mx;
    rowx[2 * kRows + hf * kRows + r] = sm;
    named_barrier(bar_pair, 64);
    mx = fmaxf(mx, rowx[(1 - hf) * kRows + r]);
    sm += rowx[2 * kRows + (1 - hf) * kRows + r];
    int e2 = 0;
    if (mx > 0.f) frexpf(mx, &e2);
    const float sigma = ldexpf(1.0f, 10 - e2);           // |sigma q'| < 1024
    rowc = a.scale_log2 / sigma;
    qs = sm * a.scale_log2;
#pragma unroll
    for (int c = 0; c < 8; ++c) {                        // 16-byte chunk c: slots 8c .. 8c + 7
      uint32_t x[4], y[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x0 = v[8 * c + 2 * k] * sigma, x1 = v[8 * c + 2 * k + 1] * sigma;
        const __half2 h2 = __floats2half2_rn(x0, x1);
        const float2 hb = __half22float2(h2);
        const __half2 l2 = __floats2half2_rn(x0 - hb.x, x1 - hb.y);
        x[k] = *reinterpret_cast<const uint32_t*>(&h2);
        y[k] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      const int off = hf * kHalfBytes + r * 128 + ((c ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(qh + off) = make_uint4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<uint4*>(ql + off) = make_uint4(y[0], y[1], y[2], y[3]);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < kConvWarps) {
    // ------------------------------------------------------------- converters
    const int t = threadIdx.x;                           // position t of each tile
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      bool ok = mbar_wait(&bars->full, i & 1, abort);
      uint32_t wk[4 * BITS], wv[4 * BITS];
      if (ok) {
        load_code_row<BITS>(stage, t, wk);
        load_code_row<BITS>(stage + kN * C::kCode, t, wv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->cfree);
      const int pos = (tile0 + i) * kN + t;
      float ks = 0.f, kz = 0.f, vs = 0.f, vz = 0.f;
      bool valid = false;
      if (pos < ctx) {
        const long long row = a.rows.row(b, kv, pos);
        if (row >= 0) {
          valid = true;
          uint32_t km, vm;
          if (KIND == WUSHKV_QUEST_INT) {
            km = __ldg(a.k_meta + row);
            vm = __ldg(a.v_meta + row);
          } else {
            km = __ldg(reinterpret_cast<const uint32_t*>(a.k_meta) + row);
            vm = __ldg(reinterpret_cast<const uint32_t*>(a.v_meta) + row);
          }
          meta_of<KIND>(km, BITS, ks, kz);
          meta_of<KIND>(vm, BITS, vs, vz);
        } else {
          report(a.status, WUSHKV_STATUS_BAD_PAGE);
        }
      }
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      if (i >= 2) ok = mbar_wait(&bars->kvfree[buf], ((i - 2) >> 1) & 1, abort) && ok;
      float* mt = reinterpret_cast<float*>(meta + buf * C::kMetaBytes);
      mt[t] = ks;
      mt[kN + t] = kz;
      mt[2 * kN + t] = vs;
      mt[3 * kN + t] = vz;
      if (lane == 0) reinterpret_cast<uint32_t*>(mt + 4 * kN)[warp] = vmask;
      if (ok) {
        if (!valid) {
#pragma unroll
          for (int q = 0; q < 4 * BITS; ++q) { wk[q] = 0u; wv[q] = 0u; }
        }
        store_code_row<BITS>(kb + buf * 2 * kHalfBytes, t, wk);
        store_code_row<BITS>(vb + buf * 2 * kHalfBytes, t, wv);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->conv[buf]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- loads + MMAs
    // The whole warp walks the tiles (the paged copies use several lanes); lane 0 waits
    // and issues the MMAs, the other lanes follow it through __syncwarp.
    constexpr uint32_t kIdS = idesc(kFmtF32, kFmtF16, kFmtF16, 0, 0, 128, 128);
    constexpr uint32_t kIdPV = idesc(kFmtF32, kFmtF16, kFmtF16, 0, 1, 128, 128);
    const uint32_t qh_a = smem_u32(qh), ql_a = smem_u32(ql), kb_a = smem_u32(kb), vb_a = smem_u32(vb);
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = mbar_wait(bar, parity, abort);
      return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    };
    auto pv = [&](int j) {
      if (!(ok = ok && wait_all(&bars->pfull, j & 1))) return;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t vbase = vb_a + (j & 1) * 2 * kHalfBytes;
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_f16_ts(tmem + kColO, tmem + kColP + pl * 64 + ks * 8,
                       make_desc(vbase + ks * 2048, kHalfBytes, 1024, 2), kIdPV, (j > 0 || pl > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->pvdone);
        mma_commit(&bars->kvfree[j & 1]);
      }
      __syncwarp();
    };
    for (int i = 0; i < n && ok; ++i) {
      const int buf = i & 1;
      if (i + 1 < n) {                                   // the next tile's codes, once these are read
        if (!(ok = wait_all(&bars->cfree, i & 1))) break;
        issue_load(i + 1);
      }
      if (!(ok = wait_all(&bars->conv[buf], (i >> 1) & 1))) break;
      if (i >= 2 && !(ok = wait_all(&bars->sfree[buf], ((i - 2) >> 1) & 1))) break;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t kbase = kb_a + buf * 2 * kHalfBytes;
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * kHalfBytes + (ks & 3) * 32;
            mma_f16_ss(tmem + kColS + buf * 128, desc_kmajor_sw128((pl ? ql_a : qh_a) + off),
                       desc_kmajor_sw128(kbase + off), kIdS, (pl | ks) != 0);
          }
        mma_commit(&bars->sfull[buf]);
      }
      __syncwarp();
      if (i >= 1) pv(i - 1);
    }
    if (ok && n > 0) pv(n - 1);
    // no copy may land after the CTA has exited, even after a timeout
    if (lane == 0 && !ok && issued > 0) {
      volatile int no_abort = 0;
      mbar_wait(&bars->full, (issued - 1) & 1, &no_abort);
    }
  } else {
    // ------------------------------------------------------------- softmax
    float m_ref = -CUDART_INF_F, l = 0.f, z = 0.f;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      ok = ok && mbar_wait(&bars->sfull[buf], (i >> 1) & 1, abort);
      ok = ok && mbar_wait(&bars->conv[buf], (i >> 1) & 1, abort);
      tc_fence_after();
      const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
      uint32_t raw[64];
      tmem_ld32(tmem + lanes + kColS + buf * 128 + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(raw));
      tmem_ld32(tmem + lanes + kColS + buf * 128 + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->sfree[buf]);
      const float* mt = reinterpret_cast<const float*>(meta + buf * C::kMetaBytes);
      const uint32_t vm0 = reinterpret_cast<const uint32_t*>(mt + 4 * kN)[2 * hf];
      const uint32_t vm1 = reinterpret_cast<const uint32_t*>(mt + 4 * kN)[2 * hf + 1];
      const int pos0 = (tile0 + i) * kN + 64 * hf;
      float s[64];
      float mloc = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(mt + 64 * hf + j);
        const float4 z4 = *reinterpret_cast<const float4*>(mt + kN + 64 * hf + j);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w}, zz[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int jj = j + e;
          const bool vis = (((jj < 32 ? vm0 >> jj : vm1 >> (jj - 32)) & 1u) != 0u) && pos0 + jj <= p_last;
          const float x = fmaf(kk[e] * rowc, __uint_as_float(raw[jj]), zz[e] * qs);
          s[jj] = vis ? x : -CUDART_INF_F;
          mloc = fmaxf(mloc, s[jj]);
        }
      }
      // tile maximum of the row (both halves)
      rowx[4 * kRows + (i & 1) * 2 * kRows + hf * kRows + r] = mloc;
      named_barrier(bar_pair, 64);
      const float m_tile = fmaxf(mloc, rowx[4 * kRows + (i & 1) * 2 * kRows + (1 - hf) * kRows + r]);
      float m_new = m_ref;
      if (m_tile != -CUDART_INF_F && (m_ref == -CUDART_INF_F || m_tile > m_ref + kLazy)) m_new = m_tile;
      const bool rescale = m_new != m_ref && m_ref != -CUDART_INF_F;
      const float corr = rescale ? ex2_approx(m_ref - m_new) : 1.f;
      const float mref = m_new == -CUDART_INF_F ? 0.f : m_new;
      // P' and O are free once the previous tile's PV MMA is done; O is rescaled when the
      // reference moved
      if (i >= 1) ok = mbar_wait(&bars->pvdone, (i - 1) & 1, abort) && ok;
      tc_fence_after();
      // tensor-memory loads and stores are warp-collective: the warp rescales when any
      // of its rows moved its reference (corr = 1 for the others)
      ok = __all_sync(0xffffffffu, ok);
      if (__any_sync(0xffffffffu, rescale) && ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 16) {
          uint32_t ov[16];
          tmem_ld16(tmem + lanes + kColO + 64 * hf + c0, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
          tmem_st16(tmem + lanes + kColO + 64 * hf + c0, ov);
        }
      }
      // P' = e * scale in fp16 hi + lo, 32 positions at a time
      float lt = 0.f, zt = 0.f;
#pragma unroll
      for (int jc = 0; jc < 64; jc += 32) {
        uint32_t ph[16], plo[16];
#pragma unroll
        for (int j = jc; j < jc + 32; j += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(mt + 2 * kN + 64 * hf + j);
          const float4 w4 = *reinterpret_cast<const float4*>(mt + 3 * kN + 64 * hf + j);
          const float vv[4] = {v4.x, v4.y, v4.z, v4.w}, ww[4] = {w4.x, w4.y, w4.z, w4.w};
          float pp[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float ex = ex2_approx(s[j + e] - mref);
            lt += ex;
            zt = fmaf(ex, ww[e], zt);
            pp[e] = ex * vv[e];
          }
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const __half2 h2 = __floats2half2_rn(pp[e], pp[e + 1]);
            const float2 hb = __half22float2(h2);
            const __half2 l2 = __floats2half2_rn(pp[e] - hb.x, pp[e + 1] - hb.y);
            ph[(j - jc + e) >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
            plo[(j - jc + e) >> 1] = *reinterpret_cast<const uint32_t*>(&l2);
          }
        }
        tmem_st16(tmem + lanes + kColP + 32 * hf + jc / 2, ph);
        tmem_st16(tmem + lanes + kColP + 64 + 32 * hf + jc / 2, plo);
      }
      l = fmaf(l, corr, lt);
      z = fmaf(z, corr, zt);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pfull);
      m_ref = m_new;
    }
    // ---- split partial of the row: m (log2 domain), l, o + z
    uint32_t o[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) o[e] = 0u;
    if (n > 0) {
      ok = ok && mbar_wait(&bars->pvdone, (n - 1) & 1, abort);
      tc_fence_after();
      const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
      tmem_ld32(tmem + lanes + kColO + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(o));
      tmem_ld32(tmem + lanes + kColO + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
      tmem_ld_wait();
      tc_fence_before();
    }
    rowx[hf * kRows + r] = l;
    rowx[2 * kRows + hf * kRows + r] = z;
    named_barrier(bar_pair, 64);
    const float l_tot = l + rowx[(1 - hf) * kRows + r];
    const float z_tot = z + rowx[2 * kRows + (1 - hf) * kRows + r];
    if (row_ok) {
      float* dst = a.ws + ((((size_t)b * a.n_q + qi) * a.hq + qh_idx) * a.num_splits + split) * kPartialStride;
#pragma unroll
      for (int e = 0; e < 64; ++e) dst[4 + slot_channel<BITS>(64 * hf + e)] = __uint_as_float(o[e]) + z_tot;
      if (hf == 0) {
        dst[0] = m_ref;
        dst[1] = l_tot;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort) report(a.status, WUSHKV_STATUS_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// Tensor map over one side's codes ([planes][rows][16 * BITS bytes], boxes of box_rows rows,
// swizzled as stage_swizzle reads them).
template <int BITS>
bool chunk_code_map(CUtensorMap* m, const uint8_t* base, int rows, int planes, int box_rows) {
  const uint64_t dims[3] = {(uint64_t)(16 * BITS), (uint64_t)rows, (uint64_t)planes};
  const uint64_t strides[2] = {(uint64_t)(16 * BITS), (uint64_t)rows * (16 * BITS)};
  const uint32_t box[3] = {(uint32_t)(16 * BITS), (uint32_t)box_rows, 1};
  const CUtensorMapSwizzle sw = BITS == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                : BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, sw);
}

template <int BITS>
cudaError_t launch_bits(const wushkv_cache& c, const FaArgs& a, int batch, cudaStream_t stream) {
  CUtensorMap km, vm;
  const bool paged = c.block_table != nullptr;
  const int rows = paged ? c.page_size : c.capacity;
  const int planes = paged ? c.num_pages * c.num_kv_heads : c.batch * c.num_kv_heads;
  if (!chunk_code_map<BITS>(&km, c.k_codes, rows, planes, a.box_rows) ||
      !chunk_code_map<BITS>(&vm, c.v_codes, rows, planes, a.box_rows))
    return cudaErrorInvalidValue;
  const dim3 grid(a.num_splits, a.hkv * a.row_blocks, batch);
  if (c.qp.kind == WUSHKV_QUEST_INT) {
    auto kern = chunk_fa_kernel<BITS, WUSHKV_QUEST_INT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FaCfg<BITS>::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, FaCfg<BITS>::kSmem, stream>>>(km, vm, a);
  } else {
    auto kern = chunk_fa_kernel<BITS, WUSHKV_PCT_AFFINE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FaCfg<BITS>::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, FaCfg<BITS>::kSmem, stream>>>(km, vm, a);
  }
  return cudaGetLastError();
}

int row_blocks_of(int n_q, int g) { return (n_q * g + kRows - 1) / kRows; }

// Split count when the caller passes 0: one CTA per SM, so the modelled time is the
// waves of CTAs over the SMs times (tiles per split + 2, for a CTA's set-up and partial).
int auto_chunk_splits(const wushkv_cache& c, int num_q_heads, int n_q) {
  const long long ctas = (long long)c.batch * c.num_kv_heads * row_blocks_of(n_q, num_q_heads / c.num_kv_heads);
  const int tiles = (c.capacity + kN - 1) / kN;
  const long long slots = num_sms(nullptr);
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= tiles && s <= 256; ++s) {
    const long long waves = (ctas * s + slots - 1) / slots;
    const long long cost = waves * ((tiles + s - 1) / s + 2);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = s; }
  }
  return best;
}

}  // namespace

size_t chunk_workspace_bytes(const wushkv_cache& c, int num_q_heads, int n_q, int num_splits) {
  const int s = num_splits > 0 ? num_splits : auto_chunk_splits(c, num_q_heads, n_q);
  return (size_t)c.batch * n_q * num_q_heads * s * kPartialStride * sizeof(float);
}

cudaError_t launch_chunk_attention(const wushkv_cache& c, const float* q_t, int n_q, int num_q_heads,
                                   const int32_t* ctx_len, float softmax_scale, float* out, void* workspace,
                                   int num_splits, int32_t* status, cudaStream_t stream) {
  FaArgs a{};
  a.k_meta = c.k_meta;
  a.v_meta = c.v_meta;
  a.rows = CacheRows::of(c);
  a.q = q_t;
  a.ctx_len = ctx_len;
  a.ws = static_cast<float*>(workspace);
  a.status = status;
  a.n_q = n_q;
  a.hq = num_q_heads;
  a.hkv = c.num_kv_heads;
  a.capacity = c.capacity;
  a.num_splits = num_splits > 0 ? num_splits : auto_chunk_splits(c, num_q_heads, n_q);
  a.row_blocks = row_blocks_of(n_q, num_q_heads / c.num_kv_heads);
  a.box_rows = c.block_table != nullptr ? (c.page_size < kN ? c.page_size : kN) : kN;
  a.scale_log2 = softmax_scale * kLog2e;
  cudaError_t e;
  switch (c.qp.bits) {
    case 2: e = launch_bits<2>(c, a, c.batch, stream); break;
    case 3: e = launch_bits<3>(c, a, c.batch, stream); break;
    default: e = launch_bits<4>(c, a, c.batch, stream); break;
  }
  if (e != cudaSuccess) return e;
  return launch_combine_partials(a.ws, c.batch * n_q * num_q_heads, a.num_splits, out, stream);
}

}  // namespace wushkv
