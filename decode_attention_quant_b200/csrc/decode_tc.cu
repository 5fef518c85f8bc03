// Split-K GQA decode attention directly over the packed cache, on the tensor cores.
//
// WUSH-KV serves grouped-query attention over a 2-bit cache (ai4snews summary,
// paragraph 5) at long context (paragraph 4).  The codes are small integers, so
// both contractions run exactly as integer MMAs (tcgen05.mma kind::i8, int32
// accumulate) and the fp16 meta is applied afterwards:
//   scores  s_t = tau * (scale_t * sum_c q'_c code_tc + zero_t * sum_c q'_c)
//           sum_c q'_c code_tc = (M / 2^30) * sum_c qi_c (f_c code_tc), where the key
//           codes are widened by masking alone, so byte c holds f_c code_tc with a
//           power of two f_c (see key_shift), and qi_c = rne(q'_c 2^30 / (M f_c)), M =
//           max |q'|, is split into four int8 limbs qi = l0 + 2^8 l1 + 2^16 l2 + 2^24 l3;
//   values  o_c = sum_t p_t (zero_t + scale_t code_tc)
//               = (F / 65535) * sum_t pi_t code_tc + sum_t p_t zero_t,
//           with p_t scale_t rounded to 16-bit integers pi = u0 + 2^8 u1 (per tile and
//           head, F = the tile's largest p_t scale_t) split into two uint8 limbs.
// (QuEST: scale = Delta, zero = -(2^(b-1) - 1/2) Delta.)  The softmax is online in the
// log2 domain across 256-token tiles.
//
// One CTA = one (sequence, KV head, split); tiles of 256 tokens, five warps:
//   warp 0      one thread: TMA copies of each tile's packed K and V codes into a
//               ring of stages (swizzled so the row reads are bank-conflict free), and every MMA, each issued when the mbarrier of the
//               event it needs completes (key codes widened; probabilities written).
//   warps 1-4   token warps.  Thread = tokens r and 128 + r of the tile (lane r of
//               the two M = 128 score MMAs) while widening codes to u8 (K codes into
//               tensor memory as A of the score MMAs, V codes into channel-major
//               shared memory as A of the value MMAs) and while turning scores into
//               probability limbs (B of the value MMAs); thread = channel while
//               accumulating the value MMAs' int32 result.  They signal the issuing
//               thread by mbarrier arrivals and meet each other only to share each
//               tile's maxima.
// Per tile i the token warps run: softmax(i) -> [value MMAs(i)]; widen K(i+1) ->
// [score MMAs(i+1)]; accumulate(i); widen V(i+1).  Every buffer is single: each is
// rewritten only after the event that ends its last read.  Two tokens per thread
// halve the per-tile work (waits, maxima exchange, rescaling, accumulation) per
// token.  Up to three CTAs run per SM (2-bit codes, g <= 4: two stages, ~73 KB shared
// memory and 128 TMEM columns each); wider codes or groups run two (4-bit, g = 16: one).
// 2- and 4-bit codes are widened to bytes by masking alone (one logic op per 4
// codes), which permutes channels inside each 16 (8) channel block and leaves a
// power-of-two factor on each channel; the query limbs and the output channels use
// the same permutation, the query limbs divide the key factor out and the split
// partial divides the value factor out, so both contractions are unchanged.
#include <math_constants.h>

#include <cmath>

#include "sm100.cuh"
#include "tmap.h"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"
#include "wushkv_quant.cuh"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kHalf = 128;              // tokens of one MMA (M) = one sweep of the 128 TMEM lanes
constexpr int kTile = 2 * kHalf;        // tokens per pipeline step: two per token-warp thread
constexpr int kThreads = 160;
constexpr int kPartialStride = 132;     // m (log2 domain), l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQScale = 1073741824.0f;  // 2^30: query integers up to 2^30 before the key factor
constexpr uint32_t kBarTok = 1;         // named barrier of the four token warps
constexpr int kSmemPerSm = 233472;      // bytes of shared memory per SM, 1 KB of it reserved per CTA

__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ constexpr int pow2cols(int x) { return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512; }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int BITS, int G>
struct Cfg {
  static constexpr int kCode = 16 * BITS;                  // packed bytes per token row
  static constexpr int kStage = 2 * kTile * kCode;         // K then V codes of one tile
  static constexpr int NK = round16(4 * G);                // score MMA N (4 limbs per head)
  static constexpr int NV = round16(2 * G);                // value MMA N (2 limbs per head)
  static constexpr int kColAk = 0;                         // 2 halves x 32 columns (u8 x 128 channels)
  static constexpr int kColS = 64;                         // 2 halves x NK
  static constexpr int kColO = 64 + 2 * NK;                // NV
  static constexpr int kCols = pow2cols(64 + 2 * NK + NV);
  // shared memory (offsets from a 1024-byte aligned base): stages, then the widened V
  // codes of both halves (channel-major, 128-byte swizzled), the probability limbs of
  // both halves, the query limbs, barriers and reduction scratch
  static constexpr int kFixed = 2 * kHalf * 128 + 2 * NV * 128 + NK * 128 + 2048 + 1024;
  // as many resident CTAs per SM (up to 3) as leave room for a double-buffered ring
  static constexpr int ring(int ctas) { return (kSmemPerSm / ctas - 1024 - kFixed) / kStage; }
  // (g = 8 would need more than the 128 registers three CTAs leave a thread: two)
  static constexpr int kCtas = (ring(3) >= 2 && G <= 4) ? 3 : ring(2) >= 2 ? 2 : 1;
  static constexpr int kSmemPerCta = kSmemPerSm / kCtas - 1024;
  static constexpr int kStages = cmin(4, ring(kCtas));
  static constexpr int kOffStage = 0;
  static constexpr int kOffAv = (kOffStage + kStages * kStage + 1023) / 1024 * 1024;
  static constexpr int kOffBv = kOffAv + 2 * kHalf * 128;
  static constexpr int kOffBk = kOffBv + 2 * NV * 128;
  static constexpr int kOffMisc = kOffBk + NK * 128;
  static constexpr int kMiscBytes = 2048;
  static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;
  static_assert(kStages >= 2, "too little shared memory for a double-buffered ring");
  static_assert(kSmem <= kSmemPerCta, "the CTAs must fit on an SM");
};

struct DecArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint16_t* k_meta;
  const uint16_t* v_meta;
  int hkv, hq, capacity, num_splits;
  const float* q;          // [B][Hq][128]
  const int32_t* ctx_len;
  float scale_log2;        // softmax scale * log2(e)
  float* ws;               // [B][Hq][S][132]
  int32_t* status;
  CacheRows rows;          // (sequence, head, position) -> row, contiguous or paged
  int box_rows;            // rows of one code box: the tile (contiguous) or min(page, tile)
};

struct Misc {
  uint64_t full[4];           // stage filled (bulk copies)
  uint64_t kw;                // 4 token warps: key codes of the tile widened
  uint64_t pr;                // 4 token warps: probabilities written (value codes widened before)
  uint64_t kdone;             // score MMAs of the tile done
  uint64_t vdone;             // value MMAs of the tile done
  uint32_t tmem_base;
  int abort;
  float4 red[2][33];          // per tile parity: head maxima and the value-scale maximum, per token warp
  float c1[16], c2[16];       // per head: qscale * softmax_scale * log2 e, sum(q') * softmax_scale * log2 e
};

// position p of a widened code row <-> channel
template <int BITS>
__device__ __forceinline__ int channel_of(int p) {
  if (BITS == 2) return (p & ~15) | ((p & 3) << 2) | ((p >> 2) & 3);
  if (BITS == 4) return (p & ~7) | ((p & 3) << 1) | ((p >> 2) & 1);
  return p;
}

// TMA swizzle of a stage's code rows: 2-bit rows (32 B) use the 32-byte pattern, 4-bit
// rows (64 B) the 64-byte one (16-byte chunk index XOR address bits 7.. of the row), so
// the 16-byte reads of eight consecutive rows hit distinct banks; 3-bit rows (48 B) are
// conflict-free unswizzled.
template <int BITS>
__host__ __device__ constexpr int code_swizzle(int row) {
  return BITS == 2 ? ((row >> 2) & 1) : BITS == 4 ? ((row >> 1) & 3) : 0;
}

// Packed row `row` of a stage's code tile (16*BITS bytes per row) -> 4*BITS words.
template <int BITS>
__device__ __forceinline__ void load_row(const uint8_t* tile, int row, uint32_t (&w)[4 * BITS]) {
  const uint8_t* p = tile + row * (16 * BITS);
  const int sw = code_swizzle<BITS>(row);
#pragma unroll
  for (int q = 0; q < BITS; ++q) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + 16 * (q ^ sw));
    w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
  }
}

template <int BITS>
__device__ __forceinline__ void widen_words(const uint32_t (&w)[4 * BITS], uint32_t (&u)[32]) {
  constexpr int kWords = 4 * BITS;
  if (BITS == 2) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) u[4 * j + k] = (w[j] >> (2 * k)) & 0x03030303u;
  } else if (BITS == 4) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
      for (int k = 0; k < 2; ++k) u[2 * j + k] = (w[j] >> (4 * k)) & 0x0F0F0F0Fu;
  } else {
#pragma unroll
    for (int g = 0; g < 32; ++g) {              // codes 4g..4g+3: 12 bits at bit 12g
      const int bit = 12 * g, wi = bit >> 5, sh = bit & 31;
      const uint32_t hi = (wi + 1 < kWords) ? w[wi + 1] : 0u;
      const uint32_t f = __funnelshift_r(w[wi], hi, sh) & 0xFFFu;
      const uint32_t a = (f & 0x3Fu) | ((f & 0xFC0u) << 10);
      u[g] = (a & 0x00070007u) | ((a & 0x00380038u) << 5);
    }
  }
}

// Codes widened by masking alone: byte p then holds code * 2^key_shift(channel_of(p))
// (2-bit: 4^((p >> 2) & 3); 4-bit: 16^((p >> 2) & 1); 3-bit: the shifted form above,
// factor 1).  Bytes stay <= 240, so every MMA limb column fits int32 (score: 128 * 240 *
// 128 per channel sum; value: 255 * 240 * 256 per tile).
template <int BITS>
__device__ __forceinline__ void widen_words_scaled(const uint32_t (&w)[4 * BITS], uint32_t (&u)[32]) {
  if (BITS == 3) {
    widen_words<BITS>(w, u);
    return;
  }
  if (BITS == 2) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) u[4 * j + k] = w[j] & (0x03030303u << (2 * k));
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
      for (int k = 0; k < 2; ++k) u[2 * j + k] = w[j] & (0x0F0F0F0Fu << (4 * k));
  }
}

// log2 of the factor the masked widening leaves on channel c (2-bit: 4^(c & 3);
// 4-bit: 16^(c & 1); 3-bit: none), for key and value codes alike
template <int BITS>
__device__ __forceinline__ int key_shift(int c) {
  if (BITS == 2) return 2 * (c & 3);
  if (BITS == 4) return 4 * (c & 1);
  return 0;
}

template <int BITS>
__device__ __forceinline__ float value_scale_of(int p) {
  if (BITS == 2) return (float)(1 << (2 * ((p >> 2) & 3)));
  if (BITS == 4) return (float)(1 << (4 * ((p >> 2) & 1)));
  return 1.f;
}

template <int KIND>
__device__ __forceinline__ void meta_pair(uint32_t raw, int bits, float& scale, float& zero) {
  if (KIND == WUSHKV_QUEST_INT) {
    scale = f16_bits_to_f32((uint16_t)raw);
    zero = -((float)(1 << (bits - 1)) - 0.5f) * scale;
  } else {
    scale = f16_bits_to_f32((uint16_t)(raw & 0xffffu));
    zero = f16_bits_to_f32((uint16_t)(raw >> 16));
  }
}

template <int KIND>
__device__ __forceinline__ uint32_t load_meta(const uint16_t* meta, size_t row) {
  if (KIND == WUSHKV_QUEST_INT) return (uint32_t)__ldg(meta + row);
  return __ldg(reinterpret_cast<const uint32_t*>(meta) + row);
}

// byte (row n, column k) of a K-major operand stored as 128-byte rows, 128B-swizzled
__device__ __forceinline__ int kmajor_off(int n, int k) {
  return (n >> 3) * 1024 + (n & 7) * 128 + ((((k >> 4) ^ (n & 7)) & 7) << 4) + (k & 15);
}

template <int BITS, int KIND, int G>
__global__ void __launch_bounds__(kThreads, Cfg<BITS, G>::kCtas)
    decode_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, DecArgs a) {
  using C = Cfg<BITS, G>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage = smem + C::kOffStage;
  uint8_t* av = smem + C::kOffAv;
  uint8_t* bv = smem + C::kOffBv;
  uint8_t* bk = smem + C::kOffBk;
  Misc* ms = reinterpret_cast<Misc*>(smem + C::kOffMisc);
  volatile int* abort = &ms->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  int L = __ldg(a.ctx_len + b);
  if (L > a.capacity) {
    if (split == 0 && kv == 0 && threadIdx.x == 0) report(a.status, WUSHKV_STATUS_CTX_OVERFLOW);
    L = a.capacity;
  }
  if (L < 0) L = 0;
  const int tiles_all = (L + kTile - 1) / kTile;
  const int per = (tiles_all + a.num_splits - 1) / a.num_splits;
  const int tile0 = split * per;
  const int n = max(0, min(per, tiles_all - tile0));
  const size_t pair = (size_t)b * a.hkv + kv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&ms->full[s], 1);
    mbar_init(&ms->kw, 4);
    mbar_init(&ms->pr, 4);
    mbar_init(&ms->kdone, 1);
    mbar_init(&ms->vdone, 1);
    ms->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem_base, C::kCols);
    tmem_relinquish();
  }
  if (warp >= 1) {
    // query limbs (B of the score MMA): thread = code position p (channel channel_of(p))
    const int p = threadIdx.x - 32;
    const int c = channel_of<BITS>(p);
    const int wq = p >> 5;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float qv = a.q[((size_t)b * a.hq + kv * G + h) * kHeadDim + c];
      float mx = fabsf(qv), sm = qv;
#pragma unroll
      for (int off = 16; off; off >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
      mx = warp_max(mx);
      if (lane == 0) {
        reinterpret_cast<float*>(&ms->red[0][h])[wq] = mx;
        reinterpret_cast<float*>(&ms->red[1][h])[wq] = sm;
      }
    }
    named_barrier(kBarTok, 128);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float qv = a.q[((size_t)b * a.hq + kv * G + h) * kHeadDim + c];
      const float4 m4 = ms->red[0][h];
      const float mx = fmaxf(fmaxf(m4.x, m4.y), fmaxf(m4.z, m4.w));
      // the key byte of channel c carries 2^key_shift(c): divide it out of q' exactly
      const float inv = mx > 0.f ? kQScale / mx * __int_as_float((127 - key_shift<BITS>(c)) << 23) : 0.f;
      const int qi = __float2int_rn(qv * inv);              // |qi| <= 2^30
      const int l0 = (int)(int8_t)(qi & 0xff);
      const int r1 = (qi - l0) >> 8;
      const int l1 = (int)(int8_t)(r1 & 0xff);
      const int r2 = (r1 - l1) >> 8;
      const int l2 = (int)(int8_t)(r2 & 0xff);
      const int l3 = (r2 - l2) >> 8;                        // |l3| <= 64
      bk[kmajor_off(h, p)] = (uint8_t)l0;
      bk[kmajor_off(G + h, p)] = (uint8_t)l1;
      bk[kmajor_off(2 * G + h, p)] = (uint8_t)l2;
      bk[kmajor_off(3 * G + h, p)] = (uint8_t)l3;
      if (p == 0) {
        const float4 s4 = ms->red[1][h];
        ms->c1[h] = (mx > 0.f ? mx / kQScale : 0.f) * a.scale_log2;
        ms->c2[h] = ((s4.x + s4.y) + (s4.z + s4.w)) * a.scale_log2;
      }
    }
    for (int nrow = 4 * G; nrow < C::NK; ++nrow) bk[kmajor_off(nrow, p)] = 0;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // -------------------------------------------------- bulk loads + MMA issue
    // One thread, in the order the token warps produce: the value MMAs of tile i once
    // every token warp has written P(i) (its value codes were widened before), which
    // also frees tile i's stage for tile i + S; the score MMAs of tile i+1 once every
    // token warp has widened its key codes.
    if (lane == 0) {
      constexpr uint32_t kIdK = idesc(kFmtS32, kFmtU8, kFmtS8, 0, 0, 128, C::NK);
      constexpr uint32_t kIdV = idesc(kFmtS32, kFmtU8, kFmtU8, 1, 1, 128, C::NV);
      const uint32_t bk_addr = smem_u32(bk), bv_addr = smem_u32(bv), av_addr = smem_u32(av);
      tma_prefetch(&kmap);
      tma_prefetch(&vmap);
      int issued = 0;
      // a tile's K and V code rows, one 3-D box each ([pair][token][byte], swizzled);
      // rows past the capacity arrive as zeros, rows past the context are never used
      // paged caches: page of position t (-1 past the capacity)
      auto page_at = [&](int t) {
        return t < a.capacity ? __ldg(a.rows.block_table + (size_t)b * a.rows.pages_per_seq + (t >> a.rows.page_shift))
                              : -1;
      };
      int pf_tile = -1, pf_page = -1;
      auto load = [&](int i) {
        const int s = i % S;
        const int t0 = (tile0 + i) * kTile;
        mbar_arrive_expect_tx(&ms->full[s], 2 * kTile * C::kCode);
        if (a.rows.block_table == nullptr) {
          tma_load_3d(stage + s * C::kStage, &kmap, &ms->full[s], 0, t0, (int)pair);
          tma_load_3d(stage + s * C::kStage + kTile * C::kCode, &vmap, &ms->full[s], 0, t0, (int)pair);
        } else {
          // one box per page the tile touches ([page * Hkv + h][row in page][byte]); rows
          // past the capacity or in a page outside the pool come from an out-of-range
          // coordinate and arrive as zeros
          const int nb = kTile / a.box_rows;
          const int oob = a.rows.num_pages * a.hkv;
          for (int sb = 0; sb < nb; ++sb) {
            const int t = t0 + sb * a.box_rows;
            const int page = (nb == 1 && pf_tile == i) ? pf_page : page_at(t);
            const bool in = page >= 0 && page < a.rows.num_pages;
            const int c1 = in ? (t & ((1 << a.rows.page_shift) - 1)) : 0;
            const int c2 = in ? page * a.hkv + kv : oob;
            const int off = sb * a.box_rows * C::kCode;
            tma_load_3d(stage + s * C::kStage + off, &kmap, &ms->full[s], 0, c1, c2);
            tma_load_3d(stage + s * C::kStage + kTile * C::kCode + off, &vmap, &ms->full[s], 0, c1, c2);
          }
          if (nb == 1 && i + 1 < n) {        // the next tile's page, read while this one loads
            pf_tile = i + 1;
            pf_page = page_at((tile0 + i + 1) * kTile);
          }
        }
        ++issued;
      };
      auto score_mma = [&]() {
        tc_fence_after();
#pragma unroll
        for (int hb = 0; hb < 2; ++hb)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_i8_ts(tmem + C::kColS + hb * C::NK, tmem + C::kColAk + hb * 32 + ks * 8,
                      desc_kmajor_sw128(bk_addr + ks * 32), kIdK, ks > 0);
        mma_commit(&ms->kdone);
      };
      auto value_mma = [&]() {
        tc_fence_after();
#pragma unroll
        for (int hb = 0; hb < 2; ++hb)
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const uint64_t adesc = make_desc(av_addr + hb * kHalf * 128 + kq * 4096, 16384, 1024, 2);
            const uint64_t bdesc = make_desc(bv_addr + hb * C::NV * 128 + kq * 512, 128, 2048, 0);
            mma_i8_ss(tmem + C::kColO, adesc, bdesc, kIdV, (hb | kq) > 0);
          }
        mma_commit(&ms->vdone);
      };
      for (int i = 0; i < n && i < S; ++i) load(i);
      bool ok = n > 0 && mbar_wait(&ms->kw, 0, abort);
      if (ok) score_mma();
      for (int i = 0; ok && i < n; ++i) {
        if (!(ok = mbar_wait(&ms->pr, i & 1, abort))) break;
        value_mma();
        if (i + S < n) load(i + S);
        if (i + 1 < n) {
          if (!(ok = mbar_wait(&ms->kw, (i + 1) & 1, abort))) break;
          score_mma();
        }
      }
      // no copy may land after the CTA has exited, even after a timeout
      volatile int no_abort = 0;
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait(&ms->full[i % S], (i / S) & 1, &no_abort);
    }
  } else {
    // ------------------------------------------------------------- token warps
    // Thread = tokens r and 128 + r of the tile (TMEM lane r of both score halves)
    // while widening and in the softmax; channel position r while accumulating.
    // Each token warp signals the issuing thread with one mbarrier arrival per event
    // and meets the other token warps only to share each tile's maxima.  After a
    // failed (timed-out) wait a warp skips work but keeps arriving, so every phase
    // still completes.
    const int qd = warp & 3;                 // TMEM lane quarter
    const int r = 32 * qd + lane;
    const uint32_t lanes = (uint32_t)(32 * qd) << 16;
    bool ok = true;
    float m_run[G], l_run[G], z_run[G], o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; z_run[h] = 0.f; o[h] = 0.f; }
    uint32_t kmeta[2] = {0u, 0u}, vmeta[2] = {0u, 0u};
    bool page_ok[2] = {true, true};         // the tile's rows r, r + 128 sit in valid pages
    // paged caches: this thread's two meta rows for the next tile, looked up one tile
    // ahead so the block-table load is off the meta load's path
    long long next_row[2] = {0, 0};
    auto lookup_rows = [&](int i) {
      if (a.rows.block_table == nullptr || i >= n) return;
      const int t = (tile0 + i) * kTile + r;
#pragma unroll
      for (int j = 0; j < 2; ++j)
        next_row[j] = t + kHalf * j < L ? a.rows.row(b, kv, t + kHalf * j) : -1;
    };
    float c1[G], c2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { c1[h] = ms->c1[h]; c2[h] = ms->c2[h]; }
    const int rx4 = (r & 7) << 4;

    // key codes of tile i -> TMEM A (lane = token), and the tile's meta
    auto widen_k = [&](int i) {
      const int s = i % S;
      const int t = (tile0 + i) * kTile + r;
      long long rows_i[2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
        rows_i[j] = a.rows.block_table == nullptr ? a.rows.row(b, kv, t + kHalf * j) : next_row[j];
      lookup_rows(i + 1);
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if (t + kHalf * j < L) {
          const long long mrow = rows_i[j];
          page_ok[j] = mrow >= 0;
          if (mrow >= 0) {
            kmeta[j] = load_meta<KIND>(a.k_meta, (size_t)mrow);
            vmeta[j] = load_meta<KIND>(a.v_meta, (size_t)mrow);
          } else {
            report(a.status, WUSHKV_STATUS_BAD_PAGE);
          }
        }
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->full[s], (i / S) & 1, abort));
      if (ok) {
        uint32_t w[2][4 * BITS];                // both rows' loads in flight before widening
#pragma unroll
        for (int j = 0; j < 2; ++j) load_row<BITS>(stage + s * C::kStage, r + kHalf * j, w[j]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t wv[32];
          widen_words_scaled<BITS>(w[j], wv);
          tmem_st32(tmem + lanes + C::kColAk + 32 * j, wv);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->kw);
    };
    // value codes of tile i -> channel-major shared A of the value MMA (published by
    // the arrival on pr after the tile's probabilities)
    auto widen_v = [&](int i) {
      const int s = i % S;
      if (ok) {
        uint32_t w[2][4 * BITS];                // both rows' loads in flight before the stores
#pragma unroll
        for (int j = 0; j < 2; ++j) load_row<BITS>(stage + s * C::kStage + kTile * C::kCode, r + kHalf * j, w[j]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t wv[32];
          widen_words_scaled<BITS>(w[j], wv);
          uint8_t* arow = av + j * kHalf * 128 + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(arow + ((c << 4) ^ rx4)) =
                make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
    };

    lookup_rows(0);
    if (n > 0) {
      widen_k(0);
      widen_v(0);
    }
    for (int i = 0; i < n; ++i) {
      const int u = i & 1;
      const int tb = (tile0 + i) * kTile + r;
      const bool valid[2] = {tb < L && page_ok[0], tb + kHalf < L && page_ok[1]};
      float ks[2], kz[2], vs[2], vz[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        meta_pair<KIND>(kmeta[j], BITS, ks[j], kz[j]);
        meta_pair<KIND>(vmeta[j], BITS, vs[j], vz[j]);
        if (!valid[j]) { vs[j] = 0.f; vz[j] = 0.f; }
      }
      // ---- scores of tile i (both halves)
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->kdone, u, abort));
      tc_fence_after();
      float s2[2][G];
      constexpr bool kOneWait = 2 * C::NK <= 32;   // both halves' limbs in flight together
      uint32_t dd[kOneWait ? 2 : 1][C::NK];
      if (kOneWait) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int c0 = 0; c0 < C::NK; c0 += 16)
            tmem_ld16(tmem + lanes + C::kColS + j * C::NK + c0,
                      *reinterpret_cast<uint32_t(*)[16]>(dd[kOneWait ? j : 0] + c0));
        tmem_ld_wait();
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t* d = dd[kOneWait ? j : 0];
        if (!kOneWait) {
#pragma unroll
          for (int c0 = 0; c0 < C::NK; c0 += 16)
            tmem_ld16(tmem + lanes + C::kColS + j * C::NK + c0, *reinterpret_cast<uint32_t(*)[16]>(d + c0));
          tmem_ld_wait();
        }
        // |limb sum| <= 128 * 240 * 128, so two limbs combine exactly in int32; the fp32
        // steps run on pairs of heads (packed f32x2 arithmetic, same rounding)
        if constexpr (G % 2 == 0) {
          const uint64_t ks2 = pk2(ks[j], ks[j]), kz2 = pk2(kz[j], kz[j]), big2 = pk2(65536.0f, 65536.0f);
#pragma unroll
          for (int h = 0; h < G; h += 2) {
            const int lo0 = (int)d[h] + (int)d[G + h] * 256, lo1 = (int)d[h + 1] + (int)d[G + h + 1] * 256;
            const int hi0 = (int)d[2 * G + h] + (int)d[3 * G + h] * 256;
            const int hi1 = (int)d[2 * G + h + 1] + (int)d[3 * G + h + 1] * 256;
            const uint64_t si = fma2_rn(pk2((float)hi0, (float)hi1), big2, pk2((float)lo0, (float)lo1));
            float a0, a1;
            unpk2(fma2_rn(ks2, mul2_rn(si, pk2(c1[h], c1[h + 1])), mul2_rn(kz2, pk2(c2[h], c2[h + 1]))), a0, a1);
            s2[j][h] = valid[j] ? a0 : -CUDART_INF_F;
            s2[j][h + 1] = valid[j] ? a1 : -CUDART_INF_F;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int lo = (int)d[h] + (int)d[G + h] * 256;
            const int hi = (int)d[2 * G + h] + (int)d[3 * G + h] * 256;
            const float si = fmaf((float)hi, 65536.0f, (float)lo);
            const float dot = fmaf(ks[j], si * c1[h], kz[j] * c2[h]);
            s2[j][h] = valid[j] ? dot : -CUDART_INF_F;
          }
        }
      }
      // ---- tile maxima: per head the largest score; the largest value scale
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = warp_max(fmaxf(s2[0][h], s2[1][h]));
        if (lane == 0) reinterpret_cast<float*>(&ms->red[u][h])[qd] = mt;
      }
      {
        const float vm = warp_max(fmaxf(vs[0], vs[1]));
        if (lane == 0) reinterpret_cast<float*>(&ms->red[u][32])[qd] = vm;
      }
      named_barrier(kBarTok, 128);              // the four token warps' maxima are published
      const float4 v4 = ms->red[u][32];
      const float vmax = max3f(v4.x, v4.y, fmaxf(v4.z, v4.w));
      // limb scale: e * scale * vq <= 65520 (1 + 2^-21) < 65536 for e = 2^(s - mt) <= 1
      const float vq = vmax > 0.f ? __fdividef(65520.0f, vmax) : 0.f;
      float corr[G], ch[G], mt[G], lt[G], zt[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 t4 = ms->red[u][h];
        mt[h] = max3f(t4.x, t4.y, fmaxf(t4.z, t4.w));
        const float mn = fmaxf(m_run[h], mt[h]);
        corr[h] = ex2_approx(m_run[h] - mn);  // 0 on the first tile
        ch[h] = ex2_approx(mt[h] - mn);
        m_run[h] = mn;
        lt[h] = 0.f;
        zt[h] = 0.f;
      }
      // ---- probabilities relative to the tile maximum, e = 2^(s - mt) (p = ch e): sums
      // in fp32; e x scale as 16-bit limbs (B of the value MMA, token-major: a token's 2G
      // limb bytes are one 16-byte row, N block of 16 = 2 KB).  Rows past the context
      // have s = -inf, so e = 0.
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float vsq = vs[j] * vq;
        uint32_t pb[G];
        // round e * scale * vq to an integer <= 65535 held in the low 16 bits of the float's
        // pattern; pairs of heads share the packed f32x2 steps
        if constexpr (G % 2 == 0) {
          const uint64_t vz2 = pk2(vz[j], vz[j]), vsq2 = pk2(vsq, vsq), mg2 = pk2(12582912.0f, 12582912.0f);
#pragma unroll
          for (int h = 0; h < G; h += 2) {
            const uint64_t e2 = pk2(ex2_approx(s2[j][h] - mt[h]), ex2_approx(s2[j][h + 1] - mt[h + 1]));
            unpk2(add2_rn(pk2(lt[h], lt[h + 1]), e2), lt[h], lt[h + 1]);
            unpk2(fma2_rn(e2, vz2, pk2(zt[h], zt[h + 1])), zt[h], zt[h + 1]);
            float p0, p1;
            unpk2(fma2_rn(e2, vsq2, mg2), p0, p1);
            pb[h] = __float_as_uint(p0);
            pb[h + 1] = __float_as_uint(p1);
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float e = ex2_approx(s2[j][h] - mt[h]);
            lt[h] += e;
            zt[h] = fmaf(e, vz[j], zt[h]);
            pb[h] = __float_as_uint(fmaf(e, vsq, 12582912.0f));
          }
        }
        uint8_t* bcol = bv + j * C::NV * 128 + r * 16;
#pragma unroll
        for (int nb = 0; nb < C::NV / 16; ++nb) {   // rows 16 nb .. 16 nb + 15 of this token
          uint32_t wds[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t wv = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int nrow = 16 * nb + 4 * q + e;   // row: limb 0 of heads 0..G-1, then limb 1
              uint32_t byte = 0;
              if (nrow < G) byte = pb[nrow] & 0xffu;
              else if (nrow < 2 * G) byte = (pb[nrow - G] >> 8) & 0xffu;
              wv |= byte << (8 * e);
            }
            wds[q] = wv;
          }
          *reinterpret_cast<uint4*>(bcol + nb * 2048) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->pr);
      float fs[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        l_run[h] = fmaf(l_run[h], corr[h], ch[h] * lt[h]);
        z_run[h] = fmaf(z_run[h], corr[h], ch[h] * zt[h]);
        fs[h] = ch[h] * vmax * (1.0f / 65520.0f);
      }
      // ---- next tile's key codes, this tile's value result, next tile's value codes
      if (i + 1 < n) widen_k(i + 1);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->vdone, u, abort));
      tc_fence_after();
      {
        uint32_t d[C::NV];
#pragma unroll
        for (int c0 = 0; c0 < C::NV; c0 += 16)
          tmem_ld16(tmem + lanes + C::kColO + c0, *reinterpret_cast<uint32_t(*)[16]>(d + c0));
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // each limb column is <= 255 * 240 * 256 (exact int32); their combination can
          // pass 2^31 when attention is flat over the tile, so it is formed in fp32
          const float di = fmaf((float)(int)d[G + h], 256.0f, (float)(int)d[h]);
          o[h] = fmaf(o[h], corr[h], fs[h] * di);
        }
      }
      tc_fence_before();
      if (i + 1 < n) widen_v(i + 1);
    }

    // ---- split partial: m, l, o + z (z = sum p zero, the same for every channel).
    // The widened value codes of channel position r carry a factor value_scale_of(r).
    named_barrier(kBarTok, 128);              // every token warp is past its last read of red[]
    const float vfix = 1.0f / value_scale_of<BITS>(r);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float l = l_run[h], z = z_run[h];
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, off);
        z += __shfl_xor_sync(0xffffffffu, z, off);
      }
      if (lane == 0) {
        reinterpret_cast<float*>(&ms->red[0][h])[qd] = l;
        reinterpret_cast<float*>(&ms->red[1][h])[qd] = z;
      }
    }
    named_barrier(kBarTok, 128);
    const int c = channel_of<BITS>(r);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4 l4 = ms->red[0][h];
      const float4 z4 = ms->red[1][h];
      float* dst = a.ws + (((size_t)b * a.hq + kv * G + h) * a.num_splits + split) * kPartialStride;
      dst[4 + c] = fmaf(o[h], vfix, (z4.x + z4.y) + (z4.z + z4.w));
      if (r == 0) {
        dst[0] = m_run[h];
        dst[1] = (l4.x + l4.y) + (l4.z + l4.w);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ms->abort) report(a.status, WUSHKV_STATUS_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
}

// out[b][h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s   (log2-domain partials).
// One pass over the splits in batches of sixteen whose loads are all in flight at once
// (the automatic split counts of the workloads fit one or two batches), rescaling the
// running sums whenever a batch raises the maximum.
constexpr int kCombineBatch = 16;
__global__ void __launch_bounds__(kHeadDim) combine_log2_kernel(const float* __restrict__ ws, int num_splits,
                                                               float* __restrict__ out) {
  const size_t bh = blockIdx.x;
  const int c = threadIdx.x;
  const float* p = ws + bh * num_splits * kPartialStride;
  float mx = -CUDART_INF_F, l = 0.f, o = 0.f;
  for (int s0 = 0; s0 < num_splits; s0 += kCombineBatch) {
    float mv[kCombineBatch], lv[kCombineBatch], ov[kCombineBatch];
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) {
      const bool in = s0 + k < num_splits;
      const float* ps = p + (size_t)(s0 + k) * kPartialStride;
      mv[k] = in ? __ldg(ps) : -CUDART_INF_F;
      lv[k] = in ? __ldg(ps + 1) : 0.f;
      ov[k] = in ? __ldg(ps + 4 + c) : 0.f;
    }
    float bm = mv[0];
#pragma unroll
    for (int k = 1; k < kCombineBatch; ++k) bm = fmaxf(bm, mv[k]);
    const float nm = fmaxf(mx, bm);
    if (nm == -CUDART_INF_F) continue;            // nothing seen yet
    const float sc = exp2f(mx - nm);              // 0 while mx is still -inf
    l *= sc;
    o *= sc;
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) {
      if (mv[k] == -CUDART_INF_F) continue;       // empty split (or past the end)
      const float w = exp2f(mv[k] - nm);
      l = fmaf(w, lv[k], l);
      o = fmaf(w, ov[k], o);
    }
    mx = nm;
  }
  out[bh * kHeadDim + c] = l > 0.f ? o / l : 0.f;
}

// Tensor map over one side's codes: [planes][rows][16*BITS bytes] (planes = sequence x
// head rows of `rows` positions, or page x head), boxes of box_rows rows, swizzled as
// code_swizzle describes.
template <int BITS>
bool code_map(CUtensorMap* m, const uint8_t* base, int rows, int planes, int box_rows) {
  const uint64_t dims[3] = {(uint64_t)(16 * BITS), (uint64_t)rows, (uint64_t)planes};
  const uint64_t strides[2] = {(uint64_t)(16 * BITS), (uint64_t)rows * (16 * BITS)};
  const uint32_t box[3] = {(uint32_t)(16 * BITS), (uint32_t)box_rows, 1};
  const CUtensorMapSwizzle sw = BITS == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                : BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, sw);
}

template <int BITS, int KIND, int G>
cudaError_t launch_g(const DecArgs& a, int batch, float* out, cudaStream_t stream) {
  using C = Cfg<BITS, G>;
  auto kern = decode_tc_kernel<BITS, KIND, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  CUtensorMap km, vm;
  // contiguous: [B * Hkv][capacity][bytes]; paged: [num_pages * Hkv][page_size][bytes]
  const bool paged = a.rows.block_table != nullptr;
  const int rows = paged ? (1 << a.rows.page_shift) : a.capacity;
  const int planes = paged ? a.rows.num_pages * a.hkv : batch * a.hkv;
  if (!code_map<BITS>(&km, a.k_codes, rows, planes, a.box_rows) || !code_map<BITS>(&vm, a.v_codes, rows, planes, a.box_rows))
    return cudaErrorInvalidValue;
  dim3 grid(a.num_splits, a.hkv, batch);
  kern<<<grid, kThreads, C::kSmem, stream>>>(km, vm, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_log2_kernel<<<batch * a.hq, kHeadDim, 0, stream>>>(a.ws, a.num_splits, out);
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

// Resident decode CTAs per SM for a cache's bit width and group size (Cfg::kCtas).
int ctas_per_sm(int bits, int g) {
  static_assert(Cfg<2, 4>::kCtas == 3 && Cfg<2, 8>::kCtas == 2 && Cfg<2, 16>::kCtas == 2 && Cfg<3, 1>::kCtas == 2 &&
                    Cfg<3, 16>::kCtas == 2 && Cfg<4, 8>::kCtas == 2 && Cfg<4, 16>::kCtas == 1,
                "keep ctas_per_sm in step with Cfg");
  if (bits == 2 && g <= 4) return 3;
  return (bits == 4 && g >= 16) ? 1 : 2;
}

}  // namespace

// Split count when the caller passes 0.  Time is modelled as (waves of CTAs over
// SMs x resident CTAs per SM) x (tiles per split + 1, the +1 for a CTA's set-up and its
// partial); the count with the least modelled time wins, the smaller on ties.
int auto_num_splits(const wushkv_cache& c, int num_q_heads) {
  const long long pairs = (long long)c.batch * c.num_kv_heads;
  const int tiles = (c.capacity + kTile - 1) / kTile;
  const int g = num_q_heads / c.num_kv_heads;
  const long long slots = (long long)ctas_per_sm(c.qp.bits, g) * num_sms(nullptr);
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= tiles && s <= 256; ++s) {
    const long long waves = (pairs * s + slots - 1) / slots;
    const long long cost = waves * ((tiles + s - 1) / s + 1);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = s; }
  }
  return best;
}

// Combine of log2-domain split partials ([rows][splits][132]) into out [rows][128].
cudaError_t launch_combine_partials(const float* ws, int rows, int num_splits, float* out, cudaStream_t stream) {
  combine_log2_kernel<<<rows, kHeadDim, 0, stream>>>(ws, num_splits, out);
  return cudaGetLastError();
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
  a.scale_log2 = softmax_scale * kLog2e;
  a.ws = static_cast<float*>(workspace);
  a.status = status;
  a.rows = CacheRows::of(c);
  a.box_rows = c.block_table != nullptr ? (c.page_size < kTile ? c.page_size : kTile) : kTile;
  switch (c.qp.bits) {
    case 2: return launch_bits<2>(a, c.qp.kind, c.batch, out, stream);
    case 3: return launch_bits<3>(a, c.qp.kind, c.batch, out, stream);
    default: return launch_bits<4>(a, c.qp.kind, c.batch, out, stream);
  }
}

}  // namespace wushkv
