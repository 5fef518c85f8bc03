// Split-K GQA decode attention directly over the packed cache, on the tensor cores.
//
// WUSH-KV serves grouped-query attention over a 2-bit cache (ai4snews summary,
// paragraph 5) at long context (paragraph 4).  The codes are small integers, so
// both contractions run exactly as integer MMAs (tcgen05.mma kind::i8, int32
// accumulate) and the fp16 meta is applied afterwards:
//   scores  s_t = tau * (scale_t * sum_c q'_c code_tc + zero_t * sum_c q'_c)
//           sum_c q'_c code_tc = (M / (2^22 - 1)) * sum_c qi_c code_tc, with q' rounded
//           to 23-bit integers qi = l0 + 2^8 l1 + 2^16 l2 split into three int8 limbs;
//   values  o_c = sum_t p_t (zero_t + scale_t code_tc)
//               = (F / 65535) * sum_t pi_t code_tc + sum_t p_t zero_t,
//           with p_t scale_t rounded to 16-bit integers pi = u0 + 2^8 u1 (per tile and
//           head, F = the tile's largest p_t scale_t) split into two uint8 limbs.
// (QuEST: scale = Delta, zero = -(2^(b-1) - 1/2) Delta.)  The softmax is online in the
// log2 domain across 128-token tiles.
//
// One CTA = one (sequence, KV head, split), five warps:
//   warp 0      one thread: bulk copies of each tile's packed K and V codes into a
//               4-stage ring, and every MMA, each issued when the mbarrier of the
//               event it needs completes (tile widened; probabilities written).
//   warps 1-4   token warps.  Thread = token of the tile while widening codes to u8
//               (K codes into tensor memory as A of the score MMA, V codes into
//               channel-major shared memory as A of the value MMA) and while turning
//               scores into probability limbs (B of the value MMA); thread = channel
//               while accumulating the value MMA's int32 result.  They signal the
//               issuing thread by mbarrier arrivals and meet each other only to share
//               each tile's per-head maxima.
// Per tile i the token warps run: softmax(i) -> [value MMA(i)]; accumulate(i-1);
// widen(i+1) -> [score MMA(i+1)], so each MMA has a whole phase to complete before
// its result is read.  Small CTAs (160 threads, ~72 KB shared memory, 128 TMEM
// columns) let three run per SM, keeping about 96 KB of code reads in flight per SM.
// 2- and 4-bit key codes are widened to bytes with two logic ops per 4 codes, which
// permutes channels inside each 16 (8) channel block; the query limbs and the output
// channels use the same permutation, so the contraction is unchanged.  Value codes
// are widened by masking alone (see widen_row_scaled).
#include <math_constants.h>

#include <cmath>

#include "sm100.cuh"
#include "tmap.h"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kTile = 128;
constexpr int kThreads = 160;
constexpr int kStages = 4;
constexpr int kPartialStride = 132;   // m (log2 domain), l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQScale = 4194303.0f; // 2^22 - 1
constexpr uint32_t kBarTok = 1;       // named barrier of the four token warps

__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ constexpr int pow2cols(int x) { return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512; }

template <int BITS, int G>
struct Cfg {
  static constexpr int kCode = 16 * BITS;                  // packed bytes per token row
  static constexpr int kStage = 2 * kTile * kCode;         // K and V codes of one tile
  static constexpr int NK = round16(3 * G);                // score MMA N (3 limbs per head)
  static constexpr int NV = round16(2 * G);                // value MMA N (2 limbs per head)
  static constexpr int kColAk = 0;                         // 2 x 32 columns (u8 x 128 channels)
  static constexpr int kColS = 64;                         // NK
  static constexpr int kColO = 64 + NK;                    // 2 x NV
  static constexpr int kCols = pow2cols(64 + NK + 2 * NV);
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int kOffStage = 0;
  static constexpr int kOffAv = (kOffStage + kStages * kStage + 1023) / 1024 * 1024;   // 2 x 16 KB
  static constexpr int kOffBv = kOffAv + 2 * kTile * 128;                              // 2 x NV x 128 bytes
  static constexpr int kOffBk = kOffBv + 2 * NV * 128;                                 // NK rows
  static constexpr int kOffMisc = kOffBk + NK * 128;
  static constexpr int kMiscBytes = 2048;
  static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;
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
};

struct Misc {
  uint64_t full[kStages];     // stage filled (bulk copies)
  uint64_t kw;                // 4 token warps: tile widened (its stage is free again)
  uint64_t pr;                // 4 token warps: probabilities of the tile written
  uint64_t mx;                // 4 token warps: per-warp tile maxima published
  uint64_t kdone;             // score MMA done
  uint64_t vdone[2];          // value MMA done, per tile parity
  uint32_t tmem_base;
  int abort;
  float4 red[2][32];          // per tile parity and value (head maxima), the 4 token warps' partials
  float c1[16], c2[16];       // per head: qscale * softmax_scale * log2 e, sum(q') * softmax_scale * log2 e
};

// position p of a widened code row <-> channel
template <int BITS>
__device__ __forceinline__ int channel_of(int p) {
  if (BITS == 2) return (p & ~15) | ((p & 3) << 2) | ((p >> 2) & 3);
  if (BITS == 4) return (p & ~7) | ((p & 3) << 1) | ((p >> 2) & 1);
  return p;
}

// Packed row (16*BITS bytes at `row`) -> 32 words of four u8 codes (K order as above).
template <int BITS>
__device__ __forceinline__ void load_row(const uint8_t* row, uint32_t (&w)[4 * BITS]) {
#pragma unroll
  for (int q = 0; q < BITS; ++q) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * q);
    w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
  }
}

template <int BITS>
__device__ __forceinline__ void widen_row(const uint8_t* row, uint32_t (&u)[32]) {
  constexpr int kWords = 4 * BITS;
  uint32_t w[kWords];
  load_row<BITS>(row, w);
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

// Value codes are widened by masking alone: byte p then holds code * value_scale_of(p)
// (2-bit: 4^((p >> 2) & 3); 4-bit: 16^((p >> 2) & 1); 3-bit: 1).  Position p is an
// output channel of the value MMA, so the power of two is divided out exactly once,
// from the split partial.  Largest int32 sum per tile: 65535 * 240 * 128 < 2^31.
template <int BITS>
__device__ __forceinline__ void widen_row_scaled(const uint8_t* row, uint32_t (&u)[32]) {
  if (BITS == 3) {
    widen_row<BITS>(row, u);
    return;
  }
  uint32_t w[4 * BITS];
  load_row<BITS>(row, w);
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
__global__ void __launch_bounds__(kThreads, (G <= 8 ? 3 : 2)) decode_tc_kernel(DecArgs a) {
  using C = Cfg<BITS, G>;
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
    for (int s = 0; s < kStages; ++s) mbar_init(&ms->full[s], 1);
    mbar_init(&ms->kw, 4);
    mbar_init(&ms->pr, 4);
    mbar_init(&ms->mx, 4);
    mbar_init(&ms->kdone, 1);
    mbar_init(&ms->vdone[0], 1);
    mbar_init(&ms->vdone[1], 1);
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
      const float inv = mx > 0.f ? kQScale / mx : 0.f;
      const int qi = __float2int_rn(qv * inv);              // |qi| <= 2^22 - 1
      const int l0 = (int)(int8_t)(qi & 0xff);
      const int r1 = (qi - l0) >> 8;
      const int l1 = (int)(int8_t)(r1 & 0xff);
      const int l2 = (r1 - l1) >> 8;                        // |l2| <= 64
      bk[kmajor_off(h, p)] = (uint8_t)l0;
      bk[kmajor_off(G + h, p)] = (uint8_t)l1;
      bk[kmajor_off(2 * G + h, p)] = (uint8_t)l2;
      if (p == 0) {
        const float4 s4 = ms->red[1][h];
        ms->c1[h] = (mx > 0.f ? mx / kQScale : 0.f) * a.scale_log2;
        ms->c2[h] = ((s4.x + s4.y) + (s4.z + s4.w)) * a.scale_log2;
      }
    }
    for (int nrow = 3 * G; nrow < C::NK; ++nrow) bk[kmajor_off(nrow, p)] = 0;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // -------------------------------------------------- bulk loads + MMA issue
    // One thread, in the order the token warps produce: value MMA(i) once every
    // token warp has written P(i); score MMA(i+1) once every token warp has widened
    // tile i+1, which also frees that tile's stage for tile i+1+kStages.
    if (lane == 0) {
      constexpr uint32_t kIdK = idesc(kFmtS32, kFmtU8, kFmtS8, 0, 0, 128, C::NK);
      constexpr uint32_t kIdV = idesc(kFmtS32, kFmtU8, kFmtU8, 1, 1, 128, C::NV);
      const uint32_t bk_addr = smem_u32(bk), bv_addr = smem_u32(bv), av_addr = smem_u32(av);
      int issued = 0;
      auto load = [&](int i) {
        const int s = i % kStages;
        const int t0 = (tile0 + i) * kTile;
        const uint32_t bytes = (uint32_t)min(kTile, L - t0) * C::kCode;
        mbar_arrive_expect_tx(&ms->full[s], 2 * bytes);
        const size_t off = (pair * a.capacity + t0) * C::kCode;
        bulk_load(stage + s * C::kStage, a.k_codes + off, bytes, &ms->full[s]);
        bulk_load(stage + s * C::kStage + kTile * C::kCode, a.v_codes + off, bytes, &ms->full[s]);
        ++issued;
      };
      auto score_mma = [&](int i) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_i8_ts(tmem + C::kColS, tmem + C::kColAk + (i & 1) * 32 + ks * 8,
                    desc_kmajor_sw128(bk_addr + ks * 32), kIdK, ks > 0);
        mma_commit(&ms->kdone);
      };
      auto value_mma = [&](int i) {
        const int u = i & 1;
        tc_fence_after();
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const uint64_t adesc = make_desc(av_addr + u * kTile * 128 + kq * 4096, 16384, 1024, 2);
          const uint64_t bdesc = make_desc(bv_addr + u * C::NV * 128 + kq * 512, 128, 2048, 0);
          mma_i8_ss(tmem + C::kColO + u * C::NV, adesc, bdesc, kIdV, kq > 0);
        }
        mma_commit(&ms->vdone[u]);
      };
      for (int i = 0; i < n && i < kStages; ++i) load(i);
      bool ok = n > 0 && mbar_wait(&ms->kw, 0, abort);
      if (ok) {
        score_mma(0);
        if (kStages < n) load(kStages);
      }
      for (int i = 0; ok && i < n; ++i) {
        if (!(ok = mbar_wait(&ms->pr, i & 1, abort))) break;
        value_mma(i);
        if (i + 1 < n) {
          if (!(ok = mbar_wait(&ms->kw, (i + 1) & 1, abort))) break;
          score_mma(i + 1);
          if (i + 1 + kStages < n) load(i + 1 + kStages);
        }
      }
      // no copy may land after the CTA has exited, even after a timeout
      volatile int no_abort = 0;
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait(&ms->full[i % kStages], (i / kStages) & 1, &no_abort);
    }
  } else {
    // ------------------------------------------------------------- token warps
    // Each token warp signals the issuer with one mbarrier arrival per event (tile
    // widened, probabilities written) and meets the other token warps only to share
    // each tile's per-head maxima.  After a failed (timed-out) wait a warp skips work
    // but keeps arriving, so every phase still completes.
    const int qd = warp & 3;                 // TMEM lane quarter
    const int r = 32 * qd + lane;            // token row while widening / in softmax; channel position while accumulating
    const uint32_t lanes = (uint32_t)(32 * qd) << 16;
    bool ok = true;
    float m_run[G], l_run[G], z_run[G], o[G], corr_prev[G], fs_prev[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; z_run[h] = 0.f; o[h] = 0.f; corr_prev[h] = 0.f; fs_prev[h] = 0.f;
    }
    uint32_t kmeta_n = 0, vmeta_n = 0, kmeta_c = 0, vmeta_c = 0;
    float c1[G], c2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { c1[h] = ms->c1[h]; c2[h] = ms->c2[h]; }
    const int rx4 = (r & 7) << 4;

    // widen tile i's codes: K -> TMEM A (lanes = tokens), V -> channel-major shared A
    auto widen = [&](int i) {
      const int s = i % kStages;
      const int u = i & 1;
      const int t = (tile0 + i) * kTile + r;
      if (t < L) {
        kmeta_n = load_meta<KIND>(a.k_meta, pair * a.capacity + t);
        vmeta_n = load_meta<KIND>(a.v_meta, pair * a.capacity + t);
      }
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->full[s], (i / kStages) & 1, abort));
      if (ok) {
        uint32_t wv[32];
        widen_row<BITS>(stage + s * C::kStage + r * C::kCode, wv);
        tmem_st32(tmem + lanes + C::kColAk + u * 32, wv);
        widen_row_scaled<BITS>(stage + s * C::kStage + kTile * C::kCode + r * C::kCode, wv);
        uint8_t* arow = av + u * kTile * 128 + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(arow + ((j << 4) ^ rx4)) =
              make_uint4(wv[4 * j], wv[4 * j + 1], wv[4 * j + 2], wv[4 * j + 3]);
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->kw);
    };

    // accumulate the value MMA of tile i into o (thread = channel position r)
    auto accumulate = [&](int i) {
      const int u = i & 1;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->vdone[u], (i >> 1) & 1, abort));
      tc_fence_after();
      uint32_t d[C::NV];
#pragma unroll
      for (int c0 = 0; c0 < C::NV; c0 += 16)
        tmem_ld16(tmem + lanes + C::kColO + u * C::NV + c0, *reinterpret_cast<uint32_t(*)[16]>(d + c0));
      tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int di = (int)d[h] + (int)d[G + h] * 256;
        o[h] = fmaf(o[h], corr_prev[h], fs_prev[h] * (float)di);
      }
      tc_fence_before();
    };

    if (n > 0) widen(0);
    for (int i = 0; i < n; ++i) {
      kmeta_c = kmeta_n;
      vmeta_c = vmeta_n;
      const int u = i & 1;
      const bool valid = (tile0 + i) * kTile + r < L;
      // ---- scores of tile i
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->kdone, i & 1, abort));
      tc_fence_after();
      uint32_t d[C::NK];
#pragma unroll
      for (int c0 = 0; c0 < C::NK; c0 += 16)
        tmem_ld16(tmem + lanes + C::kColS + c0, *reinterpret_cast<uint32_t(*)[16]>(d + c0));
      tmem_ld_wait();
      float ks, kz, vs, vz;
      meta_pair<KIND>(kmeta_c, BITS, ks, kz);
      meta_pair<KIND>(vmeta_c, BITS, vs, vz);
      float s2[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int si = (int)d[h] + (int)d[G + h] * 256 + (int)d[2 * G + h] * 65536;
        const float dot = fmaf(ks, (float)si * c1[h], kz * c2[h]);
        s2[h] = valid ? dot : -CUDART_INF_F;
      }
      // ---- tile maxima per head: the largest score and the largest log2(p x value scale)
      const float lvs = valid && vs > 0.f ? lg2_approx(vs) : -CUDART_INF_F;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = warp_max(s2[h]);
        const float mu = warp_max(s2[h] + lvs);
        if (lane == 0) {
          reinterpret_cast<float*>(&ms->red[u][h])[qd] = mt;
          reinterpret_cast<float*>(&ms->red[u][G + h])[qd] = mu;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->mx);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&ms->mx, i & 1, abort));
      float corr[G], fpt[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 t4 = ms->red[u][h];
        const float4 u4 = ms->red[u][G + h];
        const float mt = max3f(t4.x, t4.y, fmaxf(t4.z, t4.w));
        const float mu = max3f(u4.x, u4.y, fmaxf(u4.z, u4.w));
        const float mn = fmaxf(m_run[h], mt);
        corr[h] = ex2_approx(m_run[h] - mn);  // 0 on the first tile
        m_run[h] = mn;
        fpt[h] = ex2_approx(mu - mn) * 1.000244140625f;   // widened against approximate log2/exp2
      }
      // ---- probabilities: l, z in fp32; p x scale as 16-bit limbs (B of the value MMA,
      // token-major: this token's 2G limb bytes are one 16-byte row, N block of 16 = 2 KB)
      bool moved = false;
#pragma unroll
      for (int h = 0; h < G; ++h) moved |= corr[h] != 1.f;
      if (moved) {                            // uniform across the CTA: the running max moved
#pragma unroll
        for (int h = 0; h < G; ++h) { l_run[h] *= corr[h]; z_run[h] *= corr[h]; }
      }
      uint32_t pb[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = valid ? ex2_approx(s2[h] - m_run[h]) : 0.f;
        l_run[h] += p;
        z_run[h] = fmaf(p, vz, z_run[h]);
        const float fq = fpt[h] > 0.f ? __fdividef(65535.0f, fpt[h]) : 0.f;
        // round to an integer <= 65535 held in the low 16 bits of the float's pattern
        pb[h] = __float_as_uint(fmaf(p * vs, fq, 12582912.0f));
      }
      uint8_t* bcol = bv + u * C::NV * 128 + r * 16;
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
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->pr);
      // ---- previous tile's value result, then widen the next tile
      if (i >= 1) accumulate(i - 1);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        corr_prev[h] = corr[h];
        fs_prev[h] = fpt[h] * (1.0f / 65535.0f);
      }
      if (i + 1 < n) widen(i + 1);
    }
    if (n > 0) accumulate(n - 1);

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
        reinterpret_cast<float*>(&ms->red[0][G + h])[qd] = z;
      }
    }
    named_barrier(kBarTok, 128);
    const int c = channel_of<BITS>(r);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4 l4 = ms->red[0][h];
      const float4 z4 = ms->red[0][G + h];
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

// out[b][h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s   (log2-domain partials)
__global__ void __launch_bounds__(kHeadDim) combine_log2_kernel(const float* __restrict__ ws, int num_splits,
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
      const float w = exp2f(ms - mx);
      l = fmaf(w, p[s * kPartialStride + 1], l);
      o = fmaf(w, p[s * kPartialStride + 4 + c], o);
    }
  }
  out[bh * kHeadDim + c] = l > 0.f ? o / l : 0.f;
}

template <int BITS, int KIND, int G>
cudaError_t launch_g(const DecArgs& a, int batch, float* out, cudaStream_t stream) {
  using C = Cfg<BITS, G>;
  auto kern = decode_tc_kernel<BITS, KIND, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, a.hkv, batch);
  kern<<<grid, kThreads, C::kSmem, stream>>>(a);
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

}  // namespace

// Split count when the caller passes 0: the smallest count whose CTAs fill whole
// waves of (SMs x resident CTAs per SM) to >= 95%, keeping >= 4 tiles per split; a
// small problem gets one tile per CTA.
int auto_num_splits(const wushkv_cache& c, int num_q_heads) {
  const int pairs = c.batch * c.num_kv_heads;
  const int tiles = (c.capacity + kTile - 1) / kTile;
  const int g = num_q_heads / c.num_kv_heads;
  const int per_sm = (g <= 8 && c.qp.bits == 2) ? 3 : 2;
  const int slots = per_sm * num_sms(nullptr);
  if ((long long)pairs * tiles <= slots) return tiles;
  const int max_s = tiles >= 4 ? tiles / 4 : 1;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= max_s && s <= 256; ++s) {
    const double w = (double)pairs * s / slots;
    const double eff = w / std::ceil(w);
    if (eff >= 0.95) return s;
    if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
  }
  return best;
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
  switch (c.qp.bits) {
    case 2: return launch_bits<2>(a, c.qp.kind, c.batch, out, stream);
    case 3: return launch_bits<3>(a, c.qp.kind, c.batch, out, stream);
    default: return launch_bits<4>(a, c.qp.kind, c.batch, out, stream);
  }
}

}  // namespace wushkv
