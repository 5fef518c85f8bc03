// Per-group clipped quantizers of WUSH-KV, one 128-value group per thread.
//
// QuEST-INT-style symmetric grid and OSCAR-style percentile-clipped affine grid
// (ai4snews summary "WUSH-KV cuts 2-bit KV-cache perplexity ...", paragraphs 3-5;
// arXiv abstract).  The grids, as this library reads them:
//   QuEST: Delta = fp16(alpha * sqrt(sum x^2 / 128) * 2^(1-b)),
//          code = clamp(floor(x / Delta) + 2^(b-1), 0, 2^b - 1)
//   affine: lo, hi = values of ascending rank r_lo, r_hi; scale = fp16((hi-lo)/(2^b-1)),
//          zero = fp16(lo), code = clamp(rne((x - zero) / scale), 0, 2^b - 1)
// Codes must equal the exact-arithmetic decision for the given fp32 value x, so
// every fast step carries a bracket and falls back to exact comparisons when the
// bracket does not settle the answer:
//   * sum of squares: fp32 chains of 16 terms (relative error < 17 * 2^-24);
//     if fp16(pre * (1 -+ 1e-6)) disagree, the group's sum is redone in fp64.
//   * codes: the quotient is evaluated with the reciprocal widened by 2^-20 on both
//     sides; where the two roundings differ the group's codes are recomputed by
//     exact threshold comparisons (fp32 for QuEST, fp64 for affine thresholds).
//   * QuEST codes of bf16 inputs (loaders with kBf16Exact) need no bracket: a bf16
//     value (8 significant bits) and a threshold j*Delta (fp16 step times a small
//     integer, <= 15 significant bits) are either equal or at least 2^-16 apart
//     relative to the threshold, far outside the 2^-20 widening.  So one
//     round-down product with the reciprocal widened away from zero's side (up for
//     x >= 0, down for x < 0) lands on the exact floor, ties included.
#pragma once
#include "wushkv_common.cuh"

namespace wushkv {

constexpr float kMagic = 12582912.0f;       // 1.5 * 2^23: integers live in the low mantissa bits
constexpr int32_t kMagicBits = 0x4B400000;
constexpr float kWidenDn = 0.999999046325683594f;  // 1 - 2^-20 (exact in fp32)
constexpr float kWidenUp = 1.00000095367431641f;   // 1 + 2^-20 (exact in fp32)
constexpr double kStepMargin = 1.0e-6;

template <int BITS>
__device__ __forceinline__ void put_code(uint32_t (&w)[4 * BITS], int i, uint32_t c) {
  const int o = BITS * i;
  const int wi = o >> 5;
  const int sh = o & 31;
  w[wi] |= c << sh;
  if (sh + BITS > 32) w[wi + 1] |= c >> (32 - sh);
}

// Same as put_code for an index only known at run time (selects over the words so the
// array stays in registers).
template <int BITS>
__device__ __forceinline__ void put_code_dyn(uint32_t (&w)[4 * BITS], int i, uint32_t c) {
  const int o = BITS * i;
  const int wi = o >> 5;
  const int sh = o & 31;
  const uint32_t lo = c << sh;
  const uint32_t hi = (sh + BITS > 32) ? (c >> (32 - sh)) : 0u;
#pragma unroll
  for (int q = 0; q < 4 * BITS; ++q) {
    if (q == wi) w[q] |= lo;
    if (q == wi + 1) w[q] |= hi;
  }
}

template <int BITS>
__device__ __forceinline__ void clear_words(uint32_t (&w)[4 * BITS]) {
#pragma unroll
  for (int i = 0; i < 4 * BITS; ++i) w[i] = 0u;
}

// alpha * RMS * 2^(1-b) in fp64 from a sum of squares (same operation order as the
// plain definition: sqrt of the mean, times alpha, times a power of two).
__device__ __forceinline__ double quest_pre(double sumsq, double alpha, int bits) {
  const double rms = sqrt(sumsq * (1.0 / 128.0));
  return alpha * rms * ldexp(1.0, 1 - bits);
}

// The quantizers read a group as four chunks of 32 values through a loader
// `ld(c, v)` (c = 0..3, v = float[32]): once for the statistics, once for the codes,
// and again only in the rare exact fallbacks.  Re-reading from shared or tensor
// memory keeps the register footprint at one chunk; each chunk's 32 codes are exactly
// BITS packed words, written to `dst` (the group's cache row, or nullptr to drop them)
// as soon as they are known.  Loaders may be warp-collective (tensor-memory loads), so
// every lane of the calling warp runs the same loads: there is no early exit,
// degenerate groups are handled arithmetically, and the fallbacks run for the whole
// warp when any lane needs them (exact results are always valid).
constexpr int kChunk = 32;
constexpr int kNumChunks = kHeadDim / kChunk;

template <int BITS>
__device__ __forceinline__ void store_chunk(uint8_t* dst, int c, const uint32_t (&wc)[BITS]) {
  if (dst == nullptr) return;
  uint8_t* p = dst + c * 4 * BITS;
  if constexpr (BITS == 2) {
    asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(wc[0]), "r"(wc[1]) : "memory");
  } else if constexpr (BITS == 4) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(wc[0]), "r"(wc[1]), "r"(wc[2]),
                 "r"(wc[3])
                 : "memory");
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) reinterpret_cast<uint32_t*>(p)[k] = wc[k];
  }
}

// code i (0..31) of a chunk into the chunk's BITS words
template <int BITS>
__device__ __forceinline__ void put_chunk_code(uint32_t (&wc)[BITS], int i, uint32_t code) {
  const int o = BITS * i, wi = o >> 5, sh = o & 31;
  wc[wi] |= code << sh;
  if (sh + BITS > 32) wc[wi + 1] |= code >> (32 - sh);
}

// ---------------------------------------------------------------------------- QuEST
template <int BITS, class Loader>
__device__ __forceinline__ void quest_quantize(Loader& ld, double alpha, uint8_t* dst, uint16_t& delta_bits,
                                               int32_t& flags) {
  constexpr int kHalf = 1 << (BITS - 1);
  constexpr int kMaxCode = (1 << BITS) - 1;
  const unsigned mask = __activemask();
  float s[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) s[k] = 0.f;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
#pragma unroll
    for (int i = 0; i < kChunk; ++i) s[i & 7] = fmaf(v[i], v[i], s[i & 7]);
  }
  const double sum_fast = (((double)s[0] + (double)s[1]) + ((double)s[2] + (double)s[3])) +
                          (((double)s[4] + (double)s[5]) + ((double)s[6] + (double)s[7]));
  if (!isfinite(sum_fast)) flags |= WUSHKV_STATUS_NONFINITE;
  const double pre_fast = quest_pre(sum_fast, alpha, BITS);
  uint16_t h = f64_to_f16_bits(pre_fast * (1.0 - kStepMargin));
  const bool ambiguous = h != f64_to_f16_bits(pre_fast * (1.0 + kStepMargin));
  if (__any_sync(mask, ambiguous)) {  // fp64 sum of the exact squares
    double sum = 0.0;
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
#pragma unroll
      for (int i = 0; i < kChunk; ++i) sum = fma((double)v[i], (double)v[i], sum);
    }
    h = f64_to_f16_bits(quest_pre(sum, alpha, BITS));
  }
  delta_bits = h;
  const float delta = f16_bits_to_f32(h);
  if (isinf(delta)) flags |= WUSHKV_STATUS_META_OVERFLOW;
  // Delta == 0 (or overflowed): a zero reciprocal puts every value at code 2^(b-1)
  const float inv = (delta == 0.f || isinf(delta)) ? 0.f : __frcp_rn(delta);
  const float inv_dn = __fmul_rd(inv, kWidenDn);
  const float inv_up = __fmul_ru(inv, kWidenUp);
  const float m = kMagic + (float)kHalf;
  if constexpr (Loader::kBf16Exact) {
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
      uint32_t wc[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        const float y = __fmaf_rd(v[i], v[i] < 0.f ? inv_dn : inv_up, m);
        const int32_t code = min(max(f2i(y) - kMagicBits, 0), kMaxCode);
        put_chunk_code<BITS>(wc, i, (uint32_t)code);
      }
      store_chunk<BITS>(dst, c, wc);
    }
    return;
  }
  uint32_t mism = 0u;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
    uint32_t wc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      const float y1 = __fmaf_rd(v[i], inv_dn, m);
      const float y2 = __fmaf_rd(v[i], inv_up, m);
      mism |= f2u(y1) ^ f2u(y2);
      const int32_t code = min(max(f2i(y1) - kMagicBits, 0), kMaxCode);
      put_chunk_code<BITS>(wc, i, (uint32_t)code);
    }
    store_chunk<BITS>(dst, c, wc);
  }
  if (__any_sync(mask, mism != 0u)) {  // exact: count the thresholds j*Delta (exact in fp32)
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
      uint32_t wc[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        uint32_t code = 0;
#pragma unroll
        for (int j = -(kHalf - 1); j < kHalf; ++j) code += (v[i] >= (float)j * delta) ? 1u : 0u;
        if (inv == 0.f) code = kHalf;
        put_chunk_code<BITS>(wc, i, code);
      }
      store_chunk<BITS>(dst, c, wc);
    }
  }
}

// ------------------------------------------------------------------ percentile affine
// The KSEL smallest (ascending) and KSEL largest (descending) values seen so far.
template <int KSEL>
__device__ __forceinline__ void select_update(float v, float (&lo)[KSEL], float (&hi)[KSEL]) {
#pragma unroll
  for (int k = KSEL - 1; k >= 1; --k) {
    lo[k] = fminf(lo[k], fmaxf(lo[k - 1], v));
    hi[k] = fmaxf(hi[k], fminf(hi[k - 1], v));
  }
  lo[0] = fminf(lo[0], v);
  hi[0] = fmaxf(hi[0], v);
}

template <int KSEL>
__device__ __forceinline__ float pick(const float (&a)[KSEL], int idx) {
  float r = a[0];
#pragma unroll
  for (int k = 1; k < KSEL; ++k) r = (idx == k) ? a[k] : r;
  return r;
}

template <int BITS, int KSEL, class Loader>
__device__ __forceinline__ void affine_quantize(Loader& ld, int rank_lo, int rank_hi, uint8_t* dst,
                                                uint16_t& scale_bits, uint16_t& zero_bits, int32_t& flags) {
  constexpr int kMaxCode = (1 << BITS) - 1;
  const unsigned mask = __activemask();
  float lo_k[KSEL], hi_k[KSEL];
#pragma unroll
  for (int k = 0; k < KSEL; ++k) {
    lo_k[k] = __int_as_float(0x7f800000);
    hi_k[k] = __int_as_float(0xff800000);
  }
  float fsum = 0.f;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      select_update<KSEL>(v[i], lo_k, hi_k);
      fsum += v[i];
    }
  }
  if (!isfinite(fsum)) flags |= WUSHKV_STATUS_NONFINITE;
  const float lo = pick<KSEL>(lo_k, rank_lo);
  const float hi = pick<KSEL>(hi_k, kHeadDim - 1 - rank_hi);
  const double scale_pre = ((double)hi - (double)lo) / (double)kMaxCode;
  scale_bits = f64_to_f16_bits(scale_pre);
  zero_bits = f32_to_f16_bits(lo);
  const float sc = f16_bits_to_f32(scale_bits);
  const float z = f16_bits_to_f32(zero_bits);
  if (isinf(sc) || isinf(z)) flags |= WUSHKV_STATUS_META_OVERFLOW;
  // scale == 0: a zero reciprocal puts every value at code 0 (x_hat = zero)
  const float inv = (sc == 0.f || isinf(sc)) ? 0.f : __frcp_rn(sc);
  const float inv_dn = __fmul_rd(inv, kWidenDn);
  const float inv_up = __fmul_ru(inv, kWidenUp);
  uint32_t mism = 0u;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
    uint32_t wc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      const float d = __fsub_rn(v[i], z);
      const float y1 = __fmaf_rn(d, inv_dn, kMagic);
      const float y2 = __fmaf_rn(d, inv_up, kMagic);
      mism |= f2u(y1) ^ f2u(y2);
      const int32_t code = min(max(f2i(y1) - kMagicBits, 0), kMaxCode);
      put_chunk_code<BITS>(wc, i, (uint32_t)code);
    }
    store_chunk<BITS>(dst, c, wc);
  }
  if (__any_sync(mask, mism != 0u)) {  // exact: thresholds zero + (j + 1/2) scale are exact in fp64
    const double zd = (double)z, sd = (double)sc;
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
      uint32_t wc[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        const double xd = (double)v[i];
        uint32_t code = 0;
#pragma unroll
        for (int j = 0; j < kMaxCode; ++j) {
          const double t = zd + ((double)j + 0.5) * sd;
          code += (xd > t || (xd == t && (j & 1))) ? 1u : 0u;
        }
        if (inv == 0.f) code = 0;
        put_chunk_code<BITS>(wc, i, code);
      }
      store_chunk<BITS>(dst, c, wc);
    }
  }
}

// Loader over a group held in a shared-memory row of fp32 values.
struct SmemRowLoader {
  static constexpr bool kBf16Exact = false;   // fp32 rows: any value
  const float* row;
  __device__ __forceinline__ void operator()(int c, float (&v)[kChunk]) const {
#pragma unroll
    for (int i = 0; i < kChunk; ++i) v[i] = row[c * kChunk + i];
  }
};

}  // namespace wushkv
