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

// Two fp32 values in one 64-bit register pair (element 0 in the low word) for the
// sm_100a packed f32x2 arithmetic, which does two fp32 operations per instruction with
// the same rounding as the scalar ones.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpk2(uint64_t x, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fma2_rm(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

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
  // eight fp32 chains of 16 squares each (two per packed accumulator for bf16 rows, whose
  // values are unpacked into fresh registers anyway)
  float s[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) s[k] = 0.f;
  if constexpr (Loader::kBf16Exact) {
    uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
#pragma unroll
      for (int i = 0; i < kChunk / 2; ++i) {
        const uint64_t p = pk2(v[2 * i], v[2 * i + 1]);
        acc2[i & 3] = fma2_rn(p, p, acc2[i & 3]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) unpk2(acc2[k], s[2 * k], s[2 * k + 1]);
  } else {
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
#pragma unroll
      for (int i = 0; i < kChunk; ++i) s[i & 7] = fmaf(v[i], v[i], s[i & 7]);
    }
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
  // y = round-down(x * inv + 2^23 * 1.5 + 2^(b-1)) holds floor(x / Delta) + 2^(b-1) in its
  // low mantissa bits; clamping y to [1.5 * 2^23, 1.5 * 2^23 + 2^b - 1] in fp32 leaves
  // exactly the code there
  const float m = kMagic + (float)kHalf;
  const float ylo = kMagic, yhi = kMagic + (float)kMaxCode;
  const uint64_t m2 = pk2(m, m);
  if constexpr (Loader::kBf16Exact) {
#pragma unroll 1
    for (int c = 0; c < kNumChunks; ++c) {
      float v[kChunk];
      ld(c, v);
      uint32_t wc[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
      for (int i = 0; i < kChunk / 2; ++i) {
        const uint64_t y2 = fma2_rm(pk2(v[2 * i], v[2 * i + 1]),
                                    pk2(v[2 * i] < 0.f ? inv_dn : inv_up, v[2 * i + 1] < 0.f ? inv_dn : inv_up), m2);
        float ya, yb;
        unpk2(y2, ya, yb);
        put_chunk_code<BITS>(wc, 2 * i, f2u(fminf(fmaxf(ya, ylo), yhi)) & (uint32_t)kMaxCode);
        put_chunk_code<BITS>(wc, 2 * i + 1, f2u(fminf(fmaxf(yb, ylo), yhi)) & (uint32_t)kMaxCode);
      }
      store_chunk<BITS>(dst, c, wc);
    }
    return;
  }
  const uint64_t dn2 = pk2(inv_dn, inv_dn), up2 = pk2(inv_up, inv_up);
  uint32_t mism = 0u;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
    uint32_t wc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
    for (int i = 0; i < kChunk / 2; ++i) {
      const uint64_t p = pk2(v[2 * i], v[2 * i + 1]);
      const uint64_t y1 = fma2_rm(p, dn2, m2);
      const uint64_t y2 = fma2_rm(p, up2, m2);
      const uint64_t dif = y1 ^ y2;
      mism |= (uint32_t)dif | (uint32_t)(dif >> 32);
      float ya, yb;
      unpk2(y1, ya, yb);
      put_chunk_code<BITS>(wc, 2 * i, f2u(fminf(fmaxf(ya, ylo), yhi)) & (uint32_t)kMaxCode);
      put_chunk_code<BITS>(wc, 2 * i + 1, f2u(fminf(fmaxf(yb, ylo), yhi)) & (uint32_t)kMaxCode);
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

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f_q(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Three smallest (lo, ascending) and three largest (hi, descending) values so far, updated
// with four more values at once: the four are sorted by a five-comparator network, then
// each end is merged; the k-th smallest of two sorted lists A, B is the least over splits
// i + j = k of max(A[i-1], B[j-1]) (and symmetrically for the largest).
__device__ __forceinline__ void select_update4(float v0, float v1, float v2, float v3, float (&lo)[3],
                                               float (&hi)[3]) {
  float a = fminf(v0, v1), b = fmaxf(v0, v1), c = fminf(v2, v3), d = fmaxf(v2, v3);
  const float s0 = fminf(a, c), t2 = fmaxf(a, c);
  const float t1 = fminf(b, d), s3 = fmaxf(b, d);
  const float s1 = fminf(t1, t2), s2 = fmaxf(t1, t2);     // s0 <= s1 <= s2 <= s3
  const float n2 = fminf(min3f(lo[2], s2, fmaxf(lo[1], s0)), fmaxf(lo[0], s1));
  const float n1 = min3f(lo[1], s1, fmaxf(lo[0], s0));
  lo[0] = fminf(lo[0], s0);
  lo[1] = n1;
  lo[2] = n2;
  const float m2 = fmaxf(max3f_q(hi[2], s1, fminf(hi[1], s3)), fminf(hi[0], s2));
  const float m1 = max3f_q(hi[1], s2, fminf(hi[0], s3));
  hi[0] = fmaxf(hi[0], s3);
  hi[1] = m1;
  hi[2] = m2;
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
  static_assert(KSEL == 3, "the four-at-a-time selection keeps three values at each end");
  uint64_t fsum2 = 0ull;                  // packed sum, only to detect NaN / Inf inputs
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
#pragma unroll
    for (int i = 0; i < kChunk; i += 4) {
      select_update4(v[i], v[i + 1], v[i + 2], v[i + 3], lo_k, hi_k);
      fsum2 = fma2_rn(pk2(v[i], v[i + 1]), pk2(1.f, 1.f), fsum2);
      fsum2 = fma2_rn(pk2(v[i + 2], v[i + 3]), pk2(1.f, 1.f), fsum2);
    }
  }
  {
    float fa, fb;
    unpk2(fsum2, fa, fb);
    if (!isfinite(fa + fb)) flags |= WUSHKV_STATUS_NONFINITE;
  }
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
  // y = rne((x - zero) * inv) + 1.5 * 2^23; clamped to [1.5 * 2^23, 1.5 * 2^23 + 2^b - 1]
  // its low mantissa bits are the code
  const uint64_t z2 = pk2(z, z), dn2 = pk2(inv_dn, inv_dn), up2 = pk2(inv_up, inv_up), m2 = pk2(kMagic, kMagic);
  const float ylo = kMagic, yhi = kMagic + (float)kMaxCode;
  uint32_t mism = 0u;
#pragma unroll 1
  for (int c = 0; c < kNumChunks; ++c) {
    float v[kChunk];
    ld(c, v);
    uint32_t wc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wc[k] = 0u;
#pragma unroll
    for (int i = 0; i < kChunk / 2; ++i) {
      const uint64_t d = sub2_rn(pk2(v[2 * i], v[2 * i + 1]), z2);
      const uint64_t y1 = fma2_rn(d, dn2, m2);
      const uint64_t y2 = fma2_rn(d, up2, m2);
      const uint64_t dif = y1 ^ y2;
      mism |= (uint32_t)dif | (uint32_t)(dif >> 32);
      float ya, yb;
      unpk2(y1, ya, yb);
      put_chunk_code<BITS>(wc, 2 * i, f2u(fminf(fmaxf(ya, ylo), yhi)) & (uint32_t)kMaxCode);
      put_chunk_code<BITS>(wc, 2 * i + 1, f2u(fminf(fmaxf(yb, ylo), yhi)) & (uint32_t)kMaxCode);
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
