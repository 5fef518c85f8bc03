// Causal attention of a chunk of n_q <= 16 queries per sequence over the packed cache,
// on the tensor cores with the chunk's rows on the MMA's M side.
//
// WUSH-KV runs its perplexity evaluation with every sequence fed in 16-token forward
// chunks (ai4snews summary, paragraph 3).  The chunk's tokens are appended first, so
// every key and value is read in packed form: query i of sequence b sits at position
// p_i = ctx - n_q + i (ctx = min(ctx_len[b], capacity)) and attends positions 0 .. p_i.
//
// One CTA = (split of the positions, KV head, block of 128 folded rows, sequence); row
// f = i * g + h is query i of head h.  512 threads; per 128-position tile:
//   converters (warps 0-3): load the tile's packed K and V codes and meta one tile ahead
//     (lane 4i + k takes quarter k of the packed rows of positions i, 8 + i, ...; thread
//     t the meta of position t), turn the codes into exact fp16 (the code ORed into the
//     mantissa of 1024, minus 1024; fp16 subnormals would save the subtraction, but the
//     MMAs lose precision on subnormal operands) and store them with stmatrix into a
//     three-stage ring of 128-byte-swizzled K-major operands: keys as [position][slot],
//     values transposed as [slot][position] (a K-major B runs the value MMAs about 1.7x
//     faster than an MN-major one); the meta as fp32;
//   issuer (warp 12, one thread): S = Q' K^T as two fp16 MMAs with q' in tensor memory
//     (split into fp16 hi + lo, so the products carry 22 bits of q'), fp32 accumulation;
//     then O += P' V as two fp16 MMAs with P' in tensor memory;
//   softmax (warps 4-11, thread = row and half of the tile's positions): scores
//     s = tau log2e (scale_t q'.c + zero_t sum q') in the log2 domain, causal mask, the
//     tile maximum, e = 2^(s - m) against a running reference m that moves only when the
//     maximum passes it by 2^8 (then O, l and z are rescaled), l = sum e, z = sum e * zero,
//     and P' = e * scale * 2^-E in fp16 hi + lo.
// The softmax warpgroups take most of the register file (setmaxnreg); warps 13-15 only
// give theirs up.  E is the running maximum exponent of the value scales seen so far
// (from the converters), which keeps P' <= 2^8 inside fp16 for any scale; O is rescaled
// by an exact power of two when it grows.  The split partial (m, l, O 2^E + z) goes to
// the workspace; a combine pass merges splits.  Codes are converted in pairs straight
// from the lane's quarter of the packed row, which permutes the channels (slot_channel);
// the query and the output use the same order.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "sm100.cuh"
#include "tmap.h"
#include "wushkv_common.cuh"
#include "wushkv_launch.h"
#include "wushkv_quant.cuh"

namespace wushkv {
namespace {

using namespace sm100;

constexpr int kN = 128;                         // cached positions per tile
constexpr int kRows = 128;                      // folded rows per CTA = TMEM lanes
constexpr int kStages = 3;                      // K/V operand ring
constexpr int kConvWarps = 4;
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = kConvWarps + kSoftWarps;
constexpr int kThreads = 512;                   // four warpgroups
constexpr int kRegsConv = 104, kRegsSoft = 184, kRegsMma = 40;
static_assert(128 * kRegsConv + 256 * kRegsSoft + 128 * kRegsMma <= 65536, "register split over the launch's");
constexpr int kPartialStride = 132;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;                   // log2 headroom of the running reference
constexpr int kHalfBytes = 16384;               // [128 rows][64 x 16-bit], 128-byte swizzled
constexpr int kNoScale = -126;                  // value-scale exponent before any valid position

constexpr int kColS = 0;                        // 128 columns: scores
constexpr int kColQ = 128;                      // q' hi (64 columns) then q' lo (64)
constexpr int kColP = 256;                      // P' hi (64 columns) then P' lo (64)
constexpr int kColO = 384;                      // 128 columns
constexpr int kCols = 512;

struct FaBars {
  uint64_t conv[kStages], kvfree[kStages];   // operand stages: written / released by the PV MMAs
  uint64_t sfull, sfree;                      // scores: computed / read by the softmax warps
  uint64_t pfull, pvdone;                     // P' written (and O rescaled) / PV MMAs done
  uint64_t drain;                             // MMAs in flight at a timeout
  uint32_t tmem_base;
  int abort;
};

// Shared memory (operand stages 1 KB aligned for the 128-byte swizzle).
constexpr int kOffKb = 0;                                  // B of S: [stage][2 halves][128 pos][128 B]
constexpr int kOffVb = kOffKb + kStages * 2 * kHalfBytes;  // B of PV: [stage][2 halves][128 slots][128 B]
constexpr int kOffMeta = kOffVb + kStages * 2 * kHalfBytes;
// per stage: ks, kz, vs * 2^-E, vz [128] fp32; 4 validity words; E; padding
constexpr int kMetaWords = 4 * kN + 8;
constexpr int kMetaBytes = 4 * kMetaWords;
constexpr int kOffRow = kOffMeta + kStages * kMetaBytes;   // row exchange [8][128] fp32
constexpr int kOffScl = kOffRow + 8 * kRows * 4;           // converter warps' scale maxima [stage][4]
constexpr int kOffBar = kOffScl + 64;
constexpr int kSmem = kOffBar + (int)sizeof(FaBars) + 1024;
static_assert(kSmem <= 227 * 1024, "one CTA per SM");

struct FaArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint16_t* k_meta;
  const uint16_t* v_meta;
  CacheRows rows;
  const float* q;              // [B][n_q][Hq][128]
  const int32_t* ctx_len;
  float* ws;                   // partials [(b, i, h)][splits][132]
  int32_t* status;
  int n_q, hq, hkv, capacity, num_splits, row_blocks;
  float scale_log2;            // softmax scale * log2 e
};

// Channel held by slot s (of 128) of a converted row.  Slot pair (8c + 2k, 8c + 2k + 1)
// is pair c of quarter k of the packed row: 2-bit words 2k, 2k + 1 hold channels
// 32k .. 32k + 31, pair c = word 2k + c / 8 shifted by 2 (c mod 8), so channels
// (16 (2k + c / 8) + c mod 8, + 8); 4-bit words 4k .. 4k + 3, pair c = word 4k + c / 4
// shifted by 4 (c mod 4): channels (8 (4k + c / 4) + c mod 4, + 4); 3-bit bits 96k ..
// 96k + 95 hold channels 32k .. 32k + 31 in order.
template <int BITS>
__host__ __device__ __forceinline__ int slot_channel(int s) {
  const int k = (s >> 1) & 3, c = s >> 3, e = s & 1;
  if (BITS == 2) return 32 * k + 16 * (c >> 3) + (c & 7) + 8 * e;
  if (BITS == 4) return 32 * k + 8 * (c >> 2) + (c & 3) + 4 * e;
  return 32 * k + 2 * c + e;
}

// Words of quarter k of a packed row: 2-bit 2, 3-bit 3, 4-bit 4.
template <int BITS>
struct Quarter {
  static constexpr int W = BITS;
  uint32_t k[W], v[W];
};

template <int BITS>
__device__ __forceinline__ void load_quarter(const uint8_t* codes, long long row, int kq, uint32_t (&w)[BITS]) {
  const uint8_t* p = codes + row * (16 * BITS) + 4 * BITS * kq;
  if (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x; w[1] = v.y;
  } else if (BITS == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else {
#pragma unroll
    for (int q = 0; q < BITS; ++q) w[q] = __ldg(reinterpret_cast<const uint32_t*>(p) + q);
  }
}

// fp16 pair (1024 + a, 1024 + b) -> (a, b), exact for small integers
__device__ __forceinline__ uint32_t unbias2(uint32_t x) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&x), __halves2half2(__ushort_as_half(0x6400),
                                                                                    __ushort_as_half(0x6400)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Pair c of a quarter as an exact fp16 pair (slot order, see slot_channel).
template <int BITS>
__device__ __forceinline__ uint32_t code_pair_f16(const uint32_t (&w)[BITS], int c) {
  if (BITS == 2) return unbias2(((w[c >> 3] >> (2 * (c & 7))) & 0x00030003u) | 0x64006400u);
  if (BITS == 4) return unbias2(((w[c >> 2] >> (4 * (c & 3))) & 0x000F000Fu) | 0x64006400u);
  const int bit = 6 * c, wi = bit >> 5, sh = bit & 31;   // channels 2c, 2c + 1 of the quarter
  const uint32_t hi = (wi + 1 < BITS) ? w[wi + 1] : 0u;
  const uint32_t f = __funnelshift_r(w[wi], hi, sh);
  return unbias2(((f & 7u) | ((f & 0x38u) << 13)) | 0x64006400u);
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

// fp32 2^e for e in [-126, 127] (exact)
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// The raw meta of one position (zero where the position is not valid).
template <int KIND>
struct PosMeta {
  uint32_t km, vm;
  bool valid;

  __device__ __forceinline__ void load(const FaArgs& a, int b, int kv, int pos, int ctx) {
    valid = false;
    km = 0u;
    vm = 0u;
    if (pos < ctx) {
      const long long row = a.rows.row(b, kv, pos);
      if (row >= 0) {
        valid = true;
        if (KIND == WUSHKV_QUEST_INT) {
          km = __ldg(a.k_meta + row);
          vm = __ldg(a.v_meta + row);
        } else {
          km = __ldg(reinterpret_cast<const uint32_t*>(a.k_meta) + row);
          vm = __ldg(reinterpret_cast<const uint32_t*>(a.v_meta) + row);
        }
      } else {
        report(a.status, WUSHKV_STATUS_BAD_PAGE);
      }
    }
  }
};

// Quarter kq of the K and V rows of positions base + 8m (m = 0..3), zero where not valid.
template <int BITS>
__device__ __forceinline__ void load_quarters(const FaArgs& a, int b, int kv, int base, int ctx, int kq,
                                              Quarter<BITS> (&f)[4]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int pos = base + 8 * m;
    long long row = -1;
    if (pos < ctx) row = a.rows.row(b, kv, pos);
    if (row >= 0) {
      load_quarter<BITS>(a.k_codes, row, kq, f[m].k);
      load_quarter<BITS>(a.v_codes, row, kq, f[m].v);
    } else {
#pragma unroll
      for (int q = 0; q < BITS; ++q) { f[m].k[q] = 0u; f[m].v[q] = 0u; }
    }
  }
}

template <int BITS, int KIND>
__global__ void __launch_bounds__(kThreads, 1) chunk_fa_kernel(const FaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kb = smem + kOffKb;
  uint8_t* vb = smem + kOffVb;
  float* meta = reinterpret_cast<float*>(smem + kOffMeta);
  float* rowx = reinterpret_cast<float*>(smem + kOffRow);
  uint32_t* sclx = reinterpret_cast<uint32_t*>(smem + kOffScl);
  FaBars* bars = reinterpret_cast<FaBars*>(smem + kOffBar);
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

  if (threadIdx.x == 0) {
    for (int j = 0; j < kStages; ++j) {
      mbar_init(&bars->conv[j], kConvWarps);
      mbar_init(&bars->kvfree[j], 1);
    }
    mbar_init(&bars->sfull, 1);
    mbar_init(&bars->sfree, kSoftWarps);
    mbar_init(&bars->pfull, kSoftWarps);
    mbar_init(&bars->pvdone, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // Softmax warps: row r of this block, half hf of each tile's positions (and of the
  // query's slots while preparing the query operand).
  const int r = 32 * (warp & 3) + lane;
  const int hf = (warp - kConvWarps) >> 2;
  const int f = rb * kRows + r;
  const bool row_ok = f < R;
  const int qi = row_ok ? f / g : 0;
  const int qh_idx = row_ok ? kv * g + f % g : 0;
  const int p_last = ctx - a.n_q + qi;                 // last visible position of this row
  const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
  const uint32_t bar_pair = 2 + (warp & 3);              // the two softmax warps of a lane quarter
  float rowc = 0.f, qs = 0.f;                            // per row: tau log2e / sigma, tau log2e sum q'
  if (warp >= kConvWarps && warp < kMmaWarp) {
    // q' row: slots 64 hf .. 64 hf + 63 hold channels 32k + 16 hf .. 32k + 16 hf + 15
    // (k = 0..3), loaded as 16 float4 -> sigma q' in fp16 hi + lo, slot order, into
    // tensor memory as the A operand of the score MMAs
    const float4* qrow = reinterpret_cast<const float4*>(a.q + (((size_t)b * a.n_q + qi) * a.hq + qh_idx) * kHeadDim);
    float ch[64];                                        // ch[16k + j] = channel 32k + 16 hf + j
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float4 v4 = row_ok ? __ldg(qrow + 8 * (m >> 2) + 4 * hf + (m & 3)) : make_float4(0.f, 0.f, 0.f, 0.f);
      ch[4 * m] = v4.x; ch[4 * m + 1] = v4.y; ch[4 * m + 2] = v4.z; ch[4 * m + 3] = v4.w;
    }
    float mx = 0.f, sm = 0.f;
#pragma unroll
    for (int s = 0; s < 64; ++s) {
      mx = fmaxf(mx, fabsf(ch[s]));
      sm += ch[s];
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
    for (int c = 0; c < 2; ++c) {                        // slots 32c .. 32c + 31 -> 16 columns
      uint32_t x[16], y[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        // slot 64 hf + s0 holds channel slot_channel(s0) + 16 hf
        const int s0 = 32 * c + 2 * k;
        const int c0 = slot_channel<BITS>(s0), c1 = slot_channel<BITS>(s0 + 1);
        const float x0 = ch[16 * (c0 >> 5) + (c0 & 15)] * sigma, x1 = ch[16 * (c1 >> 5) + (c1 & 15)] * sigma;
        const __half2 h2 = __floats2half2_rn(x0, x1);
        const float2 hb = __half22float2(h2);
        const __half2 l2 = __floats2half2_rn(x0 - hb.x, x1 - hb.y);
        x[k] = *reinterpret_cast<const uint32_t*>(&h2);
        y[k] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      tmem_st16(tmem + lanes + kColQ + 32 * hf + 16 * c, x);
      tmem_st16(tmem + lanes + kColQ + 64 + 32 * hf + 16 * c, y);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Each role runs entirely inside its branch, which starts by resizing its registers.
  if (warp < kConvWarps) {
    // ------------------------------------------------------------- converters
    regs_dec<kRegsConv>();
    const int t = threadIdx.x;                           // meta: position t of each tile
    const int i8 = lane >> 2, kq = lane & 3;             // codes: positions 32 warp + 8m + i8, quarter kq
    const uint32_t kb_a = smem_u32(kb), vb_a = smem_u32(vb);
    PosMeta<KIND> cur, nxt;
    Quarter<BITS> fc[4], fn[4];
    if (n > 0) {
      cur.load(a, b, kv, tile0 * kN + t, ctx);
      load_quarters<BITS>(a, b, kv, tile0 * kN + 32 * warp + i8, ctx, kq, fc);
    }
    int e_cur = kNoScale;                                // running value-scale exponent
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int st = i % kStages;
      if (i + 1 < n) {
        nxt.load(a, b, kv, (tile0 + i + 1) * kN + t, ctx);
        load_quarters<BITS>(a, b, kv, (tile0 + i + 1) * kN + 32 * warp + i8, ctx, kq, fn);
      }
      float ks = 0.f, kz = 0.f, vs = 0.f, vz = 0.f;
      if (cur.valid) {
        meta_of<KIND>(cur.km, BITS, ks, kz);
        meta_of<KIND>(cur.vm, BITS, vs, vz);
      }
      // the tile's largest value scale (scales are >= 0, so their bits order like them)
      const uint32_t smax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(vs)));
      const uint32_t vmask = __ballot_sync(0xffffffffu, cur.valid);
      if (lane == 0) sclx[st * 4 + warp] = smax;
      named_barrier(1, 32 * kConvWarps);
      const float tmax = __uint_as_float(max(max(sclx[st * 4], sclx[st * 4 + 1]),
                                             max(sclx[st * 4 + 2], sclx[st * 4 + 3])));
      if (tmax > 0.f) {
        int et = 0;
        frexpf(tmax, &et);                               // tmax < 2^et (fp16 scales: et <= 16)
        e_cur = min(max(e_cur, et), 126);                // 2^-E stays a normal fp32
      }
      if (i >= kStages) ok = mbar_wait(&bars->kvfree[st], ((i - kStages) / kStages) & 1, abort) && ok;
      float* mt = meta + st * kMetaWords;
      mt[t] = ks;
      mt[kN + t] = kz;
      mt[2 * kN + t] = vs * exp2i(-e_cur);
      mt[3 * kN + t] = vz;
      uint32_t* mw = reinterpret_cast<uint32_t*>(mt + 4 * kN);
      if (lane == 0) mw[warp] = vmask;
      if (t == 0) mw[4] = (uint32_t)e_cur;
      if (ok) {
        // keys: matrix (8 positions x slots 8c .. 8c + 7) -> rows = positions;
        // values: the same matrix transposed -> rows = slots, 8 positions per row
        const uint32_t kst = kb_a + st * 2 * kHalfBytes, vst = vb_a + st * 2 * kHalfBytes;
        const int mj = lane >> 3, mr = lane & 7;         // this lane's row address: matrix mj, row mr
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int p0 = 32 * warp + 8 * m;              // first position of the group
#pragma unroll
          for (int cg = 0; cg < 4; ++cg) {
            const int c = 4 * cg + mj;                   // chunk (8 slots) of this lane's row address
            const uint32_t ka = kst + (c >> 3) * kHalfBytes + (p0 + mr) * 128 + (((c & 7) ^ mr) << 4);
            const int nrow = 8 * c + mr;
            const uint32_t va = vst + (p0 >> 6) * kHalfBytes + nrow * 128 + ((((p0 & 63) >> 3) ^ (nrow & 7)) << 4);
            stmatrix_x4(ka, code_pair_f16<BITS>(fc[m].k, 4 * cg), code_pair_f16<BITS>(fc[m].k, 4 * cg + 1),
                        code_pair_f16<BITS>(fc[m].k, 4 * cg + 2), code_pair_f16<BITS>(fc[m].k, 4 * cg + 3));
            stmatrix_x4_trans(va, code_pair_f16<BITS>(fc[m].v, 4 * cg), code_pair_f16<BITS>(fc[m].v, 4 * cg + 1),
                              code_pair_f16<BITS>(fc[m].v, 4 * cg + 2), code_pair_f16<BITS>(fc[m].v, 4 * cg + 3));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->conv[st]);
      cur = nxt;
#pragma unroll
      for (int m = 0; m < 4; ++m) fc[m] = fn[m];
    }
  } else if (warp >= kMmaWarp) {
    // ------------------------------------------------------------- MMA issue
    // The whole warp walks the tiles; lane 0 waits and issues, the others follow it.
    regs_dec<kRegsMma>();
    if (warp == kMmaWarp) {
    constexpr uint32_t kIdS = idesc(kFmtF32, kFmtF16, kFmtF16, 0, 0, 128, 128);
    constexpr uint32_t kIdPV = idesc(kFmtF32, kFmtF16, kFmtF16, 0, 0, 128, 128);
    const uint32_t kb_a = smem_u32(kb), vb_a = smem_u32(vb);
    bool ok = true, issued = false;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = mbar_wait(bar, parity, abort);
      return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    };
    auto pv = [&](int j) {
      if (!(ok = ok && wait_all(&bars->pfull, j & 1))) return;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t vbase = vb_a + (j % kStages) * 2 * kHalfBytes;
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_f16_ts(tmem + kColO, tmem + kColP + pl * 64 + k * 8,
                       desc_kmajor_sw128(vbase + (k >> 2) * kHalfBytes + (k & 3) * 32), kIdPV,
                       (j > 0 || pl > 0 || k > 0) ? 1u : 0u);
        mma_commit(&bars->pvdone);
        mma_commit(&bars->kvfree[j % kStages]);
        issued = true;
      }
      __syncwarp();
    };
    for (int i = 0; i < n && ok; ++i) {
      const int st = i % kStages;
      if (!(ok = wait_all(&bars->conv[st], (i / kStages) & 1))) break;
      if (i >= 1 && !(ok = wait_all(&bars->sfree, (i - 1) & 1))) break;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t kbase = kb_a + st * 2 * kHalfBytes;
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_f16_ts(tmem + kColS, tmem + kColQ + pl * 64 + k * 8,
                       desc_kmajor_sw128(kbase + (k >> 2) * kHalfBytes + (k & 3) * 32), kIdS, (pl | k) != 0);
        mma_commit(&bars->sfull);
        issued = true;
      }
      __syncwarp();
      if (i >= 1) pv(i - 1);
    }
    if (ok && n > 0) pv(n - 1);
    // no MMA may still run when the tensor memory is released, even after a timeout
    if (lane == 0 && issued && *abort) {
      volatile int no_abort = 0;
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &no_abort);
    }
    __syncwarp();
    }
  } else {
    // ------------------------------------------------------------- softmax
    regs_inc<kRegsSoft>();
    const uint64_t rowc2 = pk2(rowc, rowc);
    const uint64_t qs2 = pk2(qs, qs);
    // QuEST: zero = -c0 * scale, so s = scale * (rowc * raw - c0 * qs)
    const float c0 = (float)(1 << (BITS - 1)) - 0.5f;
    const uint64_t cq2 = pk2(-c0 * qs, -c0 * qs);
    float m_ref = -CUDART_INF_F, l = 0.f, z = 0.f;
    int e_prev = kNoScale;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int st = i % kStages;
      ok = ok && mbar_wait(&bars->sfull, i & 1, abort);
      ok = ok && mbar_wait(&bars->conv[st], (i / kStages) & 1, abort);
      tc_fence_after();
      uint32_t raw[64];
      tmem_ld32(tmem + lanes + kColS + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(raw));
      tmem_ld32(tmem + lanes + kColS + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->sfree);
      const float* mt = meta + st * kMetaWords;
      const uint32_t* mw = reinterpret_cast<const uint32_t*>(mt + 4 * kN);
      const uint32_t vm0 = mw[2 * hf], vm1 = mw[2 * hf + 1];
      const int e_t = (int)mw[4];
      const int pos0 = (tile0 + i) * kN + 64 * hf;
      // x = s - base, base = the reference (0 before the row has seen a position)
      const float base = m_ref == -CUDART_INF_F ? 0.f : m_ref;
      const uint64_t nb2 = pk2(-base, -base);
      float x[64];
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(mt + 64 * hf + j);
        const uint64_t r01 = pk2(__uint_as_float(raw[j]), __uint_as_float(raw[j + 1]));
        const uint64_t r23 = pk2(__uint_as_float(raw[j + 2]), __uint_as_float(raw[j + 3]));
        uint64_t x01, x23;
        if (KIND == WUSHKV_QUEST_INT) {
          x01 = fma2_rn(pk2(k4.x, k4.y), fma2_rn(rowc2, r01, cq2), nb2);
          x23 = fma2_rn(pk2(k4.z, k4.w), fma2_rn(rowc2, r23, cq2), nb2);
        } else {
          const float4 z4 = *reinterpret_cast<const float4*>(mt + kN + 64 * hf + j);
          x01 = fma2_rn(mul2_rn(pk2(k4.x, k4.y), r01), rowc2, fma2_rn(pk2(z4.x, z4.y), qs2, nb2));
          x23 = fma2_rn(mul2_rn(pk2(k4.z, k4.w), r23), rowc2, fma2_rn(pk2(z4.z, z4.w), qs2, nb2));
        }
        unpk2(x01, x[j], x[j + 1]);
        unpk2(x23, x[j + 2], x[j + 3]);
      }
      // causal mask and page validity, only where the tile reaches them
      if (!(__all_sync(0xffffffffu, pos0 + 63 <= p_last) && (vm0 & vm1) == 0xffffffffu)) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const bool vis = (((j < 32 ? vm0 >> j : vm1 >> (j - 32)) & 1u) != 0u) && pos0 + j <= p_last;
          x[j] = vis ? x[j] : -CUDART_INF_F;
        }
      }
      float mloc = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < 64; j += 2) mloc = max3f(mloc, x[j], x[j + 1]);
      // tile maximum of the row (both halves), relative to base
      rowx[4 * kRows + (i & 1) * 2 * kRows + hf * kRows + r] = mloc;
      named_barrier(bar_pair, 64);
      const float m_t = fmaxf(mloc, rowx[4 * kRows + (i & 1) * 2 * kRows + (1 - hf) * kRows + r]);
      float shift = 0.f, corr = 1.f;
      if (m_t != -CUDART_INF_F) {
        if (m_ref == -CUDART_INF_F) {
          shift = m_t;
          m_ref = m_t;
        } else if (m_t > kLazy) {
          shift = m_t;
          corr = ex2_approx(-m_t);
          m_ref += m_t;
        }
      }
      if (__any_sync(0xffffffffu, shift != 0.f)) {
        const uint64_t s2 = pk2(-shift, -shift);
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          uint64_t v2 = pk2(x[j], x[j + 1]);
          v2 = add2_rn(v2, s2);
          unpk2(v2, x[j], x[j + 1]);
        }
      }
      // O carries the value scales times 2^-E: it grows by an exact power of two with E
      const float corr_o = corr * (e_t > e_prev && i > 0 ? exp2i(max(e_prev - e_t, -126)) : 1.f);
      e_prev = e_t;
      // P' and O are free once the previous tile's PV MMAs are done
      if (i >= 1) ok = mbar_wait(&bars->pvdone, (i - 1) & 1, abort) && ok;
      tc_fence_after();
      // tensor-memory loads and stores are warp-collective: the warp rescales when any
      // of its rows needs it (factor 1 for the others)
      ok = __all_sync(0xffffffffu, ok);
      if (i > 0 && __any_sync(0xffffffffu, corr_o != 1.f) && ok) {
        const uint64_t c2 = pk2(corr_o, corr_o);
#pragma unroll 1
        for (int c0i = 0; c0i < 64; c0i += 16) {
          uint32_t ov[16];
          tmem_ld16(tmem + lanes + kColO + 64 * hf + c0i, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const uint64_t o2 = mul2_rn(pk2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), c2);
            float o0, o1;
            unpk2(o2, o0, o1);
            ov[e] = __float_as_uint(o0);
            ov[e + 1] = __float_as_uint(o1);
          }
          tmem_st16(tmem + lanes + kColO + 64 * hf + c0i, ov);
        }
      }
      // e = 2^x; l, z; P' = e * scale * 2^-E in fp16 hi + lo, 32 positions at a time
      uint64_t la = pk2(0.f, 0.f), lb = la, za = la, zb = la;
#pragma unroll
      for (int jc = 0; jc < 64; jc += 32) {
        uint32_t ph[16], plo[16];
#pragma unroll
        for (int j = jc; j < jc + 32; j += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(mt + 2 * kN + 64 * hf + j);
          const float4 w4 = *reinterpret_cast<const float4*>(mt + 3 * kN + 64 * hf + j);
          const uint64_t e01 = pk2(ex2_approx(x[j]), ex2_approx(x[j + 1]));
          const uint64_t e23 = pk2(ex2_approx(x[j + 2]), ex2_approx(x[j + 3]));
          la = add2_rn(la, e01);
          lb = add2_rn(lb, e23);
          za = fma2_rn(e01, pk2(w4.x, w4.y), za);
          zb = fma2_rn(e23, pk2(w4.z, w4.w), zb);
          const uint64_t p01 = mul2_rn(e01, pk2(v4.x, v4.y));
          const uint64_t p23 = mul2_rn(e23, pk2(v4.z, v4.w));
          float p0, p1, p2, p3;
          unpk2(p01, p0, p1);
          unpk2(p23, p2, p3);
          const __half2 h01 = __floats2half2_rn(p0, p1), h23 = __floats2half2_rn(p2, p3);
          const float2 b01 = __half22float2(h01), b23 = __half22float2(h23);
          float d0, d1, d2, d3;
          unpk2(sub2_rn(p01, pk2(b01.x, b01.y)), d0, d1);
          unpk2(sub2_rn(p23, pk2(b23.x, b23.y)), d2, d3);
          const __half2 l01 = __floats2half2_rn(d0, d1), l23 = __floats2half2_rn(d2, d3);
          ph[(j - jc) >> 1] = *reinterpret_cast<const uint32_t*>(&h01);
          ph[((j - jc) >> 1) + 1] = *reinterpret_cast<const uint32_t*>(&h23);
          plo[(j - jc) >> 1] = *reinterpret_cast<const uint32_t*>(&l01);
          plo[((j - jc) >> 1) + 1] = *reinterpret_cast<const uint32_t*>(&l23);
        }
        tmem_st16(tmem + lanes + kColP + 32 * hf + jc / 2, ph);
        tmem_st16(tmem + lanes + kColP + 64 + 32 * hf + jc / 2, plo);
      }
      float l0, l1, l2, l3, z0, z1, z2, z3;
      unpk2(la, l0, l1);
      unpk2(lb, l2, l3);
      unpk2(za, z0, z1);
      unpk2(zb, z2, z3);
      l = fmaf(l, corr, (l0 + l1) + (l2 + l3));
      z = fmaf(z, corr, (z0 + z1) + (z2 + z3));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pfull);
    }
    // ---- split partial of the row: m (log2 domain), l, O 2^E + z
    uint32_t o[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) o[e] = 0u;
    if (n > 0) {
      ok = ok && mbar_wait(&bars->pvdone, (n - 1) & 1, abort);
      tc_fence_after();
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
    const float oscale = exp2i(min(max(e_prev, -126), 127));
    if (row_ok) {
      float* dst = a.ws + ((((size_t)b * a.n_q + qi) * a.hq + qh_idx) * a.num_splits + split) * kPartialStride;
#pragma unroll
      for (int e = 0; e < 64; ++e)
        dst[4 + slot_channel<BITS>(64 * hf + e)] = fmaf(__uint_as_float(o[e]), oscale, z_tot);
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

template <int BITS>
cudaError_t launch_bits(const wushkv_cache& c, const FaArgs& a, int batch, cudaStream_t stream) {
  const dim3 grid(a.num_splits, a.hkv * a.row_blocks, batch);
  if (c.qp.kind == WUSHKV_QUEST_INT) {
    auto kern = chunk_fa_kernel<BITS, WUSHKV_QUEST_INT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kSmem, stream>>>(a);
  } else {
    auto kern = chunk_fa_kernel<BITS, WUSHKV_PCT_AFFINE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kSmem, stream>>>(a);
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
  a.k_codes = c.k_codes;
  a.v_codes = c.v_codes;
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
