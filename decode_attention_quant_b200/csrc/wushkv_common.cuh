// Shared device helpers of the WUSH-KV kernels (sm_100a).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/wushkv.h"

namespace wushkv {

constexpr int kHeadDim = 128;

// OR a status bit into the caller's optional device word.
__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }
__device__ __forceinline__ int32_t f2i(float f) { return __float_as_int(f); }

// fp64 -> fp16 with one round-to-nearest-even (the PTX conversion instruction).
__device__ __forceinline__ uint16_t f64_to_f16_bits(double d) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(d));
  return h;
}
__device__ __forceinline__ uint16_t f32_to_f16_bits(float f) {
  return __half_as_ushort(__float2half_rn(f));
}
__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 ld_global_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Row of the codes / meta arrays that holds position t of sequence b, KV head h, in the
// contiguous layout ([batch][Hkv][capacity]) or the paged one ([num_pages][Hkv][page_size],
// page from the block table); -1 when the block table points outside the pool.
struct CacheRows {
  const int32_t* block_table;   // nullptr: contiguous
  int pages_per_seq, page_shift, num_pages, hkv, capacity;

  static CacheRows of(const wushkv_cache& c) {
    CacheRows r{};
    r.block_table = c.block_table;
    r.pages_per_seq = c.pages_per_seq;
    r.num_pages = c.num_pages;
    r.hkv = c.num_kv_heads;
    r.capacity = c.capacity;
    int shift = 0;
    while (c.block_table != nullptr && (1 << shift) < c.page_size) ++shift;
    r.page_shift = shift;
    return r;
  }
  __device__ __forceinline__ long long row(int b, int h, int t) const {
    if (block_table == nullptr) return ((long long)b * hkv + h) * capacity + t;
    const int page = __ldg(block_table + (size_t)b * pages_per_seq + (t >> page_shift));
    if (page < 0 || page >= num_pages) return -1;
    return (((long long)page * hkv + h) << page_shift) + (t & ((1 << page_shift) - 1));
  }
};

// Two bf16 packed in a 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace wushkv
