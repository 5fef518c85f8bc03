// Decode attention without caller-provided scratch: the split-K partials live in a
// fixed array of this library's device memory instead of a workspace the caller
// allocates.  Everything else (checks, kernels, results) is wushkv_decode_attention.
//
// Who needs it: a caller that cannot hand the library scratch memory, such as a
// plugin inside a host runtime that owns every device allocation and offers no
// allocator to extensions, or a serving loop that forbids allocation after start-up
// so that its device-memory footprint stays fixed.
//
// Sharing rules: every call on a device uses the same array.  Calls keep whatever
// the last call left there; nothing in it has to start at zero, because the decode
// kernel writes every partial (m, l, o) of every split before the combine kernel
// reads it.  Two calls that may run at the same time on one device (different
// streams, or different host threads without ordering) race on the array.
#include <atomic>
#include <mutex>

#include "wushkv_launch.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[WUSHKV_DECODE_STATIC_SCRATCH_BYTES];

std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_decode_scratch on the current device, looked up once per device.
int scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return wushkv::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return WUSHKV_ERR_UNSUPPORTED;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e == cudaSuccess && p == nullptr) e = cudaErrorInvalidSymbol;
      if (e != cudaSuccess) return wushkv::record_cuda_error(e);
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return WUSHKV_OK;
}

}  // namespace

extern "C" {

int wushkv_decode_attention_noalloc(const wushkv_cache* cache, const float* q_t, int32_t num_q_heads,
                                    const int32_t* ctx_len, float softmax_scale, float* out,
                                    int32_t num_splits, int32_t* status, void* stream) {
  const size_t need = wushkv_decode_workspace_bytes(cache, num_q_heads, num_splits);
  if (need == 0) {
    // The cache, the head counts or num_splits are invalid: the regular entry's own
    // checks say which, before they ever look at the (absent) workspace.
    return wushkv_decode_attention(cache, q_t, num_q_heads, ctx_len, softmax_scale, out, nullptr, 0,
                                   num_splits, status, stream);
  }
  if (need > (size_t)WUSHKV_DECODE_STATIC_SCRATCH_BYTES) return WUSHKV_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != WUSHKV_OK) return rc;
  return wushkv_decode_attention(cache, q_t, num_q_heads, ctx_len, softmax_scale, out, scratch,
                                 (size_t)WUSHKV_DECODE_STATIC_SCRATCH_BYTES, num_splits, status, stream);
}

}  // extern "C"
