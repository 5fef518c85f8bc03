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
//
// The array's device address belongs to the CUDA context that loaded this module.
// It is looked up once per context (the first call after a context is made current
// on a device, e.g. the first call on that device, or the first after the primary
// context was reset by cudaDeviceReset) and cached with the context handle.
#include <cuda.h>

#include <mutex>

#include "wushkv_launch.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[WUSHKV_DECODE_STATIC_SCRATCH_BYTES];

struct ScratchSlot {
  CUcontext ctx;   // context the address was looked up in
  void* ptr;       // device address of g_decode_scratch in that context
};
ScratchSlot g_slots[kMaxDevices];
std::mutex g_setup_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_decode_scratch in the current device's current context.
int scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return wushkv::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return WUSHKV_ERR_UNSUPPORTED;
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return wushkv::record_cuda_error(cudaErrorNotSupported);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return wushkv::record_cuda_error(cudaErrorDeviceUninitialized);
  if (ctx == nullptr) {
    // no context current on this thread yet: make the device's primary context current
    // (the one the kernels below run in), then read its handle
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return wushkv::record_cuda_error(e);
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return wushkv::record_cuda_error(cudaErrorDeviceUninitialized);
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchSlot& s = g_slots[dev];
  if (s.ptr == nullptr || s.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e == cudaSuccess && p == nullptr) e = cudaErrorInvalidSymbol;
    if (e != cudaSuccess) return wushkv::record_cuda_error(e);
    s.ctx = ctx;
    s.ptr = p;
  }
  *out = s.ptr;
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
