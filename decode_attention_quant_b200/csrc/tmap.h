// Host helpers: TMA tensor-map encoding through the runtime's driver entry point (the
// library does not link libcuda directly), and a per-device SM count cache.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace wushkv {

// Encode a tiled tensor map; returns false if the driver entry point is unavailable
// or the driver rejects the layout.
bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                  const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                  CUtensorMapSwizzle swizzle);

int num_sms(cudaError_t* err);

}  // namespace wushkv
