// tensor_map.h -- TMA tensor-map creation and device queries (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dart {

// Tiled bf16 tensor map with 128-byte swizzle.  dims[0] is the contiguous
// dimension; strides_bytes[i] is the byte stride of dims[i + 1] (each a
// multiple of 16).  Returns false if the driver rejects the description.
bool encode_tile_map_bf16(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box);

// The same for fp32 elements (box[0] * 4 must not exceed the 128-byte swizzle span).
bool encode_tile_map_f32(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                         const uint64_t* strides_bytes, const uint32_t* box);

// Number of SMs of the current device (0 on error).
int sm_count();

}  // namespace dart
