// TMA tensor maps for the tcgen05 and decode kernels: bf16 elements, 128-byte
// swizzle, zero fill out of bounds. The driver's encoder is looked up once per
// process (thread-safe), through the runtime's driver entry point.
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace qsa {

// True when the driver's tensor-map encoder is available.
bool tmap_available();

// Encodes a rank-dimensional bf16 map: dims[0] is the contiguous dimension,
// strides_bytes[i] is the stride of dimension i + 1, box the copied tile. Returns
// CUDA_SUCCESS, the driver's error, or CUDA_ERROR_NOT_SUPPORTED without an encoder.
CUresult encode_tmap_bf16(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims,
                          const uint64_t *strides_bytes, const uint32_t *box);

}  // namespace qsa
