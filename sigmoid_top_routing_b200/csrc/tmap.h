// Tensor-map (TMA descriptor) construction shared by the kernels' launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Row-major 2D matrix of `rows` rows x `inner` elements of `dtype` (1, 2 or 4
// bytes), boxes of box_inner x box_rows, optionally 128-byte swizzled, zero
// fill out of bounds.  cudaErrorNotSupported without the driver entry point,
// cudaErrorInvalidValue when the driver rejects the description.
cudaError_t make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                         uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows, bool swizzle128);

}  // namespace moe
