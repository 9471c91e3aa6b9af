// Host-side helpers for the tensor-core kernels: TMA tensor-map encoding
// (through the driver entry point, so the library needs no -lcuda) and the
// device-side counter of bounded waits that gave up.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// 2-D row-major tensor of `rows` x `cols` elements of `dtype` (row stride
// `row_stride` elements), tiled into boxes of box_rows x box_cols with the
// given swizzle.  Out-of-range elements of a box read as zero.
kda_status_t make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                          uint64_t rows, uint64_t cols, uint64_t row_stride, uint32_t box_rows, uint32_t box_cols,
                          CUtensorMapSwizzle swizzle);

// 3-D tensor (d2, d1, d0) with d0 contiguous; strides in elements.
kda_status_t make_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                          uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                          uint32_t box1, uint32_t box2, CUtensorMapSwizzle swizzle);

// N-D tensor (rank <= 5): dims[0] contiguous, strides[i] (elements) for dims[i+1],
// box[i] elements per dimension.
kda_status_t make_tmap_nd(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, int rank,
                          const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                          CUtensorMapSwizzle swizzle);

// Device address of this library's wait-timeout counter on the current device.
unsigned int *device_timeout_counter();

}  // namespace kda
