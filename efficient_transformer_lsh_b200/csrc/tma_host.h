// Host helpers: TMA tensor-map encoding (driver entry point, no -lcuda) and
// the SM count of the current device.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsh {

// Encodes a 2D bf16/f16 tensor map with 128-byte swizzle: `inner` elements
// per row (contiguous), `rows` rows `row_bytes` apart, box of box_inner x
// box_rows. Out-of-range elements of a box read as zero. Returns false if
// the driver rejects it (alignment, sizes).
bool encode_tmap_2d_16bit(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                          uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows);

// Encodes a 4D bf16 tensor map with 128-byte swizzle: dims[0] elements
// innermost (contiguous), strides[i] = bytes between steps of dimension i+1,
// box of box[0..3] elements. Out-of-range elements of a box read as zero.
// Returns false if the driver rejects it.
bool encode_tmap_4d_16bit(CUtensorMap* map, const void* base, const uint64_t dims[4],
                          const uint64_t strides[3], const uint32_t box[4]);

// Multiprocessor count of the current device (cached per device).
int sm_count();

}  // namespace lsh
