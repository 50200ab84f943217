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

// Multiprocessor count of the current device (cached per device).
int sm_count();

}  // namespace lsh
