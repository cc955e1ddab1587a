// Host helper: 2-D tiled TMA tensor maps (cuTensorMapEncodeTiled), reached
// through the runtime's driver entry point so the library does not link the
// driver library itself.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace tq {

// A row-major matrix of `rows` rows, `cols` elements per row (16-bit
// elements), row stride `row_bytes` (a multiple of 16), read in boxes of
// box_cols x box_rows elements with no swizzle; reads outside the matrix give
// zeros.  Returns TQ_OK or TQ_ECUDA (message set).
int make_tmap_2d_u16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                     uint32_t box_cols, uint32_t box_rows, bool swizzle128 = false);
// (swizzle128: boxes of 64 elements x box_rows written with 128-byte swizzle - row r of a box
// at r * 128 bytes with its 16-byte chunks XOR-ed by r % 8 - into a 1024-byte aligned buffer.)

}  // namespace tq
