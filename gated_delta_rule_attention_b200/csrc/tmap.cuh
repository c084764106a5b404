// tmap.cuh -- host helper that encodes 2-D TMA tensor maps.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace la {

// A 2-D row-major tensor of `rows` rows x `inner` elements (row pitch in bytes), copied
// in boxes of box_rows x box_inner elements.  swizzle128 selects the 128-byte swizzle
// (box_inner * elem_bytes must then be <= 128).  Out-of-range box rows read as zero
// and are clipped on store.  Returns false if the driver call is unavailable or
// rejects the arguments (base and pitch must be 16-byte aligned).
bool make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                  uint32_t elem_bytes, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128);

// A 3-D row-major tensor [outer][rows][inner] (pitches in bytes), boxes of
// 1 x box_rows x box_inner.  Rows outside [0, rows) of a box read as zero and are
// clipped on store, so a box never spills into the next outer index.
bool make_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                  uint32_t elem_bytes, uint64_t inner, uint64_t rows, uint64_t outer,
                  uint64_t row_pitch, uint64_t outer_pitch, uint32_t box_inner, uint32_t box_rows,
                  bool swizzle128);

}  // namespace la
