// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled reached through the
// runtime's driver entry-point query, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s2 {

// Tiled bf16 maps with 128-byte swizzle (loads and stores use the same maps).
//   rank 2: rows of `inner` elements, `rows` rows, row pitch `pitch_bytes`; box
//           box_inner x box_rows.
//   rank 3: adds a middle dimension of `mid` entries with pitch `mid_pitch_bytes`; the box
//           takes one entry of it.
// Returns cudaSuccess or cudaErrorInvalidValue (encode failed or entry point missing).
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows);
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                              uint64_t rows, uint64_t mid_pitch_bytes, uint64_t pitch_bytes,
                              uint32_t box_inner, uint32_t box_rows);

// Rank-2 map of any element type and swizzle (e.g. fp32 rows with 128-byte swizzle, or
// bf16 rows of 32 bytes with 32-byte swizzle). Same return values.
cudaError_t make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, CUtensorMapSwizzle swizzle,
                         const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
                         uint32_t box_inner, uint32_t box_rows);

}  // namespace s2
