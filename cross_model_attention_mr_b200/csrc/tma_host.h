// Host-side creation of TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mr {

// 2D bf16 tensor map over a row-major [rows][cols] array with `row_bytes` between rows, a box of
// box_cols x box_rows elements and 128-byte swizzle (box_cols * 2 must be <= 128).
// Returns false if the driver entry point is unavailable or rejects the map.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                       uint32_t box_cols, uint32_t box_rows);

}  // namespace mr
