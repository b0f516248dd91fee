// Host-side TMA tensor-map construction (driver entry point fetched through the runtime,
// so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace spr {

// 2D bf16 tensor [rows][cols] row-major (cols * 2 bytes a multiple of 16), boxes of
// box_rows x box_cols elements with 128-byte swizzle (box_cols * 2 == 128). Out-of-range
// rows read as zero. Returns false if the driver rejects the map.
bool make_tmap_bf16_sw128(CUtensorMap* m, const void* ptr, long long rows, int cols, int box_rows, int box_cols);

}  // namespace spr
