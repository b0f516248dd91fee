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

// 3D fp32 tensor [planes][rows][cols] row-major (cols * 4 bytes a multiple of 16), boxes of
// 32 columns x box_rows rows x 1 plane with 128-byte swizzle; used for tiled stores, which
// skip the part of a box outside the tensor.
bool make_tmap_f32_3d_sw128(CUtensorMap* m, void* ptr, int cols, int rows, int planes, int box_rows);

}  // namespace spr
