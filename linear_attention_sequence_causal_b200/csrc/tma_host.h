// Host-side creation of TMA tensor maps through the driver entry point (no libcuda link).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace based {

// 3-D bf16 tensor [z][y][x] (x contiguous, rows of x_bytes), tiles of box_x x box_y x 1
// with 128-byte swizzle and zero fill outside the tensor. Returns false on failure.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z,
                       uint32_t box_x, uint32_t box_y);

// The same with the 32-, 64- or 128-byte swizzle (box_x * 2 bytes must not exceed it).
bool make_tmap_bf16_3d_swizzle(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z,
                               uint32_t box_x, uint32_t box_y, int swizzle_bytes);

}  // namespace based
