// Host creation of TMA tensor maps (cuTensorMapEncodeTiled, reached through the runtime's driver
// entry-point query so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sac {

// 2D bf16 tensor [rows, cols] with the given row stride (bytes, multiple of 16), box
// [box_rows, box_cols] (box_cols * 2 bytes <= 128 for the 128-byte swizzle), 128-byte swizzle.
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint64_t row_stride_bytes, uint32_t box_rows, uint32_t box_cols);

}  // namespace sac
