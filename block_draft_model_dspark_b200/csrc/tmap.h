// Tensor-map encoding shared by the TMA kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace dspark {
namespace tc {

// Row-major bf16 [rows, cols] matrix (cols * 2 a multiple of 16 bytes, ptr
// 16-byte aligned), box of box_rows x 64 columns, 128-byte swizzle, L2
// promotion of 256 bytes, out-of-range elements read as zero. False when the
// driver entry point is missing or the encoder refuses the shape.
bool make_tmap(CUtensorMap* tm, const void* ptr, int64_t rows, int64_t cols, int box_rows);

}  // namespace tc
}  // namespace dspark
