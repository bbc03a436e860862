// TMA tensor maps (library-internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace spear {

// 2-D row-major tensor [rows][cols] of `elem`-byte elements at `ptr`, copied in
// boxes of box_cols x box_rows; out-of-range elements of a box read as zero.
cudaError_t make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw);
// rank-D tensor: dims innermost first, strides in bytes of dims 1..rank-1.
cudaError_t make_map_nd(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int rank, const uint64_t *dims,
                        const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw);
bool tensor_maps_available();

}  // namespace spear
