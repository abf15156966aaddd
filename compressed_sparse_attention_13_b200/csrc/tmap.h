// TMA tensor-map encoding shared by the tensor-core kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace csa {

// Tiled map over a tensor of `rank` dimensions (innermost first): dims in
// elements, strides in bytes for dimensions 1.. (rank - 1 of them), box in
// elements.  Rows outside the tensor read as zero.  False if the driver's
// encoder is unavailable or rejects the description.
bool encode_tile_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle);

}  // namespace csa
