// 2-D TMA tensor maps (cuTensorMapEncodeTiled) for the kernels' weight and
// activation streams.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace q4k {

// A row-major 2-D tensor of `outer` rows of `inner` elements, rows `row_bytes`
// apart, copied in boxes of box_inner x box_outer elements; elements outside the
// tensor read as zero.
cudaError_t encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                      uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swizzle);

}  // namespace q4k
