// tmap.h -- host helper that encodes TMA tensor maps through the driver
// entry point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ret {

// Encode a tiled bf16 tensor map.  dims[0] is the innermost (contiguous)
// dimension; strides_bytes[i] is the byte stride of dimension i + 1.
// Returns false (and records an error message) on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);
// The same for an fp32 tensor.
bool make_tmap_f32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

}  // namespace ret
