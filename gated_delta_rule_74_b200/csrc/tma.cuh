// Host-side TMA tensor maps for the kernels' tile loads (not part of the C ABI).
// The driver's encoder is reached through the runtime's entry-point query, so the
// library links no driver library.  Every map covers this GPU's own memory and is
// used by plain tile loads only (no cluster multicast).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// A 3-D tiled map over a [d2][d1][d0] tensor (d0 contiguous; strides in bytes for
// d1 and d2), with boxes of box0 x 1 x box2 elements.  swizzle128: the 128-byte
// swizzle of the tensor cores' shared-memory operands (box0 * element size must
// then be 128).  Returns false if the driver rejects the map (the caller falls
// back to plain loads).
bool make_tile_map_3d(CUtensorMap* map, bool fp32, const void* base, uint64_t d0, uint64_t d1,
                      uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                      uint32_t box2, bool swizzle128);

}  // namespace kda
