// tmap.h -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled),
// reached through the runtime's driver entry point, so the library does not
// link against libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace wildcat {

// A 3-D tensor [d2][d1][d0] of `elem_bytes`-byte elements, innermost d0
// contiguous, row stride s1 and slab stride s2 in bytes (multiples of 16), a
// box of (b0, b1, 1) elements with 128-byte swizzling (b0 * elem_bytes must
// be 128).  Out-of-range box elements read as zero and are not written.
// Returns false when the driver entry point is missing or the encode fails.
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1);

}  // namespace wildcat
