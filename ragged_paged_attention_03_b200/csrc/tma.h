// tma.h -- host-side creation of TMA tensor maps.
//
// cuTensorMapEncodeTiled is a driver-API function; it is resolved at run time
// through cudaGetDriverEntryPoint so that the library does not link against
// libcuda and still loads on machines without a GPU driver.
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace rpa {

// A bf16 tensor map of rank 3 (innermost dimension first).  dims[i]
// elements, strides_bytes[i] for dimensions 1 and 2, box[i] elements per
// copy, 128-byte swizzle when swizzle128 is set.  Returns false when the
// driver entry point is unavailable or rejects the description.
bool make_tmap_bf16_3d(CUtensorMap *map, const void *base, const uint64_t dims[3],
                       const uint64_t strides_bytes[2], const uint32_t box[3], bool swizzle128);

}  // namespace rpa
