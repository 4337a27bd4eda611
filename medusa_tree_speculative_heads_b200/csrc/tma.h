// Host-side construction of TMA tensor maps (driver entry point fetched at
// run time through the runtime, so the library links no driver stub) and the
// device-side helpers that use them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace medusa {

// bf16 tensor map of rank 2 or 3 with a 128-byte swizzle, zero fill out of
// bounds.  dims[0] is the innermost (contiguous) dimension; strides_bytes[i]
// is the byte stride of dims[i+1]; box[i] the tile extent per dimension
// (box[0] * 2 bytes must be 128 for the swizzle).  Returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                    const uint32_t* box);

}  // namespace medusa
