// Host-side TMA tensor-map encoding (driver entry point fetched at run time,
// so the library links only against the CUDA runtime).
#pragma once
#include <cuda.h>
#include <cstdint>

namespace pl {

// Encode a tiled fp16 tensor map with 128-byte swizzle and zero OOB fill.
// dims/box are innermost-first; strides_bytes has rank-1 entries (dims 1..).
// Returns 0 on success, a CUresult (or -1 when the entry point is missing).
int encode_f16_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);
// Same for fp16 or fp32 elements and a 32-, 64- or 128-byte swizzle.
int encode_tmap(CUtensorMap* m, bool f32, const void* base, int rank, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

}  // namespace pl
