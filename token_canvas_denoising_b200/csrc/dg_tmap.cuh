// TMA tensor-map helpers (host side).
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace dg {

// Encode a bf16 tiled tensor map. dims[0] is the innermost (contiguous)
// extent in elements; strides_bytes has rank-1 entries (bytes between
// consecutive indices of dims[1..]), each a multiple of 16; box[i] <= 256 and
// box[0] * 2 bytes <= 128 when swizzle128 is set. Returns false (with the last
// error message set) on failure.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// The same for an 8-bit element type (e4m3 codes), encoded as unsigned bytes:
// dims[0] and box[0] count bytes.
bool encode_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// The calling thread's current CUDA context (driver handle), or false when
// none can be read. Used to key per-context caches of device addresses.
bool current_context(void** ctx);

}  // namespace dg
