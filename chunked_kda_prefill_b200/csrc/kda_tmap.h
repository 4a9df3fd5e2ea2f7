// kda_tmap.h -- host helper: encode a 3-D bf16 TMA tensor map with 128-byte swizzle.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace kda {

// dims = {d0 (innermost, elements), d1, d2}; strides_bytes = {stride of d1, stride of d2};
// box = {b0, b1, b2} elements.  Out-of-bounds elements of a box read as zero.
bool encode_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3],
                    const uint64_t strides_bytes[2], const uint32_t box[3]);

}  // namespace kda
