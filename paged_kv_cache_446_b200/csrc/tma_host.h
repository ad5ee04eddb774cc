// Host helper shared by the kernels that stage tiles with tensor-map TMA.
#pragma once

#include <cuda.h>

namespace pkv {

// Encodes a tiled tensor map over global memory at `base` (128-byte swizzle, no interleave,
// 256-byte L2 promotion, out-of-range elements read as zero). Returns false when the driver entry
// point is unavailable or rejects the description.
bool encode_tiled(CUtensorMap* m, CUtensorMapDataType t, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box);

}  // namespace pkv
