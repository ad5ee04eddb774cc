// Host helper shared by the kernels that stage tiles with tensor-map TMA.
#pragma once

#include <cuda.h>

namespace pkv {

// Encodes a tiled tensor map over global memory at `base` (128-byte swizzle, no interleave,
// 256-byte L2 promotion, out-of-range elements read as zero). Returns false when the driver entry
// point is unavailable or rejects the description.
bool encode_tiled(CUtensorMap* m, CUtensorMapDataType t, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box);

// Encodes the map the split-K items read one KV block through: a pool of `rows` rows of 128
// 16-bit elements seen as (64 columns, rows, 2 halves), the halves 128 bytes apart, with a box of
// 64 x 16 rows x 2 halves. One copy then brings both 64-column halves of a block's 16 rows, laid
// out in shared memory as two 2 KiB halves with the 128-byte swizzle -- what two copies of a
// 64 x 16 box over the plain (128 columns, rows) view would bring.
bool encode_block_halves(CUtensorMap* m, CUtensorMapDataType t, const void* base, long long rows);

}  // namespace pkv
