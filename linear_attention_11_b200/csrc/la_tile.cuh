// la_tile.cuh -- tile layout constants and helpers shared by the prefill
// kernels (device side).
#pragma once

#include "la_internal.h"
#include "la_ptx.cuh"

namespace la {

constexpr int kQBytes = kTileRows * kHeadDim * 2;  // 32 KB: 128 rows x 128 bf16
constexpr int kHalf = kTileRows * 128;             // one 64-column block of a 128-row tile
constexpr int kSBytes = kHeadDim * kHeadDim * 2;   // bf16 copy of the state
constexpr uint32_t kColS = 384;

// Store 32 fp32 values (bits) of row r, columns [32*blk, 32*blk+32), as bf16
// into a 128-row tile laid out as two 64-column blocks of 128-byte swizzled
// rows (the layout the bulk tensor copies and the MMA descriptors both use).
__device__ __forceinline__ void store_row32_sw128(uint32_t base, int r, int blk,
                                                  const uint32_t (&v)[32]) {
  const uint32_t row = base + (uint32_t)((blk >> 1) * kHalf + r * 128);
  const int c0 = (blk & 1) * 4;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t chunk = (uint32_t)((c0 + m) ^ (r & 7));
    st_shared_v4(row + chunk * 16,
                 pack_bf16x2(__uint_as_float(v[8 * m + 0]), __uint_as_float(v[8 * m + 1])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 2]), __uint_as_float(v[8 * m + 3])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 4]), __uint_as_float(v[8 * m + 5])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 6]), __uint_as_float(v[8 * m + 7])));
  }
}


}  // namespace la
