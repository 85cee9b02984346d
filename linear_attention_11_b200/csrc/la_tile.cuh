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

// fp32 state tile as the bulk tensor copies of a d x d state lay it out with
// 128-byte swizzle: four boxes of 32 columns, each 128 rows x 128 bytes, the
// 16-byte chunk j of row r at chunk j ^ (r & 7).
constexpr int kStateBoxBytes = kHeadDim * 128;  // 16 KB
constexpr int kStateBytes = 4 * kStateBoxBytes;  // 64 KB

// Row r, columns [16*q, 16*q+16) <-> v[16].
__device__ __forceinline__ void load_state_row16(uint32_t base, int r, int q, uint32_t (&v)[16]) {
  const uint32_t row = base + (uint32_t)((q >> 1) * kStateBoxBytes + r * 128);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int j = (q & 1) * 4 + m;
    ld_shared_v4(row + (uint32_t)((j ^ (r & 7)) * 16), v[4 * m], v[4 * m + 1], v[4 * m + 2],
                 v[4 * m + 3]);
  }
}

__device__ __forceinline__ void store_state_row16(uint32_t base, int r, int q,
                                                  const uint32_t (&v)[16]) {
  const uint32_t row = base + (uint32_t)((q >> 1) * kStateBoxBytes + r * 128);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int j = (q & 1) * 4 + m;
    st_shared_v4(row + (uint32_t)((j ^ (r & 7)) * 16), v[4 * m], v[4 * m + 1], v[4 * m + 2],
                 v[4 * m + 3]);
  }
}

// As store_row32_sw128 for the 16 columns [16*q, 16*q+16) of row r.
__device__ __forceinline__ void store_row16_sw128(uint32_t base, int r, int q,
                                                  const uint32_t (&v)[16]) {
  const uint32_t row = base + (uint32_t)((q >> 2) * kHalf + r * 128);
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const uint32_t chunk = (uint32_t)(((q & 3) * 2 + m) ^ (r & 7));
    st_shared_v4(row + chunk * 16,
                 pack_bf16x2(__uint_as_float(v[8 * m + 0]), __uint_as_float(v[8 * m + 1])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 2]), __uint_as_float(v[8 * m + 3])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 4]), __uint_as_float(v[8 * m + 5])),
                 pack_bf16x2(__uint_as_float(v[8 * m + 6]), __uint_as_float(v[8 * m + 7])));
  }
}

// Shared memory of the main kernel: a ring of Q tiles, a separate ring of K/V
// tiles, the bf16 state copy, and (at T = 64) a dedicated output staging tile.
// Q(i) is released once Q(i) S has been issued and completed; K/V(i) once the
// state update of tile i has; so copies of later tiles start early and more
// bytes stay in flight.  At T = 128 there is no room for a separate staging
// tile and the output goes through the Q slot (released after its store has
// read it).
// With kStage (persistent kernel, one span per sequence) a 64 KB fp32 state
// tile follows, through which entering states arrive and final states leave
// by bulk tensor copies.
template <int T, int QST, int KVST, bool DedicatedO = (T == 64), bool Stage = false,
          bool HalfKV = false>
struct MainLayout {
  static constexpr bool kDedicatedO = DedicatedO;
  static constexpr bool kStage = Stage;
  static constexpr int kKBytes = T * kHeadDim * 2;
  // bytes per K/V slot: a K and a V tile, or one of them (HalfKV: K and V
  // tiles take separate slots of one ring)
  static constexpr int kKVBytes = HalfKV ? kKBytes : 2 * kKBytes;
  static constexpr int kKVOff = QST * kQBytes;
  static constexpr int kSOff = kKVOff + KVST * kKVBytes;
  static constexpr int kOOff = kSOff + kSBytes;
  static constexpr int kStOff = kOOff + (kDedicatedO ? kQBytes : 0);
  static constexpr int kBarOff = kStOff + (kStage ? kStateBytes : 0);
  // q_full[QST], q_empty[QST], kv_full[KVST], kv_empty[KVST], a_full[2],
  // p_full[2], o_full[2], o_empty[2], s_full, sb_full, mma_done, store_ready,
  // ostage_free, st_full, st_empty, stage_done
  static constexpr int kNumBars = 2 * QST + 2 * KVST + 16;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024
};

}  // namespace la
