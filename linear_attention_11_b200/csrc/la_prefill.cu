// la_prefill.cu -- tensor-core kernels of the bf16 prefill (sm_100a).
//
// Sources, cited by page title and section:
//   [VGX]  "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
//          "Lightning Attention：长上下文为什么突然变得便宜了", the causal
//          chunkwise sketch: per block, inter = Q_b S, intra =
//          tril(Q_b K_b^T) V_b, O_b = inter + intra, then S += K_b^T V_b.
//   [MX01] "MiniMax-01与Lightning Attention": section 1.1 (grouped kv heads),
//          section 2.3 (tiles processed against a running state).
//
// Two kernels:
//   span_states_kernel   one CTA per (batch, kv head, span): the span's
//                        K^T V = sum of K_c^T V_c over its chunks (fp32).
//   prefill_main_kernel  one CTA per (batch, kv head, head subset, span): the
//                        chunk loop of [VGX] over the span, starting from the
//                        state that enters it (prepared by the scan kernel).
//
// Main-kernel tile: 128 rows = HPT query heads of one kv group x T tokens
// (T = 64, HPT = 2 or T = 128, HPT = 1); d = 128.  Per tile c:
//   A   = Q_c K_c^T           tcgen05 M=128 N=T  K=128  (SS) -> TMEM
//   P   = bf16(tril(A))       TMEM -> registers -> TMEM (math warps)
//   O   = Q_c bf16(S)         tcgen05 M=128 N=128 K=128 (SS) -> TMEM
//   O  += P V_c               tcgen05 M=128 N=128 K=T   (A from TMEM)
//   S  += K_c^T V_c           tcgen05 M=128 N=128 K=T   (SS, both MN-major)
//   O  -> bf16 -> smem -> bulk tensor store
// The masked product is "tril" including the diagonal (torch's default, as in
// the [VGX] sketch).  Q, K, V arrive by bulk tensor copies (TMA) with 128-byte
// swizzle; rows beyond N read as zero and stores beyond N are clipped, which
// handles the short last chunk.
//
// Warp roles (192 threads): warp 0 issues the copies, warp 1 owns the tensor
// memory and issues the MMAs, warps 2-5 (128 threads, one per TMEM lane) do
// the mask, the state conversion and the output epilogue.
//
// Tensor memory (512 columns, fp32 unless noted):
//   [  0,128)  O buffer 0     (the score tile A of even tiles lives here first)
//   [128,256)  O buffer 1     (A of odd tiles)
//   [256,256+T) P buffers 0/1 (bf16 pairs, T/2 columns each)
//   [384,512)  S, the running d x d state (lane = key feature, column = value feature)
#include <cuda.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_ptx.cuh"

namespace la {
namespace {

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

struct MainParams {
  const float* ws;
  unsigned* status;
  int Hq, Hkv, G, nsub, nspan, tiles_total;
};

template <int T, int STAGES>
struct MainLayout {
  static constexpr int kKBytes = T * kHeadDim * 2;
  static constexpr int kStageBytes = kQBytes + 2 * kKBytes;
  static constexpr int kSOff = STAGES * kStageBytes;
  static constexpr int kBarOff = kSOff + kSBytes;
  static constexpr int kNumBars = 2 * STAGES + 9;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024
};

template <int T, int STAGES>
__global__ void __launch_bounds__(192, 1)
    prefill_main_kernel(const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_o, const MainParams p) {
  using L = MainLayout<T, STAGES>;
  constexpr int HPT = kTileRows / T;
  constexpr uint32_t kStageTx = L::kStageBytes;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, T, 0, 0);
  constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, 1, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* a_full = bars + 2 * STAGES + 0;
  uint64_t* p_full = bars + 2 * STAGES + 1;
  uint64_t* o_full = bars + 2 * STAGES + 2;
  uint64_t* o_empty = bars + 2 * STAGES + 3;  // two barriers
  uint64_t* s_full = bars + 2 * STAGES + 5;
  uint64_t* sb_full = bars + 2 * STAGES + 6;
  uint64_t* mma_done = bars + 2 * STAGES + 7;
  uint64_t* store_ready = bars + 2 * STAGES + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);

  const uint32_t sQ0 = base;
  const uint32_t sS = base + L::kSOff;
  auto sQ = [&](int s) { return sQ0 + (uint32_t)(s * L::kStageBytes); };
  auto sK = [&](int s) { return sQ(s) + (uint32_t)kQBytes; };
  auto sV = [&](int s) { return sQ(s) + (uint32_t)(kQBytes + L::kKBytes); };

  // ---- work item
  int idx = blockIdx.x;
  const int hs = idx % p.nsub;
  idx /= p.nsub;
  const int j = idx % p.nspan;
  const int bg = idx / p.nspan;  // b * Hkv + g
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int tile_begin = (int)(((int64_t)j * p.tiles_total) / p.nspan);
  const int tile_end = (int)(((int64_t)(j + 1) * p.tiles_total) / p.nspan);
  const int ntiles = tile_end - tile_begin;
  const int head0 = g * p.G + hs * HPT;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 2);  // MMA commit + output-store release
    }
    mbar_init(a_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(&o_empty[0], 128);
    mbar_init(&o_empty[1], 128);
    mbar_init(s_full, 1);
    mbar_init(sb_full, 128);
    mbar_init(mma_done, 1);
    mbar_init(store_ready, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      prefetch_tmap(&map_o);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();  // re-read by the other head subsets
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, p.status, abort_flag))
          break;
        mbar_arrive_expect_tx(&full[s], kStageTx);
        const int c1 = (tile_begin + i) * T;
        uint8_t* q_dst = sm + (sQ(s) - base);
#pragma unroll
        for (int hh = 0; hh < HPT; ++hh) {
          tma_load_3d(q_dst + hh * T * 128, &map_q, &full[s], 0, c1, b * p.Hq + head0 + hh, pol_q);
          tma_load_3d(q_dst + kHalf + hh * T * 128, &map_q, &full[s], 64, c1,
                      b * p.Hq + head0 + hh, pol_q);
        }
        uint8_t* k_dst = sm + (sK(s) - base);
        uint8_t* v_dst = sm + (sV(s) - base);
        tma_load_3d(k_dst, &map_k, &full[s], 0, c1, bg, pol_kv);
        tma_load_3d(k_dst + T * 128, &map_k, &full[s], 64, c1, bg, pol_kv);
        tma_load_3d(v_dst, &map_v, &full[s], 0, c1, bg, pol_kv);
        tma_load_3d(v_dst + T * 128, &map_v, &full[s], 64, c1, bg, pol_kv);
        issued = i + 1;
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        const uint32_t ob = (uint32_t)(i & 1);
        const uint32_t ocol = ob * 128;
        const uint32_t pcol = 256 + ob * (T / 2);
        if (!mbar_wait(&full[s], (i / STAGES) & 1, p.status, abort_flag)) break;
        if (i >= 2 && !mbar_wait(&o_empty[ob], ((i >> 1) - 1) & 1, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t q_addr = sQ(s), k_addr = sK(s), v_addr = sV(s);
        // A = Q K^T  (both K-major; 16-element k-steps inside 128-byte rows)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint64_t da = smem_desc_sw128(q_addr + (kk >> 2) * kHalf + koff, 16, 1024);
          const uint64_t db = smem_desc_sw128(k_addr + (kk >> 2) * (T * 128) + koff, 16, 1024);
          mma_ss(tmem + ocol, da, db, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(a_full);
        if (!mbar_wait(p_full, i & 1, p.status, abort_flag)) break;
        if (!mbar_wait(sb_full, i & 1, p.status, abort_flag)) break;
        tc_fence_after();
        // O = Q S   (S: MN-major, 16 key rows of 128 B per k-step)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da =
              smem_desc_sw128(q_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t db = smem_desc_sw128(sS + kk * 2048, kHalf, 1024);
          mma_ss(tmem + ocol, da, db, IDESC_QS, kk > 0 ? 1u : 0u);
        }
        // O += P V  (P from TMEM, 8 columns = 16 bf16 per k-step; V MN-major)
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
          mma_ts(tmem + ocol, tmem + pcol + kk * 8, db, IDESC_PV, 1u);
        }
        mma_commit(o_full);
        // S += K^T V  (K as MN-major A, V as MN-major B)
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint64_t da = smem_desc_sw128(k_addr + kk * 2048, T * 128, 1024);
          const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
          mma_ss(tmem + kColS, da, db, IDESC_KV, 1u);
        }
        mma_commit(s_full);
        mma_commit(&empty[s]);
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = tile row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int t_in = r % T;
    const int mt = threadIdx.x - 64;
    bool ok = true;

    // Entering state of this span: fp32 rows -> TMEM S, bf16 copy -> smem.
    {
      const float4* src = reinterpret_cast<const float4*>(
          p.ws + ((size_t)bg * p.nspan + j) * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim);
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 f = __ldg(src + blk * 8 + i);
          v[4 * i + 0] = __float_as_uint(f.x);
          v[4 * i + 1] = __float_as_uint(f.y);
          v[4 * i + 2] = __float_as_uint(f.z);
          v[4 * i + 3] = __float_as_uint(f.w);
        }
        tmem_st32(tmem + lane_base + kColS + blk * 32, v);
        store_row32_sw128(sS, r, blk, v);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sb_full);
    }

    for (int i = 0; i < ntiles && ok; ++i) {
      const int s = i % STAGES;
      const uint32_t ob = (uint32_t)(i & 1);
      const uint32_t ocol = ob * 128;
      const uint32_t pcol = 256 + ob * (T / 2);

      // ---- causal mask of the score tile -> P (bf16 in TMEM)
      if (!warp_wait(a_full, i & 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int blk = 0; blk < T / 32; ++blk) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_base + ocol + blk * 32, a);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int s0 = blk * 32 + 2 * m;
          const float f0 = (s0 <= t_in) ? __uint_as_float(a[2 * m]) : 0.0f;
          const float f1 = (s0 + 1 <= t_in) ? __uint_as_float(a[2 * m + 1]) : 0.0f;
          pk[m] = pack_bf16x2(f0, f1);
        }
        tmem_st16(tmem + lane_base + pcol + blk * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);

      // ---- the previous tile's output store has read its smem: free that stage
      if (mt == 0 && i > 0) {
        bulk_wait_group_read<0>();
        mbar_arrive(&empty[(i - 1) % STAGES]);
      }

      // ---- bf16 copy of the updated state for the next tile's Q S
      if (i + 1 < ntiles) {
        if (!warp_wait(s_full, i & 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + kColS + blk * 32, v);
          tmem_wait_ld();
          store_row32_sw128(sS, r, blk, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sb_full);
      }

      // ---- output epilogue: TMEM -> bf16 -> this stage's Q buffer -> store
      if (!warp_wait(o_full, i & 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t stage_q = sQ(s);
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + ocol + blk * 32, v);
        tmem_wait_ld();
        store_row32_sw128(stage_q, r, blk, v);
      }
      tc_fence_before();
      mbar_arrive(&o_empty[ob]);
      fence_proxy_async_smem();
      mbar_arrive(store_ready);
      if (warp == 2) {
        // every math thread has written its row of the staging tile
        if (!warp_wait(store_ready, i & 1, p.status, abort_flag)) { ok = false; break; }
      }
      if (mt == 0) {
        const int c1 = (tile_begin + i) * T;
        const uint8_t* src = sm + (stage_q - base);
#pragma unroll
        for (int hh = 0; hh < HPT; ++hh) {
          tma_store_3d(&map_o, src + hh * T * 128, 0, c1, b * p.Hq + head0 + hh);
          tma_store_3d(&map_o, src + kHalf + hh * T * 128, 64, c1, b * p.Hq + head0 + hh);
        }
        bulk_commit_group();
      }
    }
    if (mt == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Span states: ws[bg][j] = sum over the span's tiles of K_c^T V_c.
struct SpanParams {
  float* ws;
  unsigned* status;
  int nspan, tiles_total;
};

template <int T, int STAGES>
struct SpanLayout {
  static constexpr int kKBytes = T * kHeadDim * 2;
  static constexpr int kStageBytes = 2 * kKBytes;
  static constexpr int kBarOff = STAGES * kStageBytes;
  static constexpr int kMiscOff = kBarOff + (2 * STAGES + 1) * 8;
  static constexpr int kBytes = kMiscOff + 16 + 1024;
};

template <int T, int STAGES>
__global__ void __launch_bounds__(192, 1)
    span_states_kernel(const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, const SpanParams p) {
  using L = SpanLayout<T, STAGES>;
  constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, 1, 1);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* done = full + 2 * STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);

  const int j = blockIdx.x % p.nspan;
  const int bg = blockIdx.x / p.nspan;
  const int tile_begin = (int)(((int64_t)j * p.tiles_total) / p.nspan);
  const int tile_end = (int)(((int64_t)(j + 1) * p.tiles_total) / p.nspan);
  const int ntiles = tile_end - tile_begin;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto sK = [&](int s) { return base + (uint32_t)(s * L::kStageBytes); };
  auto sV = [&](int s) { return sK(s) + (uint32_t)L::kKBytes; };

  if (warp == 0) {
    if (elect_one()) {
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      const uint64_t pol = policy_evict_normal();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, p.status, abort_flag))
          break;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        const int c1 = (tile_begin + i) * T;
        uint8_t* k_dst = sm + (sK(s) - base);
        uint8_t* v_dst = sm + (sV(s) - base);
        tma_load_3d(k_dst, &map_k, &full[s], 0, c1, bg, pol);
        tma_load_3d(k_dst + T * 128, &map_k, &full[s], 64, c1, bg, pol);
        tma_load_3d(v_dst, &map_v, &full[s], 0, c1, bg, pol);
        tma_load_3d(v_dst + T * 128, &map_v, &full[s], 64, c1, bg, pol);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], (i / STAGES) & 1, p.status, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint64_t da = smem_desc_sw128(sK(s) + kk * 2048, T * 128, 1024);
          const uint64_t db = smem_desc_sw128(sV(s) + kk * 2048, T * 128, 1024);
          mma_ss(tmem, da, db, IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(done);
      mbar_wait_drain(done, 0);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float4* dst =
        reinterpret_cast<float4*>(p.ws + ((size_t)bg * p.nspan + j) * (kHeadDim * kHeadDim) +
                                  (size_t)r * kHeadDim);
    if (ntiles == 0) {
#pragma unroll 4
      for (int i = 0; i < 32; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else if (warp_wait(done, 0, p.status, abort_flag)) {
      tc_fence_after();
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + blk * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[blk * 8 + i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]),
                                         __uint_as_float(v[4 * i + 3]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_span_states(const PrefillGeometry& g, const CUtensorMap& k,
                               const CUtensorMap& v, float* ws, unsigned* status,
                               cudaStream_t stream) {
  SpanParams p{ws, status, g.nspan, g.tiles_total};
  const dim3 grid((unsigned)(g.B * g.Hkv * g.nspan));
  cudaError_t e;
  if (g.tile == 64) {
    using L = SpanLayout<64, 4>;
    if ((e = set_smem(span_states_kernel<64, 4>, L::kBytes)) != cudaSuccess) return e;
    span_states_kernel<64, 4><<<grid, 192, L::kBytes, stream>>>(k, v, p);
  } else {
    using L = SpanLayout<128, 3>;
    if ((e = set_smem(span_states_kernel<128, 3>, L::kBytes)) != cudaSuccess) return e;
    span_states_kernel<128, 3><<<grid, 192, L::kBytes, stream>>>(k, v, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_prefill_main(const PrefillGeometry& g, const PrefillMaps& maps,
                                const float* ws, unsigned* status, cudaStream_t stream) {
  const int nsub = g.G / g.heads_per_tile;
  MainParams p{ws, status, g.Hq, g.Hkv, g.G, nsub, g.nspan, g.tiles_total};
  const dim3 grid((unsigned)(g.B * g.Hkv * g.nspan * nsub));
  cudaError_t e;
  if (g.tile == 64) {
    using L = MainLayout<64, 3>;
    if ((e = set_smem(prefill_main_kernel<64, 3>, L::kBytes)) != cudaSuccess) return e;
    prefill_main_kernel<64, 3><<<grid, 192, L::kBytes, stream>>>(maps.q, maps.k, maps.v, maps.o, p);
  } else {
    using L = MainLayout<128, 2>;
    if ((e = set_smem(prefill_main_kernel<128, 2>, L::kBytes)) != cudaSuccess) return e;
    prefill_main_kernel<128, 2><<<grid, 192, L::kBytes, stream>>>(maps.q, maps.k, maps.v, maps.o,
                                                                  p);
  }
  return cudaGetLastError();
}

}  // namespace la
