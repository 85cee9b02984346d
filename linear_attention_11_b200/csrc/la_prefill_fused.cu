// la_prefill_fused.cu -- the bf16 prefill as one persistent kernel (sm_100a).
//
// Same arithmetic as la_prefill.cu (the causal chunkwise form of
// "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
// "Lightning Attention：长上下文为什么突然变得便宜了": per chunk
// O_c = Q_c S + tril(Q_c K_c^T) V_c, then S += K_c^T V_c), scheduled so that
// K and V cross HBM about once.
//
// The sequence of every (batch, kv head) is cut into `nspan` spans.  Work items
// come in rounds, one round per span index j:
//   A(bg, j)      span-state item: Agg_j = sum over span j of K_c^T V_c, then
//                 the chained prefix P_{j+1} = P_j + Agg_j ("the state entering
//                 span j+1"), published with a GPU-scope release flag; the last
//                 span writes the final state instead.
//   M(bg, hs, j)  chunk-loop item for HPT query heads: waits for P_j, then runs
//                 the chunk loop of span j from it.
// Round j holds every A(., j) followed by every M(., ., j).  M(bg, ., j) reads
// the same K, V tiles A(bg, j) has just read, so the second read is served by
// L2 (A loads K, V with an evict-last hint; Q and O stream with evict-first).
//
// Scheduling: one CTA per SM; each CTA's copy warp takes item indices from a
// global atomic counter and hands them to the MMA warp and the math warps
// through a two-slot queue in shared memory.  An item only ever waits for
// items with smaller indices, which were taken earlier by running CTAs, so
// the smallest unfinished item can always proceed (no deadlock whatever the
// residency).  Every wait -- mbarrier or global flag -- is bounded.
//
// Roles and tensor memory as in la_prefill.cu:
//   warp 0  copies (TMA) and the item queue
//   warp 1  tensor memory owner, MMA issue
//   warps 2-5  mask, state conversion, output epilogue, span-state prefix
//   TMEM: [0,256) two O buffers (score tiles alias them), [256,256+T) two P
//   buffers, [384,512) the state S (also the span aggregate of A items).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"
#include "la_ptx.cuh"
#include "la_tile.cuh"

namespace la {
namespace {

constexpr int kQueue = 2;  // item queue depth

struct FusedParams {
  float* prefix;       // [B*Hkv][nspan][128*128]: state entering each span
  unsigned* ready;     // [B*Hkv*nspan]: prefix[bg][j] published
  unsigned* counter;   // next item index
  float* S;            // nullable: initial state in, final state out
  unsigned* status;
  int Hq, Hkv, G, nsub, nspan, tiles_total;
  int units_a;         // B*Hkv
  int units_m;         // B*Hkv*nsub
  int total_items;     // nspan * (units_a + units_m)
};

struct Item {
  int is_a, bg, hs, j, tile_begin, ntiles;
};

__device__ __forceinline__ Item decode_item(const FusedParams& p, int idx) {
  Item it;
  const int per_round = p.units_a + p.units_m;
  const int r = idx / per_round, x = idx % per_round;
  it.j = r;
  if (x < p.units_a) {
    it.is_a = 1;
    it.bg = x;
    it.hs = 0;
  } else {
    const int y = x - p.units_a;
    it.is_a = 0;
    it.bg = y / p.nsub;
    it.hs = y % p.nsub;
  }
  it.tile_begin = (int)(((int64_t)r * p.tiles_total) / p.nspan);
  it.ntiles = (int)(((int64_t)(r + 1) * p.tiles_total) / p.nspan) - it.tile_begin;
  return it;
}

template <int T, int STAGES>
struct FusedLayout {
  static constexpr int kKBytes = T * kHeadDim * 2;
  static constexpr int kStageBytes = kQBytes + 2 * kKBytes;
  static constexpr int kSOff = STAGES * kStageBytes;
  static constexpr int kBarOff = kSOff + kSBytes;
  // full[S], empty[S], a_full, p_full, o_full, o_empty[2], s_full, sb_full,
  // mma_done, store_ready, a_done, s_free, flag_bar, item_full[Q], item_empty[Q]
  static constexpr int kNumBars = 2 * STAGES + 12 + 2 * kQueue;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 32 + 1024;
};

template <int T, int STAGES>
__global__ void __launch_bounds__(192, 1)
    prefill_fused_kernel(const __grid_constant__ CUtensorMap map_q,
                         const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v,
                         const __grid_constant__ CUtensorMap map_o, const FusedParams p) {
  using L = FusedLayout<T, STAGES>;
  constexpr int HPT = kTileRows / T;
  constexpr uint32_t kTxM = L::kStageBytes;       // Q + K + V
  constexpr uint32_t kTxA = 2 * L::kKBytes;       // K + V
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, T, 0, 0);
  constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, 1, 1);
  constexpr int D2 = kHeadDim * kHeadDim;

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
  uint64_t* o_empty = bars + 2 * STAGES + 3;  // two
  uint64_t* s_full = bars + 2 * STAGES + 5;
  uint64_t* sb_full = bars + 2 * STAGES + 6;
  uint64_t* mma_done = bars + 2 * STAGES + 7;
  uint64_t* store_ready = bars + 2 * STAGES + 8;
  uint64_t* a_done = bars + 2 * STAGES + 9;
  uint64_t* s_free = bars + 2 * STAGES + 10;
  uint64_t* flag_bar = bars + 2 * STAGES + 11;
  uint64_t* item_full = bars + 2 * STAGES + 12;
  uint64_t* item_empty = item_full + kQueue;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);
  volatile int* items = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 8);  // [kQueue]

  const uint32_t sS = base + L::kSOff;
  auto sQ = [&](int s) { return base + (uint32_t)(s * L::kStageBytes); };
  auto sK = [&](int s) { return sQ(s) + (uint32_t)kQBytes; };
  auto sV = [&](int s) { return sQ(s) + (uint32_t)(kQBytes + L::kKBytes); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 2);  // MMA commit + (output-store release | MMA arrive)
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
    mbar_init(a_done, 1);
    mbar_init(s_free, 128);
    mbar_init(flag_bar, 128);
    for (int i = 0; i < kQueue; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 1 + 128);  // MMA thread + every math thread
    }
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
    // ------------------------------------------------------------ copies + queue
    if (elect_one()) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      prefetch_tmap(&map_o);
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol_kv_m = policy_evict_normal();
      int lt = 0;  // tiles loaded by this CTA
      for (int k = 0;; ++k) {
        const int slot = k % kQueue;
        if (k >= kQueue &&
            !mbar_wait(&item_empty[slot], ((k / kQueue) - 1) & 1, p.status, abort_flag))
          break;
        const int idx = (int)atomicAdd(p.counter, 1u);
        const bool done = idx >= p.total_items;
        items[slot] = done ? -1 : idx;
        mbar_arrive(&item_full[slot]);
        if (done) break;
        const Item it = decode_item(p, idx);
        const int b = it.bg / p.Hkv, g = it.bg % p.Hkv;
        const int head0 = g * p.G + it.hs * HPT;
        bool ok = true;
        for (int i = 0; i < it.ntiles; ++i, ++lt) {
          const int s = lt % STAGES;
          if (lt >= STAGES &&
              !mbar_wait(&empty[s], ((lt / STAGES) - 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          const int c1 = (it.tile_begin + i) * T;
          uint8_t* k_dst = sm + (sK(s) - base);
          uint8_t* v_dst = sm + (sV(s) - base);
          if (it.is_a) {
            mbar_arrive_expect_tx(&full[s], kTxA);
            tma_load_3d(k_dst, &map_k, &full[s], 0, c1, it.bg, pol_keep);
            tma_load_3d(k_dst + T * 128, &map_k, &full[s], 64, c1, it.bg, pol_keep);
            tma_load_3d(v_dst, &map_v, &full[s], 0, c1, it.bg, pol_keep);
            tma_load_3d(v_dst + T * 128, &map_v, &full[s], 64, c1, it.bg, pol_keep);
          } else {
            mbar_arrive_expect_tx(&full[s], kTxM);
            uint8_t* q_dst = sm + (sQ(s) - base);
#pragma unroll
            for (int hh = 0; hh < HPT; ++hh) {
              tma_load_3d(q_dst + hh * T * 128, &map_q, &full[s], 0, c1, b * p.Hq + head0 + hh,
                          pol_stream);
              tma_load_3d(q_dst + kHalf + hh * T * 128, &map_q, &full[s], 64, c1,
                          b * p.Hq + head0 + hh, pol_stream);
            }
            tma_load_3d(k_dst, &map_k, &full[s], 0, c1, it.bg, pol_kv_m);
            tma_load_3d(k_dst + T * 128, &map_k, &full[s], 64, c1, it.bg, pol_kv_m);
            tma_load_3d(v_dst, &map_v, &full[s], 0, c1, it.bg, pol_kv_m);
            tma_load_3d(v_dst + T * 128, &map_v, &full[s], 64, c1, it.bg, pol_kv_m);
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        for (int i = (lt > STAGES ? lt - STAGES : 0); i < lt; ++i)
          mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (elect_one()) {
      int lt = 0, mtc = 0;
      for (int k = 0;; ++k) {
        const int slot = k % kQueue;
        if (!mbar_wait(&item_full[slot], (k / kQueue) & 1, p.status, abort_flag)) break;
        const int idx = items[slot];
        mbar_arrive(&item_empty[slot]);
        if (idx < 0) break;
        const Item it = decode_item(p, idx);
        bool ok = true;
        if (it.is_a) {
          // the state columns are free once the math warps are done with item k-1
          if (k >= 1 && !mbar_wait(s_free, (k - 1) & 1, p.status, abort_flag)) break;
          for (int i = 0; i < it.ntiles; ++i, ++lt) {
            const int s = lt % STAGES;
            if (!mbar_wait(&full[s], (lt / STAGES) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {
              const uint64_t da = smem_desc_sw128(sK(s) + kk * 2048, T * 128, 1024);
              const uint64_t db = smem_desc_sw128(sV(s) + kk * 2048, T * 128, 1024);
              mma_ss(tmem + kColS, da, db, IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
            mbar_arrive(&empty[s]);
          }
          if (!ok) break;
          mma_commit(a_done);
        } else {
          for (int i = 0; i < it.ntiles; ++i, ++lt, ++mtc) {
            const int s = lt % STAGES;
            const uint32_t ob = (uint32_t)(mtc & 1);
            const uint32_t ocol = ob * 128;
            const uint32_t pcol = 256 + ob * (T / 2);
            if (!mbar_wait(&full[s], (lt / STAGES) & 1, p.status, abort_flag)) { ok = false; break; }
            if (mtc >= 2 &&
                !mbar_wait(&o_empty[ob], ((mtc >> 1) - 1) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = sQ(s), k_addr = sK(s), v_addr = sV(s);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // A = Q K^T
              const uint32_t koff = (uint32_t)((kk & 3) * 32);
              const uint64_t da = smem_desc_sw128(q_addr + (kk >> 2) * kHalf + koff, 16, 1024);
              const uint64_t db = smem_desc_sw128(k_addr + (kk >> 2) * (T * 128) + koff, 16, 1024);
              mma_ss(tmem + ocol, da, db, IDESC_QK, kk > 0 ? 1u : 0u);
            }
            mma_commit(a_full);
            if (!mbar_wait(p_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
            if (!mbar_wait(sb_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // O = Q S
              const uint64_t da =
                  smem_desc_sw128(q_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
              const uint64_t db = smem_desc_sw128(sS + kk * 2048, kHalf, 1024);
              mma_ss(tmem + ocol, da, db, IDESC_QS, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {  // O += P V
              const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
              mma_ts(tmem + ocol, tmem + pcol + kk * 8, db, IDESC_PV, 1u);
            }
            mma_commit(o_full);
            if (i + 1 < it.ntiles) {  // S += K^T V (not needed after the span's last tile)
#pragma unroll
              for (int kk = 0; kk < T / 16; ++kk) {
                const uint64_t da = smem_desc_sw128(k_addr + kk * 2048, T * 128, 1024);
                const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
                mma_ss(tmem + kColS, da, db, IDESC_KV, 1u);
              }
              mma_commit(s_full);
            }
            mma_commit(&empty[s]);
          }
          if (!ok) break;
        }
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = tile row = state row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int t_in = r % T;
    const int mt = threadIdx.x - 64;
    const uint64_t pol_stream = policy_evict_first();
    int lt = 0, mtc = 0, kvc = 0, ac = 0, fb = 0;
    bool ok = true;

    // all 128 math threads have written their rows; the first thread of warp 2
    // then publishes the flag (release, GPU scope)
    auto publish = [&](unsigned* flag) -> bool {
      __threadfence();
      mbar_arrive(flag_bar);
      bool good = true;
      if (warp == 2) {
        good = warp_wait(flag_bar, fb & 1, p.status, abort_flag);
        if (good && lane == 0) {
          __threadfence();
          st_release_gpu(flag, 1u);
        }
      }
      ++fb;
      return good;
    };

    for (int k = 0; ok; ++k) {
      const int slot = k % kQueue;
      if (!warp_wait(&item_full[slot], (k / kQueue) & 1, p.status, abort_flag)) break;
      const int idx = items[slot];
      mbar_arrive(&item_empty[slot]);
      if (idx < 0) break;
      const Item it = decode_item(p, idx);
      const int b = it.bg / p.Hkv, g = it.bg % p.Hkv;
      const int head0 = g * p.G + it.hs * HPT;
      float* pre = p.prefix + (size_t)it.bg * p.nspan * D2;

      if (it.is_a) {
        // ---------------------------------------------- span-state item
        if (it.j == 0) {  // P_0 = S0 (or zero), for the chunk loops of span 0
          float4* dst = reinterpret_cast<float4*>(pre + (size_t)r * kHeadDim);
          const float4* s0 = p.S ? reinterpret_cast<const float4*>(
                                       p.S + (size_t)it.bg * D2 + (size_t)r * kHeadDim)
                                 : nullptr;
#pragma unroll 8
          for (int i = 0; i < 32; ++i) dst[i] = s0 ? __ldcg(s0 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          if (!publish(p.ready + (size_t)it.bg * p.nspan)) { ok = false; break; }
        }
        if (!warp_wait(a_done, ac & 1, p.status, abort_flag)) { ok = false; break; }
        ++ac;
        lt += it.ntiles;
        tc_fence_after();
        if (!warp_wait_flag(p.ready + (size_t)it.bg * p.nspan + it.j, p.status, abort_flag)) {
          ok = false;
          break;
        }
        const bool last = it.j + 1 == p.nspan;
        const float4* src = reinterpret_cast<const float4*>(pre + (size_t)it.j * D2 +
                                                            (size_t)r * kHeadDim);
        float4* dst = last ? (p.S ? reinterpret_cast<float4*>(p.S + (size_t)it.bg * D2 +
                                                              (size_t)r * kHeadDim)
                                  : nullptr)
                           : reinterpret_cast<float4*>(pre + (size_t)(it.j + 1) * D2 +
                                                       (size_t)r * kHeadDim);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + kColS + blk * 32, v);
          tmem_wait_ld();
          if (dst) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 a = __ldcg(src + blk * 8 + i);
              dst[blk * 8 + i] = make_float4(a.x + __uint_as_float(v[4 * i + 0]),
                                             a.y + __uint_as_float(v[4 * i + 1]),
                                             a.z + __uint_as_float(v[4 * i + 2]),
                                             a.w + __uint_as_float(v[4 * i + 3]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(s_free);
        if (!last && !publish(p.ready + (size_t)it.bg * p.nspan + it.j + 1)) { ok = false; break; }
        continue;
      }

      // ------------------------------------------------ chunk-loop item
      if (!warp_wait_flag(p.ready + (size_t)it.bg * p.nspan + it.j, p.status, abort_flag)) {
        ok = false;
        break;
      }
      {
        const float4* src = reinterpret_cast<const float4*>(pre + (size_t)it.j * D2 +
                                                            (size_t)r * kHeadDim);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 f = __ldcg(src + blk * 8 + i);
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
      for (int i = 0; i < it.ntiles; ++i, ++lt, ++mtc) {
        const int s = lt % STAGES;
        const uint32_t ob = (uint32_t)(mtc & 1);
        const uint32_t ocol = ob * 128;
        const uint32_t pcol = 256 + ob * (T / 2);

        // causal mask of the score tile -> P (bf16 in TMEM)
        if (!warp_wait(a_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
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

        // the previous tile's output store has read its smem: free that stage
        if (mt == 0 && i > 0) {
          bulk_wait_group_read<0>();
          mbar_arrive(&empty[(lt - 1) % STAGES]);
        }

        // bf16 copy of the updated state for the next tile's Q S
        if (i + 1 < it.ntiles) {
          if (!warp_wait(s_full, kvc & 1, p.status, abort_flag)) { ok = false; break; }
          ++kvc;
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

        // output epilogue: TMEM -> bf16 -> this stage's Q buffer -> store
        if (!warp_wait(o_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
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
          if (!warp_wait(store_ready, mtc & 1, p.status, abort_flag)) { ok = false; break; }
        }
        if (mt == 0) {
          const int c1 = (it.tile_begin + i) * T;
          const uint8_t* srcq = sm + (stage_q - base);
#pragma unroll
          for (int hh = 0; hh < HPT; ++hh) {
            tma_store_3d_hint(&map_o, srcq + hh * T * 128, 0, c1, b * p.Hq + head0 + hh,
                              pol_stream);
            tma_store_3d_hint(&map_o, srcq + kHalf + hh * T * 128, 64, c1, b * p.Hq + head0 + hh,
                              pol_stream);
          }
          bulk_commit_group();
        }
      }
      if (!ok) break;
      if (mt == 0) {  // the item's last store has read its smem: free that stage
        bulk_wait_group_read<0>();
        mbar_arrive(&empty[(lt - 1) % STAGES]);
      }
      tc_fence_before();
      mbar_arrive(s_free);
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

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

size_t fused_workspace_bytes(int B, int Hkv, int nspan) {
  const size_t states = (size_t)B * Hkv * nspan * kHeadDim * kHeadDim * sizeof(float);
  const size_t flags = ((size_t)B * Hkv * nspan + 1) * sizeof(unsigned);
  return states + ((flags + 255) & ~(size_t)255);
}

cudaError_t launch_prefill_fused(const PrefillGeometry& g, const PrefillMaps& maps, float* S,
                                 void* workspace, unsigned* status, int num_sms,
                                 cudaStream_t stream) {
  const int nsub = g.G / g.heads_per_tile;
  const size_t states = (size_t)g.B * g.Hkv * g.nspan * kHeadDim * kHeadDim * sizeof(float);
  const size_t nflags = (size_t)g.B * g.Hkv * g.nspan;
  FusedParams p;
  p.prefix = static_cast<float*>(workspace);
  p.ready = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + states);
  p.counter = p.ready + nflags;
  p.S = S;
  p.status = status;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.G = g.G;
  p.nsub = nsub;
  p.nspan = g.nspan;
  p.tiles_total = g.tiles_total;
  p.units_a = g.B * g.Hkv;
  p.units_m = g.B * g.Hkv * nsub;
  p.total_items = g.nspan * (p.units_a + p.units_m);
  cudaError_t e = cudaMemsetAsync(p.ready, 0, (nflags + 1) * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  const int grid = std::min(num_sms, p.total_items);
  if (g.tile == 64) {
    using L = FusedLayout<64, 3>;
    if ((e = set_smem(prefill_fused_kernel<64, 3>, L::kBytes)) != cudaSuccess) return e;
    prefill_fused_kernel<64, 3><<<grid, 192, L::kBytes, stream>>>(maps.q, maps.k, maps.v, maps.o, p);
  } else {
    using L = FusedLayout<128, 2>;
    if ((e = set_smem(prefill_fused_kernel<128, 2>, L::kBytes)) != cudaSuccess) return e;
    prefill_fused_kernel<128, 2><<<grid, 192, L::kBytes, stream>>>(maps.q, maps.k, maps.v, maps.o,
                                                                   p);
  }
  return cudaGetLastError();
}

}  // namespace la
