// la_prefill_fused.cu -- the bf16 prefill as one persistent kernel (sm_100a).
//
// Same arithmetic as la_prefill.cu (the causal chunkwise form of
// "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
// "Lightning Attention：长上下文为什么突然变得便宜了": per chunk
// O_c = Q_c S + tril(Q_c K_c^T) V_c, then S += K_c^T V_c), scheduled so that
// K and V cross HBM about once.
//
// The sequence of every (batch, kv head) is cut into `nspan` spans.  Two kinds
// of work items:
//   A(bg, j)      span-state item: Agg_j = sum over span j of K_c^T V_c, then
//                 the chained prefix P_{j+1} = P_j + Agg_j (the state entering
//                 span j+1), published with a GPU-scope release flag; the last
//                 span writes the final state instead.  A(bg, 0) first
//                 publishes P_0 = S0 (or zero).
//   M(bg, hs, j)  chunk-loop item for HPT query heads: waits for P_j, then runs
//                 the chunk loop of span j from it.
// Item order: A(., 0..L-1), then for each j: A(., j+L), M(., ., j).  The state
// items run L rounds ahead of the chunk loops that need them, and the chunk
// loops of span j re-read K, V shortly after A(., j) read them (A loads K, V
// with an evict-last hint, Q and O stream with evict-first), so the second
// read is mostly served by L2.
//
// Scheduling: one CTA per SM; a scheduler lane takes item indices from a
// global atomic counter and hands them to the copy lanes, the MMA warp and the
// math warps through a queue in shared memory.  An item only waits for items
// with smaller indices, which were taken earlier by running CTAs, so the
// smallest unfinished item can always proceed.  Every wait is bounded.
//
// Roles (320 threads) and tensor memory as in the main kernel of la_prefill.cu:
//   warp 0  lane 0 Q copies, lane 1 K/V copies, lane 2 the item queue
//   warp 1  tensor memory owner, MMA issue
//   warps 2-5 (WG1)  causal mask, half of the state conversions
//   warps 6-9 (WG2)  output epilogue and stores, the other half
//   both warpgroups: entering states and span-state prefixes (half rows each)
//   TMEM: [0,256) two O buffers (score tiles alias them), [256,256+T) two P
//   buffers, [384,512) the state S (also the aggregate of A items).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"
#include "la_ptx.cuh"
#include "la_tile.cuh"

namespace la {
namespace {

constexpr int kQueue = 4;                   // item queue depth
constexpr int kQueueConsumers = 2 + 1 + 256;  // copy lanes, MMA thread, math warps

struct FusedParams {
  float* prefix;       // [B*Hkv][nspan][128*128]: state entering each span
  unsigned* ready;     // [B*Hkv*nspan]: prefix[bg][j] published
  unsigned* counter;   // next item index
  float* S;            // nullable: initial state in, final state out
  unsigned* status;
  int Hq, Hkv, G, nsub, nspan, tiles_total;
  int units_a;         // B*Hkv
  int units_m;         // B*Hkv*nsub
  int lookahead;       // rounds the state items run ahead (1..nspan)
  int total_items;     // nspan * (units_a + units_m)
};

struct Item {
  int is_a, bg, hs, j, tile_begin, ntiles;
};

__device__ __forceinline__ Item decode_item(const FusedParams& p, int idx) {
  Item it;
  const int UA = p.units_a, UM = p.units_m, n = p.nspan, L = p.lookahead;
  int x;
  if (idx < L * UA) {  // the first L rounds of state items
    it.is_a = 1;
    it.j = idx / UA;
    x = idx % UA;
  } else {
    const int i2 = idx - L * UA;
    const int full_blocks = n - L;  // blocks holding A(., j+L) and M(., ., j)
    if (i2 < full_blocks * (UA + UM)) {
      const int j = i2 / (UA + UM);
      const int y = i2 % (UA + UM);
      if (y < UA) {
        it.is_a = 1;
        it.j = j + L;
        x = y;
      } else {
        it.is_a = 0;
        it.j = j;
        x = y - UA;
      }
    } else {
      const int i3 = i2 - full_blocks * (UA + UM);
      it.is_a = 0;
      it.j = full_blocks + i3 / UM;
      x = i3 % UM;
    }
  }
  if (it.is_a) {
    it.bg = x;
    it.hs = 0;
  } else {
    it.bg = x / p.nsub;
    it.hs = x % p.nsub;
  }
  it.tile_begin = (int)(((int64_t)it.j * p.tiles_total) / n);
  it.ntiles = (int)(((int64_t)(it.j + 1) * p.tiles_total) / n) - it.tile_begin;
  return it;
}

template <int T, int QST, int KVST>
struct FusedLayout {
  static constexpr bool kDedicatedO = (T == 64);
  static constexpr int kKBytes = T * kHeadDim * 2;
  static constexpr int kKVBytes = 2 * kKBytes;
  static constexpr int kKVOff = QST * kQBytes;
  static constexpr int kSOff = kKVOff + KVST * kKVBytes;
  static constexpr int kOOff = kSOff + kSBytes;
  static constexpr int kBarOff = kOOff + (kDedicatedO ? kQBytes : 0);
  // q_full/q_empty[QST], kv_full/kv_empty[KVST], a_full, p_full, o_full[2],
  // o_empty[2], s_full, sb_full, mma_done, store_ready, ostage_free, a_done,
  // s_free, flag_bar, item_full/item_empty[kQueue]
  static constexpr int kNumBars = 2 * QST + 2 * KVST + 14 + 2 * kQueue;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 32 + 1024;
};

template <int T, int QST, int KVST>
__global__ void __launch_bounds__(320, 1)
    prefill_fused_kernel(const __grid_constant__ CUtensorMap map_q,
                         const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v,
                         const __grid_constant__ CUtensorMap map_o, const FusedParams p) {
  using L = FusedLayout<T, QST, KVST>;
  constexpr int HPT = kTileRows / T;
  constexpr bool kDedicatedO = L::kDedicatedO;
  constexpr bool kLookahead = KVST >= 3;
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
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + QST;
  uint64_t* kv_full = q_empty + QST;
  uint64_t* kv_empty = kv_full + KVST;
  uint64_t* a_full = kv_empty + KVST;
  uint64_t* p_full = a_full + 1;
  uint64_t* o_full = p_full + 1;    // two
  uint64_t* o_empty = o_full + 2;   // two
  uint64_t* s_full = o_empty + 2;
  uint64_t* sb_full = s_full + 1;
  uint64_t* mma_done = sb_full + 1;
  uint64_t* store_ready = mma_done + 1;
  uint64_t* ostage_free = store_ready + 1;
  uint64_t* a_done = ostage_free + 1;
  uint64_t* s_free = a_done + 1;
  uint64_t* flag_bar = s_free + 1;
  uint64_t* item_full = flag_bar + 1;
  uint64_t* item_empty = item_full + kQueue;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);
  volatile int* items = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 8);  // [kQueue]

  const uint32_t sS = base + L::kSOff;
  auto sQ = [&](int i) { return base + (uint32_t)((i % QST) * kQBytes); };
  auto sK = [&](int i) { return base + (uint32_t)(L::kKVOff + (i % KVST) * L::kKVBytes); };
  auto sV = [&](int i) { return sK(i) + (uint32_t)L::kKBytes; };
  auto sO = [&](int i) { return kDedicatedO ? base + (uint32_t)L::kOOff : sQ(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QST; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], kDedicatedO ? 1 : 2);
    }
    for (int i = 0; i < KVST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(p_full, 128);
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&o_empty[0], 128);
    mbar_init(&o_empty[1], 128);
    mbar_init(s_full, 1);
    mbar_init(sb_full, 256);
    mbar_init(mma_done, 1);
    mbar_init(store_ready, 128);
    mbar_init(ostage_free, 1);
    mbar_init(a_done, 1);
    mbar_init(s_free, 256);
    mbar_init(flag_bar, 256);
    for (int i = 0; i < kQueue; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], kQueueConsumers);
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

  // Take item k from the queue (every consumer walks the same sequence).
  auto take = [&](int k, bool warp_uniform) -> int {
    const int slot = k % kQueue;
    const bool ok = warp_uniform ? warp_wait(&item_full[slot], (k / kQueue) & 1, p.status, abort_flag)
                                 : mbar_wait(&item_full[slot], (k / kQueue) & 1, p.status, abort_flag);
    if (!ok) return -2;
    const int idx = items[slot];
    mbar_arrive(&item_empty[slot]);
    return idx;
  };

  if (warp == 0) {
    if (lane == 2) {
      // ------------------------------------------------------------ item queue
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
      }
    } else if (lane == 0) {
      // ------------------------------------------------------------ Q copies
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_o);
      const uint64_t pol = policy_evict_first();
      int qt = 0;
      for (int k = 0;; ++k) {
        const int idx = take(k, false);
        if (idx < 0) break;
        const Item it = decode_item(p, idx);
        if (it.is_a) continue;
        const int b = it.bg / p.Hkv, g = it.bg % p.Hkv;
        const int head0 = g * p.G + it.hs * HPT;
        bool ok = true;
        for (int i = 0; i < it.ntiles; ++i, ++qt) {
          const int s = qt % QST;
          if (qt >= QST && !mbar_wait(&q_empty[s], ((qt / QST) - 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&q_full[s], kQBytes);
          const int c1 = (it.tile_begin + i) * T;
          uint8_t* q_dst = sm + (sQ(qt) - base);
#pragma unroll
          for (int hh = 0; hh < HPT; ++hh) {
            tma_load_3d(q_dst + hh * T * 128, &map_q, &q_full[s], 0, c1, b * p.Hq + head0 + hh, pol);
            tma_load_3d(q_dst + kHalf + hh * T * 128, &map_q, &q_full[s], 64, c1,
                        b * p.Hq + head0 + hh, pol);
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int i = (qt > QST ? qt - QST : 0); i < qt; ++i)
          mbar_wait_drain(&q_full[i % QST], (i / QST) & 1);
      }
    } else if (lane == 1) {
      // ------------------------------------------------------------ K/V copies
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      const uint64_t pol_keep = policy_evict_last();   // state items: re-read soon
      const uint64_t pol_norm = policy_evict_normal();  // chunk loops: other head subsets
      int kvt = 0;
      for (int k = 0;; ++k) {
        const int idx = take(k, false);
        if (idx < 0) break;
        const Item it = decode_item(p, idx);
        const uint64_t pol = it.is_a ? pol_keep : pol_norm;
        bool ok = true;
        for (int i = 0; i < it.ntiles; ++i, ++kvt) {
          const int s = kvt % KVST;
          if (kvt >= KVST &&
              !mbar_wait(&kv_empty[s], ((kvt / KVST) - 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], L::kKVBytes);
          const int c1 = (it.tile_begin + i) * T;
          uint8_t* k_dst = sm + (sK(kvt) - base);
          uint8_t* v_dst = sm + (sV(kvt) - base);
          tma_load_3d(k_dst, &map_k, &kv_full[s], 0, c1, it.bg, pol);
          tma_load_3d(k_dst + T * 128, &map_k, &kv_full[s], 64, c1, it.bg, pol);
          tma_load_3d(v_dst, &map_v, &kv_full[s], 0, c1, it.bg, pol);
          tma_load_3d(v_dst + T * 128, &map_v, &kv_full[s], 64, c1, it.bg, pol);
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int i = (kvt > KVST ? kvt - KVST : 0); i < kvt; ++i)
          mbar_wait_drain(&kv_full[i % KVST], (i / KVST) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (elect_one()) {
      int qt = 0, kvt = 0, mtc = 0;
      bool ok = true;
      // scores of chunk-loop tile (q tile qt, kv tile kvt, M tile mtc)
      auto issue_qk = [&](int q_i, int kv_i, int m_i) -> bool {
        const uint32_t ob = (uint32_t)(m_i & 1);
        if (!mbar_wait(&q_full[q_i % QST], (q_i / QST) & 1, p.status, abort_flag)) return false;
        if (!mbar_wait(&kv_full[kv_i % KVST], (kv_i / KVST) & 1, p.status, abort_flag)) return false;
        if (m_i >= 2 && !mbar_wait(&o_empty[ob], ((m_i >> 1) - 1) & 1, p.status, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q_addr = sQ(q_i), k_addr = sK(kv_i);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint64_t da = smem_desc_sw128(q_addr + (kk >> 2) * kHalf + koff, 16, 1024);
          const uint64_t db = smem_desc_sw128(k_addr + (kk >> 2) * (T * 128) + koff, 16, 1024);
          mma_ss(tmem + ob * 128, da, db, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(a_full);
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int idx = take(k, false);
        if (idx < 0) break;
        const Item it = decode_item(p, idx);
        if (it.is_a) {
          // the state columns are free once the math warps are done with item k-1
          if (k >= 1 && !mbar_wait(s_free, (k - 1) & 1, p.status, abort_flag)) break;
          for (int i = 0; i < it.ntiles; ++i, ++kvt) {
            if (!mbar_wait(&kv_full[kvt % KVST], (kvt / KVST) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {
              const uint64_t da = smem_desc_sw128(sK(kvt) + kk * 2048, T * 128, 1024);
              const uint64_t db = smem_desc_sw128(sV(kvt) + kk * 2048, T * 128, 1024);
              mma_ss(tmem + kColS, da, db, IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&kv_empty[kvt % KVST]);
          }
          if (!ok) break;
          mma_commit(a_done);
          continue;
        }
        // chunk-loop item
        if (!issue_qk(qt, kvt, mtc)) break;
        for (int i = 0; i < it.ntiles; ++i, ++qt, ++kvt, ++mtc) {
          const uint32_t ob = (uint32_t)(mtc & 1);
          const uint32_t ocol = ob * 128;
          const uint32_t pcol = 256 + ob * (T / 2);
          if (!mbar_wait(p_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
          if (!mbar_wait(sb_full, mtc & 1, p.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q_addr = sQ(qt), k_addr = sK(kvt), v_addr = sV(kvt);
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
          mma_commit(&o_full[ob]);
          mma_commit(&q_empty[qt % QST]);
          if (i + 1 < it.ntiles) {
            if (kLookahead && !issue_qk(qt + 1, kvt + 1, mtc + 1)) { ok = false; break; }
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {  // S += K^T V
              const uint64_t da = smem_desc_sw128(k_addr + kk * 2048, T * 128, 1024);
              const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
              mma_ss(tmem + kColS, da, db, IDESC_KV, 1u);
            }
            mma_commit(s_full);
            mma_commit(&kv_empty[kvt % KVST]);
            if (!kLookahead && !issue_qk(qt + 1, kvt + 1, mtc + 1)) { ok = false; break; }
          } else {
            mma_commit(&kv_empty[kvt % KVST]);
          }
        }
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warpgroups
    const bool wg1 = warp < 6;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = tile row = state row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int t_in = r % T;
    const int blk0 = wg1 ? 0 : 2;  // state column blocks (of 32) this warpgroup owns
    const bool store_thread = (warp == 6 && lane == 0);
    const uint64_t pol_stream = policy_evict_first();
    int mtc = 0, kvc = 0, ac = 0, fb = 0;
    bool ok = true;

    // All 256 math threads have written their part; warp 2 then publishes the
    // flag (release, GPU scope).
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

    auto convert_state = [&]() -> bool {
      if (!warp_wait(s_full, kvc & 1, p.status, abort_flag)) return false;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(tmem + lane_base + kColS + blk0 * 32, v0);
      tmem_ld32(tmem + lane_base + kColS + (blk0 + 1) * 32, v1);
      tmem_wait_ld();
      store_row32_sw128(sS, r, blk0, v0);
      store_row32_sw128(sS, r, blk0 + 1, v1);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sb_full);
      return true;
    };

    auto mask_tile = [&](int m_i) -> bool {
      const uint32_t ob = (uint32_t)(m_i & 1);
      const uint32_t ocol = ob * 128;
      const uint32_t pcol = 256 + ob * (T / 2);
      if (!warp_wait(a_full, m_i & 1, p.status, abort_flag)) return false;
      tc_fence_after();
      uint32_t a[T / 32][32];
#pragma unroll
      for (int blk = 0; blk < T / 32; ++blk) tmem_ld32(tmem + lane_base + ocol + blk * 32, a[blk]);
      tmem_wait_ld();
#pragma unroll
      for (int blk = 0; blk < T / 32; ++blk) {
        uint32_t pk[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int s0 = blk * 32 + 2 * m;
          const float f0 = (s0 <= t_in) ? __uint_as_float(a[blk][2 * m]) : 0.0f;
          const float f1 = (s0 + 1 <= t_in) ? __uint_as_float(a[blk][2 * m + 1]) : 0.0f;
          pk[m] = pack_bf16x2(f0, f1);
        }
        tmem_st16(tmem + lane_base + pcol + blk * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      return true;
    };

    for (int k = 0; ok; ++k) {
      const int idx = take(k, true);
      if (idx < 0) break;
      const Item it = decode_item(p, idx);
      const int b = it.bg / p.Hkv, g = it.bg % p.Hkv;
      const int head0 = g * p.G + it.hs * HPT;
      float* pre = p.prefix + (size_t)it.bg * p.nspan * D2;
      const size_t row_off = (size_t)r * kHeadDim + (size_t)blk0 * 32;  // this thread's half row

      if (it.is_a) {
        // ---------------------------------------------- span-state item
        if (it.j == 0) {  // P_0 = S0 (or zero) for the chunk loops of span 0
          float4* dst = reinterpret_cast<float4*>(pre + row_off);
          const float4* s0 =
              p.S ? reinterpret_cast<const float4*>(p.S + (size_t)it.bg * D2 + row_off) : nullptr;
#pragma unroll 8
          for (int i = 0; i < 16; ++i) dst[i] = s0 ? __ldcg(s0 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          if (!publish(p.ready + (size_t)it.bg * p.nspan)) { ok = false; break; }
        }
        if (!warp_wait(a_done, ac & 1, p.status, abort_flag)) { ok = false; break; }
        ++ac;
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_base + kColS + blk0 * 32, v0);
        tmem_ld32(tmem + lane_base + kColS + (blk0 + 1) * 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free);  // done with the state columns
        if (!warp_wait_flag(p.ready + (size_t)it.bg * p.nspan + it.j, p.status, abort_flag)) {
          ok = false;
          break;
        }
        const bool last = it.j + 1 == p.nspan;
        const float4* src = reinterpret_cast<const float4*>(pre + (size_t)it.j * D2 + row_off);
        float4* dst = last ? (p.S ? reinterpret_cast<float4*>(p.S + (size_t)it.bg * D2 + row_off)
                                  : nullptr)
                           : reinterpret_cast<float4*>(pre + (size_t)(it.j + 1) * D2 + row_off);
        if (dst) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 a0 = __ldcg(src + i), a1 = __ldcg(src + 8 + i);
            dst[i] = make_float4(a0.x + __uint_as_float(v0[4 * i + 0]),
                                 a0.y + __uint_as_float(v0[4 * i + 1]),
                                 a0.z + __uint_as_float(v0[4 * i + 2]),
                                 a0.w + __uint_as_float(v0[4 * i + 3]));
            dst[8 + i] = make_float4(a1.x + __uint_as_float(v1[4 * i + 0]),
                                     a1.y + __uint_as_float(v1[4 * i + 1]),
                                     a1.z + __uint_as_float(v1[4 * i + 2]),
                                     a1.w + __uint_as_float(v1[4 * i + 3]));
          }
        }
        if (!last && !publish(p.ready + (size_t)it.bg * p.nspan + it.j + 1)) { ok = false; break; }
        continue;
      }

      // ------------------------------------------------ chunk-loop item
      if (!warp_wait_flag(p.ready + (size_t)it.bg * p.nspan + it.j, p.status, abort_flag)) {
        ok = false;
        break;
      }
      {
        const float4* src = reinterpret_cast<const float4*>(pre + (size_t)it.j * D2 + row_off);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 f = __ldcg(src + bb * 8 + i);
            v[4 * i + 0] = __float_as_uint(f.x);
            v[4 * i + 1] = __float_as_uint(f.y);
            v[4 * i + 2] = __float_as_uint(f.z);
            v[4 * i + 3] = __float_as_uint(f.w);
          }
          tmem_st32(tmem + lane_base + kColS + (blk0 + bb) * 32, v);
          store_row32_sw128(sS, r, blk0 + bb, v);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sb_full);
      }
      const int m_first = mtc;
      if (wg1) {
        if (!mask_tile(mtc)) { ok = false; break; }
        for (int i = 0; i < it.ntiles; ++i, ++mtc) {
          if (i + 1 < it.ntiles) {
            if (kLookahead) {
              if (!mask_tile(mtc + 1) || !convert_state()) { ok = false; break; }
            } else {
              if (!convert_state() || !mask_tile(mtc + 1)) { ok = false; break; }
            }
            ++kvc;
          }
        }
        if (!ok) break;
        // the last tile's Q S has read the bf16 state before the next item rewrites it
        const int last = m_first + it.ntiles - 1;
        if (!warp_wait(&o_full[last & 1], (last >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
      } else {
        for (int i = 0; i < it.ntiles; ++i, ++mtc) {
          const uint32_t ob = (uint32_t)(mtc & 1);
          const uint32_t ocol = ob * 128;
          if (i + 1 < it.ntiles) {
            if (!convert_state()) { ok = false; break; }
            ++kvc;
          }
          if (!warp_wait(&o_full[ob], (mtc >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          if (kDedicatedO && mtc > 0 &&
              !warp_wait(ostage_free, (mtc - 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t stage_o = sO(mtc);  // chunk-loop tiles are the only Q tiles: qt == mtc
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            uint32_t v0[32], v1[32];
            tmem_ld32(tmem + lane_base + ocol + (2 * bb) * 32, v0);
            tmem_ld32(tmem + lane_base + ocol + (2 * bb + 1) * 32, v1);
            tmem_wait_ld();
            store_row32_sw128(stage_o, r, 2 * bb, v0);
            store_row32_sw128(stage_o, r, 2 * bb + 1, v1);
          }
          tc_fence_before();
          mbar_arrive(&o_empty[ob]);
          fence_proxy_async_smem();
          mbar_arrive(store_ready);
          if (warp == 6) {
            if (!warp_wait(store_ready, mtc & 1, p.status, abort_flag)) { ok = false; break; }
          }
          if (store_thread) {
            const int c1 = (it.tile_begin + i) * T;
            const uint8_t* src = sm + (stage_o - base);
#pragma unroll
            for (int hh = 0; hh < HPT; ++hh) {
              tma_store_3d_hint(&map_o, src + hh * T * 128, 0, c1, b * p.Hq + head0 + hh,
                                pol_stream);
              tma_store_3d_hint(&map_o, src + kHalf + hh * T * 128, 64, c1,
                                b * p.Hq + head0 + hh, pol_stream);
            }
            bulk_commit_group();
            bulk_wait_group_read<0>();
            if (kDedicatedO)
              mbar_arrive(ostage_free);
            else
              mbar_arrive(&q_empty[mtc % QST]);
          }
        }
        if (!ok) break;
      }
      tc_fence_before();
      mbar_arrive(s_free);
    }
    if (store_thread) bulk_wait_group<0>();
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
                                 void* workspace, unsigned* status, int num_sms, int lookahead,
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
  p.lookahead = std::max(1, std::min(lookahead, g.nspan));
  p.total_items = g.nspan * (p.units_a + p.units_m);
  cudaError_t e = cudaMemsetAsync(p.ready, 0, (nflags + 1) * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  const int grid = std::min(num_sms, p.total_items);
  if (g.tile == 64) {
    using L = FusedLayout<64, 2, 3>;
    static_assert(L::kBytes <= 232448, "shared memory");
    if ((e = set_smem(prefill_fused_kernel<64, 2, 3>, L::kBytes)) != cudaSuccess) return e;
    prefill_fused_kernel<64, 2, 3><<<grid, 320, L::kBytes, stream>>>(maps.q, maps.k, maps.v, maps.o,
                                                                     p);
  } else {
    using L = FusedLayout<128, 2, 2>;
    static_assert(L::kBytes <= 232448, "shared memory");
    if ((e = set_smem(prefill_fused_kernel<128, 2, 2>, L::kBytes)) != cudaSuccess) return e;
    prefill_fused_kernel<128, 2, 2><<<grid, 320, L::kBytes, stream>>>(maps.q, maps.k, maps.v,
                                                                      maps.o, p);
  }
  return cudaGetLastError();
}

}  // namespace la
