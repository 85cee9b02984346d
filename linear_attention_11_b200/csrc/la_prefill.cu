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
//                        state that enters it (prepared by the scan kernel),
//                        causal or anti-causal; the backward passes run it.
//                        The forward prefill runs the persistent schedule of
//                        the same tile arithmetic (la_prefill_persist.cu).
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
// Warp roles of the main kernel (320 threads): warp 0 issues the copies, warp 1
// owns the tensor memory and issues the MMAs, warps 2-5 (one thread per TMEM
// lane) mask the score tiles, warps 6-9 write the output tiles; both
// warpgroups convert half of the state.  The span-state kernel uses 192
// threads (one epilogue warpgroup).
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
#include "la_tile.cuh"

namespace la {
namespace {

struct MainParams {
  const float* ws;
  unsigned* status;
  int Hq, Hkv, G, nsub, nspan, tiles_total;
  int qdiv;     // query rows of head h come from head h / qdiv of the query tensor
  int reverse;  // 1: anti-causal (s >= t), tiles of a span walked from the end
};

template <int T, int QST, int KVST>
__global__ void __launch_bounds__(320, 1)
    prefill_main_kernel(const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_o, const MainParams p) {
  using L = MainLayout<T, QST, KVST>;
  constexpr int HPT = kTileRows / T;
  constexpr bool kDedicatedO = L::kDedicatedO;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, T, 0, 0);
  constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, 1, 1);
  constexpr bool kLookahead = KVST >= 3;

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
  uint64_t* o_full = p_full + 1;    // two: tile i completes o_full[i & 1]
  uint64_t* o_empty = o_full + 2;   // two
  uint64_t* s_full = o_empty + 2;
  uint64_t* sb_full = s_full + 1;
  uint64_t* mma_done = sb_full + 1;
  uint64_t* store_ready = mma_done + 1;
  uint64_t* ostage_free = store_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);

  const uint32_t sS = base + L::kSOff;
  auto sQ = [&](int i) { return base + (uint32_t)((i % QST) * kQBytes); };
  auto sK = [&](int i) { return base + (uint32_t)(L::kKVOff + (i % KVST) * L::kKVBytes); };
  auto sV = [&](int i) { return sK(i) + (uint32_t)L::kKBytes; };
  auto sO = [&](int i) { return kDedicatedO ? base + (uint32_t)L::kOOff : sQ(i); };

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
  // i-th tile this CTA processes (the span is walked backwards in reverse mode)
  auto tile_at = [&](int i) { return p.reverse ? tile_end - 1 - i : tile_begin + i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QST; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], kDedicatedO ? 1 : 2);  // MMA commit (+ output-store release)
    }
    for (int i = 0; i < KVST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(p_full, 128);       // mask warpgroup
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&o_empty[0], 128);  // epilogue warpgroup
    mbar_init(&o_empty[1], 128);
    mbar_init(s_full, 1);
    mbar_init(sb_full, 256);      // both warpgroups convert half of the state
    mbar_init(mma_done, 1);
    mbar_init(store_ready, 128);
    mbar_init(ostage_free, 1);
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
    // ------------------------------------------------------------ copies
    // Lane 0 streams the Q tiles, lane 1 the K/V tiles, each through its own
    // ring, so a K/V copy never waits behind a Q slot (and vice versa).
    if (lane == 0) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_o);
      const uint64_t pol_q = policy_evict_first();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % QST;
        if (i >= QST && !mbar_wait(&q_empty[s], ((i / QST) - 1) & 1, p.status, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[s], kQBytes);
        const int c1 = tile_at(i) * T;
        uint8_t* q_dst = sm + (sQ(i) - base);
#pragma unroll
        for (int hh = 0; hh < HPT; ++hh) {
          const int qh = (b * p.Hq + head0 + hh) / p.qdiv;
          tma_load_3d(q_dst + hh * T * 128, &map_q, &q_full[s], 0, c1, qh, pol_q);
          tma_load_3d(q_dst + kHalf + hh * T * 128, &map_q, &q_full[s], 64, c1, qh, pol_q);
        }
        issued = i + 1;
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        for (int i = (issued > QST ? issued - QST : 0); i < issued; ++i)
          mbar_wait_drain(&q_full[i % QST], (i / QST) & 1);
      }
    } else if (lane == 1) {
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      const uint64_t pol_kv = policy_evict_last();  // re-read by the other head subsets
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % KVST;
        if (i >= KVST && !mbar_wait(&kv_empty[s], ((i / KVST) - 1) & 1, p.status, abort_flag))
          break;
        mbar_arrive_expect_tx(&kv_full[s], L::kKVBytes);
        const int c1 = tile_at(i) * T;
        uint8_t* k_dst = sm + (sK(i) - base);
        uint8_t* v_dst = sm + (sV(i) - base);
        tma_load_3d(k_dst, &map_k, &kv_full[s], 0, c1, bg, pol_kv);
        tma_load_3d(k_dst + T * 128, &map_k, &kv_full[s], 64, c1, bg, pol_kv);
        tma_load_3d(v_dst, &map_v, &kv_full[s], 0, c1, bg, pol_kv);
        tma_load_3d(v_dst + T * 128, &map_v, &kv_full[s], 64, c1, bg, pol_kv);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > KVST ? issued - KVST : 0); i < issued; ++i)
          mbar_wait_drain(&kv_full[i % KVST], (i / KVST) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order per tile i:  QS(i) PV(i) | QK(i+1) | KV(i) with a 3-deep K/V ring:
    // the next tile's scores go before this tile's state update, so its causal
    // mask overlaps the update.  With 2 K/V slots the next tile's copy is
    // usually still in flight, so the update goes first: QS(i) PV(i) KV(i) |
    // QK(i+1).
    if (elect_one()) {
      auto issue_qk = [&](int i) -> bool {
        const uint32_t ob = (uint32_t)(i & 1);
        if (!mbar_wait(&q_full[i % QST], (i / QST) & 1, p.status, abort_flag)) return false;
        if (!mbar_wait(&kv_full[i % KVST], (i / KVST) & 1, p.status, abort_flag)) return false;
        if (i >= 2 && !mbar_wait(&o_empty[ob], ((i >> 1) - 1) & 1, p.status, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q_addr = sQ(i), k_addr = sK(i);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // A = Q K^T, both K-major
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint64_t da = smem_desc_sw128(q_addr + (kk >> 2) * kHalf + koff, 16, 1024);
          const uint64_t db = smem_desc_sw128(k_addr + (kk >> 2) * (T * 128) + koff, 16, 1024);
          mma_ss(tmem + ob * 128, da, db, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(a_full);
        return true;
      };
      bool ok = ntiles > 0 && issue_qk(0);
      for (int i = 0; i < ntiles && ok; ++i) {
        const uint32_t ob = (uint32_t)(i & 1);
        const uint32_t ocol = ob * 128;
        const uint32_t pcol = 256 + ob * (T / 2);
        if (!mbar_wait(p_full, i & 1, p.status, abort_flag)) break;
        if (!mbar_wait(sb_full, i & 1, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t q_addr = sQ(i), k_addr = sK(i), v_addr = sV(i);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // O = Q S (S: MN-major, 16 key rows per k-step)
          const uint64_t da =
              smem_desc_sw128(q_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t db = smem_desc_sw128(sS + kk * 2048, kHalf, 1024);
          mma_ss(tmem + ocol, da, db, IDESC_QS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {  // O += P V (P from TMEM)
          const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
          mma_ts(tmem + ocol, tmem + pcol + kk * 8, db, IDESC_PV, 1u);
        }
        mma_commit(&o_full[ob]);
        mma_commit(&q_empty[i % QST]);  // Q(i) read by QK(i) and QS(i), both done then
        if (i + 1 < ntiles) {
          if (kLookahead && !issue_qk(i + 1)) break;
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk) {  // S += K^T V (both MN-major)
            const uint64_t da = smem_desc_sw128(k_addr + kk * 2048, T * 128, 1024);
            const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
            mma_ss(tmem + kColS, da, db, IDESC_KV, 1u);
          }
          mma_commit(s_full);
          mma_commit(&kv_empty[i % KVST]);
          if (!kLookahead && !issue_qk(i + 1)) break;
        } else {
          mma_commit(&kv_empty[i % KVST]);
        }
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warpgroups
    // WG1 (warps 2-5): causal mask; WG2 (warps 6-9): output epilogue and stores.
    // Both convert half of the state (WG1 columns 0-63, WG2 columns 64-127).
    const bool wg1 = warp < 6;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = tile row = state row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int t_in = r % T;
    const int diag_blk = t_in / 32;  // the 32-column score block holding this warp's diagonal
    const int blk0 = wg1 ? 0 : 2;  // state column blocks this warpgroup converts
    const bool store_thread = (warp == 6 && lane == 0);
    const bool reverse = p.reverse != 0;
    bool ok = true;

    // Entering state of this span (this warpgroup's half of the row).  The
    // kernel may start before the scan has finished (programmatic dependent
    // launch); only the workspace read waits for it.
    griddep_wait();
    {
      const float4* src = reinterpret_cast<const float4*>(
          p.ws + ((size_t)bg * p.nspan + j) * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim);
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const int blk = blk0 + bb;
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

    // half of the bf16 state copy for the next tile's Q S
    auto convert_state = [&](int i) -> bool {
      if (!warp_wait(s_full, i & 1, p.status, abort_flag)) return false;
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

    if (wg1) {
      auto mask_tile = [&](int i) -> bool {
        const uint32_t ob = (uint32_t)(i & 1);
        const uint32_t ocol = ob * 128;
        const uint32_t pcol = 256 + ob * (T / 2);
        if (!warp_wait(a_full, i & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        // 64 score columns per round (a whole 128-column row would take 128
        // registers and spill).  At T = 128 a 32-column block that lies
        // entirely on the masked side of this warp's 32 rows is not read at
        // all (at T = 64 skipping measured slower).  Rounds are not unrolled:
        // overlapping them would bring the 128 registers back.
#pragma unroll 1
        for (int h = 0; h < T / 64; ++h) {
          uint32_t a[2][32];
          bool need[2];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * h + bb;
            need[bb] = T == 64 || (reverse ? (blk >= diag_blk) : (blk <= diag_blk));
            if (need[bb]) tmem_ld32(tmem + lane_base + ocol + blk * 32, a[bb]);
          }
          tmem_wait_ld();
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * h + bb;
            uint32_t pk[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int s0 = blk * 32 + 2 * m;
              const bool keep0 = need[bb] && (reverse ? (s0 >= t_in) : (s0 <= t_in));
              const bool keep1 = need[bb] && (reverse ? (s0 + 1 >= t_in) : (s0 + 1 <= t_in));
              const float f0 = keep0 ? __uint_as_float(a[bb][2 * m]) : 0.0f;
              const float f1 = keep1 ? __uint_as_float(a[bb][2 * m + 1]) : 0.0f;
              pk[m] = pack_bf16x2(f0, f1);
            }
            tmem_st16(tmem + lane_base + pcol + blk * 16, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        return true;
      };
      ok = ntiles > 0 && mask_tile(0);
      for (int i = 0; i < ntiles && ok; ++i) {
        if (i + 1 < ntiles) {
          // the MMA order decides which of the two is ready first
          if (kLookahead) {
            if (!mask_tile(i + 1) || !convert_state(i)) { ok = false; break; }
          } else {
            if (!convert_state(i) || !mask_tile(i + 1)) { ok = false; break; }
          }
        }
      }
    } else {
      for (int i = 0; i < ntiles && ok; ++i) {
        const uint32_t ob = (uint32_t)(i & 1);
        const uint32_t ocol = ob * 128;
        if (i + 1 < ntiles && !convert_state(i)) { ok = false; break; }
        // output epilogue: TMEM -> bf16 -> staging tile -> bulk store
        if (!warp_wait(&o_full[ob], (i >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
        if (kDedicatedO && i > 0 && !warp_wait(ostage_free, (i - 1) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t stage_o = sO(i);
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
          if (!warp_wait(store_ready, i & 1, p.status, abort_flag)) { ok = false; break; }
        }
        if (store_thread) {
          const int c1 = tile_at(i) * T;
          const uint8_t* src = sm + (stage_o - base);
#pragma unroll
          for (int hh = 0; hh < HPT; ++hh) {
            tma_store_3d(&map_o, src + hh * T * 128, 0, c1, b * p.Hq + head0 + hh);
            tma_store_3d(&map_o, src + kHalf + hh * T * 128, 64, c1, b * p.Hq + head0 + hh);
          }
          bulk_commit_group();
          bulk_wait_group_read<0>();  // the store has read the staging tile
          if (kDedicatedO)
            mbar_arrive(ostage_free);
          else
            mbar_arrive(&q_empty[i % QST]);
        }
      }
      if (store_thread) bulk_wait_group<0>();
    }
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
  int nrun;  // spans computed per (batch, kv head): nspan, or nspan - 1 (the last one skipped)
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

  griddep_launch_dependents();  // the scan may be scheduled; it waits for this grid
  const int j = blockIdx.x % p.nrun;
  const int bg = blockIdx.x / p.nrun;
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
                               cudaStream_t stream, bool skip_last) {
  const int nrun = g.nspan - (skip_last ? 1 : 0);
  if (nrun <= 0) return cudaSuccess;
  SpanParams p{ws, status, g.nspan, g.tiles_total, nrun};
  const dim3 grid((unsigned)(g.B * g.Hkv * nrun));
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

template <typename K>
cudaError_t launch_dependent(K kernel, dim3 grid, int threads, int smem, cudaStream_t stream,
                             const PrefillMaps& maps, const MainParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, maps.q, maps.k, maps.v, maps.o, p);
}

cudaError_t launch_prefill_main(const PrefillGeometry& g, const PrefillMaps& maps,
                                const float* ws, unsigned* status, cudaStream_t stream, int qdiv,
                                int reverse) {
  const int nsub = g.G / g.heads_per_tile;
  MainParams p{ws, status, g.Hq, g.Hkv, g.G, nsub, g.nspan, g.tiles_total, qdiv, reverse};
  const dim3 grid((unsigned)(g.B * g.Hkv * g.nspan * nsub));
  cudaError_t e;
  if (g.tile == 64) {
    using L = MainLayout<64, 2, 3>;
    static_assert(L::kBytes <= 232448, "shared memory");
    if ((e = set_smem(prefill_main_kernel<64, 2, 3>, L::kBytes)) != cudaSuccess) return e;
    return launch_dependent(prefill_main_kernel<64, 2, 3>, grid, 320, L::kBytes, stream, maps, p);
  }
  using L = MainLayout<128, 2, 2>;
  static_assert(L::kBytes <= 232448, "shared memory");
  if ((e = set_smem(prefill_main_kernel<128, 2, 2>, L::kBytes)) != cudaSuccess) return e;
  return launch_dependent(prefill_main_kernel<128, 2, 2>, grid, 320, L::kBytes, stream, maps, p);
}

}  // namespace la
