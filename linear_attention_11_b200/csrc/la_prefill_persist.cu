// la_prefill_persist.cu -- the chunk loop of the prefill as a persistent
// tensor-core kernel.
//
// Per 128-row tile it computes the causal chunk form of "如何理解MiniMax股价创
// 历史新高？拆解国产大模型技术底座", section "Lightning Attention：长上下文为什么
// 突然变得便宜了": O_c = Q_c S + tril(Q_c K_c^T) V_c, then S += K_c^T V_c, with
// grouped kv heads as in "MiniMax-01与Lightning Attention", section 1.1.
// Tile: 128 rows = HPT query heads x T tokens (T = 64, HPT = 2, or T = 128,
// HPT = 1), d = 128:
//   A  = Q_c K_c^T      tcgen05 M=128 N=T  K=128 (SS) -> TMEM score buffer
//   P  = bf16(tril(A))  TMEM -> registers -> TMEM, over its own scores
//   O  = Q_c bf16(S)    tcgen05 M=128 N=128 K=128 (SS)
//   O += P V_c          tcgen05 M=128 N=128 K=T (A from TMEM)
//   S += K_c^T V_c      tcgen05 M=128 N=128 K=T (SS, both MN-major)
//   O -> bf16 -> smem -> bulk tensor store (clipped at N; loads past N read 0)
// Schedule:
//   - one CTA per SM walks a list of work items, item = one span of one
//     (batch, kv head) sequence, items dealt round-robin; the copy, MMA and
//     math pipelines run on across item boundaries, so the fill of one item
//     overlaps the drain of the one before;
//   - an item covers every query head of its kv group: per chunk step the
//     group's G / HPT tiles (HPT heads each) share one K/V tile and one state,
//     and the state update follows the last of them;
//   - the math warps read each item's entering state at the item boundary
//     (span-state workspace, caller's initial state, or zero), prefetched into
//     L2 one item ahead; with one span per sequence the CTA that owns the
//     whole sequence writes the final state (tensor memory after the last
//     chunk's update) at the item's end, in place if asked.
//
// Roles (320 threads): warp 0 lane 0 streams Q tiles, lane 1 K/V tiles (and
// the L2 prefetch), lane 2 staged states; warp 1 owns the tensor memory and
// issues the MMAs; warps 2-5 mask score tiles, warps 6-9 store output tiles;
// both warpgroups handle half of the state columns.  TMEM: O buffers at
// columns 0 and 128, score buffers from 256 (two of 64 columns at T = 64, one
// of 128 at T = 128; each tile's P is written over the first half of its
// scores), state at 384.  With the scores apart from the output, Q S of a
// tile is issued before its mask is done, and at T = 64 the next tile's
// scores go ahead of P V, so the tensor pipe does not wait for the mask.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"
#include "la_ptx.cuh"
#include "la_tile.cuh"

namespace la {
namespace {

struct PersistParams {
  const float* ws;  // entering state of item it at ws[it * ws_stride] (d x d fp32); nullptr: zero
  float* s_out;     // final state of sequence bg at s_out[bg], written by its last span's item
  unsigned* status;
  int Hq, Hkv, G, nsub, nspan, tiles_total, items;
  int ws_stride;     // spans cut into this many sub-spans in the workspace
};

// kStage: entering and final states pass through a 64 KB fp32 tile in shared
// memory by bulk tensor copies (map_s over the states, [units, 128, 128]),
// loaded an item ahead by a third copy lane; without it the math warps read
// and write them row by row.  kDedO: a dedicated output staging tile (else
// the output goes through the Q slot).  kHalfKV: K and V tiles take separate
// slots of the K/V ring (used at T = 128 with several tiles per chunk step,
// where the 32 KB this saves holds a third Q slot).
template <int T, int QST, int KVST, bool kDedO, bool kStage, bool kHalfKV>
__global__ void __launch_bounds__(320, 1)
    prefill_persist_kernel(const __grid_constant__ CUtensorMap map_q,
                           const __grid_constant__ CUtensorMap map_k,
                           const __grid_constant__ CUtensorMap map_v,
                           const __grid_constant__ CUtensorMap map_o,
                           const __grid_constant__ CUtensorMap map_s, const PersistParams p) {
  using L = MainLayout<T, QST, KVST, kDedO, kStage, kHalfKV>;
  constexpr int HPT = kTileRows / T;
  constexpr bool kDedicatedO = L::kDedicatedO;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, T, 0, 0);
  constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, 1, 1);
  constexpr int NSC = T == 64 ? 2 : 1;  // score buffers
  // T = 128: P handed over, and multiplied by V, in two halves of 64 keys
  constexpr int NPH = T == 128 ? 2 : 1;
  constexpr int kDD = kHeadDim * kHeadDim;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + QST;
  uint64_t* kv_full = q_empty + QST;
  uint64_t* kv_empty = kv_full + KVST;
  uint64_t* a_full = kv_empty + KVST;  // two: tile i's scores complete a_full[i % NSC]
  uint64_t* p_full = a_full + 2;       // two: tile i's P complete p_full[i % NSC]
  uint64_t* o_full = p_full + 2;    // two: tile i completes o_full[i & 1]
  uint64_t* o_empty = o_full + 2;   // two
  uint64_t* s_full = o_empty + 2;   // one completion per chunk step (state update)
  uint64_t* sb_full = s_full + 1;   // one completion per state version (bf16 copy ready)
  uint64_t* mma_done = sb_full + 1;
  uint64_t* store_ready = mma_done + 1;
  uint64_t* ostage_free = store_ready + 1;
  uint64_t* st_full = ostage_free + 1;   // staged entering state of the CTA's k-th item landed
  uint64_t* st_empty = st_full + 1;      // staging tile free again (read, final state stored)
  uint64_t* stage_done = st_empty + 1;   // math warps done with the staging tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);

  const uint32_t sS = base + L::kSOff;
  const uint32_t sSt = base + L::kStOff;
  const bool staged = kStage && p.ws != nullptr;
  auto sQ = [&](int i) { return base + (uint32_t)((i % QST) * kQBytes); };
  // K/V ring: slot c % KVST holds chunk step c's K and V tiles; with
  // kHalfKV the tiles take slots apart, copy 2c (K) and 2c + 1 (V) of the
  // ring, so a K tile can be refilled while the V tile of its step is in use
  auto kcopy = [&](int c) { return kHalfKV ? 2 * c : c; };
  auto vcopy = [&](int c) { return kHalfKV ? 2 * c + 1 : c; };
  auto sK = [&](int c) {
    return base + (uint32_t)(L::kKVOff + (kcopy(c) % KVST) * L::kKVBytes);
  };
  auto sV = [&](int c) {
    return kHalfKV ? base + (uint32_t)(L::kKVOff + (vcopy(c) % KVST) * L::kKVBytes)
                   : sK(c) + (uint32_t)L::kKBytes;
  };
  auto sO = [&](int i) { return kDedicatedO ? base + (uint32_t)L::kOOff : sQ(i); };
  // TMEM column of tile i's score buffer (its P over the first T / 2 columns)
  auto scol = [&](int i) { return (uint32_t)(256 + (i % NSC) * T); };

  // item it: sequence bg = it / nspan, chunk steps [tb, te) of span it % nspan
  auto span_of = [&](int it, int& bg, int& tb, int& te) {
    const int j = it % p.nspan;
    bg = it / p.nspan;
    tb = (int)(((int64_t)j * p.tiles_total) / p.nspan);
    te = (int)(((int64_t)(j + 1) * p.tiles_total) / p.nspan);
  };
  const int stride = (int)gridDim.x;
  auto next_item = [&](int it) { return it + stride < p.items ? it + stride : -1; };

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&o_empty[0], 128);
    mbar_init(&o_empty[1], 128);
    mbar_init(s_full, 1);
    mbar_init(sb_full, 256);
    mbar_init(mma_done, 1);
    mbar_init(store_ready, 128);
    mbar_init(ostage_free, 1);
    mbar_init(st_full, 1);
    mbar_init(st_empty, 1);
    mbar_init(stage_done, 256);
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
    if (lane == 0) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_o);
      const uint64_t pol_q = policy_evict_first();
      int i = 0;
      bool go = true;
      for (int it = blockIdx.x; it < p.items && go; it += stride) {
        int bg, tb, te;
        span_of(it, bg, tb, te);
        const int b = bg / p.Hkv, g = bg % p.Hkv;
        for (int n = 0; n < te - tb && go; ++n) {
          const int cs = tb + n;
          for (int hs = 0; hs < p.nsub; ++hs, ++i) {
            const int s = i % QST;
            if (i >= QST && !mbar_wait(&q_empty[s], ((i / QST) - 1) & 1, p.status, abort_flag)) {
              go = false;
              break;
            }
            mbar_arrive_expect_tx(&q_full[s], kQBytes);
            uint8_t* q_dst = sm + (sQ(i) - base);
#pragma unroll
            for (int hh = 0; hh < HPT; ++hh) {
              const int qh = b * p.Hq + g * p.G + hs * HPT + hh;
              tma_load_3d(q_dst + hh * T * 128, &map_q, &q_full[s], 0, cs * T, qh, pol_q);
              tma_load_3d(q_dst + kHalf + hh * T * 128, &map_q, &q_full[s], 64, cs * T, qh,
                          pol_q);
            }
          }
        }
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        for (int k = (i > QST ? i - QST : 0); k < i; ++k) mbar_wait_drain(&q_full[k % QST], (k / QST) & 1);
      }
    } else if (lane == 1) {
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      const uint64_t pol_kv = policy_evict_first();
      int gc = 0;
      bool go = true;
      int u = 0;  // copies into the ring so far
      for (int it = blockIdx.x; it < p.items && go; it += stride) {
        int bg, tb, te;
        span_of(it, bg, tb, te);
        const int nx = next_item(it);
        if (!staged && p.ws && nx >= 0)  // next item's entering state, read at this item's end
          prefetch_l2_bulk(p.ws + (size_t)nx * p.ws_stride * kDD, (uint32_t)(kDD * sizeof(float)));
        for (int n = 0; n < te - tb && go; ++n, ++gc) {
          const int cs = tb + n;
#pragma unroll
          for (int part = 0; part < (kHalfKV ? 2 : 1); ++part, ++u) {
            const int s = u % KVST;
            if (u >= KVST &&
                !mbar_wait(&kv_empty[s], ((u / KVST) - 1) & 1, p.status, abort_flag)) {
              go = false;
              break;
            }
            mbar_arrive_expect_tx(&kv_full[s], L::kKVBytes);
            if (!kHalfKV || part == 0) {
              uint8_t* k_dst = sm + (sK(gc) - base);
              tma_load_3d(k_dst, &map_k, &kv_full[s], 0, cs * T, bg, pol_kv);
              tma_load_3d(k_dst + T * 128, &map_k, &kv_full[s], 64, cs * T, bg, pol_kv);
            }
            if (!kHalfKV || part == 1) {
              uint8_t* v_dst = sm + (sV(gc) - base);
              tma_load_3d(v_dst, &map_v, &kv_full[s], 0, cs * T, bg, pol_kv);
              tma_load_3d(v_dst + T * 128, &map_v, &kv_full[s], 64, cs * T, bg, pol_kv);
            }
          }
        }
      }
      if (*abort_flag) {
        for (int k = (u > KVST ? u - KVST : 0); k < u; ++k)
          mbar_wait_drain(&kv_full[k % KVST], (k / KVST) & 1);
      }
    } else if (lane == 2 && staged) {
      // entering state of the CTA's k-th item into the staging tile, once the
      // tile is free (item k-1's state read and its final state stored)
      prefetch_tmap(&map_s);
      griddep_wait();
      const uint64_t pol_s = policy_evict_first();
      int k = 0;
      for (int it = blockIdx.x; it < p.items; it += stride, ++k) {
        if (k >= 1 && !mbar_wait(st_empty, (k - 1) & 1, p.status, abort_flag)) break;
        mbar_arrive_expect_tx(st_full, kStateBytes);
        uint8_t* dst = sm + (sSt - base);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_3d(dst + bx * kStateBoxBytes, &map_s, st_full, 32 * bx, 0, it, pol_s);
      }
      if (*abort_flag && k > 0) mbar_wait_drain(st_full, (k - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per tile i (chunk step gc, head subset hs): QS(i) into output buffer
    // i & 1 (once the epilogue of tile i - 2 has read it; at a chunk step's
    // first tile, once the state copy of the step is in), then P V(i) once
    // the mask has written P(i); after the last head subset of a chunk step
    // the state update KV(gc).  The scores of tile i + 1 go into their own
    // buffer: at T = 64 (two score buffers) right after QS(i), ahead of P V(i),
    // so the next mask overlaps P V and the update; at T = 128 (one buffer,
    // whose P(i) P V(i) still reads) after P V(i), so the next mask overlaps
    // QS(i + 1).  At an item's end the update goes first, so the state
    // hand-over to the next item does not wait for that item's first tiles.
    // With K and V apart (kHalfKV) the update of a chunk step goes right
    // after the last tile's QS, ahead of its P V: the update is then K's last
    // reader and releases K's slot, V's goes after that P V.
    if (elect_one()) {
      // wait for the K (or K/V) tile of chunk step c, or its V tile
      auto wait_k = [&](int c) {
        const int u = kcopy(c);
        return mbar_wait(&kv_full[u % KVST], (u / KVST) & 1, p.status, abort_flag);
      };
      auto wait_v = [&](int c) {
        const int u = vcopy(c);
        return mbar_wait(&kv_full[u % KVST], (u / KVST) & 1, p.status, abort_flag);
      };
      auto issue_qk = [&](int i, int gci) -> bool {
        if (!mbar_wait(&q_full[i % QST], (i / QST) & 1, p.status, abort_flag)) return false;
        if (!wait_k(gci)) return false;
        tc_fence_after();
        const uint32_t q_addr = sQ(i), k_addr = sK(gci);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // A = Q K^T, both K-major
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint64_t da = smem_desc_sw128(q_addr + (kk >> 2) * kHalf + koff, 16, 1024);
          const uint64_t db = smem_desc_sw128(k_addr + (kk >> 2) * (T * 128) + koff, 16, 1024);
          mma_ss(tmem + scol(i), da, db, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&a_full[i % NSC]);
        return true;
      };
      auto issue_kv = [&](int gci) -> bool {
        if (kHalfKV && !wait_v(gci)) return false;
        tc_fence_after();
        const uint32_t k_addr = sK(gci), v_addr = sV(gci);
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {  // S += K^T V (both MN-major)
          const uint64_t da = smem_desc_sw128(k_addr + kk * 2048, T * 128, 1024);
          const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
          mma_ss(tmem + kColS, da, db, IDESC_KV, 1u);
        }
        mma_commit(s_full);
        // the K tile's last reader (with kHalfKV; else the K/V slot's, as the
        // update follows the step's last P V)
        mma_commit(&kv_empty[kcopy(gci) % KVST]);
        return true;
      };
      int i = 0, gc = 0;
      bool ok = issue_qk(0, 0);
      for (int it = blockIdx.x; it < p.items && ok; it += stride) {
        int bg, tb, te;
        span_of(it, bg, tb, te);
        const bool last_item = next_item(it) < 0;
        for (int n = 0; n < te - tb && ok; ++n) {
          for (int hs = 0; hs < p.nsub && ok; ++hs) {
            const uint32_t ob = (uint32_t)(i & 1);
            const uint32_t ocol = ob * 128;
            const bool last_hs = hs == p.nsub - 1;
            const bool item_end = last_hs && n == te - tb - 1;
            const bool has_next = !(last_item && item_end);
            const int gnext = last_hs ? gc + 1 : gc;  // chunk step of tile i + 1
            if (hs == 0 && !mbar_wait(sb_full, gc & 1, p.status, abort_flag)) { ok = false; break; }
            if (i >= 2 && !mbar_wait(&o_empty[ob], ((i >> 1) - 1) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = sQ(i), v_addr = sV(gc);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // O = Q S (S: MN-major, 16 key rows per k-step)
              const uint64_t da =
                  smem_desc_sw128(q_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
              const uint64_t db = smem_desc_sw128(sS + kk * 2048, kHalf, 1024);
              mma_ss(tmem + ocol, da, db, IDESC_QS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&q_empty[i % QST]);  // QK(i) and QS(i) were Q(i)'s readers
            // (not with staged states: their items are a tile or two long)
            const bool early = NSC == 2 && !kStage && !item_end;
            if (early && !issue_qk(i + 1, gnext)) { ok = false; break; }
            // with K and V apart the step's update goes before its last P V,
            // which frees the K slot (its last reader) a tile earlier
            if (kHalfKV && last_hs && !issue_kv(gc)) { ok = false; break; }
            if (kHalfKV && !wait_v(gc)) { ok = false; break; }
#pragma unroll
            for (int ph = 0; ph < NPH && ok; ++ph) {  // O += P V (P from TMEM), half by half
              uint64_t* pf = NPH == 2 ? &p_full[ph] : &p_full[i % NSC];
              if (!mbar_wait(pf, (i / NSC) & 1, p.status, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kk = ph * (T / 16 / NPH); kk < (ph + 1) * (T / 16 / NPH); ++kk) {
                const uint64_t db = smem_desc_sw128(v_addr + kk * 2048, T * 128, 1024);
                mma_ts(tmem + ocol, tmem + scol(i) + kk * 8, db, IDESC_PV, 1u);
              }
            }
            if (!ok) break;
            mma_commit(&o_full[ob]);
            if (kHalfKV && last_hs) mma_commit(&kv_empty[vcopy(gc) % KVST]);  // V's last reader
            if (!kHalfKV && last_hs && !issue_kv(gc)) { ok = false; break; }
            if (!early && has_next && !issue_qk(i + 1, gnext)) { ok = false; break; }
            if (last_hs) ++gc;
            ++i;
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
    const int diag_blk = t_in / 32;
    const int blk0 = wg1 ? 0 : 2;  // state column blocks this warpgroup handles
    const bool store_thread = (warp == 6 && lane == 0);
    bool ok = true;

    // This warpgroup's half of row r of item it's entering state -> tensor
    // memory and the bf16 copy; then signal the state version.
    auto load_state = [&](int it) {
      const float* st = p.ws ? p.ws + (size_t)it * p.ws_stride * kDD : nullptr;
      const float4* src =
          st ? reinterpret_cast<const float4*>(st + (size_t)r * kHeadDim) : nullptr;
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const int blk = blk0 + bb;
        uint32_t v[32];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (src) f = src[blk * 8 + m];  // plain loads: the state may be updated in place
          v[4 * m + 0] = __float_as_uint(f.x);
          v[4 * m + 1] = __float_as_uint(f.y);
          v[4 * m + 2] = __float_as_uint(f.z);
          v[4 * m + 3] = __float_as_uint(f.w);
        }
        tmem_st32(tmem + lane_base + kColS + blk * 32, v);
        store_row32_sw128(sS, r, blk, v);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sb_full);
    };

    // Staged states: this warpgroup's half of row r of the next entering state
    // from the staging tile into tensor memory and the bf16 copy (have_in),
    // and of the final state from tensor memory into the same staging slots
    // (have_out; each thread reads its own slots before writing them).
    auto stage_swap = [&](bool have_in, bool have_out) {
      // 16 columns at a time: the incoming and outgoing rows together would
      // otherwise take 64 registers and spill
#pragma unroll 1
      for (int q = 2 * blk0; q < 2 * blk0 + 4; ++q) {
        uint32_t v[16];
        if (have_in) load_state_row16(sSt, r, q, v);
        if (have_out) {
          uint32_t w[16];
          tmem_ld16(tmem + lane_base + kColS + q * 16, w);
          tmem_wait_ld();
          store_state_row16(sSt, r, q, w);
        }
        if (have_in) {
          tmem_st16(tmem + lane_base + kColS + q * 16, v);
          store_row16_sw128(sS, r, q, v);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      if (have_in) mbar_arrive(sb_full);
      mbar_arrive(stage_done);
    };

    // After the update of chunk step gc: within an item, the bf16 copy for
    // the next chunk step; at an item's end (the CTA's item k), the final state
    // out (one span per sequence) and the next item's entering state in.
    auto state_step = [&](int gc, bool item_end, int bg, int nx, int k) -> bool {
      if (!warp_wait(s_full, gc & 1, p.status, abort_flag)) return false;
      tc_fence_after();
      if (item_end && staged) {
        if (nx >= 0) {
          // the next entering state has landed (its copy was issued only after
          // the tile's previous final state had been read by its store)
          if (!warp_wait(st_full, (k + 1) & 1, p.status, abort_flag)) return false;
        } else if (p.s_out) {
          // the CTA's last item: nothing comes in to order the reuse of the
          // tile, so wait until the store of the previous final state (or the
          // first hand-over) has released it before writing this one
          if (!warp_wait(st_empty, k & 1, p.status, abort_flag)) return false;
        }
        stage_swap(nx >= 0, p.s_out != nullptr);
        return true;
      }
      if (!item_end) {
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
      }
      // the final state of sequence bg is complete at the end of its last span
      const int jspan = ((int)blockIdx.x + k * stride) % p.nspan;
      if (p.s_out && jspan == p.nspan - 1) {
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_base + kColS + blk0 * 32, v0);
        tmem_ld32(tmem + lane_base + kColS + (blk0 + 1) * 32, v1);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(p.s_out + (size_t)bg * kDD + (size_t)r * kHeadDim +
                                                blk0 * 32);
#pragma unroll
        for (int m = 0; m < 8; ++m)
          dst[m] = make_float4(__uint_as_float(v0[4 * m]), __uint_as_float(v0[4 * m + 1]),
                               __uint_as_float(v0[4 * m + 2]), __uint_as_float(v0[4 * m + 3]));
#pragma unroll
        for (int m = 0; m < 8; ++m)
          dst[8 + m] = make_float4(__uint_as_float(v1[4 * m]), __uint_as_float(v1[4 * m + 1]),
                                   __uint_as_float(v1[4 * m + 2]), __uint_as_float(v1[4 * m + 3]));
      }
      if (nx >= 0) load_state(nx);
      return true;
    };

    // The kernel may start before the kernel writing the entering states has
    // finished (programmatic dependent launch): wait before the first read.
    griddep_wait();
    if (staged) {
      ok = warp_wait(st_full, 0, p.status, abort_flag);
      if (ok) stage_swap(true, false);
    } else {
      load_state(blockIdx.x);
    }

    if (wg1) {
      auto mask_tile = [&](int i) -> bool {
        const uint32_t acol = scol(i);  // scores; P goes over their first T / 2 columns
        if (!warp_wait(&a_full[i % NSC], (i / NSC) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        // 64 score columns per round; at T = 128 blocks entirely above the
        // diagonal of this warp's rows are not read.  Round h writes P to
        // columns [32 h, 32 h + 32), which this thread read in rounds <= h.
#pragma unroll 1
        for (int h = 0; h < T / 64; ++h) {
          uint32_t a[2][32];
          bool need[2];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * h + bb;
            need[bb] = T == 64 || blk <= diag_blk;
            if (need[bb]) tmem_ld32(tmem + lane_base + acol + blk * 32, a[bb]);
          }
          tmem_wait_ld();
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * h + bb;
            uint32_t pk[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int s0 = blk * 32 + 2 * m;
              const bool keep0 = need[bb] && s0 <= t_in;
              const bool keep1 = need[bb] && s0 + 1 <= t_in;
              const float f0 = keep0 ? __uint_as_float(a[bb][2 * m]) : 0.0f;
              const float f1 = keep1 ? __uint_as_float(a[bb][2 * m + 1]) : 0.0f;
              pk[m] = pack_bf16x2(f0, f1);
            }
            tmem_st16(tmem + lane_base + acol + blk * 16, pk);
          }
          if (NPH == 2) {  // this half of P is ready for its half of P V
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[h]);
          }
        }
        if (NPH == 1) {
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_full[i % NSC]);
        }
        return true;
      };
      ok = ok && mask_tile(0);
      int i = 0, gc = 0;
      for (int it = blockIdx.x, k = 0; it < p.items && ok; it += stride, ++k) {
        int bg, tb, te;
        span_of(it, bg, tb, te);
        const int nx = next_item(it);
        for (int n = 0; n < te - tb && ok; ++n) {
          for (int hs = 0; hs < p.nsub && ok; ++hs, ++i) {
            const bool last_hs = hs == p.nsub - 1;
            const bool item_end = last_hs && n == te - tb - 1;
            const bool has_next = !(item_end && nx < 0);
            // the MMA order decides which of the two is ready first (the next
            // tile's scores ahead of the update with two score buffers inside
            // an item); one call site each (two inlined copies of either spill
            // registers at T = 128)
            const bool mask_first = NSC == 2 && !kStage && !item_end;
#pragma unroll 1
            for (int ph = 0; ph < 2 && ok; ++ph) {
              const bool do_step = last_hs && (ph == (mask_first ? 1 : 0));
              const bool do_mask = has_next && (ph == (mask_first ? 0 : 1));
              if (do_mask && !mask_tile(i + 1)) ok = false;
              if (ok && do_step && !state_step(gc, item_end, bg, nx, k)) ok = false;
            }
            if (!ok) break;
            if (last_hs) ++gc;
          }
        }
      }
    } else {
      // Warp 6, after the math warps are done with the staging tile (use c:
      // 0 = the first entering state, k + 1 = the end of item k): bulk-store
      // the final state of sequence bg from it if asked, then hand the tile
      // back to the copy lane.
      auto stage_release = [&](int c, int bg, bool store) -> bool {
        if (!warp_wait(stage_done, c & 1, p.status, abort_flag)) return false;
        if (lane == 0) {
          if (store) {
            const uint8_t* src = sm + (sSt - base);
#pragma unroll
            for (int bx = 0; bx < 4; ++bx)
              tma_store_3d(&map_s, src + bx * kStateBoxBytes, 32 * bx, 0, bg);
            bulk_commit_group();
            bulk_wait_group_read<0>();
          }
          mbar_arrive(st_empty);
        }
        __syncwarp();
        return true;
      };
      if (staged && ok && warp == 6) ok = stage_release(0, 0, false);
      int i = 0, gc = 0;
      for (int it = blockIdx.x, k = 0; it < p.items && ok; it += stride, ++k) {
        int bg, tb, te;
        span_of(it, bg, tb, te);
        const int b = bg / p.Hkv, g = bg % p.Hkv;
        const int nx = next_item(it);
        for (int n = 0; n < te - tb && ok; ++n) {
          const int cs = tb + n;
          for (int hs = 0; hs < p.nsub && ok; ++hs, ++i) {
            const bool last_hs = hs == p.nsub - 1;
            const bool item_end = last_hs && n == te - tb - 1;
            if (last_hs && !state_step(gc, item_end, bg, nx, k)) { ok = false; break; }
            if (staged && item_end && warp == 6 && !stage_release(k + 1, bg, p.s_out != nullptr)) {
              ok = false;
              break;
            }
            if (last_hs) ++gc;
            // output epilogue: TMEM -> bf16 -> staging tile -> bulk store
            const uint32_t ob = (uint32_t)(i & 1);
            const uint32_t ocol = ob * 128;
            if (!warp_wait(&o_full[ob], (i >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
            if (kDedicatedO && i > 0 &&
                !warp_wait(ostage_free, (i - 1) & 1, p.status, abort_flag)) {
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
              const uint8_t* src = sm + (stage_o - base);
#pragma unroll
              for (int hh = 0; hh < HPT; ++hh) {
                const int oh = b * p.Hq + g * p.G + hs * HPT + hh;
                tma_store_3d(&map_o, src + hh * T * 128, 0, cs * T, oh);
                tma_store_3d(&map_o, src + kHalf + hh * T * 128, 64, cs * T, oh);
              }
              bulk_commit_group();
              bulk_wait_group_read<0>();  // the store has read the staging tile
              if (kDedicatedO)
                mbar_arrive(ostage_free);
              else
                mbar_arrive(&q_empty[i % QST]);
            }
          }
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

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int T, int QST, int KVST, bool kDedO, bool kStage, bool kHalfKV = false>
cudaError_t launch_persist(dim3 grid, cudaStream_t stream, const PrefillMaps& maps,
                           const CUtensorMap& map_s, const PersistParams& p, bool dependent) {
  using L = MainLayout<T, QST, KVST, kDedO, kStage, kHalfKV>;
  static_assert(L::kBytes <= 232448, "shared memory");
  static_assert(!kHalfKV || KVST >= 3, "K and V tiles apart need three slots");
  auto kernel = prefill_persist_kernel<T, QST, KVST, kDedO, kStage, kHalfKV>;
  cudaError_t e = set_smem(kernel, L::kBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, maps.q, maps.k, maps.v, maps.o, map_s, p);
}

}  // namespace

cudaError_t launch_prefill_persist(const PrefillGeometry& g, const PrefillMaps& maps,
                                   const float* ws, float* s_out, unsigned* status, int num_ctas,
                                   cudaStream_t stream, bool dependent, bool stage_states,
                                   int ws_stride) {
  if (s_out && s_out == ws && g.nspan != 1) return cudaErrorInvalidValue;
  const int nsub = g.G / g.heads_per_tile;
  const int64_t items = (int64_t)g.B * g.Hkv * g.nspan;
  if (items <= 0 || items > 0x7fffffff || num_ctas <= 0) return cudaErrorInvalidValue;
  if (ws_stride < 1) return cudaErrorInvalidValue;
  PersistParams p{ws,      s_out,         status,     g.Hq, g.Hkv, g.G, nsub,
                  g.nspan, g.tiles_total, (int)items, ws_stride};
  const dim3 grid((unsigned)std::min<int64_t>(items, num_ctas));
  // Staged states (room for the tile: two Q slots, output through the Q
  // slot); otherwise the smem goes to the rings.
  if (stage_states && ws_stride == 1 && g.tile == 64 &&
      g.nspan == 1 && ws && (!s_out || s_out == ws)) {
    CUtensorMap map_s;
    if (!make_tmap_state(&map_s, ws, (int64_t)g.B * g.Hkv)) return cudaErrorInvalidValue;
    return launch_persist<64, 2, 2, false, true>(grid, stream, maps, map_s, p, dependent);
  }
  if (g.tile == 64) return launch_persist<64, 3, 2, true, false>(grid, stream, maps, maps.q, p, dependent);
  // 128-token tiles: with several tiles per chunk step (grouped heads), K and
  // V apart in a three-slot ring, which leaves room for a third Q slot; with
  // one tile per step, K/V tiles together in two slots
  if (nsub > 1)
    return launch_persist<128, 3, 3, false, false, true>(grid, stream, maps, maps.q, p, dependent);
  return launch_persist<128, 2, 2, false, false>(grid, stream, maps, maps.q, p, dependent);
}

}  // namespace la
