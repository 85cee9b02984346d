// la_backward_walk.cu -- dk and dv of the backward in one anti-causal walk per
// kv group (tcgen05 tensor cores), and the scan of its span states.
//
// From o_t = q_t S_t, S_t = S0 + sum_{s<=t} k_s^T v_s (the causal chunk form
// of "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
// "Lightning Attention：长上下文为什么突然变得便宜了"; grouped kv heads as in
// "MiniMax-01与Lightning Attention", section 1.1), with D_c = dSf + the sum of
// q_{t,h}^T do_{t,h} over every query head h of the group and every token t
// after chunk c:
//   dv_c = sum_h triu(K_c Q_{c,h}^T) dO_{c,h} + K_c D_c
//   dk_c = sum_h triu(V_c dO_{c,h}^T) Q_{c,h} + V_c D_c^T
//   D_{c-1} = D_c + sum_h Q_{c,h}^T dO_{c,h},   dS0 = D before the first chunk
// (triu keeps the diagonal: key token t >= row token s).  The heads of a group
// share K_c, V_c and one state, so a walk over the group's chunks, last to
// first, reads every Q and dO tile once for both gradients and sums the heads
// inside the MMAs (fp32 in tensor memory).
//
// Per 128-token chunk c of a group, per 64-token key block (head h, half j):
//   S1 = K_c Q_hj^T, S2 = V_c dO_hj^T   M=128 N=64  K=128 (SS) -> TMEM
//   P1, P2 = bf16(triu(S1)), bf16(triu(S2))   TMEM -> registers -> TMEM, each
//                                             over its own scores
//   dv += P1 dO_hj, dk += P2 Q_hj       M=128 N=128 K=64 (P from TMEM)
//   D  += Q_hj^T dO_hj                  M=128 N=128 K=64 (SS, both MN-major)
// and once per chunk, from the bf16 copy of D_c in smem (read MN-major for D,
// K-major for D^T):  dv += K_c D_c,  dk += V_c D_c^T  (M=128 N=128 K=128).
//
// Schedule: one CTA per SM walks (group, span) items round-robin, each span
// from its last chunk to its first; the entering state of a span (dSf plus
// the later spans' sums, from group_scan_kernel) is read at the item start,
// and the item of span 0 writes dS0 at its end.
// Roles (320 threads): warp 0 lane 0 streams key blocks (Q and dO of one head
// half-chunk) through a four-stage ring, lane 1 the K and V tiles of each
// chunk (K a chunk ahead, into the region the bf16 copy of D leaves once the
// chunk's first block has used it);
// warp 1 owns the tensor memory and issues the MMAs; warps 2-5 mask S1,
// convert the state and write dv rows out; warps 6-9 mask S2 and write dk
// rows out.  TMEM: dv at column 0, dk at 128, S1 (then P1) at 256, S2 (then
// P2) at 320, D at 384.  The two score streams run apart: a stream's next
// scores are issued right after the product that reads its P, so the tensor
// pipe's order keeps them off P, and one stream's mask overlaps the other
// stream's MMAs.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"
#include "la_ptx.cuh"
#include "la_tile.cuh"

namespace la {
namespace {

constexpr int kChunk = 128;                         // tokens per chunk
constexpr int kKeyBlk = 64;                         // tokens per key block
constexpr int kRing = 4;                            // key-block stages
constexpr int kChunkBytes = kChunk * kHeadDim * 2;  // 32 KB: K_c or V_c
constexpr int kBlkBytes = kKeyBlk * kHeadDim * 2;   // 16 KB: Q or dO of one block
constexpr int kBlkHalf = kKeyBlk * 128;             // 8 KB: 64 columns of a key block
constexpr uint32_t kColDv = 0, kColDk = 128, kColS1 = 256, kColS2 = 320;

// Two 32 KB regions take turns holding K_c and the bf16 copy of D: for the
// CTA's chunk n, K_n sits in region n % 2 and D's copy in region (n + 1) % 2.
// D's copy is read only by K_n D and V_n D^T at the chunk's first block, so
// K_{n+1} is loaded into its region as soon as those have run, a chunk ahead;
// the copy for chunk n + 1 then goes into K_n's region once the chunk's last
// scores and updates have run.  V_c keeps a region of its own.
struct WalkLayout {
  static constexpr int kRegOff = 0;                  // regions 0 and 1: K_c or D
  static constexpr int kVOff = 2 * kChunkBytes;
  static constexpr int kRingOff = 3 * kChunkBytes;   // stage: Q block, dO block
  static constexpr int kBarOff = kRingOff + kRing * 2 * kBlkBytes;
  // ring_full[R], ring_empty[R], k_full, v_full, d_free, v_free, a_full[2],
  // p_full[2], o_full, o_empty[2], s_full, sb_full, mma_done
  static constexpr int kNumBars = 2 * kRing + 14;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024
};
static_assert(WalkLayout::kBytes <= 232448, "shared memory");

struct WalkParams {
  __nv_bfloat16 *dk, *dv;               // [B*Hkv, N, 128]
  const float* ws;  // entering state of item it at ws[it * d * d]; nullptr: zero
  float* s_out;     // dS0 of group bg at s_out[bg] (from span 0's item); nullable
  unsigned* status;
  int64_t N;
  int Hq, Hkv, G, nspan, tiles_total, items;
};

// Position in a CTA's sequence of key blocks: item it (group bg, chunks
// [tb, te) walked from te - 1), n-th chunk of the item (chunk index cs), block
// blk of nb in the chunk (head blk / halves, half blk % halves), the CTA's
// chunk count gc and block count i.
struct Cursor {
  int it, bg, tb, te, n, cs, blk, nb, gc, i;
  bool valid;
};

__device__ __forceinline__ void span_of(const WalkParams& p, int it, int& bg, int& tb, int& te) {
  const int j = it % p.nspan;
  bg = it / p.nspan;
  tb = (int)(((int64_t)j * p.tiles_total) / p.nspan);
  te = (int)(((int64_t)(j + 1) * p.tiles_total) / p.nspan);
}

// 64-token halves of chunk cs that hold tokens (the last chunk may have one).
__device__ __forceinline__ int halves_of(const WalkParams& p, int cs) {
  return p.N - (int64_t)cs * kChunk > kKeyBlk ? 2 : 1;
}

__device__ __forceinline__ void cursor_item(const WalkParams& p, Cursor& c) {
  span_of(p, c.it, c.bg, c.tb, c.te);
  c.n = 0;
  c.cs = c.te - 1;
  c.nb = p.G * halves_of(p, c.cs);
  c.blk = 0;
}

__device__ __forceinline__ void cursor_init(const WalkParams& p, Cursor& c) {
  c.it = blockIdx.x;
  c.gc = 0;
  c.i = 0;
  c.valid = c.it < p.items;
  if (c.valid) cursor_item(p, c);
}

__device__ __forceinline__ void cursor_next(const WalkParams& p, Cursor& c) {
  ++c.i;
  if (++c.blk < c.nb) return;
  c.blk = 0;
  ++c.gc;
  if (++c.n < c.te - c.tb) {
    c.cs = c.te - 1 - c.n;
    c.nb = p.G * halves_of(p, c.cs);
    return;
  }
  c.it += (int)gridDim.x;
  c.valid = c.it < p.items;
  if (c.valid) cursor_item(p, c);
}

__global__ void __launch_bounds__(320, 1)
    bwd_walk_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_do,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const WalkParams p) {
  using L = WalkLayout;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, kKeyBlk, 0, 0);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_KD = idesc_bf16_f32(128, 128, 0, 1);
  constexpr uint32_t IDESC_VDT = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_D = idesc_bf16_f32(128, 128, 1, 1);
  constexpr int kDD = kHeadDim * kHeadDim;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBarOff);
  uint64_t* ring_full = bars;
  uint64_t* ring_empty = ring_full + kRing;
  uint64_t* k_full = ring_empty + kRing;  // K_c of a chunk landed
  uint64_t* v_full = k_full + 1;          // V_c of a chunk landed
  uint64_t* d_free = v_full + 1;          // a chunk's K_c D, V_c D^T done: D's region free
  uint64_t* v_free = d_free + 1;          // a chunk's last V_c reader done
  uint64_t* a_full = v_free + 1;     // two: S1, S2 of a block computed
  uint64_t* p_full = a_full + 2;     // two: P1, P2 of a block written over their scores
  uint64_t* o_full = p_full + 2;     // dv, dk of a chunk complete
  uint64_t* o_empty = o_full + 1;    // two: dv, dk read out
  uint64_t* s_full = o_empty + 2;    // D updated with a chunk
  uint64_t* sb_full = s_full + 1;    // bf16 copy of D (and D itself at an item start) ready
  uint64_t* mma_done = sb_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMiscOff + 4);

  // region of K_n and of D's bf16 copy for the CTA's chunk n; V_c's region
  auto sK = [&](int n) { return base + (uint32_t)(L::kRegOff + (n & 1) * kChunkBytes); };
  auto sS = [&](int n) { return base + (uint32_t)(L::kRegOff + ((n + 1) & 1) * kChunkBytes); };
  const uint32_t sV = base + L::kVOff;
  auto sQ = [&](int s) { return base + (uint32_t)(L::kRingOff + s * 2 * kBlkBytes); };
  auto sDO = [&](int s) { return sQ(s) + (uint32_t)kBlkBytes; };
  const int stride = (int)gridDim.x;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    mbar_init(k_full, 1);
    mbar_init(v_full, 1);
    mbar_init(d_free, 1);
    mbar_init(v_free, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&a_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(o_full, 1);
    mbar_init(&o_empty[0], 128);
    mbar_init(&o_empty[1], 128);
    mbar_init(s_full, 1);
    mbar_init(sb_full, 128);
    mbar_init(mma_done, 1);
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
      // key blocks: Q and dO rows [t0, t0 + 64) of head h, in cursor order
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_do);
      const uint64_t pol = policy_evict_first();
      Cursor c;
      cursor_init(p, c);
      int issued = 0;
      for (; c.valid; cursor_next(p, c)) {
        const int s = c.i % kRing;
        if (c.i >= kRing &&
            !mbar_wait(&ring_empty[s], ((c.i / kRing) - 1) & 1, p.status, abort_flag))
          break;
        const int halves = c.nb / p.G;
        const int h = c.blk / halves, j = c.blk % halves;
        const int b = c.bg / p.Hkv, g = c.bg % p.Hkv;
        const int qh = b * p.Hq + g * p.G + h;
        const int t0 = c.cs * kChunk + j * kKeyBlk;
        mbar_arrive_expect_tx(&ring_full[s], 2 * kBlkBytes);
        uint8_t* q_dst = sm + (sQ(s) - base);
        uint8_t* do_dst = sm + (sDO(s) - base);
        tma_load_3d(q_dst, &map_q, &ring_full[s], 0, t0, qh, pol);
        tma_load_3d(q_dst + kBlkHalf, &map_q, &ring_full[s], 64, t0, qh, pol);
        tma_load_3d(do_dst, &map_do, &ring_full[s], 0, t0, qh, pol);
        tma_load_3d(do_dst + kBlkHalf, &map_do, &ring_full[s], 64, t0, qh, pol);
        issued = c.i + 1;
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        for (int k = (issued > kRing ? issued - kRing : 0); k < issued; ++k)
          mbar_wait_drain(&ring_full[k % kRing], (k / kRing) & 1);
      }
    } else if (lane == 1) {
      // K_c, V_c per chunk; L2 prefetch of the next item's entering state
      // (no L2 prefetch of key blocks or K, V: measured, it raised DRAM reads
      // by 15% and slowed the walk by 10%)
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      const uint64_t pol = policy_evict_first();
      int gc = 0, k_issued = 0, v_issued = 0;
      bool go = true;
      for (int it = blockIdx.x; it < p.items && go; it += stride) {
        int bg, tb, te;
        span_of(p, it, bg, tb, te);
        const int nx = it + stride < p.items ? it + stride : -1;
        if (p.ws && nx >= 0)
          prefetch_l2_bulk(p.ws + (size_t)nx * kDD, (uint32_t)(kDD * sizeof(float)));
        for (int n = 0; n < te - tb; ++n, ++gc) {
          const int cs = te - 1 - n;
          // K_c into the region chunk gc - 1's D copy held (free once that
          // chunk's K_c D, V_c D^T have run), then V_c into its own region
          if (gc >= 1 && !mbar_wait(d_free, (gc - 1) & 1, p.status, abort_flag)) {
            go = false;
            break;
          }
          mbar_arrive_expect_tx(k_full, kChunkBytes);
          uint8_t* k_dst = sm + (sK(gc) - base);
          tma_load_3d(k_dst, &map_k, k_full, 0, cs * kChunk, bg, pol);
          tma_load_3d(k_dst + kHalf, &map_k, k_full, 64, cs * kChunk, bg, pol);
          ++k_issued;
          if (gc >= 1 && !mbar_wait(v_free, (gc - 1) & 1, p.status, abort_flag)) {
            go = false;
            break;
          }
          mbar_arrive_expect_tx(v_full, kChunkBytes);
          uint8_t* v_dst = sm + (sV - base);
          tma_load_3d(v_dst, &map_v, v_full, 0, cs * kChunk, bg, pol);
          tma_load_3d(v_dst + kHalf, &map_v, v_full, 64, cs * kChunk, bg, pol);
          ++v_issued;
        }
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        if (k_issued > 0) mbar_wait_drain(k_full, (k_issued - 1) & 1);
        if (v_issued > 0) mbar_wait_drain(v_full, (v_issued - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per block k: dv += P1(k) dO(k) (a chunk's first block starts dv once it
    // has been read out), the next block's S1, dk += P2(k) Q(k), the next
    // block's S2, at a chunk's first block K_c D and V_c D^T, then D += Q^T dO.
    // Each stream's next scores come after the product that reads its P (the
    // tensor pipe runs in issue order), and each mask has the other stream's
    // product and scores and D's update to run under it.  The bf16 copy of D
    // is waited for only before K_c D; D's first update of a chunk follows it
    // (the conversion reads D).  After K_c D, V_c D^T the region of D's copy
    // is released (the next chunk's K_c goes there); V_c's region once the
    // chunk's last S2 and V_c D^T are issued.  A next chunk's scores go at the
    // end of the block.
    if (elect_one()) {
      int inter_gc = -1;    // last chunk whose K_c D, V_c D^T are issued
      int kv_pending = -1;  // chunk whose last S2 is issued before its V_c D^T
      auto issue_s = [&](int t, const Cursor& x) -> bool {
        if (x.blk == 0 && !mbar_wait(t == 0 ? k_full : v_full, x.gc & 1, p.status, abort_flag))
          return false;
        const int s = x.i % kRing;
        if (!mbar_wait(&ring_full[s], (x.i / kRing) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t src = t == 0 ? sK(x.gc) : sV;         // K_c or V_c
        const uint32_t blk = t == 0 ? sQ(s) : sDO(s);        // Q or dO of the block
        const uint32_t dst = tmem + (t == 0 ? kColS1 : kColS2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // S1 = K_c Q^T, S2 = V_c dO^T (all K-major)
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint32_t ch = (uint32_t)(kk >> 2);
          mma_ss(dst, smem_desc_sw128(src + ch * kHalf + koff, 16, 1024),
                 smem_desc_sw128(blk + ch * kBlkHalf + koff, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&a_full[t]);
        if (t == 1 && x.blk == x.nb - 1) {  // the chunk's last score read of V_c
          if (inter_gc >= x.gc)
            mma_commit(v_free);
          else
            kv_pending = x.gc;
        }
        return true;
      };
      Cursor c;
      cursor_init(p, c);
      bool ok = !c.valid || (issue_s(0, c) && issue_s(1, c));
      while (ok && c.valid) {
        Cursor nx = c;
        cursor_next(p, nx);
        const int k = c.i, s = k % kRing;
        const bool first = c.blk == 0, last = c.blk == c.nb - 1;
        const bool nx_same = nx.valid && nx.blk != 0;  // the next block is in this chunk
        const uint32_t qa = sQ(s), doa = sDO(s);
        // dv += P1 dO
        if (!mbar_wait(&p_full[0], k & 1, p.status, abort_flag)) break;
        if (first && c.gc >= 1 && !mbar_wait(&o_empty[0], (c.gc - 1) & 1, p.status, abort_flag))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKeyBlk / 16; ++kk)
          mma_ts(tmem + kColDv, tmem + kColS1 + kk * 8,
                 smem_desc_sw128(doa + kk * 2048, kBlkHalf, 1024), IDESC_PV,
                 (first && kk == 0) ? 0u : 1u);
        if (nx_same && !issue_s(0, nx)) break;
        // dk += P2 Q
        if (!mbar_wait(&p_full[1], k & 1, p.status, abort_flag)) break;
        if (first && c.gc >= 1 && !mbar_wait(&o_empty[1], (c.gc - 1) & 1, p.status, abort_flag))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKeyBlk / 16; ++kk)
          mma_ts(tmem + kColDk, tmem + kColS2 + kk * 8,
                 smem_desc_sw128(qa + kk * 2048, kBlkHalf, 1024), IDESC_PV,
                 (first && kk == 0) ? 0u : 1u);
        if (nx_same && !issue_s(1, nx)) break;
        if (first) {  // the state's terms: dv += K_c D, dk += V_c D^T
          if (!mbar_wait(sb_full, c.gc & 1, p.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t ka = sK(c.gc), da = sS(c.gc);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)((kk & 3) * 32);
            const uint32_t ch = (uint32_t)(kk >> 2);
            mma_ss(tmem + kColDv, smem_desc_sw128(ka + ch * kHalf + koff, 16, 1024),
                   smem_desc_sw128(da + kk * 2048, kHalf, 1024), IDESC_KD, 1u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)((kk & 3) * 32);
            const uint32_t ch = (uint32_t)(kk >> 2);
            mma_ss(tmem + kColDk, smem_desc_sw128(sV + ch * kHalf + koff, 16, 1024),
                   smem_desc_sw128(da + ch * kHalf + koff, 16, 1024), IDESC_VDT, 1u);
          }
          mma_commit(d_free);  // D's copy read: its region takes the next K_c
          inter_gc = c.gc;
          if (kv_pending == c.gc) {
            mma_commit(v_free);
            kv_pending = -1;
          }
        }
#pragma unroll
        for (int kk = 0; kk < kKeyBlk / 16; ++kk)  // D += Q^T dO (both MN-major)
          mma_ss(tmem + kColS, smem_desc_sw128(qa + kk * 2048, kBlkHalf, 1024),
                 smem_desc_sw128(doa + kk * 2048, kBlkHalf, 1024), IDESC_D, 1u);
        mma_commit(&ring_empty[s]);
        if (last) {
          mma_commit(o_full);
          mma_commit(s_full);
        }
        if (nx.valid && !nx_same) {
          if (!issue_s(0, nx) || !issue_s(1, nx)) break;
        }
        c = nx;
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warpgroups
    // Warps 2-5 mask S1 into P1, convert the state and write dv; warps 6-9
    // mask S2 into P2 and write dk.  Each thread owns TMEM lane r = chunk row r.
    const bool wg1 = warp < 6;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t col_s = wg1 ? kColS1 : kColS2;
    const uint32_t col_o = wg1 ? kColDv : kColDk;
    __nv_bfloat16* const out_base = wg1 ? p.dv : p.dk;
    uint64_t* const my_empty = &o_empty[wg1 ? 0 : 1];
    bool ok = true;

    // entering state of item it -> D in tensor memory and its bf16 copy
    auto load_state = [&](int it, int gcd) {  // for the CTA's chunk gcd
      const uint32_t dcopy = sS(gcd);
      const float4* src =
          p.ws ? reinterpret_cast<const float4*>(p.ws + (size_t)it * kDD + (size_t)r * kHeadDim)
               : nullptr;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (src) f = src[blk * 8 + m];  // plain loads: dS0 may be written in place
          v[4 * m + 0] = __float_as_uint(f.x);
          v[4 * m + 1] = __float_as_uint(f.y);
          v[4 * m + 2] = __float_as_uint(f.z);
          v[4 * m + 3] = __float_as_uint(f.w);
        }
        tmem_st32(tmem + lane_base + kColS + blk * 32, v);
        store_row32_sw128(dcopy, r, blk, v);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sb_full);
    };

    // (warps 2-5) after chunk gcd's state update: the bf16 copy for the next
    // chunk, or at an item's end dS0 out (span 0) and the next item's
    // entering state in
    auto state_step = [&](int gcd, bool item_end, int done_it, int next_it) -> bool {
      if (!warp_wait(s_full, gcd & 1, p.status, abort_flag)) return false;
      tc_fence_after();
      if (!item_end) {
#pragma unroll 1
        for (int blk = 0; blk < 4; blk += 2) {
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem + lane_base + kColS + blk * 32, v0);
          tmem_ld32(tmem + lane_base + kColS + (blk + 1) * 32, v1);
          tmem_wait_ld();
          store_row32_sw128(sS(gcd + 1), r, blk, v0);
          store_row32_sw128(sS(gcd + 1), r, blk + 1, v1);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sb_full);
        return true;
      }
      if (p.s_out && done_it % p.nspan == 0) {
        float4* dst = reinterpret_cast<float4*>(p.s_out + (size_t)(done_it / p.nspan) * kDD +
                                                (size_t)r * kHeadDim);
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + kColS + blk * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int m = 0; m < 8; ++m)
            dst[blk * 8 + m] = make_float4(__uint_as_float(v[4 * m]), __uint_as_float(v[4 * m + 1]),
                                           __uint_as_float(v[4 * m + 2]),
                                           __uint_as_float(v[4 * m + 3]));
        }
      }
      tc_fence_before();
      if (next_it >= 0) load_state(next_it, gcd + 1);
      return true;
    };

    // this warpgroup's score tile of block c -> masked bf16 P over the first
    // 32 columns of the same tensor-memory buffer (every score is in
    // registers before P is written)
    const int t = wg1 ? 0 : 1;
    auto mask_block = [&](const Cursor& c) -> bool {
      const int k = c.i;
      const int halves = c.nb / p.G;
      const int j = c.blk % halves;
      if (!warp_wait(&a_full[t], k & 1, p.status, abort_flag)) return false;
      tc_fence_after();
      // key column u of the block is token 64 j + u of the chunk; row r keeps
      // u >= r - 64 j.  Rows 64..127 keep nothing of the first half.
      const int rel = r - kKeyBlk * j;
      const bool none = j == 0 && quarter >= 2;
      uint32_t pa[16], pb[16];
      if (!none) {
        uint32_t x0[32], x1[32];
        tmem_ld32(tmem + lane_base + col_s, x0);
        tmem_ld32(tmem + lane_base + col_s + 32, x1);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int u = 2 * m;
          pa[m] = pack_bf16x2(u >= rel ? __uint_as_float(x0[u]) : 0.f,
                              u + 1 >= rel ? __uint_as_float(x0[u + 1]) : 0.f);
          pb[m] = pack_bf16x2(u + 32 >= rel ? __uint_as_float(x1[u]) : 0.f,
                              u + 33 >= rel ? __uint_as_float(x1[u + 1]) : 0.f);
        }
      } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) pa[m] = pb[m] = 0u;
      }
      tmem_st16(tmem + lane_base + col_s, pa);
      tmem_st16(tmem + lane_base + col_s + 16, pb);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      return true;
    };

    // this warpgroup's accumulator of chunk gcd -> bf16 row r in registers;
    // the accumulator is released as soon as it is read, before any store
    auto read_out = [&](int gcd, uint32_t (&row_bf)[64]) -> bool {
      if (!warp_wait(o_full, gcd & 1, p.status, abort_flag)) return false;
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t x0[32], x1[32];
        tmem_ld32(tmem + lane_base + col_o + hh * 64, x0);
        tmem_ld32(tmem + lane_base + col_o + hh * 64 + 32, x1);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          row_bf[hh * 32 + m] = pack_bf16x2(__uint_as_float(x0[2 * m]), __uint_as_float(x0[2 * m + 1]));
          row_bf[hh * 32 + 16 + m] =
              pack_bf16x2(__uint_as_float(x1[2 * m]), __uint_as_float(x1[2 * m + 1]));
        }
      }
      tc_fence_before();
      mbar_arrive(my_empty);
      return true;
    };
    // quarter qt (64 bytes) of row r of chunk cs of group bg to global
    // memory (rows past N dropped)
    auto store_quarter = [&](int bg, int cs, const uint32_t (&row_bf)[64], int qt) {
      const int64_t row = (int64_t)cs * kChunk + r;
      if (row >= p.N) return;
      uint4* dst = reinterpret_cast<uint4*>(out_base + ((size_t)bg * p.N + row) * kHeadDim);
      switch (qt) {  // constant register indices in each case
#define LA_STORE_QUARTER(Q)                                                             \
  case Q:                                                                               \
    _Pragma("unroll") for (int m = 4 * Q; m < 4 * Q + 4; ++m) dst[m] =                 \
        make_uint4(row_bf[4 * m], row_bf[4 * m + 1], row_bf[4 * m + 2], row_bf[4 * m + 3]); \
    break;
        LA_STORE_QUARTER(0)
        LA_STORE_QUARTER(1)
        LA_STORE_QUARTER(2)
        LA_STORE_QUARTER(3)
#undef LA_STORE_QUARTER
        default:
          break;
      }
    };

    if (wg1) {
      griddep_wait();  // entering states come from the kernel before
      load_state(blockIdx.x, 0);
    }
    Cursor c;
    cursor_init(p, c);
    int prev_it = -1, prev_gc = -1, prev_bg = 0, prev_cs = 0;
    uint32_t row_bf[64];
    // the read-out row goes to global memory a quarter per block, after each
    // of the next four masks: stored all at once, the warpgroups' 16-byte
    // stores slowed the MMA thread's issue for the chunk's first block
    int stored = 4, out_bg = 0, out_cs = 0;
    for (; c.valid && ok; cursor_next(p, c)) {
      // the chunk before ended: the rest of the row before it goes out, its
      // accumulator is read out (the new chunk's first product waits for
      // it), then this block's mask, then the state step (the bf16 copy is
      // first used later in the block)
      const bool boundary = c.blk == 0 && prev_gc >= 0;
      if (boundary) {
        for (; stored < 4; ++stored) store_quarter(out_bg, out_cs, row_bf, stored);
        if (!read_out(prev_gc, row_bf)) { ok = false; break; }
      }
      if (!mask_block(c)) { ok = false; break; }
      if (boundary) {
        const bool item_end = c.it != prev_it;
        if (wg1 && !state_step(prev_gc, item_end, prev_it, item_end ? c.it : -1)) {
          ok = false;
          break;
        }
        stored = 0;
        out_bg = prev_bg;
        out_cs = prev_cs;
      }
      if (stored < 4) store_quarter(out_bg, out_cs, row_bf, stored++);
      prev_it = c.it;
      prev_gc = c.gc;
      prev_bg = c.bg;
      prev_cs = c.cs;
    }
    if (ok && prev_gc >= 0) {
      for (; stored < 4; ++stored) store_quarter(out_bg, out_cs, row_bf, stored);
      if (wg1) ok = state_step(prev_gc, true, prev_it, -1);
      if (ok && read_out(prev_gc, row_bf))
        for (int qt = 0; qt < 4; ++qt) store_quarter(prev_bg, prev_cs, row_bf, qt);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ent[bg][j] = dSf[bg] (nullable: 0) + sum over the group's heads h and the
// spans j' > j of wsh[b*Hq + g*G + h][j'] (span 0 of wsh is not read): the
// state entering span j of the group's backwards walk.
__global__ void __launch_bounds__(256)
    group_scan_kernel(const float4* __restrict__ wsh, const float4* __restrict__ dSf,
                      float4* __restrict__ ent, int Hq, int Hkv, int G, int nspan, int n4) {
  griddep_launch_dependents();  // the walk may start its copies
  griddep_wait();               // the span states are complete
  const int bg = blockIdx.y;
  const int b = bg / Hkv, g = bg % Hkv;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n4) return;
  float4 run = dSf ? dSf[(size_t)bg * n4 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = nspan - 1; j >= 0; --j) {
    ent[((size_t)bg * nspan + j) * n4 + e] = run;
    if (j == 0) break;
    for (int h = 0; h < G; ++h) {
      const float4 x = wsh[((size_t)(b * Hq + g * G + h) * nspan + j) * n4 + e];
      run.x += x.x;
      run.y += x.y;
      run.z += x.z;
      run.w += x.w;
    }
  }
}

}  // namespace

int walk_spans(int units, int tiles, int sms, int G) {
  // cost in chunk steps of one CTA: rounds x chunks per item, plus the span
  // pass over Q and dO (2G key tiles per chunk against the walk's 2G + 4)
  // spread over the SMs, plus a fixed cost for its two extra launches
  const double r_span = (2.0 * G) / (2.0 * G + 4.0);
  int best = 1;
  double best_cost = 1e300;
  for (int ns = 1; ns <= std::min(tiles, 256); ++ns) {
    const int64_t items = (int64_t)units * ns;
    const int64_t rounds = (items + sms - 1) / sms;
    const int per = (tiles + ns - 1) / ns;
    double cost = (double)(rounds * per);
    if (ns > 1) cost += (double)(ns - 1) / ns * units * (double)tiles * r_span / sms + 1.0;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = ns;
    }
  }
  return best;
}

cudaError_t launch_group_scan(const float* wsh, const float* dSf, float* ent, int B, int Hq,
                              int Hkv, int nspan, cudaStream_t stream) {
  const int n4 = kHeadDim * kHeadDim / 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n4 + 255) / 256), (unsigned)(B * Hkv));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, group_scan_kernel, reinterpret_cast<const float4*>(wsh),
                            reinterpret_cast<const float4*>(dSf), reinterpret_cast<float4*>(ent),
                            Hq, Hkv, Hq / Hkv, nspan, n4);
}

cudaError_t launch_bwd_walk(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                            const la_bf16* dO, la_bf16* dk, la_bf16* dv, const float* ws,
                            float* s_out, unsigned* status, int B, int Hq, int Hkv, int64_t N,
                            int nspan, int num_ctas, cudaStream_t stream, bool dependent) {
  const int tiles = (int)((N + kChunk - 1) / kChunk);
  const int64_t items = (int64_t)B * Hkv * nspan;
  if (N <= 0 || nspan < 1 || nspan > tiles || items > 0x7fffffff || num_ctas <= 0)
    return cudaErrorInvalidValue;
  CUtensorMap map_q, map_do, map_k, map_v;
  if (!make_tmap_bf16(&map_q, q, N, (int64_t)B * Hq, kKeyBlk) ||
      !make_tmap_bf16(&map_do, dO, N, (int64_t)B * Hq, kKeyBlk) ||
      !make_tmap_bf16(&map_k, k, N, (int64_t)B * Hkv, kChunk) ||
      !make_tmap_bf16(&map_v, v, N, (int64_t)B * Hkv, kChunk))
    return cudaErrorInvalidValue;
  WalkParams p;
  p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  p.ws = ws;
  p.s_out = s_out;
  p.status = status;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.nspan = nspan;
  p.tiles_total = tiles;
  p.items = (int)items;
  cudaError_t e = cudaFuncSetAttribute(bwd_walk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       WalkLayout::kBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<int64_t>(items, num_ctas));
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = WalkLayout::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, bwd_walk_kernel, map_q, map_do, map_k, map_v, p);
}

}  // namespace la
