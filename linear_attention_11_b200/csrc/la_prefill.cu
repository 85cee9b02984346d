// la_prefill.cu -- the span-state kernel of the span-parallel prefill
// (sm_100a).
//
// The chunk loop of "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座",
// section "Lightning Attention：长上下文为什么突然变得便宜了", is sequential per
// (batch, kv head).  To spread one sequence over the GPU it is cut into spans
// of whole tiles; this kernel, one CTA per (batch, kv head, span), computes
// each span's K^T V = sum of K_c^T V_c over its chunks (fp32, in tensor
// memory), the first of the three stages (span states, scan, chunk loop).
// "MiniMax-01与Lightning Attention", section 2.2: kv_sum = K^T V.
//
// Roles (192 threads): warp 0 streams K/V tiles by bulk tensor copies (128-byte
// swizzle, zero fill past N) through a ring, warp 1 owns the tensor memory and
// issues S += K_c^T V_c (tcgen05 M=128 N=128 K=T, both operands MN-major),
// warps 2-5 read the 128 x 128 fp32 result out to the workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_ptx.cuh"
#include "la_tile.cuh"

namespace la {
namespace {

// ---------------------------------------------------------------------------
// Span states: ws[bg][j] = sum over the span's tiles of K_c^T V_c.
struct SpanParams {
  float* ws;
  unsigned* status;
  int nspan, tiles_total;
  int nrun;   // spans computed per (batch, kv head): nrun of the nspan from `first` on
  int first;
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
  const int j = p.first + (int)(blockIdx.x % p.nrun);
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
                               cudaStream_t stream, bool skip_last, int parts, int first) {
  if (parts < 1 || first < 0 || (first > 0 && parts != 1)) return cudaErrorInvalidValue;
  const int nparts = g.nspan * parts;                                // sub-spans per sequence
  const int nrun = (g.nspan - (skip_last ? 1 : 0)) * parts - first;  // of them computed
  if (nrun <= 0) return cudaSuccess;
  SpanParams p{ws, status, nparts, g.tiles_total, nrun, first};
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

}  // namespace la
