// la_backward.cu -- gradients of the bf16 prefill.
//
// For a loss with gradient dO on the output and dSf on the final state, from
// o_t = q_t S_t and S_t = S0 + sum_{s<=t} k_s^T v_s (the causal chunkwise form
// of "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
// "Lightning Attention：长上下文为什么突然变得便宜了"; grouped kv heads as in
// "MiniMax-01与Lightning Attention", section 1.1):
//   dq_t = do_t S0^T + sum_{s<=t} (do_t . v_s) k_s
//        -> the forward pass itself with queries dO, keys V, values K and
//           initial state S0^T (grouped heads as in the forward);
//   dv_s = sum_{h in g} sum_{t>=s} (k_s . q_{t,h}) do_{t,h} + k_s D_s
//   dk_s = sum_{h in g} sum_{t>=s} (v_s . do_{t,h}) q_{t,h} + v_s D_s^T
//        with D_s = dSf + sum_{h in g} sum_{t > chunk of s} q_{t,h}^T do_{t,h}
//        -> one anti-causal walk per kv group over its chunks, last to first
//           (la_backward_walk.cu), spans of it in parallel: per-head span
//           sums of Q^T dO, then their scan over the group's heads and the
//           later spans gives each span's entering state;
//   dS0  = dSf + sum_{h in g} sum_t q_{t,h}^T do_{t,h}
//        -> the state after the walk's last chunk (written by span 0).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la.h"
#include "la_internal.h"

#define LA_EXPORT extern "C" __attribute__((visibility("default")))

namespace la {
namespace {

// dst[b, h] = (src && h % G == 0) ? src[b, h / G] (transposed if asked) : 0,
// for d x d fp32 states.
__global__ void place_states_kernel(const float* __restrict__ src, float* __restrict__ dst, int H,
                                    int G, int d, int transpose) {
  const size_t bh = blockIdx.y;
  const int h = (int)(bh % H);
  const size_t b = bh / H;
  const int dd = d * d;
  float* out = dst + bh * dd;
  const float* in = (src && h % G == 0) ? src + (b * (H / G) + h / G) * dd : nullptr;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < dd; e += gridDim.x * blockDim.x) {
    const int i = e / d, j = e % d;
    out[e] = in ? (transpose ? in[j * d + i] : in[e]) : 0.f;
  }
}

cudaError_t place_states(const float* src, float* dst, int B, int H, int G, int d, int transpose,
                         cudaStream_t s) {
  place_states_kernel<<<dim3(16, (unsigned)(B * H)), 256, 0, s>>>(src, dst, H, G, d, transpose);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace la

using namespace la;

LA_EXPORT la_status la_backward(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                const la_bf16* dO, const float* S0, const float* dSf, la_bf16* dq,
                                la_bf16* dk, la_bf16* dv, float* dS0, int B, int Hq, int Hkv,
                                int64_t N, int d, int chunk, la_stream stream) {
  if (!q || !k || !v || !dO || !dq || !dk || !dv) return LA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)q, (const void*)k, (const void*)v, (const void*)dO,
                        (const void*)dq, (const void*)dk, (const void*)dv, (const void*)S0,
                        (const void*)dSf, (const void*)dS0})
    if (p && !aligned16(p)) return LA_ERR_INVALID_ARG;
  la_plan plan_q;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan_q);  // dq: grouped, causal
  if (st != LA_OK) return st;
  const int G = Hq / Hkv;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned* status = device_status_ptr();
  if (!status) return LA_ERR_CUDA;
  {  // outputs must not overlap the inputs
    const size_t qb = (size_t)B * Hq * N * d * 2, kb = (size_t)B * Hkv * N * d * 2;
    const void* outs[3] = {dq, dk, dv};
    const size_t osz[3] = {qb, kb, kb};
    const void* ins[4] = {q, k, v, dO};
    const size_t isz[4] = {qb, kb, kb, qb};
    for (int i = 0; i < 3; ++i)
      for (int j = 0; j < 4; ++j) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(outs[i]), b2 = reinterpret_cast<uintptr_t>(ins[j]);
        if (a < b2 + isz[j] && b2 < a + osz[i]) return LA_ERR_INVALID_ARG;
      }
  }

  auto round = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t dd = (size_t)d * d;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LA_ERR_CUDA;
  const int tiles_w = (int)((N + 127) / 128);
  const int nspan_w = walk_spans(B * Hkv, tiles_w, sms, G);
  const size_t sq_bytes = S0 ? round((size_t)B * Hkv * dd * 4) : 0;
  const size_t wsq_bytes = forward_workspace_bytes(plan_q);
  const size_t wsq = round(wsq_bytes);
  const size_t wsh = nspan_w > 1 ? round((size_t)B * Hq * nspan_w * dd * 4) : 0;
  const size_t ent_bytes = nspan_w > 1 ? round((size_t)B * Hkv * nspan_w * dd * 4) : 0;
  const size_t total = sq_bytes + wsq + wsh + ent_bytes;
  char* pool = nullptr;
  if (!keep_pool_memory()) return LA_ERR_CUDA;
  if (cudaMallocAsync(reinterpret_cast<void**>(&pool), total, s) != cudaSuccess) return LA_ERR_CUDA;
  char* cur = pool;
  auto take = [&](size_t n) { char* p = cur; cur += n; return p; };
  float* S_q = S0 ? reinterpret_cast<float*>(take(sq_bytes)) : nullptr;
  void* ws_q = take(wsq);
  float* ws_h = wsh ? reinterpret_cast<float*>(take(wsh)) : nullptr;
  float* ent = ent_bytes ? reinterpret_cast<float*>(take(ent_bytes)) : nullptr;

  auto cu = [&](cudaError_t e) {
    if (e != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  };

  // ---- dq: the forward pass on (dO, V, K) from S0^T (from zero without S0)
  if (S0) cu(place_states(S0, S_q, B, Hkv, 1, d, 1, s));
  if (st == LA_OK)
    st = forward_dispatch(dO, v, k, dq, S_q, B, Hq, Hkv, N, plan_q, ws_q, wsq_bytes, s, false);

  // ---- dv, dk: the walk per kv group; with several spans, the per-head span
  // sums of Q^T dO (spans 1..nspan-1) and their scan give the entering states
  if (st == LA_OK && nspan_w > 1) {
    PrefillGeometry gh;
    gh.B = B;
    gh.Hq = Hq;
    gh.Hkv = Hq;
    gh.G = 1;
    gh.N = N;
    gh.tile = 128;
    gh.heads_per_tile = 1;
    gh.tiles_total = tiles_w;
    gh.nspan = nspan_w;
    CUtensorMap map_q, map_do;
    if (!make_tmap_bf16(&map_q, q, N, (int64_t)B * Hq, 128) ||
        !make_tmap_bf16(&map_do, dO, N, (int64_t)B * Hq, 128)) {
      st = LA_ERR_CUDA;
    } else {
      cu(launch_span_states(gh, map_q, map_do, ws_h, status, s, false, 1, 1));
      if (st == LA_OK) cu(launch_group_scan(ws_h, dSf, ent, B, Hq, Hkv, nspan_w, s));
      if (st == LA_OK)
        cu(launch_bwd_walk(q, k, v, dO, dk, dv, ent, dS0, status, B, Hq, Hkv, N, nspan_w, sms, s,
                           true));
    }
  } else if (st == LA_OK) {
    cu(launch_bwd_walk(q, k, v, dO, dk, dv, dSf, dS0, status, B, Hq, Hkv, N, 1, sms, s, false));
  }
  cu(cudaFreeAsync(pool, s));
  return st;
}
