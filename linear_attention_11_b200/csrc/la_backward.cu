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
//   dv_s = sum_{h in g} [ sum_{t>=s} (k_s . q_{t,h}) do_{t,h} ] + k_s dSf
//        -> an anti-causal pass per query head h with queries K (the kv head
//           of h), keys Q_h, values dO_h, state Q_h^T dO_h accumulated from
//           the end (initial dSf on the first head of each group), then a sum
//           over the heads of each group;
//   dk_s = sum_{h in g} [ sum_{t>=s} (v_s . do_{t,h}) q_{t,h} ] + v_s dSf^T
//        -> the same with queries V, keys dO_h, values Q_h, initial dSf^T;
//   dS0  = dSf + sum_{h in g} sum_t q_{t,h}^T do_{t,h}
//        -> the per-head final states of the dv pass summed over each group.
// Every pass runs the tensor-core kernels of the prefill (span states, scan,
// persistent chunk loop), the anti-causal ones in their reverse mode; the dv
// and dk walks share one set of span states (the dk walk reads them
// transposed).
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

// out[b, g, :] = sum_{h < G} part[b, g*G + h, :] over rows of `row` bf16
// elements (fp32 sum, one rounding), eight elements per thread.
__global__ void reduce_heads_kernel(const __nv_bfloat16* __restrict__ part,
                                    __nv_bfloat16* __restrict__ out, int G, size_t row,
                                    size_t total8) {
  const size_t i8 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i8 >= total8) return;
  const size_t e = i8 * 8;
  const size_t bg = e / row, off = e % row;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int h = 0; h < G; ++h) {
    const uint4 raw = *reinterpret_cast<const uint4*>(part + (bg * G + h) * row + off);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(p2[u]);
      acc[2 * u] += f.x;
      acc[2 * u + 1] += f.y;
    }
  }
  uint4 res;
  __nv_bfloat162* r2 = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
  for (int u = 0; u < 4; ++u) r2[u] = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
  *reinterpret_cast<uint4*>(out + bg * row + off) = res;
}

// out[b, g] = sum_{h < G} S[b, g*G + h] for d x d fp32 states.
__global__ void reduce_states_kernel(const float* __restrict__ S, float* __restrict__ out, int G,
                                     int dd) {
  const size_t bg = blockIdx.y;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < dd; e += gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int h = 0; h < G; ++h) acc += S[(bg * G + h) * dd + e];
    out[bg * dd + e] = acc;
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
  la_plan plan_q, plan_m;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan_q);  // dq: grouped, causal
  if (st != LA_OK) return st;
  if ((st = la_prefill_plan(B, Hq, Hq, N, d, 128, &plan_m)) != LA_OK) return st;  // per head
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
  const size_t sq_bytes = round((size_t)B * Hkv * dd * 4);
  const size_t sm_bytes = round((size_t)B * Hq * dd * 4);
  const size_t part_bytes = round((size_t)B * Hq * N * d * 2);
  const size_t wsq_bytes = forward_workspace_bytes(plan_q);
  const size_t wsq = round(wsq_bytes);
  const size_t wsm = plan_m.nspan > 1 ? round((size_t)plan_m.workspace_bytes) : 0;
  const size_t total = sq_bytes + 2 * sm_bytes + part_bytes + wsq + wsm;
  char* pool = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&pool), total, s) != cudaSuccess) return LA_ERR_CUDA;
  char* cur = pool;
  auto take = [&](size_t n) { char* p = cur; cur += n; return p; };
  float* S_q = reinterpret_cast<float*>(take(sq_bytes));
  float* S_in = reinterpret_cast<float*>(take(sm_bytes));   // dSf on each group's first head
  float* S_fin = reinterpret_cast<float*>(take(sm_bytes));  // per-head final states of the dv walk
  la_bf16* part = reinterpret_cast<la_bf16*>(take(part_bytes));
  void* ws_q = take(wsq);
  float* ws_m = wsm ? reinterpret_cast<float*>(take(wsm)) : nullptr;

  auto cu = [&](cudaError_t e) {
    if (e != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  };
  const size_t row = (size_t)N * d, total8 = (size_t)B * Hkv * row / 8;
  const unsigned red_blocks = (unsigned)((total8 + 255) / 256);
  int dev = 0, sms = 0;
  cu(cudaGetDevice(&dev));
  cu(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));

  // ---- dq: the forward pass on (dO, V, K) from S0^T
  cu(place_states(S0, S_q, B, Hkv, 1, d, 1, s));
  if (st == LA_OK)
    st = forward_dispatch(dO, v, k, dq, S_q, B, Hq, Hkv, N, plan_q, ws_q, wsq_bytes, s, false);

  // ---- dv, then dk: anti-causal walks per query head, summed over groups.
  // One state serves both: D = sum_t q_t^T do_t over the later chunks (dv
  // walk, from dSf), and its transpose (dk walk, from dSf^T), so the dk walk
  // reads the dv walk's entering states transposed.
  PrefillGeometry gm;
  gm.B = B;
  gm.Hq = Hq;
  gm.Hkv = Hq;
  gm.G = 1;
  gm.N = N;
  gm.tile = plan_m.tile;
  gm.heads_per_tile = plan_m.heads_per_tile;
  gm.tiles_total = plan_m.tiles_total;
  gm.nspan = plan_m.nspan;
  cu(place_states(dSf, S_in, B, Hq, G, d, 0, s));
  if (plan_m.nspan > 1)
    cu(cudaMemcpyAsync(S_fin, S_in, (size_t)B * Hq * dd * 4, cudaMemcpyDeviceToDevice, s));
  for (int pass = 0; pass < 2 && st == LA_OK; ++pass) {
    // dv: queries K, keys Q, values dO;  dk: queries V, keys dO, values Q
    const la_bf16* qsrc = pass == 0 ? k : v;
    const la_bf16* ksrc = pass == 0 ? q : dO;
    const la_bf16* vsrc = pass == 0 ? dO : q;
    la_bf16* dst = pass == 0 ? dv : dk;
    PrefillMaps maps;
    if (!make_tmap_bf16(&maps.q, qsrc, N, (int64_t)B * Hkv, gm.tile) ||
        !make_tmap_bf16(&maps.k, ksrc, N, (int64_t)B * Hq, gm.tile) ||
        !make_tmap_bf16(&maps.v, vsrc, N, (int64_t)B * Hq, gm.tile) ||
        !make_tmap_bf16(&maps.o, part, N, (int64_t)B * Hq, gm.tile)) {
      st = LA_ERR_CUDA;
      break;
    }
    if (plan_m.nspan > 1) {
      if (pass == 0) {  // span states of D and the reverse scan (S_fin: dSf -> final)
        cu(launch_span_states(gm, maps.k, maps.v, ws_m, status, s));
        if (st == LA_OK) cu(launch_state_scan(ws_m, S_fin, B * Hq, gm.nspan, d, s, 1));
      }
      // the dv walk may overlap the scan's tail (it waits before reading
      // states); the dk walk writes the partial sums the dv reduction reads,
      // so it starts only after it
      if (st == LA_OK)
        cu(launch_prefill_persist(gm, maps, ws_m, nullptr, status, sms, s, pass == 0, false, G,
                                  1, pass));
    } else if (st == LA_OK) {  // one span: from dSf (dSf^T), the dv walk writes the final states
      cu(launch_prefill_persist(gm, maps, S_in, pass == 0 ? S_fin : nullptr, status, sms, s, false,
                                false, G, 1, pass));
    }
    if (st == LA_OK) {
      reduce_heads_kernel<<<red_blocks, 256, 0, s>>>(
          reinterpret_cast<const __nv_bfloat16*>(part), reinterpret_cast<__nv_bfloat16*>(dst), G,
          row, total8);
      cu(cudaGetLastError());
    }
  }
  if (dS0 && st == LA_OK) {
    reduce_states_kernel<<<dim3(16, (unsigned)(B * Hkv)), 256, 0, s>>>(S_fin, dS0, G, (int)dd);
    cu(cudaGetLastError());
  }
  cu(cudaFreeAsync(pool, s));
  return st;
}
