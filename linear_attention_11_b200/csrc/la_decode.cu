// la_decode.cu -- the recurrent decode step (one new token per sequence).
//
// "MiniMax-01与Lightning Attention", section 4.1 ("Streaming" row): the kv
// state is updated incrementally and no history is kept.  For each
// (batch b, kv head g):
//     S += k^T v            (d x d fp32, in place)
//     o_h = q_h S           for the G query heads h of g
// Update first, then read, so the new token sees itself (the diagonal of the
// causal mask).
//
// The step is a pure sweep over the fp32 states (2 x 4 d^2 bytes per unit,
// about 1.2 flop/byte): HBM-bound.  One CTA of 256 threads per unit; a warp
// reads one row of S as 32 contiguous float4 (512 B, fully coalesced), each
// thread keeps its updated rows in registers for the G dot products, and the
// per-row-group partial sums are reduced through shared memory.  S is read and
// written exactly once with streaming cache hints.  The single step runs 512
// threads per CTA, the multi-step kernel 256.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kMaxGroup = 32;  // query heads per kv head supported by the decode step

template <int D, int NT>
__global__ void __launch_bounds__(NT)
    decode_step_kernel(float* __restrict__ S, const __nv_bfloat16* __restrict__ q,
                       const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                       __nv_bfloat16* __restrict__ o, int Hq, int Hkv) {
  constexpr int TPR = D / 4;                 // threads per row (one float4 each)
  constexpr int RP = NT / TPR;               // rows per pass
  constexpr int RPT = D / RP;                // rows per thread
  extern __shared__ float sh[];
  const int G = Hq / Hkv;
  float* ks = sh;                   // [D]
  float* vs = ks + D;               // [D]
  float* qs = vs + D;               // [G][D]
  float* red = qs + G * D;          // [G][RP][D]

  const int unit = blockIdx.x;      // b * Hkv + g
  const int b = unit / Hkv, g = unit % Hkv;
  const int tid = threadIdx.x;
  const __nv_bfloat16* kp = k + (size_t)unit * D;
  const __nv_bfloat16* vp = v + (size_t)unit * D;
  const __nv_bfloat16* qp = q + ((size_t)b * Hq + (size_t)g * G) * D;
  for (int i = tid; i < D; i += NT) {
    ks[i] = __bfloat162float(kp[i]);
    vs[i] = __bfloat162float(vp[i]);
  }
  for (int i = tid; i < G * D; i += NT) qs[i] = __bfloat162float(qp[i]);
  __syncthreads();

  const int tx = tid % TPR, ty = tid / TPR;
  const int col = 4 * tx;
  const float4 vv = make_float4(vs[col], vs[col + 1], vs[col + 2], vs[col + 3]);
  float4* Su = reinterpret_cast<float4*>(S + (size_t)unit * D * D);
  float4 srow[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) srow[r] = __ldcs(Su + (size_t)(ty + r * RP) * TPR + tx);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const float kr = ks[ty + r * RP];
    srow[r].x = fmaf(kr, vv.x, srow[r].x);
    srow[r].y = fmaf(kr, vv.y, srow[r].y);
    srow[r].z = fmaf(kr, vv.z, srow[r].z);
    srow[r].w = fmaf(kr, vv.w, srow[r].w);
    __stcs(Su + (size_t)(ty + r * RP) * TPR + tx, srow[r]);
  }
  for (int h = 0; h < G; ++h) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float* qh = qs + h * D;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float qr = qh[ty + r * RP];
      acc.x = fmaf(qr, srow[r].x, acc.x);
      acc.y = fmaf(qr, srow[r].y, acc.y);
      acc.z = fmaf(qr, srow[r].z, acc.z);
      acc.w = fmaf(qr, srow[r].w, acc.w);
    }
    *reinterpret_cast<float4*>(red + ((size_t)h * RP + ty) * D + col) = acc;
  }
  __syncthreads();
  __nv_bfloat16* op = o + ((size_t)b * Hq + (size_t)g * G) * D;
  for (int e = tid; e < G * D; e += NT) {
    const int h = e / D, c = e % D;
    float sum = 0.f;
#pragma unroll
    for (int y = 0; y < RP; ++y) sum += red[((size_t)h * RP + y) * D + c];
    op[e] = __float2bfloat16_rn(sum);
  }
}

// Several decode steps per launch: the state of one (batch, kv head) stays in
// registers across `steps` tokens, so it crosses HBM once per launch instead
// of once per token.  Step t: S += k_t^T v_t; o_{t,h} = q_{t,h} S, in token
// order -- the same recurrence as decode_step_kernel, applied `steps` times.
// Inputs follow the prefill layout with N = steps: q, o [B, Hq, steps, D],
// k, v [B, Hkv, steps, D].  The next step's q, k, v are loaded into registers
// while the current step computes.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_steps_kernel(float* __restrict__ S, const __nv_bfloat16* __restrict__ q,
                        const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                        __nv_bfloat16* __restrict__ o, int Hq, int Hkv, int steps) {
  constexpr int TPR = D / 4;
  constexpr int RP = kDecodeThreads / TPR;
  constexpr int RPT = D / RP;
  extern __shared__ float sh[];
  const int G = Hq / Hkv;
  const int per_step = (G + 2) * D;  // k, v, then the G query rows of one step
  float* tok = sh;                   // [per_step] current step
  float* red = tok + per_step;       // [G][RP][D]

  const int unit = blockIdx.x;  // b * Hkv + g
  const int b = unit / Hkv, g = unit % Hkv;
  const int tid = threadIdx.x;
  const __nv_bfloat16* kp = k + (size_t)unit * steps * D;
  const __nv_bfloat16* vp = v + (size_t)unit * steps * D;
  const size_t qh0 = (size_t)b * Hq + (size_t)g * G;  // first query head of the group

  // element e of step t's (k, v, q_0..q_{G-1}) record
  auto fetch = [&](int t, int e) -> float {
    if (e < D) return __bfloat162float(kp[(size_t)t * D + e]);
    if (e < 2 * D) return __bfloat162float(vp[(size_t)t * D + e - D]);
    const int h = (e - 2 * D) / D, c = (e - 2 * D) % D;
    return __bfloat162float(q[((qh0 + h) * steps + t) * D + c]);
  };
  constexpr int kMaxPer = (kMaxGroup + 2) * 128 / kDecodeThreads;  // elements per thread per step
  float nxt[kMaxPer];
  const int nper = (per_step + kDecodeThreads - 1) / kDecodeThreads;
#pragma unroll
  for (int u = 0; u < kMaxPer; ++u) {
    const int e = tid + u * kDecodeThreads;
    if (u < nper && e < per_step) nxt[u] = fetch(0, e);
  }

  const int tx = tid % TPR, ty = tid / TPR;
  const int col = 4 * tx;
  float4* Su = reinterpret_cast<float4*>(S + (size_t)unit * D * D);
  float4 srow[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) srow[r] = __ldcs(Su + (size_t)(ty + r * RP) * TPR + tx);

  for (int t = 0; t < steps; ++t) {
    __syncthreads();  // the previous step is done with tok and red
#pragma unroll
    for (int u = 0; u < kMaxPer; ++u) {
      const int e = tid + u * kDecodeThreads;
      if (u < nper && e < per_step) tok[e] = nxt[u];
    }
    __syncthreads();
    if (t + 1 < steps) {  // next step's record, in flight while this one computes
#pragma unroll
      for (int u = 0; u < kMaxPer; ++u) {
        const int e = tid + u * kDecodeThreads;
        if (u < nper && e < per_step) nxt[u] = fetch(t + 1, e);
      }
    }
    const float4 vv = make_float4(tok[D + col], tok[D + col + 1], tok[D + col + 2], tok[D + col + 3]);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float kr = tok[ty + r * RP];
      srow[r].x = fmaf(kr, vv.x, srow[r].x);
      srow[r].y = fmaf(kr, vv.y, srow[r].y);
      srow[r].z = fmaf(kr, vv.z, srow[r].z);
      srow[r].w = fmaf(kr, vv.w, srow[r].w);
    }
    for (int h = 0; h < G; ++h) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float* qh = tok + 2 * D + h * D;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float qr = qh[ty + r * RP];
        acc.x = fmaf(qr, srow[r].x, acc.x);
        acc.y = fmaf(qr, srow[r].y, acc.y);
        acc.z = fmaf(qr, srow[r].z, acc.z);
        acc.w = fmaf(qr, srow[r].w, acc.w);
      }
      *reinterpret_cast<float4*>(red + ((size_t)h * RP + ty) * D + col) = acc;
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kDecodeThreads) {
      const int h = e / D, c = e % D;
      float sum = 0.f;
#pragma unroll
      for (int y = 0; y < RP; ++y) sum += red[((size_t)h * RP + y) * D + c];
      o[((qh0 + h) * steps + t) * D + c] = __float2bfloat16_rn(sum);
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) __stcs(Su + (size_t)(ty + r * RP) * TPR + tx, srow[r]);
}

template <int D>
cudaError_t launch_decode_steps_d(float* S, const void* q, const void* k, const void* v, void* o,
                                  int B, int Hq, int Hkv, int steps, cudaStream_t stream) {
  constexpr int RP = kDecodeThreads / (D / 4);
  const int G = Hq / Hkv;
  const size_t smem = sizeof(float) * ((size_t)(G + 2) * D + (size_t)G * RP * D);
  cudaError_t e = cudaFuncSetAttribute(decode_steps_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_steps_kernel<D><<<(unsigned)(B * Hkv), kDecodeThreads, smem, stream>>>(
      S, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), Hq, Hkv, steps);
  return cudaGetLastError();
}

// 512 threads (8 rows of S per thread at d = 128): more of each state in flight
// per SM than with 256 threads, so the loads of one CTA overlap the stores of
// another; measured 92.8 against 100.3 us per step on the decode workload.
// Groups above 16 query heads keep 256 threads (the per-row-group partial sums
// of 512 threads would not fit in shared memory).
template <int D, int NT>
cudaError_t launch_decode_nt(float* S, const void* q, const void* k, const void* v, void* o,
                             int B, int Hq, int Hkv, cudaStream_t stream) {
  constexpr int RP = NT / (D / 4);
  const int G = Hq / Hkv;
  const size_t smem = sizeof(float) * ((size_t)2 * D + (size_t)G * D + (size_t)G * RP * D);
  cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<D, NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_step_kernel<D, NT><<<(unsigned)(B * Hkv), NT, smem, stream>>>(
      S, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), Hq, Hkv);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(float* S, const void* q, const void* k, const void* v, void* o, int B,
                            int Hq, int Hkv, cudaStream_t stream) {
  if (Hq / Hkv <= 16) return launch_decode_nt<D, 512>(S, q, k, v, o, B, Hq, Hkv, stream);
  return launch_decode_nt<D, 256>(S, q, k, v, o, B, Hq, Hkv, stream);
}

}  // namespace

cudaError_t launch_decode_steps(float* S, const void* q, const void* k, const void* v, void* o,
                                int B, int Hq, int Hkv, int d, int steps, cudaStream_t stream) {
  if (Hq / Hkv > kMaxGroup) return cudaErrorInvalidValue;
  if (d == 128) return launch_decode_steps_d<128>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
  return launch_decode_steps_d<64>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
}

cudaError_t launch_decode(float* S, const void* q, const void* k, const void* v, void* o, int B,
                          int Hq, int Hkv, int d, cudaStream_t stream) {
  if (Hq / Hkv > kMaxGroup) return cudaErrorInvalidValue;
  if (d == 128) return launch_decode_d<128>(S, q, k, v, o, B, Hq, Hkv, stream);
  return launch_decode_d<64>(S, q, k, v, o, B, Hq, Hkv, stream);
}

}  // namespace la
