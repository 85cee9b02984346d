// la_scan.cu -- exclusive prefix over span states (the second prefill stage).
//
// The state entering span j of a (batch, kv head) is S0 + sum_{i<j} K_i^T V_i,
// where K_i^T V_i is span i's contribution; the state after the last span is
// the final state S0 + K^T V ("MiniMax-01与Lightning Attention", section 2.2,
// kv_sum over the whole sequence).  When the chunk loop writes the final state
// itself, the last span's K^T V is never computed (nread < nspan) and only the
// entering states are written.  Elementwise fp32 adds, HBM/L2-bound: one
// thread owns two float4 of the d x d matrix of one unit and walks the spans
// in order, eight spans at a time with all their loads issued before the
// stores, so a short scan costs one round trip to memory, not one per span.
// Two float4 per thread keep the grid small (at most a few 256-thread CTAs
// per SM), so the chunk-loop kernel, launched behind it, finds room to start
// its copies early.  Launched as a programmatic dependent of the span-state
// kernel: it lets the chunk-loop kernel start its copies, then waits for the
// span states.
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_ptx.cuh"

namespace la {
namespace {

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

constexpr int kScanVec = 1;  // float4 per thread
constexpr int kScanBatch = 4;  // spans whose loads are issued together

__global__ void __launch_bounds__(256)
    state_scan_kernel(float4* __restrict__ ws, float4* __restrict__ S, int nspan, int n4,
                      int blocks_per_unit, int nread) {
  griddep_launch_dependents();  // the chunk-loop kernel may start its copies
  griddep_wait();               // the span states are complete
  const size_t unit = blockIdx.x / blocks_per_unit;
  const int p0 = (blockIdx.x % blocks_per_unit) * (blockDim.x * kScanVec) + threadIdx.x;
  float4* w = ws + unit * (size_t)nspan * n4;
  int pos[kScanVec];
  bool in[kScanVec];
  float4 carry[kScanVec];
#pragma unroll
  for (int e = 0; e < kScanVec; ++e) {
    pos[e] = p0 + e * (int)blockDim.x;
    in[e] = pos[e] < n4;
    carry[e] = (S && in[e]) ? S[unit * n4 + pos[e]] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // nread < nspan: entries from nread on were not computed (they only feed
  // the final state); the entering state of entry nread is written, no final
  for (int j = 0; j < nread; j += kScanBatch) {
    float4 x[kScanVec][kScanBatch];
#pragma unroll
    for (int e = 0; e < kScanVec; ++e)
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u)
        if (in[e] && j + u < nread) x[e][u] = w[(size_t)(j + u) * n4 + pos[e]];
#pragma unroll
    for (int e = 0; e < kScanVec; ++e)
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u)
        if (in[e] && j + u < nread) {
          w[(size_t)(j + u) * n4 + pos[e]] = carry[e];
          carry[e] = add4(carry[e], x[e][u]);
        }
  }
#pragma unroll
  for (int e = 0; e < kScanVec; ++e) {
    if (!in[e]) continue;
    if (nread < nspan)
      w[(size_t)nread * n4 + pos[e]] = carry[e];
    else if (S)
      S[unit * n4 + pos[e]] = carry[e];
  }
}

}  // namespace

cudaError_t launch_state_scan(float* ws, float* S, int units, int nspan, int d,
                              cudaStream_t stream, int nread) {
  if (nread < 0) nread = nspan;
  if (nread < 1 || nread > nspan) return cudaErrorInvalidValue;
  const int n4 = d * d / 4;
  const int bpu = (n4 + 256 * kScanVec - 1) / (256 * kScanVec);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * bpu));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, state_scan_kernel, reinterpret_cast<float4*>(ws),
                            reinterpret_cast<float4*>(S), nspan, n4, bpu, nread);
}

namespace {

// S[u] = S0[u] (or 0) + sum_{i < seg} states[i][u], one float4 per thread.
__global__ void __launch_bounds__(256)
    state_prefix_kernel(const float4* __restrict__ states, const float4* S0, float4* S,
                        int seg, size_t per_seg4) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= per_seg4) return;
  float4 acc = S0 ? S0[e] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < seg; ++i) acc = add4(acc, states[(size_t)i * per_seg4 + e]);
  S[e] = acc;
}

}  // namespace

cudaError_t launch_state_prefix(const float* states, const float* S0, float* S, int seg,
                                size_t per_seg_floats, cudaStream_t stream) {
  const size_t n4 = per_seg_floats / 4;
  state_prefix_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(states), reinterpret_cast<const float4*>(S0),
      reinterpret_cast<float4*>(S), seg, n4);
  return cudaGetLastError();
}

}  // namespace la
