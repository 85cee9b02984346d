// la_simt.cu -- fp32 prefill with plain fp32 FMA (CUDA cores), for checking
// the method at fp32 precision.  Not tuned for speed.
//
// The chunk loop of the causal chunkwise sketch in
// "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座" (section "Lightning
// Attention：长上下文为什么突然变得便宜了"), per block of `chunk` tokens:
//     O_c = Q_c S + tril(Q_c K_c^T) V_c ;   S += K_c^T V_c
// with the diagonal kept by tril and a short last block.  One CTA per
// (batch, query head) walks all blocks in order; the state lives in shared
// memory in fp32.  Query heads of one kv group recompute the same state from
// S_in; the first head of the group writes the final state to S_out (a
// different buffer, so no CTA reads a state another one has already written).
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;

template <int D>
__global__ void __launch_bounds__(kSimtThreads)
    forward_simt_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                            const float* __restrict__ v, float* __restrict__ o,
                            const float* __restrict__ S_in, float* __restrict__ S_out, int Hq,
                            int Hkv, int64_t N, int C) {
  extern __shared__ float sh[];
  constexpr int KP = D + 1;              // padded key rows (lanes read different keys)
  float* Ss = sh;                        // [D][D]
  float* Ks = Ss + D * D;                // [C][D+1]
  float* Vs = Ks + C * KP;               // [C][D]
  float* sc = Vs + C * D;                // [warps][C] scores of the warp's row
  float* qb = sc + kSimtWarps * C;       // [warps][D] the warp's query row

  const int G = Hq / Hkv;
  const int b = blockIdx.x / Hq, h = blockIdx.x % Hq, g = h / G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qh = q + ((size_t)b * Hq + h) * N * D;
  float* oh = o + ((size_t)b * Hq + h) * N * D;
  const float* kg = k + ((size_t)b * Hkv + g) * N * D;
  const float* vg = v + ((size_t)b * Hkv + g) * N * D;
  const size_t soff = ((size_t)b * Hkv + g) * D * D;

  for (int e = tid; e < D * D; e += kSimtThreads) Ss[e] = S_in ? S_in[soff + e] : 0.f;
  __syncthreads();

  for (int64_t c0 = 0; c0 < N; c0 += C) {
    const int len = (int)((N - c0) < C ? (N - c0) : C);
    for (int e = tid; e < len * D; e += kSimtThreads) {
      const int s = e / D, i = e % D;
      Ks[s * KP + i] = kg[(c0 + s) * D + i];
      Vs[s * D + i] = vg[(c0 + s) * D + i];
    }
    __syncthreads();
    float* myq = qb + warp * D;
    float* mys = sc + warp * C;
    for (int t = warp; t < len; t += kSimtWarps) {
      for (int i = lane; i < D; i += 32) myq[i] = qh[(c0 + t) * D + i];
      __syncwarp();
      for (int s = lane; s <= t; s += 32) {  // intra-block scores, s <= t
        float a = 0.f;
        for (int i = 0; i < D; ++i) a = fmaf(myq[i], Ks[s * KP + i], a);
        mys[s] = a;
      }
      __syncwarp();
      for (int jcol = lane; jcol < D; jcol += 32) {
        float acc = 0.f;
        for (int i = 0; i < D; ++i) acc = fmaf(myq[i], Ss[i * D + jcol], acc);  // Q_c S
        for (int s = 0; s <= t; ++s) acc = fmaf(mys[s], Vs[s * D + jcol], acc);  // tril(QK^T) V
        oh[(c0 + t) * D + jcol] = acc;
      }
      __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < D * D; e += kSimtThreads) {  // S += K_c^T V_c
      const int i = e / D, jcol = e % D;
      float acc = Ss[e];
      for (int s = 0; s < len; ++s) acc = fmaf(Ks[s * KP + i], Vs[s * D + jcol], acc);
      Ss[e] = acc;
    }
    __syncthreads();
  }
  if (S_out && h % G == 0)
    for (int e = tid; e < D * D; e += kSimtThreads) S_out[soff + e] = Ss[e];
}

template <int D>
cudaError_t launch_simt_d(const float* q, const float* k, const float* v, float* o,
                          const float* S_in, float* S_out, int B, int Hq, int Hkv, int64_t N,
                          int C, cudaStream_t stream) {
  const size_t smem = sizeof(float) * ((size_t)D * D + (size_t)C * (D + 1) + (size_t)C * D +
                                       (size_t)kSimtWarps * C + (size_t)kSimtWarps * D);
  cudaError_t e = cudaFuncSetAttribute(forward_simt_f32_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  forward_simt_f32_kernel<D><<<(unsigned)(B * Hq), kSimtThreads, smem, stream>>>(
      q, k, v, o, S_in, S_out, Hq, Hkv, N, C);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_simt_f32(const float* q, const float* k, const float* v, float* o,
                                    const float* S_in, float* S_out, int B, int Hq, int Hkv,
                                    int64_t N, int d, int chunk, cudaStream_t stream) {
  if (d == 128) return launch_simt_d<128>(q, k, v, o, S_in, S_out, B, Hq, Hkv, N, chunk, stream);
  return launch_simt_d<64>(q, k, v, o, S_in, S_out, B, Hq, Hkv, N, chunk, stream);
}

}  // namespace la
