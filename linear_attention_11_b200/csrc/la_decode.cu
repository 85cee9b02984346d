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
// about 1.2 flop/byte): HBM-bound.  One CTA per unit, 512 threads (256 for
// groups above 16 query heads); a warp reads one row of S as 32 contiguous
// float4 (512 B, fully coalesced), each thread keeps its updated rows in
// registers for the G dot products.  The sum over rows of o_h = q_h S runs
// across warps (the lanes of a warp hold different columns, which is what
// makes the row reads coalesced), so the per-row-group partial sums are
// reduced through shared memory rather than by warp shuffles.  S is read and
// written exactly once with streaming cache hints.  The multi-step kernel
// keeps half a state column per thread and does shuffle its dot products.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

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
// order -- the same recurrence as decode_step_kernel, applied `steps` times,
// with the same fmaf(k_r, v_c, S_rc) per element, so the state is bit for bit
// that of single steps.  Inputs follow the prefill layout with N = steps:
// q, o [B, Hq, steps, D], k, v [B, Hkv, steps, D].
//
// Two threads per state column c (2 D threads per unit), each holding half
// of the column (D / 2 rows) in registers: the update is elementwise and
// o_{t,h}[c] is a dot product over rows, so each thread sums its half and
// the pair (adjacent lanes) adds the two halves with one shuffle.  k and q
// come from shared memory as broadcast float4 reads, each half stored with a
// 4-float pad so the two halves of a warp read different banks.  Query heads
// go in passes of GB (the update rides on the first pass).  The next step's
// k, v, q are loaded into registers while the current step computes, then
// written to the other half of a double buffer: one barrier per step.
// Two CTAs per SM (128 registers at d = 128), except 2- and 8-head passes at
// d = 128, which would spill at that bound.
template <int D, int GB>
__global__ void __launch_bounds__(2 * D, (D == 128 && (GB == 8 || GB == 2)) ? 1 : 2)
    decode_steps_kernel(float* __restrict__ S, const __nv_bfloat16* __restrict__ q,
                        const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                        __nv_bfloat16* __restrict__ o, int Hq, int Hkv, int steps) {
  constexpr int R = D / 2;   // rows per thread
  constexpr int RP = R + 4;  // padded stride of one half row in shared memory
  extern __shared__ float4 sh4[];
  float* sh = reinterpret_cast<float*>(sh4);
  const int G = Hq / Hkv;
  // one step's record: k and q_0 .. q_{G-1} as [2][RP] halves, then v [D]
  const int rec = 2 * RP * (G + 1) + D;
  auto row_off = [&](int j) { return j == 1 ? 2 * RP * (G + 1) : 2 * RP * (j == 0 ? 0 : j - 1); };
  const int unit = blockIdx.x;  // b * Hkv + g
  const int b = unit / Hkv, g = unit % Hkv;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int c = (tid >> 5) * 16 + (lane >> 1);  // state column
  const int half = lane & 1;                    // rows [half * R, half * R + R)
  const size_t qh0 = (size_t)b * Hq + (size_t)g * G;  // first query head of the group

  // staging: thread tid brings element e = tid % D of the record's rows j with
  // j % 2 == tid / D (rows: 0 = k, 1 = v, 2 + h = q_h)
  const int e = tid % D, jpar = tid / D;
  const int eo = e < R ? e : RP + (e - R);  // its place in a split row
  constexpr int kMaxG = GB == 8 ? kMaxGroup : 2 * GB - 1;
  constexpr int kMaxRows = (2 + kMaxG + 1) / 2;
  __nv_bfloat16 pre[kMaxRows];
  auto row_src = [&](int j, int t) -> const __nv_bfloat16* {
    if (j == 0) return k + ((size_t)unit * steps + t) * D;
    if (j == 1) return v + ((size_t)unit * steps + t) * D;
    return q + ((qh0 + (j - 2)) * steps + t) * D;
  };
  auto fetch = [&](int t) {
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) {
      const int j = 2 * m + jpar;
      if (j < 2 + G) pre[m] = row_src(j, t)[e];
    }
  };
  auto stash = [&](float* buf) {
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) {
      const int j = 2 * m + jpar;
      if (j < 2 + G) buf[row_off(j) + (j == 1 ? e : eo)] = __bfloat162float(pre[m]);
    }
  };

  float s[R];
  const float* Su = S + (size_t)unit * D * D + (size_t)half * R * D + c;
#pragma unroll
  for (int r = 0; r < R; ++r) s[r] = __ldcs(Su + (size_t)r * D);
  fetch(0);
  stash(sh);
  __syncthreads();

  __nv_bfloat16* op = o + qh0 * steps * D + c;
  for (int t = 0; t < steps; ++t) {
    const float* buf = sh + (size_t)(t & 1) * rec;
    if (t + 1 < steps) fetch(t + 1);  // in flight while this step computes
    const float vc = buf[2 * RP * (G + 1) + c];
    const float4* k4 = reinterpret_cast<const float4*>(buf + half * RP);
    for (int hb = 0; hb < G; hb += GB) {
      float acc[GB][2];  // two partial sums per head: shorter chains
#pragma unroll
      for (int j = 0; j < GB; ++j) acc[j][0] = acc[j][1] = 0.f;
      const int nh = G - hb;  // heads left; a short last pass is predicated
#pragma unroll
      for (int r4 = 0; r4 < R / 4; ++r4) {
        if (hb == 0) {
          const float4 kk = k4[r4];
          s[4 * r4 + 0] = fmaf(kk.x, vc, s[4 * r4 + 0]);
          s[4 * r4 + 1] = fmaf(kk.y, vc, s[4 * r4 + 1]);
          s[4 * r4 + 2] = fmaf(kk.z, vc, s[4 * r4 + 2]);
          s[4 * r4 + 3] = fmaf(kk.w, vc, s[4 * r4 + 3]);
        }
#pragma unroll
        for (int j = 0; j < GB; ++j) {
          if (j < nh) {
            const float4 qq =
                reinterpret_cast<const float4*>(buf + 2 * RP * (1 + hb + j) + half * RP)[r4];
            float& a = acc[j][r4 & 1];
            a = fmaf(qq.x, s[4 * r4 + 0], a);
            a = fmaf(qq.y, s[4 * r4 + 1], a);
            a = fmaf(qq.z, s[4 * r4 + 2], a);
            a = fmaf(qq.w, s[4 * r4 + 3], a);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < GB; ++j) {
        if (j < nh) {  // uniform over the warp
          float a = acc[j][0] + acc[j][1];
          a += __shfl_xor_sync(0xffffffffu, a, 1);  // the other half of the column
          if (half == 0) op[((size_t)(hb + j) * steps + t) * D] = __float2bfloat16_rn(a);
        }
      }
    }
    if (t + 1 < steps) stash(sh + (size_t)((t + 1) & 1) * rec);
    __syncthreads();  // the next step's record is complete; this step's is no longer read
  }
  float* Sw = S + (size_t)unit * D * D + (size_t)half * R * D + c;
#pragma unroll
  for (int r = 0; r < R; ++r) __stcs(Sw + (size_t)r * D, s[r]);
}

template <int D, int GB>
cudaError_t launch_decode_steps_gb(float* S, const void* q, const void* k, const void* v, void* o,
                                   int B, int Hq, int Hkv, int steps, cudaStream_t stream) {
  const int G = Hq / Hkv;
  const size_t smem = sizeof(float) * 2 * (size_t)(2 * (D / 2 + 4) * (G + 1) + D);
  cudaError_t e = cudaFuncSetAttribute(decode_steps_kernel<D, GB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_steps_kernel<D, GB><<<(unsigned)(B * Hkv), 2 * D, smem, stream>>>(
      S, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), Hq, Hkv, steps);
  return cudaGetLastError();
}

// Heads per pass: the largest power of two up to min(G, 8), so groups of 1, 2,
// 4 and 8 heads take one pass with no predicated-off work.
template <int D>
cudaError_t launch_decode_steps_d(float* S, const void* q, const void* k, const void* v, void* o,
                                  int B, int Hq, int Hkv, int steps, cudaStream_t stream) {
  const int G = Hq / Hkv;
  if (G >= 8) return launch_decode_steps_gb<D, 8>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
  if (G >= 4) return launch_decode_steps_gb<D, 4>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
  if (G >= 2) return launch_decode_steps_gb<D, 2>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
  return launch_decode_steps_gb<D, 1>(S, q, k, v, o, B, Hq, Hkv, steps, stream);
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
