// la_internal.h -- launch helpers shared by the translation units of the
// library (host side only; not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la.h"

namespace la {

constexpr int kHeadDim = 128;   // head dim of the tensor-core path
constexpr int kTileRows = 128;  // rows of one tcgen05 M=128 tile

struct PrefillGeometry {
  int B, Hq, Hkv, G;
  int64_t N;
  int tile;            // tokens per tile (T)
  int heads_per_tile;  // HPT, tile * HPT == 128
  int tiles_total;     // ceil(N / T)
  int nspan;           // spans per (b, kv head)
};

// Tensor maps for one call: q, o over [B*Hq, N, 128]; k, v over [B*Hkv, N, 128];
// box {64, tile, 1}, 128-byte swizzle, bf16.
struct PrefillMaps {
  CUtensorMap q, k, v, o;
};

// Device address of the status word on the current device (nullptr on failure).
unsigned* device_status_ptr();

// Builds a 3-D bf16 tensor map; returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows_per_head, int64_t heads,
                    int box_rows);

cudaError_t launch_span_states(const PrefillGeometry& g, const CUtensorMap& k,
                               const CUtensorMap& v, float* ws, unsigned* status,
                               cudaStream_t stream);
// qdiv: query rows of head h come from head h / qdiv of the query tensor map;
// reverse: anti-causal pass (sum over s >= t), the tiles of every span walked
// from the end.  The forward pass is qdiv = 1, reverse = 0.  ws == nullptr
// starts every span from a zero state.  s_out (nspan == 1 only; else
// cudaErrorInvalidValue): the final state [B*Hkv, d, d] is written there; when
// s_out is ws itself (in place) and G / heads_per_tile > 1, tickets must point
// to B*Hkv zeroed counters.
cudaError_t launch_prefill_main(const PrefillGeometry& g, const PrefillMaps& maps,
                                const float* ws, unsigned* status, cudaStream_t stream,
                                int qdiv = 1, int reverse = 0, float* s_out = nullptr,
                                unsigned* tickets = nullptr);
size_t fused_workspace_bytes(int B, int Hkv, int nspan);
// The whole bf16 prefill of a plan with nspan == 1 as one chunk-loop launch
// that reads S (nullable: zero) and writes the final state back into it.
// `tickets`: device memory for B*Hkv counters (zeroed here), needed when S is
// given and a kv group spans several CTAs.  Arguments already validated.
la_status forward_single_span(const la_bf16* q, const la_bf16* k, const la_bf16* v, la_bf16* o,
                              float* S, int B, int Hq, int Hkv, int64_t N, const la_plan& plan,
                              unsigned* tickets, cudaStream_t stream);
// Workspace bytes la_forward_ws needs for `plan`: the span states, or only
// the tickets of the single-span launch.
size_t forward_workspace_bytes(const la_plan& plan, int B, int Hkv);
cudaError_t launch_prefill_fused(const PrefillGeometry& g, const PrefillMaps& maps, float* S,
                                 void* workspace, unsigned* status, int num_sms, int lookahead,
                                 cudaStream_t stream);
// reverse: ws[j] <- S0 + sum_{i>j} ws[i] (the state entering span j of a
// backwards walk); S receives S0 + sum_i ws[i] either way.
cudaError_t launch_state_scan(float* ws, float* S, int units, int nspan, int d,
                              cudaStream_t stream, int reverse = 0);
cudaError_t launch_decode(float* S, const void* q, const void* k, const void* v, void* o, int B,
                          int Hq, int Hkv, int d, cudaStream_t stream);
cudaError_t launch_decode_steps(float* S, const void* q, const void* k, const void* v, void* o,
                                int B, int Hq, int Hkv, int d, int steps, cudaStream_t stream);
cudaError_t launch_forward_simt_f32(const float* q, const float* k, const float* v, float* o,
                                    const float* S_in, float* S_out, int B, int Hq, int Hkv,
                                    int64_t N, int d, int chunk, cudaStream_t stream);
cudaError_t launch_selftest_wait(unsigned* status, int64_t timeout_ns, cudaStream_t stream);

}  // namespace la
