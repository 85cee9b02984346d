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
// Raises the release threshold of the current device's default memory pool
// once, so stream-ordered workspaces stay mapped between calls instead of
// being returned at every synchronisation (la_shutdown trims the pool).
// False if the current device cannot be queried.
bool keep_pool_memory();

// Pointer checks of a bf16 prefill call: q, k, v, o present and 16-byte
// aligned, S (nullable) aligned, o and S disjoint from each other and from
// q, k, v.  LA_OK or LA_ERR_INVALID_ARG.
la_status check_prefill_ptrs(const void* q, const void* k, const void* v, const void* o,
                             const void* S, int B, int Hq, int Hkv, int64_t N, int d);

// Builds a 3-D bf16 tensor map; returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows_per_head, int64_t heads,
                    int box_rows);
// 3-D fp32 tensor map over `units` d x d states [units, 128, 128]; box
// {32, 128, 1} (32 columns of one state), 128-byte swizzle.
bool make_tmap_state(CUtensorMap* map, const void* base, int64_t units);

// skip_last: spans 0 .. nspan-2 only (the last span's state is needed only
// for the final state).  parts: each span
// cut into `parts` sub-spans computed by separate CTAs (more CTAs when there
// are few sequences and spans); ws then holds nspan * parts states per
// sequence, in order.  first (parts == 1 only): spans before it are neither
// computed nor written (a backwards walk never needs span 0's sum).
cudaError_t launch_span_states(const PrefillGeometry& g, const CUtensorMap& k,
                               const CUtensorMap& v, float* ws, unsigned* status,
                               cudaStream_t stream, bool skip_last = false, int parts = 1,
                               int first = 0);
// Persistent chunk loop: min(B*Hkv*nspan, num_ctas) CTAs walk the items (one
// span of one (batch, kv head) sequence each, every query head of the group)
// round-robin.  ws: entering state of item bg * nspan + j (nullptr: zero);
// s_out (nullable): final states [B*Hkv, d, d], written by the items of the
// last spans; with nspan == 1 it may be ws itself.  ws_stride:
// entering state of item it at ws[it * ws_stride] (spans cut into parts).  dependent:
// launched as a programmatic dependent of the previous kernel in the stream.
// stage_states (honoured at tile 64, nspan == 1, forward, s_out null or ws):
// states pass through shared memory by bulk tensor copies, for short items
// where they are a large share of the bytes (see stage_states_pays).
cudaError_t launch_prefill_persist(const PrefillGeometry& g, const PrefillMaps& maps,
                                   const float* ws, float* s_out, unsigned* status, int num_ctas,
                                   cudaStream_t stream, bool dependent, bool stage_states,
                                   int ws_stride = 1);
// Whether staging the states pays for a one-span plan: the staged layout
// (two Q slots, output through a Q slot) streams tiles slower, so only items
// of at most four tiles use it.
bool stage_states_pays(const PrefillGeometry& g);
size_t fused_workspace_bytes(int B, int Hkv, int nspan);
// Sub-spans per span for the span-state pass of the forward: enough CTAs for
// the SMs when sequences x spans are few (1 when nspan == 1).
int span_parts(const la_plan& plan, int units, int sms);
// Workspace bytes la_forward_ws needs for `plan` (never zero): the span
// (sub-span) states, or nothing (a nominal 256 bytes) with one span per
// sequence, which runs as the persistent chunk loop alone with the state read
// and written in place.
size_t forward_workspace_bytes(const la_plan& plan);
// The whole prefill (validated arguments): one persistent chunk-loop launch
// when the plan has one span per sequence, else span states, scan and the
// persistent chunk loop; the span parts are lowered to what workspace_bytes
// holds (at least the plan's own workspace_bytes).
// final_out = false: S (nullable) supplies S0 only and is not written.
la_status forward_dispatch(const la_bf16* q, const la_bf16* k, const la_bf16* v, la_bf16* o,
                           float* S, int B, int Hq, int Hkv, int64_t N, const la_plan& plan,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream,
                           bool final_out = true);
cudaError_t launch_prefill_fused(const PrefillGeometry& g, const PrefillMaps& maps, float* S,
                                 void* workspace, unsigned* status, int num_sms, int lookahead,
                                 cudaStream_t stream);
// ws[j] <- S0 + sum_{i<j} ws[i] (the state entering entry j; S0 = *S or
// zero), and S receives S0 + sum_i ws[i].  nread < nspan: entries from nread
// on are not read, ws[nread] receives its entering state and S is only read
// (S0); nread < 0 means nspan.
cudaError_t launch_state_scan(float* ws, float* S, int units, int nspan, int d,
                              cudaStream_t stream, int nread = -1);
// S = S0 (nullable) + sum_{i < seg} states[i * per_seg_floats ...] (float4-wise).
cudaError_t launch_state_prefix(const float* states, const float* S0, float* S, int seg,
                                size_t per_seg_floats, cudaStream_t stream);
cudaError_t launch_decode(float* S, const void* q, const void* k, const void* v, void* o, int B,
                          int Hq, int Hkv, int d, cudaStream_t stream);
cudaError_t launch_decode_steps(float* S, const void* q, const void* k, const void* v, void* o,
                                int B, int Hq, int Hkv, int d, int steps, cudaStream_t stream);
cudaError_t launch_forward_simt_f32(const float* q, const float* k, const float* v, float* o,
                                    const float* S_in, float* S_out, int B, int Hq, int Hkv,
                                    int64_t N, int d, int chunk, cudaStream_t stream);
// Spans per kv group for the backward's dk/dv walk (each at least one
// 128-token chunk): the makespan of the walk plus the span pass it needs.
int walk_spans(int units, int tiles, int sms, int G);
// ent[bg][j] <- dSf[bg] (nullable: 0) + sum over the group's query heads and
// the spans after j of wsh[b*Hq + h][j'] (per-head span states of Q^T dO,
// span 0 not read); launched as a programmatic dependent of the span pass.
cudaError_t launch_group_scan(const float* wsh, const float* dSf, float* ent, int B, int Hq,
                              int Hkv, int nspan, cudaStream_t stream);
// dk, dv [B*Hkv, N, 128] of the backward in one anti-causal walk per (kv
// group, span): ws holds the entering state of item bg * nspan + j (nullable:
// zero; may be s_out when nspan == 1), s_out (nullable) receives dS0 from the
// items of span 0.  1 <= nspan <= ceil(N / 128).
cudaError_t launch_bwd_walk(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                            const la_bf16* dO, la_bf16* dk, la_bf16* dv, const float* ws,
                            float* s_out, unsigned* status, int B, int Hq, int Hkv, int64_t N,
                            int nspan, int num_ctas, cudaStream_t stream, bool dependent);
cudaError_t launch_selftest_wait(unsigned* status, int64_t timeout_ns, cudaStream_t stream);

}  // namespace la
