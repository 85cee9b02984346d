/*
 * la.h -- C ABI of the causal Lightning Attention library for B200 (sm_100a).
 *
 * Sources cited by page title and section:
 *   [MX01] "MiniMax-01与Lightning Attention": section 1.1 (128 attention heads,
 *          32 kv heads), 2.2 (linear attention by associativity, kv_sum =
 *          K^T V), 2.3 (tiled state updates), 4.1 (incremental kv state).
 *   [VGX]  "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座", section
 *          "Lightning Attention：长上下文为什么突然变得便宜了": the causal
 *          chunkwise sketch (per block: inter term Q_b S, masked intra term
 *          tril(Q_b K_b^T) V_b, then S += K_b^T V_b; the state starts at zero;
 *          the last block may be short).
 *
 * What the library computes.  For every batch b and query head h, with
 * g = floor(h / (Hq/Hkv)) the kv head h shares:
 *
 *     O[b,h,t,:] = q[b,h,t] S0[b,g] + sum_{s <= t} (q[b,h,t] . k[b,g,s]) v[b,g,s,:]
 *     S[b,g]     = S0[b,g] + sum_s k[b,g,s]^T v[b,g,s]          (final state)
 *
 * chunk by chunk as [VGX] lays it out: O_c = Q_c S_{<c} + tril(Q_c K_c^T) V_c,
 * then S += K_c^T V_c.  No softmax, no normalisation, no decay, no scaling (the
 * 1/sqrt(d) factor belongs to the inputs).  S0 is zero unless given.
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned DEVICE memory, contiguous, row-major:
 *       q, o  [B, Hq,  N, d]      k, v  [B, Hkv, N, d]      S  [B, Hkv, d, d]
 *     S[b,g][i][j] pairs key feature i with value feature j.  The library never
 *     frees, reallocates or keeps pointers to caller memory after a call.
 *   - la_bf16 is the bit pattern of a bfloat16.  Outputs have the input dtype;
 *     states are fp32; all accumulation is fp32.
 *   - Every tensor pointer must be 16-byte aligned (the bulk tensor copies
 *     require it); o must not overlap q, k, v or S.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and launch on the device current to the calling thread.
 *   - Return codes report argument validation and launch errors only.  A fault
 *     during execution surfaces at the caller's next synchronisation; a bounded
 *     device-side wait that expires sets the device status word, read with
 *     la_device_status().
 */
#ifndef LIGHTNING_B200_LA_H
#define LIGHTNING_B200_LA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, Hq % Hkv != 0, misalignment, overlap */
  LA_ERR_UNSUPPORTED = 2, /* head dim or chunk size the library does not implement */
  LA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  LA_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired (see la_device_status) */
  LA_ERR_WORKSPACE = 5    /* workspace pointer missing, misaligned or too small */
} la_status;

typedef uint16_t la_bf16; /* bfloat16 bits */
typedef void *la_stream;  /* cudaStream_t */

/* Device status word bits, set by kernels, read by la_device_status(). */
#define LA_DEV_TIMEOUT 0x1u /* a bounded mbarrier / flag wait gave up */

/* Human-readable name of a status code (static storage, never NULL). */
const char *la_status_string(la_status s);

/* Library ABI version (this header: 1). */
int la_version(void);

/* ------------------------------------------------------------------------
 * Prefill, bf16 -- the hot path.  Tensor-core (tcgen05) kernels, d == 128.
 *
 * la_forward: O only, zero initial state ([VGX] sketch; rows a1-a9 of the
 * method).  chunk is the block length of the masked intra-chunk product,
 * 64 or 128; any N >= 1 is accepted (the last chunk may be short, as in the
 * sketch's end = min(start + block, n)).
 *
 * Query heads are grouped with their kv head ([MX01] section 1.1, GQA): one
 * 128-row tensor-core tile holds 128/chunk query heads of a group times chunk
 * tokens.  A group with a single query head at chunk 64 stacks two
 * consecutive 64-token chunks into one 128-token tile with the full causal
 * mask -- the same sum in exact arithmetic, since the chunked form is exact for
 * every block length.
 *
 * Uses a workspace for the per-span states: la_forward / la_forward_state take
 * it from the device's default stream-ordered memory pool (cudaMallocAsync and
 * cudaFreeAsync on `stream`; the pool keeps the memory cached between calls),
 * la_forward_ws takes one from the caller.  The chunk loop is a persistent
 * kernel: one CTA per SM walks work items (a span of one (batch, kv head)
 * sequence with all its query heads).  When the plan has one span per
 * sequence -- many sequences or kv heads, short N -- the call is that one
 * launch: it reads the initial state and writes the final one itself, and
 * needs no workspace (la_forward_workspace_bytes returns a nominal 256).
 *
 * Errors: LA_ERR_INVALID_ARG (null or misaligned pointer, B/Hq/Hkv/N <= 0,
 * Hq % Hkv, o overlapping an input), LA_ERR_UNSUPPORTED (d != 128, chunk not
 * in {64, 128}), LA_ERR_CUDA (allocation or launch failure).
 * ---------------------------------------------------------------------- */
la_status la_forward(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o, int B,
                     int Hq, int Hkv, int64_t N, int d, int chunk, la_stream stream);

/* As la_forward, plus a state.  S (nullable) is [B,Hkv,d,d] fp32 device
 * memory: on entry the initial state S0, on return the final state
 * S0 + K^T V ([MX01] section 4.1: the state is the whole resume point, so a
 * sequence may be processed in pieces).  S == NULL means S0 = 0, no state out. */
la_status la_forward_state(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                           float *S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                           la_stream stream);

/* Bytes of workspace la_forward_ws needs for this problem on the current device. */
size_t la_forward_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int d, int chunk);

/* As la_forward_state with a caller-owned device workspace (256-byte aligned,
 * at least la_forward_workspace_bytes()); LA_ERR_WORKSPACE otherwise.  The
 * workspace must not be used by anything else until the call's work on
 * `stream` has finished. */
la_status la_forward_ws(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                        float *S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                        void *workspace, size_t workspace_bytes, la_stream stream);

/* ------------------------------------------------------------------------
 * Prefill from and to HOST memory, transfers pipelined against the compute.
 * q, k, v, o are host pointers, page-locked (cudaHostAlloc / cudaHostRegister)
 * so the copies run asynchronously, in the layouts above; S (nullable) is a
 * DEVICE state as in la_forward_state.  The sequence is processed in pieces of
 * `piece` tokens (0: about N/16; rounded up to whole tiles): piece p is copied
 * in on a copy-in stream, computed on `stream` with the state carried from
 * piece p-1 ([MX01] section 4.1: the state is the whole resume point), and
 * copied out on a copy-out stream, so the two copy directions and the compute
 * of neighbouring pieces overlap.  Same result as la_forward_state on the
 * whole sequence (up to the rounding of the bf16 state copy at piece ends).
 * Asynchronous: returns once the work is queued; the host buffers must stay
 * valid and unmodified until `stream` has reached the end of the call.  Device
 * buffers for two pieces come from the stream-ordered pool and go back to it.
 * Errors as la_forward_state; piece < 0 is LA_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------- */
la_status la_forward_host(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                          float *S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                          int64_t piece, la_stream stream);

/* ------------------------------------------------------------------------
 * The prefill as one single-pass persistent kernel (an alternative schedule
 * of the same arithmetic, slower; la_forward runs the span states, the scan
 * and the persistent chunk loop of the stages below).  Every (batch, kv head)
 * sequence is cut into `nspan` spans; span-state items (K^T V of a span, then the chained prefix: the state
 * entering the next span) and chunk-loop items (the chunk loop of one span for
 * a group of query heads, from its entering state) are taken in rounds, one
 * round per span index, so the chunk loops of a span re-read its K and V from
 * L2 right after the span-state item has read them from HBM.  The entering
 * states are published through GPU-scope flags; every wait is bounded.
 *   nspan <= 0 picks the span count for the problem and device; otherwise
 *   1 <= nspan <= ceil(N / tile) (tile = la_plan.tile).
 *   lookahead: how many rounds the span-state items run ahead of the chunk
 *   loops that need them (<= 0: 1; capped at nspan).
 *   workspace: device memory, 256-byte aligned, at least
 *   la_prefill_fused_workspace_bytes(..., nspan) bytes (entering states and
 *   flags); the call clears the flags on `stream` first (cudaMemsetAsync).
 * Errors as la_forward_ws.
 * ---------------------------------------------------------------------- */
size_t la_prefill_fused_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                                        int nspan);
la_status la_prefill_fused(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                           float *S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                           int nspan, int lookahead, void *workspace, size_t workspace_bytes,
                           la_stream stream);

/* ------------------------------------------------------------------------
 * Prefill without any device allocation.  The pages have no counterpart to
 * this entry point: it exists for callers that cannot allocate device memory
 * at call time (code inside an allocator or memory-pool callback, frameworks
 * that own every device byte, paths that must not block in the driver's
 * allocator).  Same arguments, results and errors as la_forward_state, with
 * the span-state workspace taken from one 32 MiB file-scope device array
 * instead of an allocation; every GPU that loads this part of the library
 * keeps that array until the process exits.
 *   - Limit: the span states (B * Hkv * nspan * d * d * 4 bytes) must fit in
 *     32 MiB; the span count is lowered until they do, down to one span per
 *     (batch, kv head), which runs as the single chunk-loop launch and needs
 *     no workspace, so every problem size is accepted.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress).  With lazy module loading that lookup, like
 *     the first launch of each kernel, loads the module holding the array
 *     and so allocates device memory.  Make one warm-up call per device,
 *     outside any context where allocation is forbidden and before any
 *     stream capture; calls after it allocate nothing.
 *   - All calls share the array: calls whose work overlaps on the GPU race
 *     and must be serialised by the caller.  Each call writes every entry it
 *     reads, so nothing from an earlier call needs clearing.
 * ---------------------------------------------------------------------- */
la_status la_forward_noalloc(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                             float *S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                             la_stream stream);

/* ------------------------------------------------------------------------
 * The prefill's three stages -- the scheme the la_forward* calls run -- for
 * callers that schedule or time them apart: plan, then span_states, scan,
 * main on one stream.  (The la_forward* calls refine it: without a state to
 * return they skip the last span's K^T V, they cut spans into sub-spans for
 * the first stage when sequences x spans are fewer than the SMs, and with
 * one span per sequence they run the chunk loop alone.)
 *
 * The sequence of every (batch, kv head) is cut into `nspan` spans of whole
 * chunks.  span_states writes each span's K^T V into the workspace; scan turns
 * those into the state entering each span (S0 + the spans before it) and, if S
 * is given, writes the final state; main runs the chunked loop of every span
 * from its entering state.  This split is not on the pages: the chunk loop of
 * the [VGX] sketch is sequential, and spans let one sequence fill the GPU.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t nspan;           /* spans per (batch, kv head) */
  int32_t tile;            /* tokens per 128-row tile: chunk, or 128 when stacking two 64-chunks */
  int32_t heads_per_tile;  /* query heads stacked in one tile (tile * heads_per_tile == 128) */
  int32_t tiles_total;     /* ceil(N / tile) */
  int64_t workspace_bytes; /* B * Hkv * nspan * d * d * 4 */
} la_plan;

/* Fill *plan for this problem on the current device.  Errors as la_forward. */
la_status la_prefill_plan(int B, int Hq, int Hkv, int64_t N, int d, int chunk, la_plan *plan);

/* Stage 1: ws[b,g,j] = sum over span j of K_c^T V_c (fp32, [B,Hkv,nspan,d,d]). */
la_status la_prefill_span_states(const la_bf16 *k, const la_bf16 *v, int B, int Hkv, int64_t N,
                                 int d, const la_plan *plan, float *ws, la_stream stream);

/* Stage 2, in place: ws[b,g,j] <- S0[b,g] + sum_{i<j} ws[b,g,i].  S (nullable)
 * supplies S0 on entry and receives S0 + sum_i ws[b,g,i] on return. */
la_status la_prefill_scan(float *ws, float *S, int B, int Hkv, int d, const la_plan *plan,
                          la_stream stream);

/* Stage 3: O for every span, starting each from ws[b,g,j] (the persistent
 * chunk loop: min(B * Hkv * nspan, SM count) CTAs walk the spans round-robin). */
la_status la_prefill_main(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, la_bf16 *o,
                          const float *ws, int B, int Hq, int Hkv, int64_t N, int d,
                          const la_plan *plan, la_stream stream);

/* ------------------------------------------------------------------------
 * Sequence sharding: one sequence cut into nseg consecutive segments (one per
 * GPU, say).  The state entering segment r is S0 + sum_{i<r} K_i^T V_i (the
 * state is the whole resume point of the recurrence, [MX01] section 4.1,
 * "Streaming"; K^T V of a segment is its kv_sum, section 2.2).  Each holder
 * of a segment computes its K^T V, the nseg states are exchanged (an
 * all-gather: B*Hkv*d*d*4 bytes per segment), each takes the prefix of the
 * segments before its own, and runs la_forward_state from it.
 *
 * la_segment_state: S [B,Hkv,d,d] fp32 (device, 16-byte aligned, written)
 * <- K^T V of this segment's k, v [B,Hkv,N,d] bf16; d = 128, chunk as
 * la_forward.  Errors as la_forward.
 * la_state_prefix: S [B,Hkv,d,d] <- S0 (nullable: 0) + sum_{i<seg} states[i],
 * states [nseg,B,Hkv,d,d] fp32 contiguous (segment-major, as an all-gather
 * lays it out), 0 <= seg < nseg; S may be S0 but must not overlap states.
 * LA_ERR_INVALID_ARG on bad sizes or pointers.
 * ---------------------------------------------------------------------- */
la_status la_segment_state(const la_bf16 *k, const la_bf16 *v, float *S, int B, int Hkv,
                           int64_t N, int d, int chunk, la_stream stream);
la_status la_state_prefix(const float *states, const float *S0, float *S, int nseg, int seg,
                          int B, int Hkv, int d, la_stream stream);

/* ------------------------------------------------------------------------
 * Backward of the bf16 prefill (training).  For a loss with gradient dO
 * [B,Hq,N,d] on the output and dSf [B,Hkv,d,d] (nullable = 0) on the final
 * state, with S0 (nullable = 0) the initial state of the forward call:
 *   dq_t = do_t S0^T + sum_{s<=t} (do_t . v_s) k_s
 *   dk_s = sum_{h in group} sum_{t>=s} (v_s . do_{t,h}) q_{t,h} + v_s dSf^T
 *   dv_s = sum_{h in group} sum_{t>=s} (k_s . q_{t,h}) do_{t,h} + k_s dSf
 *   dS0  = dSf + sum_{h in group} sum_t q_{t,h}^T do_{t,h}    (dS0 nullable)
 * (the chain rule through o_t = q_t S_t, S_t = S0 + sum_{s<=t} k_s^T v_s of
 * [VGX]).  dq is the forward pass itself on (dO, V, K, S0^T); dk and dv come
 * from one anti-causal walk per kv group (chunks last to first, every query
 * head of the group summed inside the tensor-core products, spans of it in
 * parallel).  dS0 may be dSf.  dq [B,Hq,N,d], dk, dv [B,Hkv,N,d] bf16 outputs
 * (no overlap with the inputs).  Scratch comes from the stream-ordered pool.
 * d = 128, chunk in {64, 128} (the chunk of the dq pass; the others use 128).
 * Errors as la_forward_state. */
la_status la_backward(const la_bf16 *q, const la_bf16 *k, const la_bf16 *v, const la_bf16 *dO,
                      const float *S0, const float *dSf, la_bf16 *dq, la_bf16 *dk, la_bf16 *dv,
                      float *dS0, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                      la_stream stream);

/* ------------------------------------------------------------------------
 * Prefill in fp32 (inputs, output and state fp32; SIMT fp32 arithmetic).
 * Same definition and arguments as la_forward_state; d in {64, 128}, chunk in
 * {64, 128}.  For checking at fp32 precision, not tuned for speed.
 * ---------------------------------------------------------------------- */
la_status la_forward_f32(const float *q, const float *k, const float *v, float *o, float *S,
                         int B, int Hq, int Hkv, int64_t N, int d, int chunk, la_stream stream);

/* ------------------------------------------------------------------------
 * Decode step: one new token per sequence on the recurrent state
 * ([MX01] section 4.1, incremental kv state; update first, then read, which
 * keeps the diagonal term of the causal mask).  For every (b, g):
 *     S[b,g] += k[b,g]^T v[b,g];   o[b,h] = q[b,h] S[b,g]  for the heads h of g.
 * S [B,Hkv,d,d] fp32 is updated in place; q, o [B,Hq,d] and k, v [B,Hkv,d]
 * are bf16.  d in {64, 128}.  Errors as la_forward.
 * ---------------------------------------------------------------------- */
la_status la_decode_step(float *S, const la_bf16 *q, const la_bf16 *k, const la_bf16 *v,
                         la_bf16 *o, int B, int Hq, int Hkv, int d, la_stream stream);

/* Several decode steps per launch for tokens that are all known in advance
 * (speculative or draft tokens, short appended segments): for t = 0..steps-1,
 *     S[b,g] += k[b,g,t]^T v[b,g,t];   o[b,h,t] = q[b,h,t] S[b,g]
 * -- la_decode_step applied `steps` times, in fp32, with each state held in
 * registers across the steps so it is read and written once per call.
 * q, o [B,Hq,steps,d] and k, v [B,Hkv,steps,d] bf16 (the prefill layout with
 * N = steps); S as la_decode_step.  Errors as la_decode_step. */
la_status la_decode_steps(float *S, const la_bf16 *q, const la_bf16 *k, const la_bf16 *v,
                          la_bf16 *o, int B, int Hq, int Hkv, int d, int steps, la_stream stream);

/* ------------------------------------------------------------------------
 * Failure detection.
 * la_device_status: synchronises the current device, then stores the device
 * status word (LA_DEV_* bits, 0 = clean) in *flags and clears it if `clear`.
 * Returns LA_ERR_TIMEOUT when LA_DEV_TIMEOUT is set, LA_ERR_CUDA if the
 * synchronisation reports a fault, else LA_OK.
 *
 * la_selftest_wait: launches one warp that waits, bounded by timeout_ns of
 * device time, on a device flag that nothing ever sets; when the limit passes
 * it records LA_DEV_TIMEOUT and returns.  Exercises the same bounded-wait
 * routine the kernels use, without faulting or hanging the GPU.
 * ---------------------------------------------------------------------- */
la_status la_device_status(unsigned int *flags, int clear);
la_status la_selftest_wait(int64_t timeout_ns, la_stream stream);

/* Returns the memory the device's default pool keeps cached for the
 * workspaces of la_forward / la_forward_state (cudaMemPoolTrimTo). */
void la_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_B200_LA_H */
