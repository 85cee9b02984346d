// la_api.cu -- the C ABI declared in include/la.h: argument validation,
// planning of the span-parallel prefill, tensor-map construction, launches,
// and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "la.h"
#include "la_internal.h"
#include "la_ptx.cuh"

#define LA_EXPORT extern "C" __attribute__((visibility("default")))

namespace la {

// Device status word (LA_DEV_* bits) and a flag nothing ever sets (waited on by
// the self-test).  One copy per device that loads the library.
__device__ unsigned g_status;
__device__ unsigned g_never_set;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device device address of g_status and SM count, looked up once.
bool device_info(unsigned** status, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return false;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    g_num_sms[dev] = n;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  if (status) *status = g_status_ptr[dev];
  if (sms) *sms = g_num_sms[dev];
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Common shape checks of the prefill entry points.
la_status check_shape(int B, int Hq, int Hkv, int64_t N, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return LA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return LA_ERR_INVALID_ARG;
  // bulk tensor copies take int32 coordinates
  if (N > (int64_t)0x7fff0000 || (int64_t)B * Hq > 0x7fffffff) return LA_ERR_INVALID_ARG;
  return LA_OK;
}

constexpr double kQBytesHost = 128.0 * 128 * 2;  // one 128-row bf16 tile (Q or O)

}  // namespace

bool keep_pool_memory() {
  static std::once_flag once[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(once[dev], [dev]() {
    cudaMemPool_t pool;
    if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
      uint64_t keep = ~0ull;
      cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    }
  });
  return true;
}

namespace {

la_status plan_impl(int B, int Hq, int Hkv, int64_t N, int d, int chunk, int sms, la_plan* out) {
  la_status st = check_shape(B, Hq, Hkv, N, d);
  if (st != LA_OK) return st;
  if (d != kHeadDim || (chunk != 64 && chunk != 128)) return LA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  int T, HPT;
  if (chunk == 64 && G % 2 == 0) {
    T = 64;
    HPT = 2;  // two query heads x 64 tokens
  } else {
    T = 128;  // one head x 128 tokens (two 64-token chunks stacked when chunk == 64)
    HPT = 1;
  }
  const int64_t tiles = (N + T - 1) / T;
  const int64_t units = (int64_t)B * Hkv;
  const int64_t nsub = G / HPT;
  // Pick the span count: the persistent chunk loop deals units * nspan items
  // (a span of one kv group, nsub tiles per chunk step) round-robin over the
  // SMs; estimated time in tile times ~ rounds * (tiles per item + a per-item
  // cost of about three tiles), plus, with more than one span, the span-state
  // pass over (nspan - 1) / nspan of K and V, at the whole GPU's bandwidth:
  // its bytes / (bytes of one tile x SMs).
  const int64_t max_span = std::min<int64_t>(tiles, 4096);
  const double kv_tile = 2.0 * T * kHeadDim * 2;                   // K and V of one chunk step
  const double tile_bytes = 2.0 * kQBytesHost + kv_tile / (double)nsub;  // Q, O + K,V share
  const double span_pass = (double)units * tiles * kv_tile / (tile_bytes * sms);
  int64_t best = 1;
  double best_cost = 1e300;
  for (int64_t ns = 1; ns <= max_span; ++ns) {
    const int64_t items = units * ns;
    if (items > 0x7fffffff) break;
    const int64_t rounds = (items + sms - 1) / sms;
    const int64_t per = (tiles + ns - 1) / ns * nsub;
    const double cost =
        (double)rounds * (double)(per + 3) + span_pass * (double)(ns - 1) / (double)ns;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = ns;
    }
  }
  out->nspan = (int32_t)best;
  out->tile = T;
  out->heads_per_tile = HPT;
  out->tiles_total = (int32_t)tiles;
  out->workspace_bytes = (int64_t)B * Hkv * best * d * d * (int64_t)sizeof(float);
  return LA_OK;
}

// Span count of the fused single-pass kernel.  Each round (one span index
// over every kv head) re-reads its K and V from L2, so a round's K+V should
// stay well inside the 126 MB L2 next to the streaming Q and O: about 24 MB.
// Enough chunk-loop items for the dynamic scheduler to balance (two per SM),
// and at least four tiles per item so per-item costs stay small.
int fused_nspan(int B, int Hkv, int G, int HPT, int64_t N, int T, int sms) {
  const int64_t tiles = (N + T - 1) / T;
  const double kv_bytes = 2.0 * 2.0 * (double)B * Hkv * (double)N * kHeadDim;
  const double round_budget = 24.0 * 1024 * 1024;
  int64_t ns = (int64_t)(kv_bytes / round_budget) + 1;
  const int64_t units_m = (int64_t)B * Hkv * (G / HPT);
  ns = std::max<int64_t>(ns, (2 * sms + units_m - 1) / units_m);
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, tiles / 4));
  ns = std::min<int64_t>(ns, tiles);
  return (int)std::max<int64_t>(1, ns);
}

// A caller-supplied plan must describe this problem.
la_status check_plan(const la_plan* p, int B, int Hq, int Hkv, int64_t N, int d) {
  if (!p) return LA_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (!((p->tile == 64 && p->heads_per_tile == 2) || (p->tile == 128 && p->heads_per_tile == 1)))
    return LA_ERR_INVALID_ARG;
  if (G % p->heads_per_tile != 0) return LA_ERR_INVALID_ARG;
  if ((int64_t)p->tiles_total != (N + p->tile - 1) / p->tile) return LA_ERR_INVALID_ARG;
  if (p->nspan < 1 || p->nspan > p->tiles_total) return LA_ERR_INVALID_ARG;
  if (p->workspace_bytes != (int64_t)B * Hkv * p->nspan * d * d * (int64_t)sizeof(float))
    return LA_ERR_INVALID_ARG;
  if ((int64_t)B * Hkv * p->nspan * (G / p->heads_per_tile) > 0x7fffffff) return LA_ERR_INVALID_ARG;
  return LA_OK;
}

PrefillGeometry geometry(const la_plan* p, int B, int Hq, int Hkv, int64_t N) {
  PrefillGeometry g;
  g.B = B;
  g.Hq = Hq;
  g.Hkv = Hkv;
  g.G = Hq / Hkv;
  g.N = N;
  g.tile = p->tile;
  g.heads_per_tile = p->heads_per_tile;
  g.tiles_total = p->tiles_total;
  g.nspan = p->nspan;
  return g;
}

la_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

}  // namespace

la_status check_prefill_ptrs(const void* q, const void* k, const void* v, const void* o,
                             const void* S, int B, int Hq, int Hkv, int64_t N, int d) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LA_ERR_INVALID_ARG;
  if (S && !aligned16(S)) return LA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)B * Hq * N * d * 2, kbytes = (size_t)B * Hkv * N * d * 2,
               sbytes = (size_t)B * Hkv * d * d * 4;
  if (overlap(o, qbytes, q, qbytes) || overlap(o, qbytes, k, kbytes) ||
      overlap(o, qbytes, v, kbytes) || overlap(o, qbytes, S, sbytes) ||
      overlap(S, sbytes, q, qbytes) || overlap(S, sbytes, k, kbytes) ||
      overlap(S, sbytes, v, kbytes))
    return LA_ERR_INVALID_ARG;
  return LA_OK;
}

unsigned* device_status_ptr() {
  unsigned* st = nullptr;
  return device_info(&st, nullptr) ? st : nullptr;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows_per_head, int64_t heads,
                    int box_rows) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows_per_head, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2,
                                 (cuuint64_t)rows_per_head * kHeadDim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_state(CUtensorMap* map, const void* base, int64_t units) {
  CUtensorMap probe;
  if (!make_tmap_bf16(&probe, base, 128, 1, 64)) return false;  // resolves the encoder once
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)kHeadDim, (cuuint64_t)units};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 4, (cuuint64_t)kHeadDim * kHeadDim * 4};
  const cuuint32_t box[3] = {32, (cuuint32_t)kHeadDim, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

__global__ void selftest_wait_kernel(unsigned* status, const unsigned* flag, int64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (*reinterpret_cast<const volatile unsigned*>(flag) == 0u) {
    if (globaltimer_ns() - t0 > (uint64_t)limit_ns) {
      if (threadIdx.x == 0) atomicOr(status, kDevTimeout);
      return;
    }
    __nanosleep(1000);
  }
}

}  // namespace

bool stage_states_pays(const PrefillGeometry& g) {
  // Measured (64 tokens x 256 sequences, two tiles per item): 0.32 ms with
  // row-by-row state I/O, 0.22 ms staged, i.e. ~3.6 us saved per item; on
  // long items the staged layout costs ~0.7 us per tile (one 32K-token span
  // per kv head: 1.54 -> 2.23 ms).
  return g.nspan == 1 && (int64_t)g.tiles_total * (g.G / g.heads_per_tile) <= 4;
}

int span_parts(const la_plan& plan, int units, int sms) {
  if (plan.nspan <= 1) return 1;
  // the forward computes the states of the first nspan - 1 spans, one CTA
  // per SM at a time; cut each span into the number of parts (at least two
  // tiles each) whose CTAs finish soonest: waves x (tiles per part + a fixed
  // cost of about three tiles per CTA: pipeline fill, state write-out), the
  // fewest parts on a tie
  const int64_t ctas = (int64_t)units * (plan.nspan - 1);
  const int64_t span_tiles = (plan.tiles_total + plan.nspan - 1) / plan.nspan;
  const int64_t max_parts = std::max<int64_t>(1, std::min<int64_t>(64, span_tiles / 2));
  int64_t best = 1, best_cost = INT64_MAX;
  for (int64_t parts = 1; parts <= max_parts; ++parts) {
    const int64_t waves = (ctas * parts + sms - 1) / sms;
    const int64_t cost = waves * ((span_tiles + parts - 1) / parts + 3);
    if (cost < best_cost) {
      best_cost = cost;
      best = parts;
    }
  }
  return (int)best;
}

size_t forward_workspace_bytes(const la_plan& plan) {
  if (plan.nspan == 1) return 256;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return (size_t)plan.workspace_bytes;
  const int64_t per_seq = (int64_t)plan.nspan * kHeadDim * kHeadDim * (int64_t)sizeof(float);
  const int units = (int)(plan.workspace_bytes / per_seq);
  return (size_t)plan.workspace_bytes * (size_t)span_parts(plan, units, sms);
}

la_status forward_persistent(const la_bf16* q, const la_bf16* k, const la_bf16* v, la_bf16* o,
                             float* S, int B, int Hq, int Hkv, int64_t N, const la_plan& plan,
                             cudaStream_t stream, bool final_out) {
  unsigned* status = nullptr;
  int sms = 0;
  if (!device_info(&status, &sms)) return LA_ERR_CUDA;
  PrefillMaps maps;
  if (!make_tmap_bf16(&maps.q, q, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.o, o, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.k, k, N, (int64_t)B * Hkv, plan.tile) ||
      !make_tmap_bf16(&maps.v, v, N, (int64_t)B * Hkv, plan.tile))
    return LA_ERR_CUDA;
  PrefillGeometry g = geometry(&plan, B, Hq, Hkv, N);
  return from_cuda(launch_prefill_persist(g, maps, S, final_out ? S : nullptr, status, sms, stream,
                                          false, stage_states_pays(g)));
}

la_status forward_dispatch(const la_bf16* q, const la_bf16* k, const la_bf16* v, la_bf16* o,
                           float* S, int B, int Hq, int Hkv, int64_t N, const la_plan& plan,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream,
                           bool final_out) {
  if (plan.nspan == 1)
    return forward_persistent(q, k, v, o, S, B, Hq, Hkv, N, plan, stream, final_out);
  // Span states, entering states (and the final state), chunk loop.
  unsigned* status = nullptr;
  int sms = 0;
  if (!device_info(&status, &sms)) return LA_ERR_CUDA;
  PrefillMaps maps;
  if (!make_tmap_bf16(&maps.q, q, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.o, o, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.k, k, N, (int64_t)B * Hkv, plan.tile) ||
      !make_tmap_bf16(&maps.v, v, N, (int64_t)B * Hkv, plan.tile))
    return LA_ERR_CUDA;
  PrefillGeometry g = geometry(&plan, B, Hq, Hkv, N);
  float* ws = static_cast<float*>(workspace);
  // span parts, as many as wanted and as the workspace holds
  int parts = span_parts(plan, B * Hkv, sms);
  const size_t per_part = (size_t)plan.workspace_bytes;
  if (per_part == 0 || workspace_bytes < per_part) return LA_ERR_WORKSPACE;
  parts = (int)std::min<size_t>((size_t)parts, workspace_bytes / per_part);
  const int nsub_spans = plan.nspan * parts;
  // Without a state to return, the last span's K^T V feeds nothing and is
  // skipped.  With one, all spans are summed by the scan: a sum of span
  // states is more accurate than the last span's updates accumulated in
  // tensor memory on top of its entering state (1M tokens: final-state rel-L2
  // 3.3e-5 against 8.6e-5), for 1/nspan more of the first pass.
  const bool final_state = S != nullptr && final_out;
  cudaError_t e = launch_span_states(g, maps.k, maps.v, ws, status, stream, !final_state, parts);
  if (e == cudaSuccess)
    e = launch_state_scan(ws, S, B * Hkv, nsub_spans, kHeadDim, stream,
                          final_state ? nsub_spans : nsub_spans - parts);
  if (e == cudaSuccess)
    e = launch_prefill_persist(g, maps, ws, nullptr, status, sms, stream, true, false, parts);
  return from_cuda(e);
}

cudaError_t launch_selftest_wait(unsigned* status, int64_t timeout_ns, cudaStream_t stream) {
  void* flag = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&flag, g_never_set);
  if (e != cudaSuccess) return e;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, static_cast<const unsigned*>(flag),
                                             timeout_ns);
  return cudaGetLastError();
}

}  // namespace la

using namespace la;

// ---------------------------------------------------------------------------
LA_EXPORT const char* la_status_string(la_status s) {
  switch (s) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
    case LA_ERR_CUDA: return "LA_ERR_CUDA";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE";
  }
  return "LA_ERR_UNKNOWN";
}

LA_EXPORT int la_version(void) { return 1; }

LA_EXPORT la_status la_prefill_plan(int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                                    la_plan* plan) {
  if (!plan) return LA_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return LA_ERR_CUDA;
  return plan_impl(B, Hq, Hkv, N, d, chunk, sms, plan);
}

LA_EXPORT size_t la_forward_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int d, int chunk) {
  la_plan p;
  if (la_prefill_plan(B, Hq, Hkv, N, d, chunk, &p) != LA_OK) return 0;
  return forward_workspace_bytes(p);
}

LA_EXPORT la_status la_prefill_span_states(const la_bf16* k, const la_bf16* v, int B, int Hkv,
                                           int64_t N, int d, const la_plan* plan, float* ws,
                                           la_stream stream) {
  la_status st = check_shape(B, Hkv, Hkv, N, d);
  if (st != LA_OK) return st;
  if (d != kHeadDim) return LA_ERR_UNSUPPORTED;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return LA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_ERR_WORKSPACE;
  if (!plan || plan->nspan < 1 || plan->nspan > plan->tiles_total) return LA_ERR_INVALID_ARG;
  if (!((plan->tile == 64 && plan->heads_per_tile == 2) ||
        (plan->tile == 128 && plan->heads_per_tile == 1)) ||
      (int64_t)plan->tiles_total != (N + plan->tile - 1) / plan->tile)
    return LA_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  if (!device_info(&status, nullptr)) return LA_ERR_CUDA;
  PrefillMaps maps;
  const int64_t heads = (int64_t)B * Hkv;
  if (!make_tmap_bf16(&maps.k, k, N, heads, plan->tile) ||
      !make_tmap_bf16(&maps.v, v, N, heads, plan->tile))
    return LA_ERR_CUDA;
  PrefillGeometry g = geometry(plan, B, Hkv, Hkv, N);
  return from_cuda(
      launch_span_states(g, maps.k, maps.v, ws, status, static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_prefill_scan(float* ws, float* S, int B, int Hkv, int d,
                                    const la_plan* plan, la_stream stream) {
  if (B <= 0 || Hkv <= 0 || d != kHeadDim) return d != kHeadDim ? LA_ERR_UNSUPPORTED
                                                                 : LA_ERR_INVALID_ARG;
  if (!plan || plan->nspan < 1) return LA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_ERR_WORKSPACE;
  if (S && !aligned16(S)) return LA_ERR_INVALID_ARG;
  return from_cuda(
      launch_state_scan(ws, S, B * Hkv, plan->nspan, d, static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_prefill_main(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                    la_bf16* o, const float* ws, int B, int Hq, int Hkv,
                                    int64_t N, int d, const la_plan* plan, la_stream stream) {
  la_status st = check_shape(B, Hq, Hkv, N, d);
  if (st != LA_OK) return st;
  if (d != kHeadDim) return LA_ERR_UNSUPPORTED;
  if ((st = check_prefill_ptrs(q, k, v, o, nullptr, B, Hq, Hkv, N, d)) != LA_OK) return st;
  if ((st = check_plan(plan, B, Hq, Hkv, N, d)) != LA_OK) return st;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_ERR_WORKSPACE;
  unsigned* status = nullptr;
  if (!device_info(&status, nullptr)) return LA_ERR_CUDA;
  PrefillMaps maps;
  if (!make_tmap_bf16(&maps.q, q, N, (int64_t)B * Hq, plan->tile) ||
      !make_tmap_bf16(&maps.o, o, N, (int64_t)B * Hq, plan->tile) ||
      !make_tmap_bf16(&maps.k, k, N, (int64_t)B * Hkv, plan->tile) ||
      !make_tmap_bf16(&maps.v, v, N, (int64_t)B * Hkv, plan->tile))
    return LA_ERR_CUDA;
  PrefillGeometry g = geometry(plan, B, Hq, Hkv, N);
  int sms = 0;
  if (!device_info(nullptr, &sms)) return LA_ERR_CUDA;
  return from_cuda(launch_prefill_persist(g, maps, ws, nullptr, status, sms,
                                          static_cast<cudaStream_t>(stream), true,
                                          stage_states_pays(g)));
}

LA_EXPORT size_t la_prefill_fused_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int d,
                                                 int chunk, int nspan) {
  la_plan plan;
  if (la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan) != LA_OK) return 0;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return 0;
  if (nspan <= 0)
    nspan = fused_nspan(B, Hkv, Hq / Hkv, plan.heads_per_tile, N, plan.tile, sms);
  if (nspan > plan.tiles_total) return 0;
  return fused_workspace_bytes(B, Hkv, nspan);
}

LA_EXPORT la_status la_prefill_fused(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                     la_bf16* o, float* S, int B, int Hq, int Hkv, int64_t N,
                                     int d, int chunk, int nspan, int lookahead, void* workspace,
                                     size_t workspace_bytes, la_stream stream) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  la_plan plan;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, o, S, B, Hq, Hkv, N, d)) != LA_OK) return st;
  unsigned* status = nullptr;
  int sms = 0;
  if (!device_info(&status, &sms)) return LA_ERR_CUDA;
  if (nspan <= 0) nspan = fused_nspan(B, Hkv, Hq / Hkv, plan.heads_per_tile, N, plan.tile, sms);
  if (nspan > plan.tiles_total) return LA_ERR_INVALID_ARG;
  if ((int64_t)nspan * ((int64_t)B * Hkv + (int64_t)B * Hkv * (Hq / Hkv / plan.heads_per_tile)) >
      0x7fffffff)
    return LA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < fused_workspace_bytes(B, Hkv, nspan))
    return LA_ERR_WORKSPACE;
  plan.nspan = nspan;
  PrefillMaps maps;
  if (!make_tmap_bf16(&maps.q, q, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.o, o, N, (int64_t)B * Hq, plan.tile) ||
      !make_tmap_bf16(&maps.k, k, N, (int64_t)B * Hkv, plan.tile) ||
      !make_tmap_bf16(&maps.v, v, N, (int64_t)B * Hkv, plan.tile))
    return LA_ERR_CUDA;
  PrefillGeometry g = geometry(&plan, B, Hq, Hkv, N);
  if (lookahead <= 0) lookahead = 1;
  return from_cuda(launch_prefill_fused(g, maps, S, workspace, status, sms, lookahead,
                                        static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_forward_ws(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                  la_bf16* o, float* S, int B, int Hq, int Hkv, int64_t N, int d,
                                  int chunk, void* workspace, size_t workspace_bytes,
                                  la_stream stream) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  la_plan plan;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, o, S, B, Hq, Hkv, N, d)) != LA_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < forward_workspace_bytes(plan))
    return LA_ERR_WORKSPACE;
  return forward_dispatch(q, k, v, o, S, B, Hq, Hkv, N, plan, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(stream));
}

LA_EXPORT la_status la_forward_state(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                     la_bf16* o, float* S, int B, int Hq, int Hkv, int64_t N,
                                     int d, int chunk, la_stream stream) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  la_plan plan;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, o, S, B, Hq, Hkv, N, d)) != LA_OK) return st;
  // Stream-ordered workspace from the device's default memory pool, kept
  // cached by the pool between calls (release threshold raised once).
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!keep_pool_memory()) return LA_ERR_CUDA;
  const size_t bytes = la_forward_workspace_bytes(B, Hq, Hkv, N, d, chunk);
  if (bytes == 0) return LA_ERR_CUDA;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, s) != cudaSuccess) return LA_ERR_CUDA;
  st = la_forward_ws(q, k, v, o, S, B, Hq, Hkv, N, d, chunk, ws, bytes, stream);
  if (cudaFreeAsync(ws, s) != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  return st;
}

LA_EXPORT la_status la_forward(const la_bf16* q, const la_bf16* k, const la_bf16* v, la_bf16* o,
                               int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                               la_stream stream) {
  return la_forward_state(q, k, v, o, nullptr, B, Hq, Hkv, N, d, chunk, stream);
}

LA_EXPORT la_status la_forward_f32(const float* q, const float* k, const float* v, float* o,
                                   float* S, int B, int Hq, int Hkv, int64_t N, int d, int chunk,
                                   la_stream stream) {
  la_status st = check_shape(B, Hq, Hkv, N, d);
  if (st != LA_OK) return st;
  if ((d != 64 && d != 128) || (chunk != 64 && chunk != 128)) return LA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (S && !aligned16(S)))
    return LA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)B * Hq * N * d * 4, kbytes = (size_t)B * Hkv * N * d * 4,
               sbytes = (size_t)B * Hkv * d * d * 4;
  if (overlap(o, qbytes, q, qbytes) || overlap(o, qbytes, k, kbytes) ||
      overlap(o, qbytes, v, kbytes) || overlap(o, qbytes, S, sbytes))
    return LA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* S_in = nullptr;
  if (S) {  // the kernel reads the initial state from a copy and writes S
    if (cudaMallocAsync(reinterpret_cast<void**>(&S_in), sbytes, s) != cudaSuccess)
      return LA_ERR_CUDA;
    if (cudaMemcpyAsync(S_in, S, sbytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
      cudaFreeAsync(S_in, s);
      return LA_ERR_CUDA;
    }
  }
  st = from_cuda(launch_forward_simt_f32(q, k, v, o, S_in, S, B, Hq, Hkv, N, d, chunk, s));
  if (S_in) cudaFreeAsync(S_in, s);
  return st;
}

LA_EXPORT la_status la_decode_step(float* S, const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                   la_bf16* o, int B, int Hq, int Hkv, int d, la_stream stream) {
  if (!S || !q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0) return LA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 32) return LA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 0x7fffffff) return LA_ERR_INVALID_ARG;
  if (!aligned16(S) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return LA_ERR_INVALID_ARG;
  const size_t sbytes = (size_t)B * Hkv * d * d * 4, qbytes = (size_t)B * Hq * d * 2,
               kbytes = (size_t)B * Hkv * d * 2;
  if (overlap(o, qbytes, S, sbytes) || overlap(o, qbytes, q, qbytes) ||
      overlap(o, qbytes, k, kbytes) || overlap(o, qbytes, v, kbytes) ||
      overlap(S, sbytes, q, qbytes) || overlap(S, sbytes, k, kbytes) ||
      overlap(S, sbytes, v, kbytes))
    return LA_ERR_INVALID_ARG;
  return from_cuda(
      launch_decode(S, q, k, v, o, B, Hq, Hkv, d, static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_decode_steps(float* S, const la_bf16* q, const la_bf16* k,
                                    const la_bf16* v, la_bf16* o, int B, int Hq, int Hkv, int d,
                                    int steps, la_stream stream) {
  if (!S || !q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || steps <= 0 || Hq % Hkv != 0)
    return LA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 32) return LA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 0x7fffffff) return LA_ERR_INVALID_ARG;
  if (!aligned16(S) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return LA_ERR_INVALID_ARG;
  const size_t sbytes = (size_t)B * Hkv * d * d * 4, qbytes = (size_t)B * Hq * steps * d * 2,
               kbytes = (size_t)B * Hkv * steps * d * 2;
  if (overlap(o, qbytes, S, sbytes) || overlap(o, qbytes, q, qbytes) ||
      overlap(o, qbytes, k, kbytes) || overlap(o, qbytes, v, kbytes) ||
      overlap(S, sbytes, q, qbytes) || overlap(S, sbytes, k, kbytes) ||
      overlap(S, sbytes, v, kbytes))
    return LA_ERR_INVALID_ARG;
  return from_cuda(launch_decode_steps(S, q, k, v, o, B, Hq, Hkv, d, steps,
                                       static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_segment_state(const la_bf16* k, const la_bf16* v, float* S, int B, int Hkv,
                                     int64_t N, int d, int chunk, la_stream stream) {
  la_plan plan;
  la_status st = la_prefill_plan(B, Hkv, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if (!k || !v || !S || !aligned16(k) || !aligned16(v) || !aligned16(S)) return LA_ERR_INVALID_ARG;
  const size_t kbytes = (size_t)B * Hkv * N * d * 2, sbytes = (size_t)B * Hkv * d * d * 4;
  if (overlap(S, sbytes, k, kbytes) || overlap(S, sbytes, v, kbytes)) return LA_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  if (!device_info(&status, nullptr)) return LA_ERR_CUDA;
  PrefillMaps maps;
  if (!make_tmap_bf16(&maps.k, k, N, (int64_t)B * Hkv, plan.tile) ||
      !make_tmap_bf16(&maps.v, v, N, (int64_t)B * Hkv, plan.tile))
    return LA_ERR_CUDA;
  plan.nspan = 1;  // the whole segment as one span: its state is K^T V, written into S
  PrefillGeometry g = geometry(&plan, B, Hkv, Hkv, N);
  return from_cuda(launch_span_states(g, maps.k, maps.v, S, status,
                                      static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_state_prefix(const float* states, const float* S0, float* S, int nseg,
                                    int seg, int B, int Hkv, int d, la_stream stream) {
  if (!states || !S || nseg < 1 || seg < 0 || seg >= nseg || B <= 0 || Hkv <= 0 || d <= 0 ||
      d % 2 != 0)
    return LA_ERR_INVALID_ARG;
  if (!aligned16(states) || !aligned16(S) || (S0 && !aligned16(S0))) return LA_ERR_INVALID_ARG;
  const size_t per = (size_t)B * Hkv * d * d;
  if (overlap(S, per * 4, states, per * 4 * nseg) || (S0 && S0 != S && overlap(S, per * 4, S0, per * 4)))
    return LA_ERR_INVALID_ARG;
  return from_cuda(launch_state_prefix(states, S0, S, seg, per, static_cast<cudaStream_t>(stream)));
}

LA_EXPORT la_status la_device_status(unsigned int* flags, int clear) {
  if (!flags) return LA_ERR_INVALID_ARG;
  *flags = 0;
  if (!device_info(nullptr, nullptr)) return LA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return LA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return LA_ERR_CUDA;
  if (clear) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return LA_ERR_CUDA;
  }
  *flags = v;
  return (v & LA_DEV_TIMEOUT) ? LA_ERR_TIMEOUT : LA_OK;
}

LA_EXPORT la_status la_selftest_wait(int64_t timeout_ns, la_stream stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return LA_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  if (!device_info(&status, nullptr)) return LA_ERR_CUDA;
  return from_cuda(launch_selftest_wait(status, timeout_ns, static_cast<cudaStream_t>(stream)));
}

LA_EXPORT void la_shutdown(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  cudaMemPool_t pool;
  if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) cudaMemPoolTrimTo(pool, 0);
}
