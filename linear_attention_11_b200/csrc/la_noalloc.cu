// la_noalloc.cu -- la_forward_noalloc: the bf16 prefill without any device
// allocation, for callers that cannot call cudaMalloc or any allocator:
// code running where allocation is forbidden or unsafe (inside a custom
// allocator or memory-pool callback, a framework that owns all device memory
// and rejects foreign allocations, or a hard-real-time path that must not
// block on the driver's allocator).
//
// The workspace that la_forward takes from the stream-ordered pool (the span
// states of the span-parallel scheme; a plan with one span per sequence needs
// none) lives instead in one file-scope device array of fixed size.  Every
// GPU that loads this part of the library holds the array until the process
// exits.  Every call uses the same array, so calls whose work overlaps on the
// GPU (other streams, other host threads) race on it and must be serialised
// by the caller.  Each call writes every workspace entry before reading it,
// so nothing left by an earlier call needs clearing.
//
// The first call on a device is not free of allocation: it looks up the
// array's device address, and with lazy module loading that lookup, like the
// first launch of each kernel, loads the module and so allocates its device
// memory (the 32 MiB array among it).  Callers make one warm-up call outside
// any restricted context; calls after it allocate nothing.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "la.h"
#include "la_internal.h"

#define LA_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

// 32 MiB of span states: B * Hkv * nspan * d * d * 4 bytes must fit.
constexpr size_t kScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the array's name as a device address).
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

LA_EXPORT la_status la_forward_noalloc(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                       la_bf16* o, float* S, int B, int Hq, int Hkv, int64_t N,
                                       int d, int chunk, la_stream stream) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  la_plan plan;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if ((st = la::check_prefill_ptrs(q, k, v, o, S, B, Hq, Hkv, N, d)) != LA_OK) return st;
  // Fewer spans if the planned span states exceed the array; a single span
  // needs none (the chunk loop reads and writes the state itself).
  const int64_t per_span = (int64_t)B * Hkv * d * d * (int64_t)sizeof(float);
  if (plan.nspan > 1 && plan.workspace_bytes > (int64_t)kScratchBytes) {
    plan.nspan = (int32_t)std::max<int64_t>(1, (int64_t)kScratchBytes / per_span);
    plan.workspace_bytes = per_span * plan.nspan;
  }
  void* ws = scratch_on_current_device();
  if (!ws) return LA_ERR_CUDA;
  return la::forward_dispatch(q, k, v, o, S, B, Hq, Hkv, N, plan, ws, kScratchBytes,
                              static_cast<cudaStream_t>(stream));
}
