// la_host.cu -- la_forward_host: the bf16 prefill from and to page-locked
// host memory, with the transfers pipelined against the compute.
//
// The sequence is cut into pieces along N.  Piece p is copied in on a copy-in
// stream, computed on the caller's stream with the state carried from piece
// p-1 (the state is the whole resume point of the recurrence: "MiniMax-01与
// Lightning Attention", section 4.1, "Streaming" row), and copied out on a
// copy-out stream, so host-to-device copies, device-to-host copies and
// compute of neighbouring pieces overlap.  Device buffers for two pieces are
// taken from the stream-ordered pool and returned at the end of the call.
// Strided host slices are moved with one cudaMemcpy2DAsync per tensor and
// piece (rows = (batch, head), row length = piece tokens x d).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "la.h"
#include "la_internal.h"

#define LA_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
cudaStream_t g_copy_in[kMaxDevices], g_copy_out[kMaxDevices];

// Two non-blocking helper streams per device, created once.
bool helper_streams(cudaStream_t* in, cudaStream_t* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_copy_in[dev]) {
    if (cudaStreamCreateWithFlags(&g_copy_in[dev], cudaStreamNonBlocking) != cudaSuccess)
      return false;
    if (cudaStreamCreateWithFlags(&g_copy_out[dev], cudaStreamNonBlocking) != cudaSuccess)
      return false;
  }
  *in = g_copy_in[dev];
  *out = g_copy_out[dev];
  return true;
}

// Copy tokens [n0, n0+len) of every (batch, head) row between a [rows, N, d]
// host tensor and a [rows, len, d] device piece.
cudaError_t copy_piece(void* dst, const void* src, size_t rows, int64_t N, int64_t n0, int64_t len,
                       int d, bool to_device, cudaStream_t s) {
  const size_t row_bytes = (size_t)len * d * 2;
  if (to_device)
    return cudaMemcpy2DAsync(dst, row_bytes, static_cast<const char*>(src) + (size_t)n0 * d * 2,
                             (size_t)N * d * 2, row_bytes, rows, cudaMemcpyHostToDevice, s);
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + (size_t)n0 * d * 2, (size_t)N * d * 2, src,
                           row_bytes, row_bytes, rows, cudaMemcpyDeviceToHost, s);
}

}  // namespace

LA_EXPORT la_status la_forward_host(const la_bf16* q, const la_bf16* k, const la_bf16* v,
                                    la_bf16* o, float* S, int B, int Hq, int Hkv, int64_t N, int d,
                                    int chunk, int64_t piece, la_stream stream) {
  if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
  la_plan plan;
  la_status st = la_prefill_plan(B, Hq, Hkv, N, d, chunk, &plan);
  if (st != LA_OK) return st;
  if (piece < 0) return LA_ERR_INVALID_ARG;
  // about sixteen pieces: the copy-in of the first and the copy-out of the
  // last piece are not overlapped, and finer pieces add per-piece costs
  // (measured, 32K tokens x 128 heads: 4 pieces 37.4 ms, 8: 34.6, 16: 33.6,
  // 32: 33.6, 64: 34.8)
  if (piece == 0) piece = std::max<int64_t>(plan.tile, (N + 15) / 16);
  piece = ((piece + plan.tile - 1) / plan.tile) * plan.tile;           // whole tiles
  piece = std::min<int64_t>(piece, N);
  const int64_t npieces = (N + piece - 1) / piece;

  cudaStream_t s = static_cast<cudaStream_t>(stream), s_in, s_out;
  if (!helper_streams(&s_in, &s_out)) return LA_ERR_CUDA;

  const size_t qrows = (size_t)B * Hq, krows = (size_t)B * Hkv;
  const size_t qbytes = qrows * piece * d * 2, kbytes = krows * piece * d * 2;
  // one workspace for every piece: the full pieces' or the shorter last one's
  const int64_t last = N - (npieces - 1) * piece;
  const size_t ws_bytes = std::max(la_forward_workspace_bytes(B, Hq, Hkv, piece, d, chunk),
                                   la_forward_workspace_bytes(B, Hq, Hkv, last, d, chunk));
  const size_t sbytes = (size_t)B * Hkv * d * d * 4;
  if (ws_bytes == 0) return LA_ERR_CUDA;
  // two piece buffers (q, k, v, o), a carried state when the caller gives none,
  // and one workspace (the pieces are computed in order on one stream)
  auto round = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t set_bytes = round(qbytes) * 2 + round(kbytes) * 2;
  const size_t total = 2 * set_bytes + round(ws_bytes) + (S ? 0 : round(sbytes));
  char* pool = nullptr;
  if (!la::keep_pool_memory()) return LA_ERR_CUDA;
  if (cudaMallocAsync(reinterpret_cast<void**>(&pool), total, s) != cudaSuccess) return LA_ERR_CUDA;
  float* carry = S;
  if (!carry) {
    carry = reinterpret_cast<float*>(pool + 2 * set_bytes + round(ws_bytes));
    if (cudaMemsetAsync(carry, 0, sbytes, s) != cudaSuccess) st = LA_ERR_CUDA;
  }
  struct Set { la_bf16 *q, *k, *v, *o; } sets[2];
  for (int b = 0; b < 2; ++b) {
    char* p = pool + b * set_bytes;
    sets[b].q = reinterpret_cast<la_bf16*>(p);
    sets[b].o = reinterpret_cast<la_bf16*>(p + round(qbytes));
    sets[b].k = reinterpret_cast<la_bf16*>(p + 2 * round(qbytes));
    sets[b].v = reinterpret_cast<la_bf16*>(p + 2 * round(qbytes) + round(kbytes));
  }
  void* ws = pool + 2 * set_bytes;

  cudaEvent_t ev[2][3];  // per buffer set: inputs in, computed, output out
  int made = 0;
  for (int b = 0; b < 2 && st == LA_OK; ++b)
    for (int e = 0; e < 3; ++e, ++made)
      if (cudaEventCreateWithFlags(&ev[b][e], cudaEventDisableTiming) != cudaSuccess) {
        st = LA_ERR_CUDA;
        break;
      }
  // the helper streams start after everything already queued on the caller's stream
  cudaEvent_t start;
  bool have_start = false;
  if (st == LA_OK && cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess) {
    have_start = true;
    if (cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(s_in, start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(s_out, start, 0) != cudaSuccess)
      st = LA_ERR_CUDA;
  } else if (st == LA_OK) {
    st = LA_ERR_CUDA;
  }

  for (int64_t p = 0; p < npieces && st == LA_OK; ++p) {
    const int b = (int)(p & 1);
    const int64_t n0 = p * piece, len = std::min<int64_t>(piece, N - n0);
    Set& bs = sets[b];
    // inputs of piece p: the set's previous compute (piece p-2) must be done
    if (p >= 2 && cudaStreamWaitEvent(s_in, ev[b][1], 0) != cudaSuccess) st = LA_ERR_CUDA;
    if (st == LA_OK &&
        (copy_piece(bs.q, q, qrows, N, n0, len, d, true, s_in) != cudaSuccess ||
         copy_piece(bs.k, k, krows, N, n0, len, d, true, s_in) != cudaSuccess ||
         copy_piece(bs.v, v, krows, N, n0, len, d, true, s_in) != cudaSuccess ||
         cudaEventRecord(ev[b][0], s_in) != cudaSuccess))
      st = LA_ERR_CUDA;
    // compute: inputs in, and the set's output of piece p-2 copied out
    if (st == LA_OK && cudaStreamWaitEvent(s, ev[b][0], 0) != cudaSuccess) st = LA_ERR_CUDA;
    if (st == LA_OK && p >= 2 && cudaStreamWaitEvent(s, ev[b][2], 0) != cudaSuccess)
      st = LA_ERR_CUDA;
    if (st == LA_OK)
      st = la_forward_ws(bs.q, bs.k, bs.v, bs.o, carry, B, Hq, Hkv, len, d, chunk, ws, ws_bytes,
                         stream);
    if (st == LA_OK && cudaEventRecord(ev[b][1], s) != cudaSuccess) st = LA_ERR_CUDA;
    // output of piece p
    if (st == LA_OK &&
        (cudaStreamWaitEvent(s_out, ev[b][1], 0) != cudaSuccess ||
         copy_piece(o, bs.o, qrows, N, n0, len, d, false, s_out) != cudaSuccess ||
         cudaEventRecord(ev[b][2], s_out) != cudaSuccess))
      st = LA_ERR_CUDA;
  }
  // the caller's stream covers every copy of the call before the buffers go back
  for (int b = 0; b < 2 && b < npieces; ++b)
    if (cudaStreamWaitEvent(s, ev[b][2], 0) != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  if (cudaFreeAsync(pool, s) != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i / 3][i % 3]);
  if (have_start) cudaEventDestroy(start);
  return st;
}
