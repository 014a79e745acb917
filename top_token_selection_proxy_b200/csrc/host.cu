// host.cu -- pivot_refine_host: PIVOT-Refine of a prefill sequence whose inputs and
// output live in host memory.  The keys and weights are copied first, then the
// queries in runs of whole groups on a copy stream; each run is indexed with the
// group-range call on the caller's stream as soon as it has landed, and its rows
// are copied back on a second copy stream while later runs are still being
// copied in or indexed.  The runs go from the sequence's end to its start: a
// group's work grows with its causal prefix, so the heaviest runs overlap the
// copies of the rest and the run indexed last, whose kernels and copy back are
// not overlapped, is the cheapest.  Every step is ordered by events; nothing
// synchronises the host.  (Group ranges: the groups of Eq. (2) are independent
// given k_I, so a run's rows equal the same rows of one whole-sequence call.)
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "kernels.cuh"

using namespace pivot;

namespace {

constexpr int kMaxChunks = 64;

// Copy streams and events of one device, created by the first call on it and kept
// until the process exits.
struct HostPipe {
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t landed[kMaxChunks] = {}, done[kMaxChunks] = {};
};

std::mutex g_pipe_mu;
HostPipe g_pipes[64];

cudaError_t pipe_setup(HostPipe& p) {
  if (p.ready) return cudaSuccess;
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&p.end, cudaEventDisableTiming)) != cudaSuccess) return e;
  for (int i = 0; i < kMaxChunks; ++i) {
    if ((e = cudaEventCreateWithFlags(&p.landed[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  p.ready = true;
  return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Device copies carved from the caller's workspace, followed by the refine workspace.
struct HostWs {
  size_t q_off, w_off, k_off, out_off, ws_off, ws_bytes, total;
};

HostWs host_ws(int64_t L, int H, int d, int k, int c, int g) {
  HostWs w{};
  size_t off = 0;
  w.q_off = off;
  off = align256(off + (size_t)L * H * d * 2);
  w.w_off = off;
  off = align256(off + (size_t)L * H * 4);
  w.k_off = off;
  off = align256(off + (size_t)L * d * 2);
  w.out_off = off;
  off = align256(off + (size_t)L * k * 4);
  w.ws_off = off;
  w.ws_bytes = pivot_workspace_size(PIVOT_OP_REFINE, L, H, d, k, c, g, PIVOT_BF16);
  w.total = w.ws_bytes ? off + w.ws_bytes : 0;
  return w;
}

}  // namespace

extern "C" {

PIVOT_API size_t pivot_refine_host_workspace_size(int64_t L, int H, int d, int k, int c, int g) {
  if (L <= 0 || H <= 0 || d <= 0 || k <= 0 || c < k || g <= 0) return 0;
  return host_ws(L, H, d, k, c, g).total;
}

PIVOT_API pivot_status pivot_refine_host(const void* q_host, const float* w_host, const void* k_host, int64_t L,
                                         int H, int d, int k, int c, int g, int chunks, int32_t* out_host, void* ws,
                                         size_t ws_bytes, pivot_stream_t stream) {
  clear_cuda_error();
  if (!q_host || !w_host || !k_host || !out_host || !ws) return PIVOT_ERR_INVALID_ARG;
  if (chunks < 1 || chunks > kMaxChunks) return PIVOT_ERR_INVALID_ARG;
  if (L <= 0 || H <= 0 || d <= 0 || k <= 0 || c < k || g <= 0) return PIVOT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PIVOT_ERR_INVALID_ARG;
  const HostWs W = host_ws(L, H, d, k, c, g);
  if (W.total == 0) return PIVOT_ERR_UNSUPPORTED_SHAPE;  // pivot_refine_range rejects these sizes
  if (ws_bytes < W.total) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  char* base = reinterpret_cast<char*>(ws);
  char* q_dev = base + W.q_off;
  float* w_dev = reinterpret_cast<float*>(base + W.w_off);
  char* k_dev = base + W.k_off;
  int32_t* out_dev = reinterpret_cast<int32_t*>(base + W.out_off);
  void* rws = base + W.ws_off;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return record_cuda_error(cudaErrorInvalidDevice, "device ordinal beyond 63");
  // the pipe's streams and events are shared by the calls on this device: enqueue one call at a time
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe& p = g_pipes[dev];
  if ((e = pipe_setup(p)) != cudaSuccess) return record_cuda_error(e, "copy streams / events");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  const size_t qrow = (size_t)H * d * 2, wrow = (size_t)H * 4, orow = (size_t)k * 4;
  const int64_t G = (L + g - 1) / g, per = (G + chunks - 1) / chunks;
  // the copies wait for earlier work on the caller's stream (it may still use the buffers)
  if ((e = cudaEventRecord(p.start, s)) != cudaSuccess) return record_cuda_error(e, "event record");
  if ((e = cudaStreamWaitEvent(p.s_in, p.start, 0)) != cudaSuccess) return record_cuda_error(e, "stream wait");
  if ((e = cudaStreamWaitEvent(p.s_out, p.start, 0)) != cudaSuccess) return record_cuda_error(e, "stream wait");
  if ((e = cudaMemcpyAsync(k_dev, k_host, (size_t)L * d * 2, cudaMemcpyHostToDevice, p.s_in)) != cudaSuccess ||
      (e = cudaMemcpyAsync(w_dev, w_host, (size_t)L * wrow, cudaMemcpyHostToDevice, p.s_in)) != cudaSuccess)
    return record_cuda_error(e, "copy in");
  const int n_runs = (int)((G + per - 1) / per);
  for (int i = 0; i < n_runs; ++i) {
    const int64_t g0 = (int64_t)(n_runs - 1 - i) * per;  // the last run first
    const int64_t g1 = std::min<int64_t>(G, g0 + per);
    const int64_t t0 = g0 * g, t1 = std::min<int64_t>(g1 * g, L);
    if ((e = cudaMemcpyAsync(q_dev + t0 * qrow, reinterpret_cast<const char*>(q_host) + t0 * qrow,
                             (size_t)(t1 - t0) * qrow, cudaMemcpyHostToDevice, p.s_in)) != cudaSuccess)
      return record_cuda_error(e, "copy in");
    if ((e = cudaEventRecord(p.landed[i], p.s_in)) != cudaSuccess) return record_cuda_error(e, "event record");
    if ((e = cudaStreamWaitEvent(s, p.landed[i], 0)) != cudaSuccess) return record_cuda_error(e, "stream wait");
    const pivot_status st =
        pivot_refine_range(q_dev + t0 * qrow, w_dev + t0 * H, k_dev, L, H, d, PIVOT_BF16, k, c, g, g0, g1,
                           out_dev + t0 * k, nullptr, nullptr, nullptr, rws, W.ws_bytes, stream);
    if (st != PIVOT_OK) return st;
    if ((e = cudaEventRecord(p.done[i], s)) != cudaSuccess) return record_cuda_error(e, "event record");
    if ((e = cudaStreamWaitEvent(p.s_out, p.done[i], 0)) != cudaSuccess) return record_cuda_error(e, "stream wait");
    if ((e = cudaMemcpyAsync(reinterpret_cast<char*>(out_host) + t0 * orow, out_dev + t0 * k,
                             (size_t)(t1 - t0) * orow, cudaMemcpyDeviceToHost, p.s_out)) != cudaSuccess)
      return record_cuda_error(e, "copy out");
  }
  // the caller's stream is ordered after the last copy out
  if ((e = cudaEventRecord(p.end, p.s_out)) != cudaSuccess) return record_cuda_error(e, "event record");
  if ((e = cudaStreamWaitEvent(s, p.end, 0)) != cudaSuccess) return record_cuda_error(e, "stream wait");
  return PIVOT_OK;
}

}  // extern "C"
