// noalloc.cu -- pivot_reuse_noalloc: PIVOT-Reuse for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: their device
// memory is owned by a pool or a planner they do not control (a serving
// engine that reserves all memory up front, a plugin host that forbids
// allocations on the request path), so they cannot call cudaMalloc, and
// they cannot size a workspace for us either.  For them this entry point
// runs the same scan kernel as pivot_reuse with its scratch (the status
// word, the work counter and the per-group candidate buffers) taken from a
// fixed static device array that every process loading this library holds
// until exit.  The pages describing PIVOT have no counterpart of this: it
// is an integration convenience, not part of the method.
//
// Limits: bf16 q/k, H = 64, d in {64, 128}, g <= 16, k + g - 1 <= 256, and
// at most 148 CTAs (one per SM up to 148).  Each candidate sub-buffer gets the
// same slack as on the workspace path (selection size + 384, rounded up to 64:
// 640 entries for the largest selection of 256).  Scratch is
//   256 B (status + counters) + 148 CTAs * 4 groups * 4 sub-buffers * 640 entries * 8 B
//   = 12,124,416 B + 256 B (about 11.6 MiB).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "kernels.cuh"

using namespace pivot;

namespace {

constexpr int kMaxSel = 256;                   // k + g - 1
constexpr int kSubCap = 640;                   // entries per (group, lane quarter) sub-buffer: kMaxSel + 384
constexpr int kMaxCtas = 148;
constexpr int kGroupsPerItem = 4;              // 256 / H with H = 64
constexpr size_t kHdrBytes = 256;              // status word + counters
constexpr size_t kSelBytes = (size_t)kMaxCtas * kGroupsPerItem * 4 * kSubCap * sizeof(uint64_t);
constexpr size_t kStaticBytes = kHdrBytes + kSelBytes;  // 12,124,416 B + 256 B
static_assert(kSubCap >= kMaxSel + 384 && kSubCap % 64 == 0, "the workspace path's sub-buffer slack");

// The scratch itself.  In host code this name is only a host-side stand-in:
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticBytes];

std::mutex g_mu;
void* g_addr[64] = {nullptr};  // device address of the array, per device ordinal

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_keys(CUtensorMap* m, const void* base, int64_t rows, int d) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" PIVOT_API pivot_status pivot_reuse_noalloc(const void* q_I, const float* w_I, const void* k_I, int64_t L,
                                                      int H, int d, pivot_dtype dt, int k, int g, int32_t* indices,
                                                      float* scores_opt, pivot_stream_t stream) {
  clear_cuda_error();
  if (!q_I || !w_I || !k_I || !indices || L <= 0 || k <= 0 || g <= 0) return PIVOT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q_I) & 15u) || (reinterpret_cast<uintptr_t>(k_I) & 15u))
    return PIVOT_ERR_INVALID_ARG;
  if (dt != PIVOT_BF16 || H != 64 || (d != 64 && d != 128) || g > 16 || L >= (int64_t)0x7FFFFFF0)
    return PIVOT_ERR_UNSUPPORTED_SHAPE;
  if (k + g - 1 > kMaxSel) return PIVOT_ERR_UNSUPPORTED_SHAPE;  // beyond the static scratch

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return record_cuda_error(cudaErrorInvalidDevice, "device ordinal beyond 63");
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {  // first call on this device: look the array up once
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return record_cuda_error(e, "cudaGetSymbolAddress");
      if (p == nullptr) return record_cuda_error(cudaErrorInvalidSymbol, "cudaGetSymbolAddress");
      g_addr[dev] = p;
    }
    base = g_addr[dev];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* hdr = reinterpret_cast<char*>(base);
  // the array keeps the previous call's contents: the status word and the work
  // counter must start at zero (the candidate buffers are written before read)
  e = cudaMemsetAsync(hdr, 0, kHdrBytes, s);
  if (e != cudaSuccess) return record_cuda_error(e, "cudaMemsetAsync");

  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return record_cuda_error(e, "cudaDeviceGetAttribute");
  if (sms <= 0) return record_cuda_error(cudaErrorInvalidValue, "multiprocessor count");
  const int n_sel = k + g - 1;
  const int64_t n_groups = (L + g - 1) / g;
  const int n_items = (int)((n_groups + kGroupsPerItem - 1) / kGroupsPerItem);
  const int grid = (int)std::min<int64_t>(std::min(sms, kMaxCtas), n_items);

  CUtensorMap kmap;
  if (!encode_keys(&kmap, k_I, L, d)) return record_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  ScanArgs a{};
  a.q = reinterpret_cast<const uint16_t*>(q_I);
  a.w = w_I;
  a.L = L;
  a.H = H;
  a.D = d;
  a.g = g;
  a.n_sel = n_sel;
  a.topk = k;
  a.nb = kGroupsPerItem;
  a.mode = EMIT_REUSE;
  a.n_groups = n_groups;
  a.n_items = n_items;
  a.out_idx = indices;
  a.out_scores = scores_opt;
  a.selbuf = reinterpret_cast<uint64_t*>(hdr + kHdrBytes);
  a.cap = 4 * kSubCap;
  a.sub_cap = kSubCap;
  a.counter = reinterpret_cast<unsigned int*>(hdr + 64);
  a.status = reinterpret_cast<int*>(hdr);
  a.timeout_ns = device_timeout_ns();  // the bound pivot_set_device_timeout_ns sets for every call
  a.debug_flags = 0;                   // the test hooks apply to the workspace entry points only
  e = launch_scan(a, &kmap, grid, s);
  return e == cudaSuccess ? PIVOT_OK : record_cuda_error(e, "scan kernel");
}
