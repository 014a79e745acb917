// api.cu -- host side of the C ABI declared in include/pivot.h: argument
// validation, workspace carving, TMA descriptors and the launch sequence of
// each entry point.  Allocates nothing; every launch goes on the caller's
// stream and no call synchronises the host (pivot_last_device_status aside).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kernels.cuh"

using namespace pivot;

namespace {

thread_local char g_cuda_err[256] = "";
uint64_t g_timeout_ns = 2000000000ull;
int g_debug_flags = 0;
cudaEvent_t g_prof[4] = {nullptr, nullptr, nullptr, nullptr};

void prof(int i, cudaStream_t s) {
  if (g_prof[0]) cudaEventRecord(g_prof[i], s);
}
void prof_rest(int from, cudaStream_t s) {
  for (int i = from; i < 4; ++i) prof(i, s);
}

constexpr size_t kHdr = 256;     // status word + counters
constexpr int kStatusOff = 0;    // int
constexpr int kCounterOff = 64;  // 4 x uint32

pivot_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", what, cudaGetErrorString(e));
  return PIVOT_ERR_CUDA;
}

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- TMA descriptor
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, d] (d contiguous), 64-column x box_rows boxes, 128-byte swizzle.
bool make_kmap(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- shapes and paths
bool tc_shape(int H, int d, pivot_dtype dt) { return dt == PIVOT_BF16 && H == 64 && (d == 64 || d == 128); }

pivot_status check_common(int64_t L, int H, int d, pivot_dtype dt, int k, int c, int g, int op) {
  if (L <= 0 || H <= 0 || d <= 0 || k <= 0 || g <= 0) return PIVOT_ERR_INVALID_ARG;
  if (dt != PIVOT_BF16 && dt != PIVOT_F32) return PIVOT_ERR_INVALID_ARG;
  if (d % 8 != 0) return PIVOT_ERR_INVALID_ARG;
  if (op == PIVOT_OP_REFINE && (c < k || c <= 0)) return PIVOT_ERR_INVALID_ARG;
  if (g > 16 || L >= (int64_t)0x7FFFFFF0 || k > 65536 || (op == PIVOT_OP_REFINE && c > 16384) || H > 1024 ||
      d > 1024)
    return PIVOT_ERR_UNSUPPORTED_SHAPE;
  return PIVOT_OK;
}

int sel_size(int op, int k, int c, int g) {
  return op == PIVOT_OP_DENSE ? k : (op == PIVOT_OP_REUSE ? k + g - 1 : c);
}
// per (group, lane quarter) sub-buffer of the scan kernel: room for a full
// selection plus slack, so that cut-backs are rare; a group owns 4 of them
int sel_sub_cap(int n_sel) { return (int)align_up((size_t)n_sel + 384, 64); }
int sel_cap(int n_sel) { return 4 * sel_sub_cap(n_sel); }

struct Carve {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

// Workspace of the prefill calls; with base == nullptr only sizes are computed.
struct PrefillWs {
  int* status;
  unsigned* counters;
  uint64_t* selbuf;
  int32_t* cand;
  uint32_t* keys;
  uint64_t* sscratch;
  float* fscratch;
  int grid, simt_grid;
  int64_t simt_per_block, simt_member_off;
  size_t bytes;
};

PrefillWs carve_prefill(void* base, int op, int64_t L, int H, int d, int k, int c, int g, pivot_dtype dt,
                        bool user_cand) {
  PrefillWs w{};
  Carve cv{reinterpret_cast<char*>(base)};
  char* hdr = cv.take<char>(kHdr);
  w.status = reinterpret_cast<int*>(hdr ? hdr + kStatusOff : nullptr);
  w.counters = reinterpret_cast<unsigned*>(hdr ? hdr + kCounterOff : nullptr);
  const int sms = num_sms();
  const int64_t gs = (op == PIVOT_OP_DENSE) ? 1 : g;
  const int64_t n_groups = (L + gs - 1) / gs;
  if (tc_shape(H, d, dt)) {
    const int nb = 256 / H;
    const int64_t n_items = (n_groups + nb - 1) / nb;
    w.grid = (int)std::min<int64_t>(sms, n_items);
    const int n_sel = sel_size(op, k, c, g);
    w.selbuf = cv.take<uint64_t>((size_t)sms * nb * sel_cap(n_sel));
    if (op == PIVOT_OP_REFINE) {
      if (!user_cand) w.cand = cv.take<int32_t>((size_t)n_groups * c);
      w.keys = cv.take<uint32_t>((size_t)L * c);
    }
  } else {
    w.simt_grid = (int)std::min<int64_t>(2 * sms, n_groups);
    w.simt_member_off = (int64_t)align_up((size_t)L, 32);
    w.simt_per_block = w.simt_member_off + (op == PIVOT_OP_REFINE ? (int64_t)align_up((size_t)c, 32) : 0);
    w.sscratch = cv.take<uint64_t>((size_t)(2 * sms) * w.simt_per_block);
    w.fscratch = cv.take<float>((size_t)(2 * sms) * ((size_t)H * d + H));
  }
  w.bytes = align_up(cv.off, 256);
  return w;
}

struct DecodeWs {
  int* status;
  unsigned* counters;
  DecodeArgs d;  // workspace pointers of the tensor-core path
  int32_t* cand;
  uint32_t* keys;
  uint64_t* sscratch;
  float* fscratch;
  int scan_grid, simt_grid;
  int64_t simt_per_block, simt_member_off;
  size_t bytes;
};

DecodeWs carve_decode(void* base, int op, int B, const int64_t* off, int H, int d, int k, int c, int g,
                      pivot_dtype dt, bool user_cand) {
  DecodeWs w{};
  Carve cv{reinterpret_cast<char*>(base)};
  char* hdr = cv.take<char>(kHdr);
  w.status = reinterpret_cast<int*>(hdr ? hdr + kStatusOff : nullptr);
  w.counters = reinterpret_cast<unsigned*>(hdr ? hdr + kCounterOff : nullptr);
  const int sms = num_sms();
  int64_t total = 0, pmax = 0, n_sets = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t P = off[b + 1] - off[b];
    total += P;
    pmax = std::max(pmax, P);
    n_sets += (P + kDecodeSetKeys - 1) / kDecodeSetKeys;
  }
  if (tc_shape(H, d, dt)) {
    const int n_sel = sel_size(op, k, c, g);
    DecodeArgs& a = w.d;
    a.n_sets = n_sets;
    w.scan_grid = (int)std::min<int64_t>(sms, n_sets);
    a.proxy = cv.take<uint16_t>((size_t)B * H * d);
    a.wbar = cv.take<float>((size_t)B * kWbarStride);
    a.set_off = cv.take<int32_t>((size_t)B + 1);
    a.scores = cv.take<uint32_t>((size_t)total);
    a.ties = cv.take<uint64_t>((size_t)total);
    a.ties2 = cv.take<uint64_t>((size_t)total);
    a.hist1 = cv.take<uint32_t>((size_t)B * 2048);
    a.sel = cv.take<uint64_t>((size_t)B * n_sel);
    if (op == PIVOT_OP_REFINE) {
      if (!user_cand) w.cand = cv.take<int32_t>((size_t)B * c);
      w.keys = cv.take<uint32_t>((size_t)B * g * c);
    }
  } else {
    w.simt_grid = std::min(B, 2 * sms);
    w.simt_member_off = (int64_t)align_up((size_t)pmax, 32);
    w.simt_per_block = w.simt_member_off + (op == PIVOT_OP_REFINE ? (int64_t)align_up((size_t)c, 32) : 0);
    w.sscratch = cv.take<uint64_t>((size_t)(2 * sms) * w.simt_per_block);
    w.fscratch = cv.take<float>((size_t)(2 * sms) * ((size_t)H * d + H));
  }
  w.bytes = align_up(cv.off, 256);
  return w;
}

pivot_status check_offsets(int B, const int64_t* off, int g) {
  if (B <= 0 || !off || off[0] != 0) return PIVOT_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (off[b + 1] - off[b] < g) return PIVOT_ERR_INVALID_ARG;
  if (off[B] >= (int64_t)0x7FFFFFF0) return PIVOT_ERR_UNSUPPORTED_SHAPE;
  return PIVOT_OK;
}

ScanArgs scan_base(const void* q, const float* w, int H, int d, int g, int n_sel, int k, int mode, int64_t n_groups,
                   int n_items, uint64_t* selbuf, int cap, unsigned* counter, int* status) {
  ScanArgs a{};
  a.q = reinterpret_cast<const uint16_t*>(q);
  a.w = w;
  a.H = H;
  a.D = d;
  a.g = g;
  a.n_sel = n_sel;
  a.topk = k;
  a.nb = 256 / H;
  a.mode = mode;
  a.n_groups = n_groups;
  a.n_items = n_items;
  a.selbuf = selbuf;
  a.cap = cap;
  a.sub_cap = cap / 4;
  a.counter = counter;
  a.status = status;
  a.timeout_ns = g_timeout_ns;
  a.debug_flags = g_debug_flags;
  return a;
}

// ---------------------------------------------------------------- prefill driver
// Shift a caller's pointer to rows [r0, ...) down by r0 rows of `row` elements, so that
// kernels indexing rows of the whole sequence land in the caller's buffer.
template <typename T>
T* rows_from(T* p, int64_t r0, int64_t row) {
  if (!p) return p;
  return reinterpret_cast<T*>(reinterpret_cast<uintptr_t>(p) - (uintptr_t)(r0 * row) * sizeof(*p));
}
const void* rows_from_bytes(const void* p, int64_t r0, int64_t row_bytes) {
  return reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(p) - (uintptr_t)(r0 * row_bytes));
}

// Prefill over groups [g_lo, g_hi) of a length-L sequence (g_hi < 0: all groups).  For a
// proper range, q / w / indices / scores hold only the range's rows, cand_opt only its
// groups, and k_I the key rows [0, min(g_hi * g, L)) the range reads.
pivot_status run_prefill(int op, const void* q, const float* w, const void* k_I, int64_t L, int H, int d,
                         pivot_dtype dt, int k, int c, int g, int32_t* indices, float* scores, int32_t* cand_opt,
                         float* cand_scores, void* ws, size_t ws_bytes, cudaStream_t s, int agg = 0,
                         int64_t g_lo = 0, int64_t g_hi = -1) {
  g_cuda_err[0] = 0;
  if (op == PIVOT_OP_DENSE) g = 1;
  if (agg < 0 || agg > 2) return PIVOT_ERR_INVALID_ARG;
  pivot_status st = check_common(L, H, d, dt, k, c, g, op);
  if (st != PIVOT_OK) return st;
  if (!q || !w || !k_I || !indices || !ws) return PIVOT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_I) || !aligned16(ws)) return PIVOT_ERR_INVALID_ARG;
  const int64_t n_groups_all = (L + g - 1) / g;
  if (g_hi < 0) g_hi = n_groups_all;
  if (g_lo < 0 || g_lo >= g_hi || g_hi > n_groups_all) return PIVOT_ERR_INVALID_ARG;
  const int64_t r_lo = g_lo * g, r_hi = std::min<int64_t>(g_hi * g, L);  // the range's query rows
  const int64_t L_keys = r_hi;                                            // key rows it reads
  const size_t esz = dt == PIVOT_BF16 ? 2 : 4;
  q = rows_from_bytes(q, r_lo, (int64_t)H * d * (int64_t)esz);
  w = rows_from(w, r_lo, H);
  indices = rows_from(indices, r_lo, k);
  scores = rows_from(scores, r_lo, k);
  cand_opt = rows_from(cand_opt, g_lo, c);
  cand_scores = rows_from(cand_scores, g_lo, c);
  const PrefillWs need = carve_prefill(nullptr, op, L, H, d, k, c, g, dt, cand_opt != nullptr);
  if (ws_bytes < need.bytes) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  const PrefillWs W = carve_prefill(ws, op, L, H, d, k, c, g, dt, cand_opt != nullptr);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  const int64_t n_groups = g_hi;  // kernels cover groups [g_lo, g_hi)

  if (!tc_shape(H, d, dt)) {
    SimtArgs a{};
    a.q = q;
    a.w = w;
    a.k = k_I;
    a.is_bf16 = dt == PIVOT_BF16;
    a.L = L;
    a.H = H;
    a.D = d;
    a.g = g;
    a.c = c;
    a.topk = k;
    a.variant = op;
    a.agg = agg;
    a.grp_base = g_lo;
    a.n_groups = n_groups;
    a.out_idx = indices;
    a.out_scores = scores;
    a.cand_out = cand_opt;
    a.cand_scores = cand_scores;
    a.scratch = W.sscratch;
    a.scratch_per_block = W.simt_per_block;
    a.member_off = W.simt_member_off;
    a.fscratch = W.fscratch;
    e = launch_simt(a, W.simt_grid, s);
    return e == cudaSuccess ? PIVOT_OK : cuda_fail(e, "simt kernel");
  }

  CUtensorMap kmap;
  if (!make_kmap(&kmap, k_I, L_keys, d, 128)) return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  const int nb = 256 / H;
  const int n_sel = sel_size(op, k, c, g);
  const int n_items = (int)((g_hi - g_lo + nb - 1) / nb);
  const int mode = op == PIVOT_OP_DENSE ? EMIT_DENSE : (op == PIVOT_OP_REUSE ? EMIT_REUSE : EMIT_CAND);
  ScanArgs a = scan_base(q, w, H, d, g, n_sel, k, mode, n_groups, n_items, W.selbuf, sel_cap(n_sel),
                         W.counters + 0, W.status);
  a.L = L;
  a.agg = agg;
  a.grp_base = g_lo;
  a.out_idx = indices;
  a.out_scores = scores;
  int32_t* cand = cand_opt ? cand_opt : W.cand;
  a.cand = cand;
  a.cand_scores = cand_scores;
  prof(0, s);
  e = launch_scan(a, &kmap, W.grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "scan kernel");
  prof(1, s);
  if (op != PIVOT_OP_REFINE) {
    prof_rest(2, s);
    return PIVOT_OK;
  }

  RefineArgs r{};
  r.q = reinterpret_cast<const uint16_t*>(q);
  r.w = w;
  r.k = reinterpret_cast<const uint16_t*>(k_I);
  r.L = L;
  r.H = H;
  r.D = d;
  r.g = g;
  r.c = c;
  r.topk = k;
  r.mc = 512 / H;
  r.cparts = 1;
  r.n_groups = n_groups;  // items count down from group g_hi - 1 to g_lo
  r.n_items = (int)((g_hi - g_lo) * ((g + r.mc - 1) / r.mc));
  r.cand = cand;
  r.key_off = nullptr;
  r.keys = W.keys;
  r.counter = W.counters + 1;
  r.status = W.status;
  r.timeout_ns = g_timeout_ns;
  CUtensorMap gmap, qmap;  // one-row boxes for the candidate gather; 256-row boxes of q rows
  if (!make_kmap(&gmap, k_I, L_keys, d, 1) || !make_kmap(&qmap, q, r_hi * H, d, 256))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  e = launch_refine(r, &gmap, &qmap, (int)std::min<int64_t>(num_sms(), r.n_items), s);
  if (e != cudaSuccess) return cuda_fail(e, "refine kernel");
  prof(2, s);

  RowSelArgs rs{};
  rs.keys = W.keys;
  rs.cand = cand;
  rs.row_base = r_lo;
  rs.n_rows = r_hi;
  rs.L = L;
  rs.key_off = nullptr;
  rs.g = g;
  rs.c = c;
  rs.topk = k;
  rs.out_idx = indices;
  rs.out_scores = scores;
  e = launch_rowselect(rs, (int)std::min<int64_t>(8 * num_sms(), r_hi - r_lo), s);
  if (e != cudaSuccess) return cuda_fail(e, "rowselect kernel");
  prof(3, s);
  return PIVOT_OK;
}

// ---------------------------------------------------------------- decode driver
pivot_status run_decode(int op, const void* q, const float* w, const void* kc, const int64_t* off_dev,
                        const int64_t* off_host, int B, int H, int d, pivot_dtype dt, int k, int c, int g,
                        int32_t* indices, float* scores, int32_t* cand_opt, float* cand_scores, void* ws,
                        size_t ws_bytes, cudaStream_t s) {
  g_cuda_err[0] = 0;
  pivot_status st = check_common(1, H, d, dt, k, c, g, op);
  if (st != PIVOT_OK) return st;
  if ((st = check_offsets(B, off_host, g)) != PIVOT_OK) return st;
  if (!q || !w || !kc || !off_dev || !indices || !ws) return PIVOT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(ws)) return PIVOT_ERR_INVALID_ARG;
  const DecodeWs need = carve_decode(nullptr, op, B, off_host, H, d, k, c, g, dt, cand_opt != nullptr);
  if (ws_bytes < need.bytes) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  const DecodeWs W = carve_decode(ws, op, B, off_host, H, d, k, c, g, dt, cand_opt != nullptr);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");

  if (!tc_shape(H, d, dt)) {
    SimtArgs a{};
    a.q = q;
    a.w = w;
    a.k = kc;
    a.is_bf16 = dt == PIVOT_BF16;
    a.L = 0;
    a.H = H;
    a.D = d;
    a.g = g;
    a.c = c;
    a.topk = k;
    a.variant = op;
    a.n_groups = B;
    a.key_off = off_dev;
    a.out_idx = indices;
    a.out_scores = scores;
    a.cand_out = cand_opt;
    a.cand_scores = cand_scores;
    a.scratch = W.sscratch;
    a.scratch_per_block = W.simt_per_block;
    a.member_off = W.simt_member_off;
    a.fscratch = W.fscratch;
    e = launch_simt(a, W.simt_grid, s);
    return e == cudaSuccess ? PIVOT_OK : cuda_fail(e, "simt kernel");
  }

  if ((int64_t)B * kSelCl > 0x7FFFFFFFLL) return PIVOT_ERR_UNSUPPORTED_SHAPE;  // selection grid
  const int n_sel = sel_size(op, k, c, g);
  int32_t* cand = cand_opt ? cand_opt : W.cand;
  DecodeArgs a = W.d;
  a.q = reinterpret_cast<const uint16_t*>(q);
  a.w = w;
  a.key_off = off_dev;
  a.B = B;
  a.H = H;
  a.D = d;
  a.g = g;
  a.n_sel = n_sel;
  a.topk = k;
  a.mode = op == PIVOT_OP_REUSE ? EMIT_REUSE : EMIT_CAND;
  a.cand = cand;
  a.cand_scores = cand_scores;
  a.out_idx = indices;
  a.out_scores = scores;
  a.status = W.status;
  a.timeout_ns = g_timeout_ns;
  CUtensorMap kmap, pmap;  // 128-key tiles of the cache; the 64-row proxy of a sequence
  if (!make_kmap(&kmap, kc, off_host[B], d, 128) || !make_kmap(&pmap, a.proxy, (int64_t)B * H, d, H))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  prof(0, s);
  e = launch_decode_scan(a, &kmap, &pmap, W.scan_grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode scan");
  prof(1, s);
  e = launch_decode_select(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode selection");
  prof(2, s);
  if (op == PIVOT_OP_REUSE) {
    prof(3, s);
    return PIVOT_OK;
  }

  RefineArgs r{};
  r.q = reinterpret_cast<const uint16_t*>(q);
  r.w = w;
  r.k = reinterpret_cast<const uint16_t*>(kc);
  r.L = 0;
  r.H = H;
  r.D = d;
  r.g = g;
  r.c = c;
  r.topk = k;
  r.mc = 512 / H;
  r.n_groups = B;
  {
    // few groups: split each group's candidate tiles so that the items cover the SMs
    const int chunks = (g + r.mc - 1) / r.mc, tiles = (c + 127) / 128;
    r.cparts = std::max(1, std::min(tiles, num_sms() / std::max(1, B * chunks)));
    r.n_items = B * chunks * r.cparts;
  }
  r.cand = cand;
  r.key_off = off_dev;
  r.keys = W.keys;
  r.counter = W.counters + 1;
  r.status = W.status;
  r.timeout_ns = g_timeout_ns;
  CUtensorMap gmap, qmap;  // one-row boxes for the candidate gather; 256-row boxes of q rows
  if (!make_kmap(&gmap, kc, off_host[B], d, 1) || !make_kmap(&qmap, q, (int64_t)B * g * H, d, 256))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  e = launch_refine(r, &gmap, &qmap, std::min(num_sms(), r.n_items), s);
  if (e != cudaSuccess) return cuda_fail(e, "refine kernel");

  RowSelArgs rs{};
  rs.keys = W.keys;
  rs.cand = cand;
  rs.n_rows = (int64_t)B * g;
  rs.L = 0;
  rs.key_off = off_dev;
  rs.g = g;
  rs.c = c;
  rs.topk = k;
  rs.out_idx = indices;
  rs.out_scores = scores;
  e = launch_rowselect(rs, (int)std::min<int64_t>(8 * num_sms(), rs.n_rows), s);
  if (e != cudaSuccess) return cuda_fail(e, "rowselect kernel");
  prof(3, s);
  return PIVOT_OK;
}

// ---------------------------------------------------------------- decode split (one long prefix over ranks)
// Shard offsets: like key offsets, but a shard may hold any number >= 1 of a sequence's keys.
pivot_status check_shard_offsets(int B, const int64_t* off) {
  if (B <= 0 || !off || off[0] != 0) return PIVOT_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (off[b + 1] - off[b] < 1) return PIVOT_ERR_INVALID_ARG;
  if (off[B] >= (int64_t)0x7FFFFFF0) return PIVOT_ERR_UNSUPPORTED_SHAPE;
  return PIVOT_OK;
}

size_t merge_ws_bytes(int op, int R, int B, int k, int c, int g) {
  const size_t n_sel = (size_t)sel_size(op, k, c, g);
  return kHdr + align_up((size_t)B * R * n_sel * 8, 256) + align_up((size_t)B * n_sel * 8, 256);
}

DecodeArgs shard_args(const DecodeWs& W, int op, const void* q, const float* w, const int64_t* off_dev, int B, int H,
                      int d, int k, int c, int g) {
  DecodeArgs a = W.d;
  a.q = reinterpret_cast<const uint16_t*>(q);
  a.w = w;
  a.key_off = off_dev;
  a.B = B;
  a.H = H;
  a.D = d;
  a.g = g;
  a.n_sel = sel_size(op, k, c, g);
  a.topk = k;
  a.status = W.status;
  a.timeout_ns = g_timeout_ns;
  return a;
}

}  // namespace

// Library-internal hooks for the other host files (hidden: not part of the C ABI).
namespace pivot {
uint64_t device_timeout_ns() { return g_timeout_ns; }
int debug_flags() { return g_debug_flags; }
void clear_cuda_error() { g_cuda_err[0] = 0; }
pivot_status record_cuda_error(cudaError_t e, const char* what) { return cuda_fail(e, what); }
}  // namespace pivot

extern "C" {

size_t pivot_workspace_size(int op, int64_t L, int H, int d, int k, int c, int g, pivot_dtype dt) {
  if (op < 0 || op > 2) return 0;
  if (op == PIVOT_OP_DENSE) g = 1;
  if (check_common(L, H, d, dt, k, c, g, op) != PIVOT_OK) return 0;
  return carve_prefill(nullptr, op, L, H, d, k, c, g, dt, false).bytes;
}

size_t pivot_varlen_workspace_size(int op, int B, const int64_t* off, int H, int d, int k, int c, int g,
                                   pivot_dtype dt) {
  if (op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) return 0;
  if (check_common(1, H, d, dt, k, c, g, op) != PIVOT_OK || check_offsets(B, off, g) != PIVOT_OK) return 0;
  return carve_decode(nullptr, op, B, off, H, d, k, c, g, dt, false).bytes;
}

pivot_status pivot_indexer_dense(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                                 pivot_dtype dt, int k, int32_t* indices, float* scores_opt, void* ws,
                                 size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_DENSE, q_I, w_I, k_I, L, H, d, dt, k, k, 1, indices, scores_opt, nullptr, nullptr,
                     ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pivot_status pivot_reuse(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                         pivot_dtype dt, int k, int g, int32_t* indices, float* scores_opt, void* ws,
                         size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REUSE, q_I, w_I, k_I, L, H, d, dt, k, k, g, indices, scores_opt, nullptr, nullptr,
                     ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pivot_status pivot_refine(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                          pivot_dtype dt, int k, int c, int g, int32_t* indices, float* scores_opt,
                          int32_t* cand_opt, float* cand_scores_opt, void* ws, size_t ws_bytes,
                          pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REFINE, q_I, w_I, k_I, L, H, d, dt, k, c, g, indices, scores_opt, cand_opt,
                     cand_scores_opt, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pivot_status pivot_reuse_varlen(const void* q, const float* w, const void* k_cache, const int64_t* key_offsets_dev,
                                const int64_t* key_offsets_host, int B, int H, int d, pivot_dtype dt, int k, int g,
                                int32_t* indices, float* scores_opt, void* ws, size_t ws_bytes,
                                pivot_stream_t stream) {
  return run_decode(PIVOT_OP_REUSE, q, w, k_cache, key_offsets_dev, key_offsets_host, B, H, d, dt, k, k, g, indices,
                    scores_opt, nullptr, nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pivot_status pivot_refine_varlen(const void* q, const float* w, const void* k_cache,
                                 const int64_t* key_offsets_dev, const int64_t* key_offsets_host, int B, int H,
                                 int d, pivot_dtype dt, int k, int c, int g, int32_t* indices, float* scores_opt,
                                 int32_t* cand_opt, float* cand_scores_opt, void* ws, size_t ws_bytes,
                                 pivot_stream_t stream) {
  return run_decode(PIVOT_OP_REFINE, q, w, k_cache, key_offsets_dev, key_offsets_host, B, H, d, dt, k, c, g,
                    indices, scores_opt, cand_opt, cand_scores_opt, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

size_t pivot_decode_shard_workspace_size(int op, int B, const int64_t* shard_offsets_host, int H, int d, int k, int c,
                                         int g) {
  if (op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) return 0;
  if (op == PIVOT_OP_REUSE) c = k;
  if (check_common(1, H, d, PIVOT_BF16, k, c, g, op) != PIVOT_OK || !tc_shape(H, d, PIVOT_BF16) ||
      check_shard_offsets(B, shard_offsets_host) != PIVOT_OK)
    return 0;
  return carve_decode(nullptr, op, B, shard_offsets_host, H, d, k, c, g, PIVOT_BF16, false).bytes;
}

pivot_status pivot_decode_shard_select(int op, const void* q, const float* w, const void* k_shard,
                                       const int64_t* shard_offsets_dev, const int64_t* shard_offsets_host,
                                       const int64_t* pos_base_dev, int B, int H, int d, pivot_dtype dt, int k, int c,
                                       int g, uint64_t* entries, void* ws, size_t ws_bytes, pivot_stream_t stream) {
  g_cuda_err[0] = 0;
  if (op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) return PIVOT_ERR_INVALID_ARG;
  if (op == PIVOT_OP_REUSE) c = k;
  pivot_status st = check_common(1, H, d, dt, k, c, g, op);
  if (st != PIVOT_OK) return st;
  if ((st = check_shard_offsets(B, shard_offsets_host)) != PIVOT_OK) return st;
  if (!q || !w || !k_shard || !shard_offsets_dev || !pos_base_dev || !entries || !ws) return PIVOT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_shard) || !aligned16(ws)) return PIVOT_ERR_INVALID_ARG;
  if (!tc_shape(H, d, dt)) return PIVOT_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)B * kSelCl > 0x7FFFFFFFLL) return PIVOT_ERR_UNSUPPORTED_SHAPE;  // selection grid
  const DecodeWs need = carve_decode(nullptr, op, B, shard_offsets_host, H, d, k, c, g, dt, false);
  if (ws_bytes < need.bytes) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  const DecodeWs W = carve_decode(ws, op, B, shard_offsets_host, H, d, k, c, g, dt, false);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  DecodeArgs a = shard_args(W, op, q, w, shard_offsets_dev, B, H, d, k, c, g);
  a.mode = EMIT_ENTRIES;
  a.pos_base = pos_base_dev;
  a.entries = entries;
  CUtensorMap kmap, pmap;
  if (!make_kmap(&kmap, k_shard, shard_offsets_host[B], d, 128) || !make_kmap(&pmap, a.proxy, (int64_t)B * H, d, H))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  if ((e = launch_decode_scan(a, &kmap, &pmap, W.scan_grid, s)) != cudaSuccess) return cuda_fail(e, "decode scan");
  if ((e = launch_decode_select(a, s)) != cudaSuccess) return cuda_fail(e, "decode selection");
  return PIVOT_OK;
}

size_t pivot_decode_merge_workspace_size(int op, int R, int B, int k, int c, int g) {
  if ((op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) || R < 1 || B < 1 || k < 1 || g < 1) return 0;
  if (op == PIVOT_OP_REUSE) c = k;
  if (c < k) return 0;
  return merge_ws_bytes(op, R, B, k, c, g);
}

pivot_status pivot_decode_merge(int op, const uint64_t* entries, int R, const int64_t* plen_offsets_dev,
                                const int64_t* plen_offsets_host, int B, int k, int c, int g, int32_t* indices,
                                float* scores_opt, int32_t* cand, float* cand_scores_opt,
                                const int64_t* pos_base_dev, const int64_t* shard_offsets_dev,
                                int32_t* cand_local_opt, void* ws, size_t ws_bytes, pivot_stream_t stream) {
  g_cuda_err[0] = 0;
  if (op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) return PIVOT_ERR_INVALID_ARG;
  if (op == PIVOT_OP_REUSE) c = k;
  if (R < 1 || k < 1 || c < k || g < 1 || g > 16) return PIVOT_ERR_INVALID_ARG;
  pivot_status st = check_offsets(B, plen_offsets_host, g);
  if (st != PIVOT_OK) return st;
  if (!entries || !plen_offsets_dev || !ws || !aligned16(ws)) return PIVOT_ERR_INVALID_ARG;
  if (op == PIVOT_OP_REUSE ? !indices : !cand) return PIVOT_ERR_INVALID_ARG;
  if (cand_local_opt && (!pos_base_dev || !shard_offsets_dev)) return PIVOT_ERR_INVALID_ARG;
  if ((int64_t)R * sel_size(op, k, c, g) >= (int64_t)0x7FFFFFF0) return PIVOT_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < merge_ws_bytes(op, R, B, k, c, g)) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  Carve cv{reinterpret_cast<char*>(ws)};
  cv.take<char>(kHdr);
  MergeArgs m{};
  m.entries = entries;
  m.R = R;
  m.B = B;
  m.g = g;
  m.n_sel = sel_size(op, k, c, g);
  m.topk = k;
  m.mode = op == PIVOT_OP_REUSE ? EMIT_REUSE : EMIT_CAND;
  m.plen_off = plen_offsets_dev;
  m.gather = cv.take<uint64_t>((size_t)B * R * m.n_sel);
  m.sel = cv.take<uint64_t>((size_t)B * m.n_sel);
  m.out_idx = indices;
  m.out_scores = scores_opt;
  m.cand = cand;
  m.cand_scores = cand_scores_opt;
  m.pos_base = pos_base_dev;
  m.shard_off = shard_offsets_dev;
  m.cand_local = cand_local_opt;
  e = launch_decode_merge(m, s);
  return e == cudaSuccess ? PIVOT_OK : cuda_fail(e, "decode merge");
}

pivot_status pivot_decode_shard_rescore(const void* q, const float* w, const void* k_shard,
                                        const int64_t* shard_offsets_dev, const int64_t* shard_offsets_host,
                                        const int64_t* pos_base_dev, const int64_t* plen_offsets_dev, int B, int H,
                                        int d, pivot_dtype dt, int k, int c, int g, const int32_t* cand_local,
                                        uint32_t* keys, void* ws, size_t ws_bytes, pivot_stream_t stream) {
  g_cuda_err[0] = 0;
  pivot_status st = check_common(1, H, d, dt, k, c, g, PIVOT_OP_REFINE);
  if (st != PIVOT_OK) return st;
  if ((st = check_shard_offsets(B, shard_offsets_host)) != PIVOT_OK) return st;
  if (!q || !w || !k_shard || !shard_offsets_dev || !pos_base_dev || !plen_offsets_dev || !cand_local || !keys || !ws)
    return PIVOT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_shard) || !aligned16(ws)) return PIVOT_ERR_INVALID_ARG;
  if (!tc_shape(H, d, dt)) return PIVOT_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < kHdr) return PIVOT_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  RefineArgs r{};
  r.q = reinterpret_cast<const uint16_t*>(q);
  r.w = w;
  r.k = reinterpret_cast<const uint16_t*>(k_shard);
  r.L = 0;
  r.H = H;
  r.D = d;
  r.g = g;
  r.c = c;
  r.topk = k;
  r.mc = 512 / H;
  r.n_groups = B;
  {
    const int chunks = (g + r.mc - 1) / r.mc, tiles = (c + 127) / 128;
    r.cparts = std::max(1, std::min(tiles, num_sms() / std::max(1, B * chunks)));
    r.n_items = B * chunks * r.cparts;
  }
  r.cand = cand_local;
  r.key_off = shard_offsets_dev;
  r.pos_base = pos_base_dev;
  r.plen_off = plen_offsets_dev;
  r.keys = keys;
  char* hdr = reinterpret_cast<char*>(ws);
  r.counter = reinterpret_cast<unsigned*>(hdr + kCounterOff) + 1;
  r.status = reinterpret_cast<int*>(hdr + kStatusOff);
  r.timeout_ns = g_timeout_ns;
  CUtensorMap gmap, qmap;
  if (!make_kmap(&gmap, k_shard, shard_offsets_host[B], d, 1) || !make_kmap(&qmap, q, (int64_t)B * g * H, d, 256))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  e = launch_refine(r, &gmap, &qmap, std::min(num_sms(), r.n_items), s);
  return e == cudaSuccess ? PIVOT_OK : cuda_fail(e, "refine kernel");
}

pivot_status pivot_decode_rowselect(const uint32_t* keys, const int32_t* cand, const int64_t* plen_offsets_dev,
                                    int B, int k, int c, int g, int32_t* indices, float* scores_opt,
                                    pivot_stream_t stream) {
  g_cuda_err[0] = 0;
  if (!keys || !cand || !plen_offsets_dev || !indices || B < 1 || k < 1 || c < k || g < 1)
    return PIVOT_ERR_INVALID_ARG;
  RowSelArgs rs{};
  rs.keys = keys;
  rs.cand = cand;
  rs.n_rows = (int64_t)B * g;
  rs.L = 0;
  rs.key_off = plen_offsets_dev;
  rs.g = g;
  rs.c = c;
  rs.topk = k;
  rs.out_idx = indices;
  rs.out_scores = scores_opt;
  const cudaError_t e =
      launch_rowselect(rs, (int)std::min<int64_t>(8 * num_sms(), rs.n_rows), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PIVOT_OK : cuda_fail(e, "rowselect kernel");
}

pivot_status pivot_last_device_status(const void* ws, pivot_stream_t stream) {
  if (!ws) return PIVOT_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream sync");
  int st = 0;
  e = cudaMemcpy(&st, reinterpret_cast<const char*>(ws) + kStatusOff, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status copy");
  if (st & DEV_ERR_TIMEOUT) return PIVOT_ERR_DEVICE_TIMEOUT;
  if (st & DEV_ERR_BOUNDS) return PIVOT_ERR_DEVICE_BOUNDS;
  return PIVOT_OK;
}

const char* pivot_status_string(pivot_status s) {
  switch (s) {
    case PIVOT_OK: return "PIVOT_OK";
    case PIVOT_ERR_INVALID_ARG: return "PIVOT_ERR_INVALID_ARG";
    case PIVOT_ERR_UNSUPPORTED_SHAPE: return "PIVOT_ERR_UNSUPPORTED_SHAPE";
    case PIVOT_ERR_WORKSPACE_TOO_SMALL: return "PIVOT_ERR_WORKSPACE_TOO_SMALL";
    case PIVOT_ERR_CUDA: return "PIVOT_ERR_CUDA";
    case PIVOT_ERR_DEVICE_TIMEOUT: return "PIVOT_ERR_DEVICE_TIMEOUT";
    case PIVOT_ERR_DEVICE_BOUNDS: return "PIVOT_ERR_DEVICE_BOUNDS";
  }
  return "PIVOT_ERR_UNKNOWN";
}

const char* pivot_last_cuda_error(void) { return g_cuda_err; }

int pivot_path(int op, int64_t L, int H, int d, int k, int c, int g, pivot_dtype dt) {
  if (op < 0 || op > 2) return -1;
  if (op == PIVOT_OP_DENSE) g = 1;
  if (check_common(L, H, d, dt, k, c, g, op) != PIVOT_OK) return -1;
  return tc_shape(H, d, dt) ? 1 : 0;
}

void pivot_set_device_timeout_ns(uint64_t ns) { g_timeout_ns = ns; }
void pivot_set_debug_flags(int flags) { g_debug_flags = flags; }

void pivot_set_profile_events(void** events, int n) {
  for (int i = 0; i < 4; ++i)
    g_prof[i] = (events && n >= 4) ? reinterpret_cast<cudaEvent_t>(events[i]) : nullptr;
}
pivot_status pivot_indexer_dense_range(const void* q_rows, const float* w_rows, const void* k_prefix, int64_t L,
                                       int H, int d, pivot_dtype dt, int k, int64_t t0, int64_t t1,
                                       int32_t* indices, float* scores_opt, void* ws, size_t ws_bytes,
                                       pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_DENSE, q_rows, w_rows, k_prefix, L, H, d, dt, k, k, 1, indices, scores_opt, nullptr,
                     nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), 0, t0, t1);
}

pivot_status pivot_reuse_range(const void* q_rows, const float* w_rows, const void* k_prefix, int64_t L, int H,
                               int d, pivot_dtype dt, int k, int g, int64_t g0, int64_t g1, int32_t* indices,
                               float* scores_opt, void* ws, size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REUSE, q_rows, w_rows, k_prefix, L, H, d, dt, k, k, g, indices, scores_opt, nullptr,
                     nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), 0, g0, g1);
}

pivot_status pivot_refine_range(const void* q_rows, const float* w_rows, const void* k_prefix, int64_t L, int H,
                                int d, pivot_dtype dt, int k, int c, int g, int64_t g0, int64_t g1,
                                int32_t* indices, float* scores_opt, int32_t* cand_opt, float* cand_scores_opt,
                                void* ws, size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REFINE, q_rows, w_rows, k_prefix, L, H, d, dt, k, c, g, indices, scores_opt,
                     cand_opt, cand_scores_opt, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), 0, g0, g1);
}

pivot_status pivot_reuse_agg(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                             pivot_dtype dt, int k, int g, int aggregation, int32_t* indices, float* scores_opt,
                             void* ws, size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REUSE, q_I, w_I, k_I, L, H, d, dt, k, k, g, indices, scores_opt, nullptr, nullptr,
                     ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), aggregation);
}

pivot_status pivot_refine_agg(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                              pivot_dtype dt, int k, int c, int g, int aggregation, int32_t* indices,
                              float* scores_opt, int32_t* cand_opt, float* cand_scores_opt, void* ws,
                              size_t ws_bytes, pivot_stream_t stream) {
  return run_prefill(PIVOT_OP_REFINE, q_I, w_I, k_I, L, H, d, dt, k, c, g, indices, scores_opt, cand_opt,
                     cand_scores_opt, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), aggregation);
}

// Guardrail work model (see pivot.h): key-row products of each path.
int pivot_guardrail_dense(int op, int64_t L, int c, int g) {
  if (L < 1 || g < 1 || (op != PIVOT_OP_REUSE && op != PIVOT_OP_REFINE) || (op == PIVOT_OP_REFINE && c < 1))
    return -1;
  const double dense = 0.5 * (double)L * (double)(L + 1);
  double pivot = 0.0;
  for (int64_t t0 = 0; t0 < L; t0 += g) {
    const int64_t t1 = std::min<int64_t>(t0 + g, L);
    const double P = (double)t1;  // the group's prefix: keys 0 .. group end
    pivot += P;
    if (op == PIVOT_OP_REFINE) pivot += (double)(t1 - t0) * std::min<double>((double)c, P);
  }
  return dense <= pivot ? 1 : 0;
}

pivot_status pivot_reuse_guarded(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                                 pivot_dtype dt, int k, int g, int32_t* indices, float* scores_opt, void* ws,
                                 size_t ws_bytes, pivot_stream_t stream, int* path_out) {
  const int use_dense = pivot_guardrail_dense(PIVOT_OP_REUSE, L, k, g);
  if (use_dense < 0) return PIVOT_ERR_INVALID_ARG;
  if (path_out) *path_out = use_dense;
  if (use_dense)
    return pivot_indexer_dense(q_I, w_I, k_I, L, H, d, dt, k, indices, scores_opt, ws, ws_bytes, stream);
  return pivot_reuse(q_I, w_I, k_I, L, H, d, dt, k, g, indices, scores_opt, ws, ws_bytes, stream);
}

pivot_status pivot_refine_guarded(const void* q_I, const float* w_I, const void* k_I, int64_t L, int H, int d,
                                  pivot_dtype dt, int k, int c, int g, int32_t* indices, float* scores_opt,
                                  int32_t* cand_opt, float* cand_scores_opt, void* ws, size_t ws_bytes,
                                  pivot_stream_t stream, int* path_out) {
  const int use_dense = pivot_guardrail_dense(PIVOT_OP_REFINE, L, c, g);
  if (use_dense < 0) return PIVOT_ERR_INVALID_ARG;
  if (path_out) *path_out = use_dense;
  if (use_dense)
    return pivot_indexer_dense(q_I, w_I, k_I, L, H, d, dt, k, indices, scores_opt, ws, ws_bytes, stream);
  return pivot_refine(q_I, w_I, k_I, L, H, d, dt, k, c, g, indices, scores_opt, cand_opt, cand_scores_opt, ws,
                      ws_bytes, stream);
}

int pivot_version(void) { return 100; }

}  // extern "C"
