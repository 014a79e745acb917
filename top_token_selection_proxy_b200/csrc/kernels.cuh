// kernels.cuh -- argument blocks and launch declarations shared by the
// kernel files and the C-ABI host code of the PIVOT indexer library.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "pivot.h"  // include/ of the repository (-I)

namespace pivot {

// What a scan work item emits once its groups' selections are final.
enum EmitMode : int {
  EMIT_DENSE = 0,   // g == 1: row t = top-k of the query's own scores (Eq. 1)
  EMIT_REUSE = 1,   // Eq. 6: each member t takes the proxy top-k under s <= t
  EMIT_CAND = 2,    // Eq. 7: write the proxy top-c candidate set C_i
  EMIT_ENTRIES = 3  // decode split: a key shard's exact top-n as packed entries (global positions)
};

// Device status word bits (written with atomicOr, read by pivot_last_device_status).
enum : int {
  DEV_ERR_TIMEOUT = 1,
  DEV_ERR_BOUNDS = 2,
};

struct ScanArgs {
  const uint16_t* q;   // bf16 bits [rows, H, D]
  const float* w;      // [rows, H]
  int64_t L;           // prefill: sequence length (query rows == key rows)
  int H, D, g;
  int n_sel;           // selection size per group
  int topk;            // k
  int nb;              // groups per work item (N = nb * H)
  int mode;            // EmitMode
  int agg;             // proxy aggregation: 0 mean of the members (Eq. 4), 1 first, 2 last query
  int64_t grp_base;    // prefill: first group of the call (items cover groups [grp_base, n_groups))
  int64_t n_groups;
  int n_items;
  // outputs
  int32_t* out_idx;    // [rows, topk]
  float* out_scores;   // [rows, topk] or null
  int32_t* cand;       // [n_groups, n_sel]
  float* cand_scores;  // [n_groups, n_sel] or null
  // workspace
  uint64_t* selbuf;    // [gridDim.x, nb, cap]: per group 4 sub-buffers of sub_cap entries
  int cap;             // = 4 * sub_cap
  int sub_cap;         // entries per (group, TMEM lane quarter) sub-buffer
  unsigned int* counter;
  int* status;
  uint64_t timeout_ns;
  int debug_flags;     // bit 0: the epilogue waits on a barrier nothing signals (timeout test)
};

struct RefineArgs {
  const uint16_t* q;     // bf16 bits [rows, H, D]
  const float* w;        // [rows, H]
  const uint16_t* k;     // bf16 bits [key rows, D]
  int64_t L;             // prefill sequence length (0 for decode)
  int H, D, g, c, topk;
  int mc;                // members per work item (mc * H <= 512)
  int cparts;            // parts the candidate tiles of a (group, member chunk) are split into
  int64_t n_groups;
  int n_items;           // n_groups * ceil(g / mc) * cparts
  const int32_t* cand;   // [n_groups, c]  (-1 padded)
  const int64_t* key_off;  // decode: [B+1]; null for prefill
  const int64_t* pos_base;  // decode, optional: [B] global position of each sequence's first key row
  const int64_t* plen_off;  // decode, optional: [B+1] offsets giving the full prefix lengths (members' positions)
  uint32_t* keys;        // [rows, c] member score keys (0 = not eligible)
  unsigned int* counter;
  int* status;
  uint64_t timeout_ns;
};

// Eq. (9): per query row, the top-k of its candidates' score keys.
struct RowSelArgs {
  const uint32_t* keys;  // [rows, c]
  const int32_t* cand;   // [n_groups, c]
  int64_t row_base;      // first row of the call (rows [row_base, n_rows))
  int64_t n_rows;
  int64_t L;             // prefill sequence length (decode: 0)
  const int64_t* key_off;  // decode: [B+1]
  int g, c, topk;
  int32_t* out_idx;
  float* out_scores;
};

struct SimtArgs {
  const void* q;       // bf16 bits or fp32 [rows, H, D]
  const float* w;
  const void* k;       // [key rows, D]
  int is_bf16;
  int64_t L;
  int H, D, g, c, topk;
  int variant;         // 0 dense, 1 reuse, 2 refine
  int agg;             // proxy aggregation as in ScanArgs
  int64_t grp_base;    // first group of the call (groups [grp_base, n_groups))
  int64_t n_groups;
  const int64_t* key_off;  // decode: [B+1] (groups are sequences), else null
  int32_t* out_idx;
  float* out_scores;
  int32_t* cand_out;   // refine: [n_groups, c] or null
  float* cand_scores;
  uint64_t* scratch;   // [gridDim.x, scratch_per_block]
  int64_t scratch_per_block;  // multiple of 32: prefix scores, then (Refine) the member entries
  int64_t member_off;         // offset of the member entries in a block's scratch (multiple of 32)
  float* fscratch;     // [gridDim.x, H*D + H] pooled proxy / member query
};


// MTP decode groups: one group of g draft rows per sequence (decode.cu).
constexpr int kDecodeSetKeys = 512;  // keys per scan set (4 tiles of 128, one per accumulator slot)
constexpr int kSelCl = 8;            // CTAs of the decode selection's cluster (one per sequence)
constexpr int kSelClThreads = 512;   // threads per CTA of that cluster
constexpr int kSelStage = 4096;      // selected entries the cluster keeps in shared memory
constexpr int kWbarStride = 80;      // floats per sequence of the permuted w-bar table (4 rows of 20)
struct DecodeArgs {
  const uint16_t* q;        // bf16 bits [B*g, H, D]
  const float* w;           // [B*g, H]
  const int64_t* key_off;   // [B+1] row offsets of each sequence in the key cache
  int B, H, D, g;
  int n_sel;                // k+g-1 (Reuse) or c (Refine)
  int topk;
  int mode;                 // EMIT_CAND, EMIT_REUSE or EMIT_ENTRIES
  int64_t n_sets;           // sum over b of ceil(P_b / kDecodeSetKeys)
  const int64_t* pos_base;  // EMIT_ENTRIES: [B] global position of each sequence's first key here
  // workspace
  uint16_t* proxy;          // [B*H, D] bf16 bits: the pooled proxies (Eq. 4)
  float* wbar;              // [B, kWbarStride] w-bar, permuted for the epilogue
  int32_t* set_off;         // [B+1] first scan set of each sequence
  uint32_t* scores;         // [sum P] order keys of the proxy scores (Eq. 5)
  uint32_t* hist1;          // [B, 2048] counts of the order keys' top 11 bits
  uint64_t* sel;            // [B, n_sel] packed selected entries (when n_sel > kSelStage)
  uint64_t* ties;           // [sum P] packed entries: level-1 lists, then the level-2 ties
  uint64_t* ties2;          // [sum P] packed entries: level-2 lists
  // outputs
  int32_t* cand;            // [B, n_sel] (Refine)
  float* cand_scores;       // or null
  int32_t* out_idx;         // [B*g, topk] (Reuse)
  float* out_scores;        // or null
  uint64_t* entries;        // [B, n_sel] (EMIT_ENTRIES; 0 pads)
  int* status;
  uint64_t timeout_ns;
};

// Decode split: the top-n of the ranks' exchanged shard entries, then the emit.
struct MergeArgs {
  const uint64_t* entries;  // [R, B, n_sel] packed entries with global positions (0 pads)
  int R, B, g, n_sel, topk, mode;  // mode: EMIT_REUSE or EMIT_CAND
  const int64_t* plen_off;  // [B+1] offsets whose differences are the full prefix lengths P_b
  uint64_t* gather;         // workspace [B, R * n_sel]
  uint64_t* sel;            // workspace [B, n_sel]
  int32_t* out_idx;         // Reuse: [B*g, topk]
  float* out_scores;
  int32_t* cand;            // Refine: [B, n_sel] global positions
  float* cand_scores;
  const int64_t* pos_base;  // optional: this rank's shard ([B] first global position, shard_off [B+1])
  const int64_t* shard_off;
  int32_t* cand_local;      // optional: [B, n_sel] C in this rank's shard rows (-1: held elsewhere)
};
// launchers (return cudaError_t of the launch)
cudaError_t launch_scan(const ScanArgs& a, const CUtensorMap* kmap, int grid, cudaStream_t s);
size_t scan_smem_bytes(int H, int D);
cudaError_t launch_refine(const RefineArgs& a, const CUtensorMap* gather_kmap, const CUtensorMap* qmap, int grid,
                          cudaStream_t s);
size_t refine_smem_bytes(int H, int D, int mc);
cudaError_t launch_simt(const SimtArgs& a, int grid, cudaStream_t s);
cudaError_t launch_rowselect(const RowSelArgs& a, int grid, cudaStream_t s);
// MTP decode batch: prep + scan (order keys and digit histogram; scan_grid <= n_sets), then
// the selection and emit (one cluster of kSelCl CTAs per sequence).
cudaError_t launch_decode_scan(const DecodeArgs& a, const CUtensorMap* kmap, const CUtensorMap* pmap, int scan_grid,
                               cudaStream_t s);
cudaError_t launch_decode_select(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_merge(const MergeArgs& a, cudaStream_t s);
size_t decode_scan_smem_bytes(int D);

// host-side library state shared by the entry-point files (defined in api.cu)
uint64_t device_timeout_ns();     // bound on every device-side wait (pivot_set_device_timeout_ns)
int debug_flags();                // pivot_set_debug_flags
void clear_cuda_error();          // start of an entry point: pivot_last_cuda_error() reads ""
pivot_status record_cuda_error(cudaError_t e, const char* what);  // remember e; returns PIVOT_ERR_CUDA

}  // namespace pivot
