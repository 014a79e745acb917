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
  EMIT_PARTIAL = 3  // decode chunk: write the chunk's top-n_sel packed entries
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
  // decode (mode EMIT_PARTIAL): item -> (sequence, key chunk)
  const int64_t* key_off;     // [B+1] row offsets of each sequence in the key tensor
  const int32_t* item_seq;    // [n_items] sequence of each item
  const int64_t* item_s0;     // [n_items] first local key of the chunk
  const int64_t* item_s1;     // [n_items] one past the last local key
  uint64_t* partial;          // [n_items, partial_stride] packed entries (EMIT_PARTIAL)
  int partial_stride;         // >= n_sel, multiple of 32 (zero padded)
  uint32_t* partial_cnt;      // [n_items]
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
  int64_t n_groups;
  int n_items;           // n_groups * ceil(g / mc)
  const int32_t* cand;   // [n_groups, c]  (-1 padded)
  const int64_t* key_off;  // decode: [B+1]; null for prefill
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

struct MergeArgs {
  const uint64_t* partial;     // [n_items, n_sel]
  const uint32_t* partial_cnt; // [n_items]
  const int32_t* seq_item0;    // [B+1] first item of each sequence
  int n_sel;                   // c (refine) or k+g-1 (reuse)
  int partial_stride;          // entries per item in `partial` (>= n_sel, zero padded)
  int B, g, topk, mode;        // mode: EMIT_CAND or EMIT_REUSE
  const int64_t* key_off;      // [B+1]
  uint64_t* scratch;           // [gridDim.x, cap]
  int cap;
  int32_t* cand;               // [B, n_sel]
  float* cand_scores;
  int32_t* out_idx;            // [B*g, topk]
  float* out_scores;
};

// launchers (return cudaError_t of the launch)
cudaError_t launch_scan(const ScanArgs& a, const CUtensorMap* kmap, int grid, cudaStream_t s);
size_t scan_smem_bytes(int H, int D);
cudaError_t launch_refine(const RefineArgs& a, const CUtensorMap* gather_kmap, const CUtensorMap* qmap, int grid,
                          cudaStream_t s);
size_t refine_smem_bytes(int H, int D, int mc);
cudaError_t launch_simt(const SimtArgs& a, int grid, cudaStream_t s);
cudaError_t launch_merge(const MergeArgs& a, int grid, cudaStream_t s);
cudaError_t launch_rowselect(const RowSelArgs& a, int grid, cudaStream_t s);
cudaError_t launch_plan_items(const int64_t* key_off, int B, int64_t chunk, int32_t* item_seq, int64_t* item_s0,
                              int64_t* item_s1, int32_t* seq_item0, cudaStream_t s);

}  // namespace pivot
