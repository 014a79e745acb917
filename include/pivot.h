/*
 * pivot.h -- C ABI of the PIVOT group-shared sparse-attention indexer for
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (PIVOT, picx.dev summary of the paper, sections
 * "Introduction and Theoretical Foundation" and "Methodology"):
 *
 *   Eq. (1)  I_{t,s} = sum_{j<H} w_{t,j} * ReLU(q_{t,j} . k_s),  T_t = TopK(I_{t,:}, k)
 *   Eq. (2)  prefill groups: positions [i*g, min(i*g+g, L))
 *   Eq. (3)  decode group: the current token and its g-1 MTP draft tokens
 *   Eq. (4)  proxy: q-bar_j = mean_t q_{t,j},  w-bar_j = mean_t w_{t,j}   (t in the group)
 *   Eq. (5)  proxy score  I-bar_s = sum_j w-bar_j ReLU(q-bar_j . k_s),  s <= last group position
 *   Eq. (6)  PIVOT-Reuse:  T_t = TopK({I-bar_s : s <= t}, k) for every member t
 *   Eq. (7)  PIVOT-Refine candidates  C = TopK({I-bar_s : s <= last group position}, c)
 *   Eq. (8)  member re-scoring  I_{t,s} for s in C
 *   Eq. (9)  T_t = TopK({I_{t,s} : s in C, s <= t}, k)
 *
 * Conventions fixed by this library where the pages are silent:
 *   - the proxy scans the prefix up to the group's LAST position; each member
 *     t then masks s <= t (so Refine with c >= L equals the dense indexer);
 *   - the pooled q-bar is rounded to nearest-even to the input dtype (it is
 *     the operand of the scan); w-bar stays fp32;
 *   - TopK order: larger score first, equal scores -> lower key index; -0.0
 *     and +0.0 are equal;
 *   - an output row holds its valid indices first, in unspecified order, and
 *     -1 in the remaining slots.  Dense and Reuse rows hold min(k, t+1)
 *     indices; Refine rows hold min(k, |C cap [0,t]|) (= min(k, t+1) when
 *     c >= k+g-1).  Indices are positions local to the sequence.
 *   - decode: sequence b holds P_b cached keys (positions 0..P_b-1, the
 *     group's own rows included); its g query rows are positions
 *     P_b-g .. P_b-1 (current token first, then the drafts).
 *
 * Memory: every tensor pointer is a DEVICE pointer owned by the caller,
 * row-major and contiguous: q_I [rows, H, d], w_I [rows, H] (fp32),
 * k_I [key rows, d], indices [rows, k] (int32), scores [rows, k] (fp32).
 * q_I and k_I are bf16 (bit patterns) or fp32 (pivot_dtype); q_I, k_I and
 * the workspace must be 16-byte aligned, and d must be a multiple of 8.
 * The library allocates nothing: scratch comes from the caller's workspace
 * (size from the *_workspace_size call for the current device).
 *
 * Execution: every call is asynchronous on `stream`; none synchronises the
 * host, except pivot_last_device_status.  Calls that share a workspace must
 * be ordered on the device (same stream or events).
 *
 * Errors are returned, never thrown; no device assert or trap is used.
 * Invalid arguments are rejected on the host before any launch.  Inputs
 * must be finite (a precondition, not checked).  Device-side waits are
 * bounded; a wait that runs out records PIVOT_ERR_DEVICE_TIMEOUT in the
 * workspace, which pivot_last_device_status reports.
 */
#ifndef PIVOT_H_
#define PIVOT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PIVOT_API __attribute__((visibility("default")))
#else
#define PIVOT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pivot_stream_t; /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum { PIVOT_BF16 = 0, PIVOT_F32 = 1 } pivot_dtype; /* dtype of q_I and k_I (w_I is fp32) */

typedef enum {
  PIVOT_OK = 0,
  PIVOT_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, k > c, misalignment ... */
  PIVOT_ERR_UNSUPPORTED_SHAPE = 2, /* g > 16, L >= 2^31, ... */
  PIVOT_ERR_WORKSPACE_TOO_SMALL = 3,
  PIVOT_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed (see pivot_last_cuda_error) */
  PIVOT_ERR_DEVICE_TIMEOUT = 5,    /* a bounded device wait ran out (reported by pivot_last_device_status) */
  PIVOT_ERR_DEVICE_BOUNDS = 6
} pivot_status;

typedef enum { PIVOT_OP_DENSE = 0, PIVOT_OP_REUSE = 1, PIVOT_OP_REFINE = 2 } pivot_op;

/* Workspace bytes needed by pivot_indexer_dense / pivot_reuse / pivot_refine
 * (op = PIVOT_OP_*) for these sizes on the CURRENT device.  c is ignored
 * unless op == PIVOT_OP_REFINE, g unless op != PIVOT_OP_DENSE.  Returns 0 for
 * arguments the call would reject. */
PIVOT_API size_t pivot_workspace_size(int op, int64_t L, int H, int d, int k, int c, int g, pivot_dtype dt);

/* Eq. (1): the dense DSA indexer, T_t for t = 0..L-1.
 * q_I [L,H,d], w_I [L,H], k_I [L,d] -> indices [L,k]; scores_opt [L,k] (or
 * NULL) receives I_{t,s} of each returned index (-inf in padded slots). */
PIVOT_API pivot_status pivot_indexer_dense(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H, int d,
                                 pivot_dtype dt, int k, int32_t *indices, float *scores_opt, void *ws,
                                 size_t ws_bytes, pivot_stream_t stream);

/* Eq. (2), (4)-(6): PIVOT-Reuse with prefill groups of g (1 <= g <= 16).
 * scores_opt receives the proxy scores I-bar_s of the returned indices. */
PIVOT_API pivot_status pivot_reuse(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H, int d,
                         pivot_dtype dt, int k, int g, int32_t *indices, float *scores_opt, void *ws,
                         size_t ws_bytes, pivot_stream_t stream);

/* Eq. (2), (4), (5), (7)-(9): PIVOT-Refine with prefill groups of g and c
 * candidates (k <= c; the pages use c = 2k).  scores_opt receives the member
 * scores I_{t,s}.  cand_opt [ceil(L/g), c] (or NULL) receives each group's
 * candidate set C_i (valid entries first, unordered, -1 padded) and
 * cand_scores_opt the proxy scores of those candidates. */
PIVOT_API pivot_status pivot_refine(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H, int d,
                          pivot_dtype dt, int k, int c, int g, int32_t *indices, float *scores_opt,
                          int32_t *cand_opt, float *cand_scores_opt, void *ws, size_t ws_bytes,
                          pivot_stream_t stream);

/* Group ranges of one prefill sequence, for splitting a sequence's groups over
 * several GPUs (the groups of Eq. (4)-(9) are independent given k_I).  Same
 * computation as pivot_indexer_dense / pivot_reuse / pivot_refine on a length-L
 * sequence, restricted to groups [g0, g1) (dense: query rows [t0, t1)); rows
 * r0 = g0*g .. r1 = min(g1*g, L) - 1 of the output are produced:
 *   q_rows [r1 + 1 - r0, H, d], w_rows [r1 + 1 - r0, H]: the range's query rows
 *     only (row r0 first);
 *   k_prefix [r1 + 1, d]: the key rows 0 .. r1 (all the range reads);
 *   indices / scores_opt [r1 + 1 - r0, k]; cand_opt / cand_scores_opt [g1 - g0, c].
 * Indices are positions in the whole sequence.  ws_bytes must cover
 * pivot_workspace_size of the whole sequence (length L).  0 <= g0 < g1 <=
 * ceil(L / g), else PIVOT_ERR_INVALID_ARG. */
PIVOT_API pivot_status pivot_indexer_dense_range(const void *q_rows, const float *w_rows, const void *k_prefix,
                                                 int64_t L, int H, int d, pivot_dtype dt, int k, int64_t t0,
                                                 int64_t t1, int32_t *indices, float *scores_opt, void *ws,
                                                 size_t ws_bytes, pivot_stream_t stream);
PIVOT_API pivot_status pivot_reuse_range(const void *q_rows, const float *w_rows, const void *k_prefix, int64_t L,
                                         int H, int d, pivot_dtype dt, int k, int g, int64_t g0, int64_t g1,
                                         int32_t *indices, float *scores_opt, void *ws, size_t ws_bytes,
                                         pivot_stream_t stream);
PIVOT_API pivot_status pivot_refine_range(const void *q_rows, const float *w_rows, const void *k_prefix, int64_t L,
                                          int H, int d, pivot_dtype dt, int k, int c, int g, int64_t g0, int64_t g1,
                                          int32_t *indices, float *scores_opt, int32_t *cand_opt,
                                          float *cand_scores_opt, void *ws, size_t ws_bytes, pivot_stream_t stream);

/* Proxy aggregation variants (PIVOT paper, Ablation Studies, "Proxy aggregation
 * (Table 2)": mean pooling against a first- or last-query proxy).  As
 * pivot_reuse / pivot_refine, with the group proxy of Eq. (4) replaced by:
 *   aggregation 0  the mean of the members (Eq. 4; the calls above),
 *               1  the first member's query and w (the earliest position),
 *               2  the last member's query and w.
 * Other values return PIVOT_ERR_INVALID_ARG. */
PIVOT_API pivot_status pivot_reuse_agg(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H, int d,
                                       pivot_dtype dt, int k, int g, int aggregation, int32_t *indices,
                                       float *scores_opt, void *ws, size_t ws_bytes, pivot_stream_t stream);
PIVOT_API pivot_status pivot_refine_agg(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H,
                                        int d, pivot_dtype dt, int k, int c, int g, int aggregation,
                                        int32_t *indices, float *scores_opt, int32_t *cand_opt,
                                        float *cand_scores_opt, void *ws, size_t ws_bytes,
                                        pivot_stream_t stream);

/* PIVOT-Refine of one prefill sequence held in HOST memory (same computation as
 * pivot_refine, Eq. (2), (4), (5), (7)-(9); the groups are independent given
 * k_I, so the sequence is indexed in runs of whole groups).  q_host [L,H,d] bf16,
 * w_host [L,H] fp32, k_host [L,d] bf16 and out_host [L,k] int32 are host
 * pointers; they should be pinned (cudaHostAlloc / cudaHostRegister), otherwise
 * the copies do not overlap.  The keys and weights are copied first, then the
 * queries in `chunks` (1..64) runs of whole groups on a copy stream, from the
 * sequence's end to its start (the groups with the longest prefixes first, so
 * the run indexed last is the cheapest); each run is indexed on `stream`
 * (pivot_refine_range) once its rows have landed, while the next run is
 * copied in and the previous run's rows are copied back on a second copy
 * stream.  ws is a DEVICE buffer of pivot_refine_host_workspace_size bytes
 * (256-byte aligned) that holds the device copies and the refine workspace.
 * Asynchronous: when the call returns the work is queued and `stream` is ordered
 * after the last copy back, so synchronise `stream` before reading out_host or
 * reusing the host buffers.  The first call on a device creates two copy
 * streams and 130 events that live until the process exits; make that call
 * before any stream capture.  Calls on one device enqueue one at a time (a
 * mutex) and share the copy streams; give concurrent calls their own ws.
 * Errors: PIVOT_ERR_INVALID_ARG (null pointer, chunks outside 1..64, c < k,
 * misaligned ws), PIVOT_ERR_UNSUPPORTED_SHAPE, PIVOT_ERR_WORKSPACE_TOO_SMALL,
 * PIVOT_ERR_CUDA (pivot_last_cuda_error says which call). */
PIVOT_API size_t pivot_refine_host_workspace_size(int64_t L, int H, int d, int k, int c, int g);
PIVOT_API pivot_status pivot_refine_host(const void *q_host, const float *w_host, const void *k_host, int64_t L,
                                         int H, int d, int k, int c, int g, int chunks, int32_t *out_host, void *ws,
                                         size_t ws_bytes, pivot_stream_t stream);

/* Guardrail (PIVOT paper, "Efficiency Results (Figure 4)": PIVOT falls back to
 * dense DSA at short context to avoid overhead).  The pages give no criterion;
 * this library uses the work model of the prefill call, in key-row products
 * q.k (each 2*H*d FLOPs):
 *   dense  sum_t (t + 1) = L (L + 1) / 2
 *   Reuse  sum_i P_i                            (the proxy scan, Eq. 5)
 *   Refine sum_i (P_i + |G_i| * min(c, P_i))    (scan + re-scoring, Eq. 5, 8)
 * with groups G_i of g consecutive positions and P_i = the group's end + 1.
 * Returns 1 when dense needs no more work than op (PIVOT_OP_REUSE or
 * PIVOT_OP_REFINE), 0 when the PIVOT variant is cheaper, -1 for invalid
 * arguments (L < 1, g < 1, c < 1 for Refine, other ops). */
PIVOT_API int pivot_guardrail_dense(int op, int64_t L, int c, int g);

/* pivot_reuse / pivot_refine behind the guardrail: when pivot_guardrail_dense
 * returns 1 the call runs pivot_indexer_dense instead (indices and scores_opt
 * then hold the dense rows; cand_opt and cand_scores_opt are not written).
 * *path_out (host pointer, may be NULL) receives 1 for dense, 0 for PIVOT.
 * ws_bytes must cover the path taken: pivot_workspace_size of PIVOT_OP_DENSE
 * or of op, as pivot_guardrail_dense says. */
PIVOT_API pivot_status pivot_reuse_guarded(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H,
                                           int d, pivot_dtype dt, int k, int g, int32_t *indices, float *scores_opt,
                                           void *ws, size_t ws_bytes, pivot_stream_t stream, int *path_out);
PIVOT_API pivot_status pivot_refine_guarded(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H,
                                            int d, pivot_dtype dt, int k, int c, int g, int32_t *indices,
                                            float *scores_opt, int32_t *cand_opt, float *cand_scores_opt, void *ws,
                                            size_t ws_bytes, pivot_stream_t stream, int *path_out);

/* Workspace bytes for the decode calls below.  key_offsets_host [B+1] is the
 * host copy of the key offsets (key_offsets_host[0] = 0, non-decreasing,
 * every P_b = key_offsets_host[b+1] - key_offsets_host[b] >= g).  On the
 * tensor-core path (bf16, H = 64, d in {64, 128}) it grows with the batch's
 * keys: 20 bytes per cached key (a 32-bit score key and room for two packed
 * selection lists) plus per-sequence proxies, histograms and the selection. */
PIVOT_API size_t pivot_varlen_workspace_size(int op, int B, const int64_t *key_offsets_host, int H, int d, int k, int c,
                                   int g, pivot_dtype dt);

/* Eq. (3)-(6): PIVOT-Reuse for a batch of B MTP decode groups.
 * q [B*g,H,d] (rows b*g..b*g+g-1 = sequence b's current token then drafts),
 * w [B*g,H], k_cache [sum P_b, d] (sequence b's keys are rows
 * key_offsets[b] .. key_offsets[b+1]-1), key_offsets_dev / key_offsets_host
 * [B+1] (same values, device and host copies) -> indices [B*g,k] of
 * positions local to each sequence.  Asynchronous on `stream`.  Returns
 * PIVOT_ERR_UNSUPPORTED_SHAPE when 8 * B exceeds 2^31 - 1 (the selection
 * grid: one 8-CTA cluster per sequence).  A device-side wait that runs out (PIVOT_ERR_DEVICE_TIMEOUT
 * from pivot_last_device_status) leaves the outputs undefined; the selection
 * then never writes past its buffers and may also flag PIVOT_ERR_DEVICE_BOUNDS. */
PIVOT_API pivot_status pivot_reuse_varlen(const void *q, const float *w, const void *k_cache, const int64_t *key_offsets_dev,
                                const int64_t *key_offsets_host, int B, int H, int d, pivot_dtype dt, int k, int g,
                                int32_t *indices, float *scores_opt, void *ws, size_t ws_bytes,
                                pivot_stream_t stream);

/* Eq. (3)-(5), (7)-(9): PIVOT-Refine for a batch of B MTP decode groups;
 * arguments as pivot_reuse_varlen plus c, cand_opt [B,c], cand_scores_opt. */
PIVOT_API pivot_status pivot_refine_varlen(const void *q, const float *w, const void *k_cache,
                                 const int64_t *key_offsets_dev, const int64_t *key_offsets_host, int B, int H,
                                 int d, pivot_dtype dt, int k, int c, int g, int32_t *indices, float *scores_opt,
                                 int32_t *cand_opt, float *cand_scores_opt, void *ws, size_t ws_bytes,
                                 pivot_stream_t stream);

/* ---- One long decode prefix split over ranks (one exchange, then one merge).
 * Eq. (3), (5)-(7) select over a group's whole prefix, and the exact top-n of
 * a set is inside the union of the exact top-n of its parts.  So rank r of R
 * holds, for every sequence b, one contiguous shard of its cached keys: rows
 * shard_offsets[b] .. shard_offsets[b+1]-1 of k_shard (at least one row), which
 * are the prefix positions pos_base[b] .. of a prefix of P_b = plen_offsets[b+1]
 * - plen_offsets[b] keys (P_b >= g).  Every rank holds all q [B*g,H,d] and w
 * [B*g,H] rows.  Steps:
 *   1. pivot_decode_shard_select (each rank): the shard's exact top-n, n = k+g-1
 *      (Reuse) or c (Refine), as packed entries [B, n] uint64 (order key << 32 |
 *      (0xFFFFFFFF - prefix position); 0 pads a shard with fewer keys);
 *   2. exchange: all-gather of the entries into [R, B, n] (rank order free);
 *   3. pivot_decode_merge (every rank): Reuse rows [B*g, k], or the candidate set
 *      C [B, c] (prefix positions) and, for this rank, C in its shard's rows;
 *   Refine adds:
 *   4. pivot_decode_shard_rescore (each rank): Eq. (8) member score keys [B*g, c]
 *      (uint32) of the candidates this rank holds, 0 for the others;
 *   5. exchange: element-wise sum of the keys over the ranks (every candidate is
 *      held by exactly one rank);
 *   6. pivot_decode_rowselect: Eq. (9), indices [B*g, k] of prefix positions.
 * The results equal pivot_reuse_varlen / pivot_refine_varlen on the whole prefix.
 * Tensor-core shape only (bf16, H = 64, d in {64, 128}), else
 * PIVOT_ERR_UNSUPPORTED_SHAPE.  All pointers are device pointers except the
 * *_host offsets; all calls are asynchronous on `stream`; the caller owns every
 * buffer.  Errors (returned before any device work): PIVOT_ERR_INVALID_ARG
 * (an op other than Reuse / Refine, null pointers, a shard without a key, a
 * prefix shorter than g, c < k, a local C without this rank's shard, a
 * misaligned q / k_shard / ws), PIVOT_ERR_UNSUPPORTED_SHAPE,
 * PIVOT_ERR_WORKSPACE_TOO_SMALL, PIVOT_ERR_CUDA (pivot_last_cuda_error says
 * which call).  Steps 1 and 4 use the library-wide bounded device waits
 * (pivot_last_device_status on their workspace reports a timeout). */

/* Step 1.  ws: pivot_decode_shard_workspace_size bytes (0: unsupported shape or
 * offsets).  op is PIVOT_OP_REUSE (c ignored) or PIVOT_OP_REFINE. */
PIVOT_API size_t pivot_decode_shard_workspace_size(int op, int B, const int64_t *shard_offsets_host, int H, int d,
                                                   int k, int c, int g);
PIVOT_API pivot_status pivot_decode_shard_select(int op, const void *q, const float *w, const void *k_shard,
                                                 const int64_t *shard_offsets_dev, const int64_t *shard_offsets_host,
                                                 const int64_t *pos_base_dev, int B, int H, int d, pivot_dtype dt,
                                                 int k, int c, int g, uint64_t *entries, void *ws, size_t ws_bytes,
                                                 pivot_stream_t stream);

/* Step 3.  entries [R, B, n] from step 2.  Reuse writes indices [B*g, k] (and
 * scores_opt); Refine writes cand [B, c] (and cand_scores_opt), and cand_local_opt
 * [B, c] (-1 where another rank holds the key) when pos_base_dev and
 * shard_offsets_dev describe this rank's shard.  ws: the bytes below. */
PIVOT_API size_t pivot_decode_merge_workspace_size(int op, int R, int B, int k, int c, int g);
PIVOT_API pivot_status pivot_decode_merge(int op, const uint64_t *entries, int R, const int64_t *plen_offsets_dev,
                                          const int64_t *plen_offsets_host, int B, int k, int c, int g,
                                          int32_t *indices, float *scores_opt, int32_t *cand, float *cand_scores_opt,
                                          const int64_t *pos_base_dev, const int64_t *shard_offsets_dev,
                                          int32_t *cand_local_opt, void *ws, size_t ws_bytes, pivot_stream_t stream);

/* Step 4.  cand_local [B, c] from step 3; keys [B*g, c]; ws: at least 256 bytes
 * (step 1's workspace will do). */
PIVOT_API pivot_status pivot_decode_shard_rescore(const void *q, const float *w, const void *k_shard,
                                                  const int64_t *shard_offsets_dev, const int64_t *shard_offsets_host,
                                                  const int64_t *pos_base_dev, const int64_t *plen_offsets_dev, int B,
                                                  int H, int d, pivot_dtype dt, int k, int c, int g,
                                                  const int32_t *cand_local, uint32_t *keys, void *ws,
                                                  size_t ws_bytes, pivot_stream_t stream);

/* Step 6.  keys [B*g, c] summed over the ranks, cand [B, c] from step 3. */
PIVOT_API pivot_status pivot_decode_rowselect(const uint32_t *keys, const int32_t *cand,
                                              const int64_t *plen_offsets_dev, int B, int k, int c, int g,
                                              int32_t *indices, float *scores_opt, pivot_stream_t stream);

/* Synchronises `stream`, then reads the device status word that the last
 * call using workspace `ws` left: PIVOT_OK, PIVOT_ERR_DEVICE_TIMEOUT or
 * PIVOT_ERR_DEVICE_BOUNDS (or PIVOT_ERR_CUDA if the sync/copy failed). */
PIVOT_API pivot_status pivot_last_device_status(const void *ws, pivot_stream_t stream);

/* Human-readable name of a status code (static string). */
PIVOT_API const char *pivot_status_string(pivot_status s);

/* Text of the last CUDA error seen by this library in the calling thread ("" if none). */
PIVOT_API const char *pivot_last_cuda_error(void);

/* Which kernel path a call with these arguments takes on the current device:
 * 1 = tcgen05 tensor-core path (bf16, H = 64, d in {64,128}), 0 = CUDA-core
 * path, -1 = the call would be rejected. */
PIVOT_API int pivot_path(int op, int64_t L, int H, int d, int k, int c, int g, pivot_dtype dt);

/* Bound (nanoseconds of wall-clock time) on every device-side wait; default
 * 2e9.  Test hooks (pivot_set_debug_flags, process-wide, 0 = normal):
 *   bit 0 (1): the scan kernel waits on a barrier that nothing signals, so
 *              the bound runs out and the timeout path is exercised without
 *              hanging the GPU;
 *   bit 1 (2): the scan visits key tiles in natural order (no sampled
 *              threshold estimate);
 *   bit 2 (4): the sampled estimate is taken at the sample's best entry, so
 *              it is too high and every long work item is scanned a second
 *              time (exercises the exact fallback).
 * Results are identical under bits 1 and 2; only the work differs. */
PIVOT_API void pivot_set_device_timeout_ns(uint64_t ns);
PIVOT_API void pivot_set_debug_flags(int flags);

/* Measurement hook: when events != NULL (n >= 4 cudaEvent_t handles created
 * by the caller), every following call records them on its stream:
 * events[0] before its first kernel, events[1] after the scan kernel,
 * events[2] after the refine kernel and events[3] after the last kernel
 * (unused slots are recorded at the same point as the previous one).  A
 * decode-batch call records events[1] after its proxies and scan, events[2]
 * after its selection and emit, events[3] after its last kernel.
 * Pass NULL to stop.  Not thread-safe; a process-wide setting. */
PIVOT_API void pivot_set_profile_events(void **events, int n);

/* PIVOT-Reuse without a workspace (the pages describing PIVOT have no
 * counterpart of this; it is an integration convenience).  For callers that
 * cannot allocate device memory, e.g. whose device memory belongs to a pool
 * or memory planner they do not control, so they can neither call cudaMalloc
 * nor hand over a workspace.  Computes exactly what pivot_reuse computes,
 * with the same arguments minus the workspace, on the tensor-core scan
 * kernel; its scratch (status word, work counter, candidate buffers) is a
 * fixed static device array of 12,124,416 B + 256 B (about 11.6 MiB) that
 * every process loading this library holds on every device it uses until
 * exit.
 * Limits: bf16 q/k, H = 64, d in {64, 128}, g <= 16 and k + g - 1 <= 256;
 * larger sizes return PIVOT_ERR_UNSUPPORTED_SHAPE without launching.  At most
 * 148 CTAs run (one per SM).
 * The first call on a device looks the array's device address up (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents: calls that overlap on the GPU (other streams, other host
 * threads) race and give undefined results, so order them.  Device-side
 * waits are bounded by pivot_set_device_timeout_ns like every other call,
 * but a wait that runs out is not reported (there is no workspace for
 * pivot_last_device_status to read); the outputs are then undefined.
 * pivot_last_cuda_error describes a PIVOT_ERR_CUDA return.  Allocates
 * nothing. */
PIVOT_API pivot_status pivot_reuse_noalloc(const void *q_I, const float *w_I, const void *k_I, int64_t L, int H,
                                           int d, pivot_dtype dt, int k, int g, int32_t *indices, float *scores_opt,
                                           pivot_stream_t stream);

PIVOT_API int pivot_version(void); /* 100 * major + minor */

#ifdef __cplusplus
}
#endif
#endif /* PIVOT_H_ */
