// select.cuh -- exact TopK machinery used by every kernel of the library.
//
// TopK order of the indexer (PIVOT, picx.dev summary, Eq. 1 "T_t = TopK"):
// larger score first; equal scores -> lower key index first; -0.0 == +0.0.
// Each (score, index) pair is packed into one uint64 whose unsigned order is
// exactly that order:
//     packed = orderkey(score) << 32 | (0xFFFFFFFF - index)
// so all packed values of one row are distinct and "the n best" is "the n
// largest packed values".  Selection is a most-significant-digit radix
// select (8-bit digits, shared-memory histogram) followed by a stream
// compaction, run by a group of NT threads that sync on one named barrier.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace pivot {

__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;  // -0.0 ties with +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ uint64_t pack_entry(uint32_t key, uint32_t idx) {
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - idx);
}
__device__ __forceinline__ uint32_t entry_idx(uint64_t p) { return 0xFFFFFFFFu - (uint32_t)p; }
__device__ __forceinline__ float entry_score(uint64_t p) { return key_score((uint32_t)(p >> 32)); }

struct alignas(16) SelSmem {  // hist is also reused as uint64 scratch (emit_reuse)
  uint32_t hist[256];
  uint32_t warp_tot[32];
  uint32_t scal[4];
};

// A group of NT threads (NT multiple of 32, tid in [0, NT)) synchronised by
// named barrier `bar` (bar 0 with NT == blockDim.x is __syncthreads).
template <int NT>
struct Group {
  int tid;
  int bar;
  __device__ __forceinline__ void sync() const { named_bar_sync(bar, NT); }
};

// Warp-aggregated append of `val` (when `pass`) to buf[*cnt ...]; the whole warp calls.
__device__ __forceinline__ void warp_append(bool pass, uint64_t val, uint64_t* buf, uint32_t* cnt) {
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, pass);
  if (m == 0u) return;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0;
  if ((int)lane_id() == leader) base = atomicAdd(cnt, (uint32_t)__popc(m));
  base = __shfl_sync(0xFFFFFFFFu, base, leader);
  if (pass) buf[base + __popc(m & lanemask_lt())] = val;
}

// Visit every slot of buf[0..n) (f(x, valid) for x = buf[i]; slots past n
// come with valid = false) with U loads in flight per thread and a trip count
// that is the same for all NT threads, so warp-synchronous code (match_any,
// ballot) may run inside f.  16-byte loads when buf is 16-byte aligned,
// 8-byte loads otherwise.
template <int NT, int U, typename F>
__device__ __forceinline__ void visit_entries(const uint64_t* buf, uint32_t n, const Group<NT>& G, F&& f) {
  if ((reinterpret_cast<uintptr_t>(buf) & 15u) != 0) {
    for (uint32_t base = 0; base < n; base += NT * U) {
      uint64_t v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t i = base + u * NT + G.tid;
        v[u] = (i < n) ? buf[i] : 0ull;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) f(v[u], base + u * NT + G.tid < n);
    }
    return;
  }
  constexpr uint32_t STEP = NT * 2 * U;
  for (uint32_t base = 0; base < n; base += STEP) {
    ulonglong2 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      if (i + 1 < n) {
        v[u] = *reinterpret_cast<const ulonglong2*>(buf + i);
      } else {
        v[u].x = (i < n) ? buf[i] : 0ull;
        v[u].y = 0ull;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      f(v[u].x, i < n);
      f(v[u].y, i + 1 < n);
    }
  }
}

// Warp-aggregated histogram increment (bin >= 256 = skip); whole warp calls.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
  if (bin < 256u && (int)lane_id() == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Returns a threshold T such that count{ buf[i] >= T } lies in [need, max_keep]
// (exactly `need` when max_keep == need).  Requires need <= n.  All NT threads
// call it and get the same T.  T == 0 keeps everything.  hist1 (optional) is
// the histogram of the top 8 bits of buf[0..n); it saves the first pass.
template <int NT>
__device__ uint64_t radix_threshold(const uint64_t* buf, uint32_t n, uint32_t need, uint32_t max_keep,
                                    SelSmem& S, const Group<NT>& G, const uint32_t* hist1 = nullptr) {
  if (n <= max_keep) return 0ull;
  uint64_t prefix = 0;
  uint32_t above = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    const uint32_t* hist = S.hist;
    if (shift == 56 && hist1 != nullptr) {
      hist = hist1;
    } else {
      for (int i = G.tid; i < 256; i += NT) S.hist[i] = 0u;
      G.sync();
      visit_entries<NT, 4>(buf, n, G, [&](uint64_t x, bool valid) {
        const bool match = valid && (shift == 56 || (x >> (shift + 8)) == prefix);
        hist_add(S.hist, match ? ((uint32_t)(x >> shift) & 255u) : 256u);
      });
      G.sync();
    }
    if (G.tid < 32) {
      const int l = G.tid;
      uint32_t loc[8], sum = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        loc[u] = hist[255 - 8 * l - u];
        sum += loc[u];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (l >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      if (above + excl < need && need <= above + incl) {
        uint32_t c = above + excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (c + loc[u] >= need) {
            S.scal[0] = 255u - 8u * l - u;
            S.scal[1] = c;
            S.scal[2] = loc[u];
            break;
          }
          c += loc[u];
        }
      }
    }
    G.sync();
    const uint32_t digit = S.scal[0];
    above = S.scal[1];
    const uint32_t h = S.scal[2];
    prefix = (prefix << 8) | digit;
    G.sync();  // everyone has read scal / hist before they are rewritten
    if (above + h <= max_keep || shift == 0) return prefix << shift;
  }
  return prefix;
}

// Block-wide min and max of 64-bit values (every thread of G calls; all get the result).
template <int NT>
__device__ __forceinline__ void group_minmax64(uint64_t& lo, uint64_t& hi, SelSmem& S, const Group<NT>& G) {
  static_assert(NT / 32 <= 64, "at most 64 warps");
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, o), h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    lo = l2 < lo ? l2 : lo;
    hi = h2 > hi ? h2 : hi;
  }
  uint64_t* sc = reinterpret_cast<uint64_t*>(S.hist);  // 128 x uint64 of scratch
  const int w = G.tid >> 5;
  if ((G.tid & 31) == 0) {
    sc[w] = lo;
    sc[64 + w] = hi;
  }
  G.sync();
  lo = sc[0];
  hi = sc[64];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) {
    lo = sc[i] < lo ? sc[i] : lo;
    hi = sc[64 + i] > hi ? sc[64 + i] : hi;
  }
  G.sync();
}

// Up to 4 disjoint segments of packed entries, read as one set.
struct Segs {
  const uint64_t* p[4];
  uint32_t n[4];
  int cnt;
};

// One warp keeps the entries >= T of seg[0..n) in place; returns the new count.
// seg must be 16-byte aligned; 2*V entries per lane are in flight per chunk.
__device__ __forceinline__ uint32_t warp_compact_ge(uint64_t* seg, uint32_t n, uint64_t T) {
  constexpr int V = 8;
  const uint32_t lane = lane_id();
  const uint32_t lt = lanemask_lt();
  uint32_t out = 0;
  for (uint32_t base = 0; base < n; base += 64 * V) {
    ulonglong2 x[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t i = base + (v * 32 + lane) * 2;
      if (i + 1 < n) {
        x[v] = *reinterpret_cast<const ulonglong2*>(seg + i);
      } else {
        x[v].x = (i < n) ? seg[i] : 0ull;
        x[v].y = 0ull;
      }
    }
    __syncwarp();
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t i = base + (v * 32 + lane) * 2;
      const bool k0 = (i < n) && x[v].x >= T;
      const bool k1 = (i + 1 < n) && x[v].y >= T;
      const uint32_t m0 = __ballot_sync(0xFFFFFFFFu, k0);
      const uint32_t m1 = __ballot_sync(0xFFFFFFFFu, k1);
      // this lane's two survivors go after the survivors of the lower lanes (order is free)
      uint32_t pos = out + __popc(m0 & lt) + __popc(m1 & lt);
      if (k0) seg[pos++] = x[v].x;
      if (k1) seg[pos] = x[v].y;
      out += __popc(m0) + __popc(m1);
    }
    __syncwarp();
  }
  return out;
}

// Copy src[0..n) to dst (both 16-byte aligned) with the NT threads of a group, 8 entries in flight each.
template <int NT>
__device__ __forceinline__ void group_copy(uint64_t* dst, const uint64_t* src, uint32_t n, const Group<NT>& G) {
  constexpr int U = 4;
  for (uint32_t base = 0; base < n; base += NT * 2 * U) {
    ulonglong2 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      if (i + 1 < n) v[u] = *reinterpret_cast<const ulonglong2*>(src + i);
      else if (i < n) v[u].x = src[i];
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      if (i + 1 < n) *reinterpret_cast<ulonglong2*>(dst + i) = v[u];
      else if (i < n) dst[i] = v[u].x;
    }
  }
}

// group_copy that also returns max(hi, the largest entry copied) to every thread's own
// view (each thread sees the maximum of what it copied; reduce across the group after).
template <int NT>
__device__ __forceinline__ uint64_t group_copy_max(uint64_t* dst, const uint64_t* src, uint32_t n, uint64_t hi,
                                                   const Group<NT>& G) {
  constexpr int U = 4;
  for (uint32_t base = 0; base < n; base += NT * 2 * U) {
    ulonglong2 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      v[u].x = v[u].y = 0ull;
      if (i + 1 < n) v[u] = *reinterpret_cast<const ulonglong2*>(src + i);
      else if (i < n) v[u].x = src[i];
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = base + (u * NT + G.tid) * 2;
      if (i + 1 < n) *reinterpret_cast<ulonglong2*>(dst + i) = v[u];
      else if (i < n) dst[i] = v[u].x;
      hi = v[u].x > hi ? v[u].x : hi;
      hi = v[u].y > hi ? v[u].y : hi;
    }
  }
  return hi;
}

// Inclusive warp scan of v.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int l = lane_id();
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (l >= o) v += t;
  }
  return v;
}

// Block-level exclusive offsets of per-thread counts: returns this thread's
// offset; *total gets the group total.  Two syncs.
template <int NT>
__device__ __forceinline__ uint32_t group_offsets(uint32_t cnt, uint32_t* total, SelSmem& S, const Group<NT>& G) {
  const uint32_t incl = warp_incl_scan(cnt);
  const int w = G.tid >> 5;
  if ((G.tid & 31) == 31) S.warp_tot[w] = incl;
  G.sync();
  uint32_t off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    const uint32_t t = S.warp_tot[i];
    if (i < w) off += t;
    tot += t;
  }
  *total = tot;
  return off + incl - cnt;
}

// ---------------------------------------------------------------- 11-bit digits

// The 2048-bin histogram is stored with one pad word after every 32 bins, so
// the digit search (thread t reads bins BPT*t .. BPT*t + BPT-1, BPT = 4 or 8)
// hits 32 distinct banks per warp instead of 32 / BPT.
constexpr int kHist11Words = 2048 + 64;
__device__ __forceinline__ uint32_t h11(uint32_t bin) { return bin + (bin >> 5); }

// Like radix_threshold, with 11-bit digits (at most 6 passes, usually 2) and a
// 2048-bin shared-memory histogram `hist` (kHist11Words words, padded layout)
// updated with plain atomics.  The
// entries are the union of the segments of sg.
// When [lo, hi] is given (lo <= every entry that can be selected, hi >= every
// entry, at least `need` entries inside), the digits start below the bits lo
// and hi share: for scores packed from a narrow range that skips the sign and
// exponent bits that all of them have in common, so one or two passes suffice.
template <int NT>
__device__ uint64_t radix11_threshold(const Segs& sg, uint32_t need, uint32_t max_keep, uint32_t* hist,
                                      SelSmem& S, const Group<NT>& G, uint64_t lo = 0ull,
                                      uint64_t hi = ~0ull) {
  static_assert(2048 % NT == 0, "NT must divide 2048");
  constexpr int BPT = 2048 / NT;  // bins per thread in the digit search
  uint32_t n = 0;
  for (int i = 0; i < sg.cnt; ++i) n += sg.n[i];
  if (n <= max_keep) return 0ull;
  int consumed = (lo == hi) ? 64 : __clzll(lo ^ hi);  // bits every entry of interest shares
  if (consumed == 64) return lo;
  uint64_t prefix = consumed ? (hi >> (64 - consumed)) : 0ull;
  uint32_t above = 0;
  while (consumed < 64) {
    const int w = (64 - consumed) < 11 ? (64 - consumed) : 11, shift = 64 - consumed - w;
    const uint32_t nb = 1u << w;
    for (uint32_t i = G.tid; i < (uint32_t)kHist11Words; i += NT) hist[i] = 0u;
    G.sync();
    for (int sgi = 0; sgi < sg.cnt; ++sgi)
      visit_entries<NT, 8>(sg.p[sgi], sg.n[sgi], G, [&](uint64_t x, bool valid) {
        if (valid && (consumed == 0 || (x >> (64 - consumed)) == prefix))
          atomicAdd(&hist[h11((uint32_t)(x >> shift) & (nb - 1u))], 1u);
      });
    G.sync();
    // thread t owns bins [nb-1 - BPT*t - (BPT-1), nb-1 - BPT*t] (descending); bins >= nb are empty
    uint32_t loc[BPT], sum = 0;
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
      const int bin = 2047 - BPT * G.tid - u - (2048 - (int)nb);
      loc[u] = (bin >= 0) ? hist[h11((uint32_t)bin)] : 0u;
      sum += loc[u];
    }
    uint32_t total;
    const uint32_t excl = group_offsets<NT>(sum, &total, S, G);
    if (above + excl < need && need <= above + excl + sum) {
      uint32_t c = above + excl;
#pragma unroll
      for (int u = 0; u < BPT; ++u) {
        if (c + loc[u] >= need) {
          S.scal[0] = (uint32_t)(2047 - BPT * G.tid - u - (2048 - (int)nb));
          S.scal[1] = c;
          S.scal[2] = loc[u];
          break;
        }
        c += loc[u];
      }
    }
    G.sync();
    const uint32_t digit = S.scal[0];
    above = S.scal[1];
    const uint32_t h = S.scal[2];
    prefix = (prefix << w) | digit;
    consumed += w;
    G.sync();
    if (above + h <= max_keep || shift == 0) return prefix << shift;
  }
  return prefix;
}

template <int NT>
__device__ __forceinline__ uint64_t radix11_threshold(const uint64_t* buf, uint32_t n, uint32_t need,
                                                      uint32_t max_keep, uint32_t* hist, SelSmem& S,
                                                      const Group<NT>& G, uint64_t lo = 0ull,
                                                      uint64_t hi = ~0ull) {
  Segs sg;
  sg.cnt = 1;
  sg.p[0] = buf;
  sg.n[0] = n;
  return radix11_threshold<NT>(sg, need, max_keep, hist, S, G, lo, hi);
}

// Stream-compact the entries >= T of src[0..n) into dst[0..m) (dst may be
// src: every chunk is fully read before any of its survivors is written, and
// survivors never move forward).  Returns m.  When hist1 is given it is
// rebuilt as the top-8-bit histogram of the survivors.
template <int NT, int V = 8>
__device__ uint32_t compact_ge(const uint64_t* src, uint64_t* dst, uint32_t n, uint64_t T, SelSmem& S,
                               const Group<NT>& G, uint32_t* hist1 = nullptr) {
  if (hist1) {
    for (int i = G.tid; i < 256; i += NT) hist1[i] = 0u;
    G.sync();
  }
  uint32_t base = 0;
  for (uint32_t c0 = 0; c0 < n; c0 += NT * V) {
    uint64_t x[V];
    uint32_t keep = 0, cnt = 0;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t i = c0 + v * NT + G.tid;
      x[v] = (i < n) ? src[i] : 0ull;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t i = c0 + v * NT + G.tid;
      const bool k = (i < n) && (x[v] >= T);
      keep |= (k ? 1u : 0u) << v;
      cnt += k ? 1u : 0u;
      if (hist1) hist_add(hist1, k ? (uint32_t)(x[v] >> 56) : 256u);
    }
    uint32_t total;
    uint32_t pos = base + group_offsets<NT>(cnt, &total, S, G);
#pragma unroll
    for (int v = 0; v < V; ++v)
      if (keep & (1u << v)) dst[pos++] = x[v];
    base += total;
    G.sync();
  }
  return base;
}

// Write the indices (and optionally scores) of the entries of buf[0..n) that
// satisfy  idx <= t_max && entry > cut  to row[0..) in arbitrary order; pad
// the rest of row[0..width) with -1.  Returns the number written.
template <int NT>
__device__ uint32_t emit_row(const uint64_t* buf, uint32_t n, uint32_t t_max, uint64_t cut, int32_t* row,
                             float* row_scores, uint32_t width, SelSmem& S, const Group<NT>& G) {
  uint32_t base = 0;
  constexpr int V = 4;
  for (uint32_t c0 = 0; c0 < n; c0 += NT * V) {
    uint64_t x[V];
    uint32_t keep = 0, cnt = 0;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t i = c0 + v * NT + G.tid;
      x[v] = (i < n) ? buf[i] : 0ull;
      const bool k = (i < n) && (entry_idx(x[v]) <= t_max) && (x[v] > cut);
      keep |= (k ? 1u : 0u) << v;
      cnt += k ? 1u : 0u;
    }
    uint32_t total;
    uint32_t pos = base + group_offsets<NT>(cnt, &total, S, G);
#pragma unroll
    for (int v = 0; v < V; ++v)
      if ((keep & (1u << v)) && pos < width) {
        row[pos] = (int32_t)entry_idx(x[v]);
        if (row_scores) row_scores[pos] = entry_score(x[v]);
        ++pos;
      }
    base += total;
    G.sync();
  }
  const uint32_t m = base < width ? base : width;
  for (uint32_t i = m + G.tid; i < width; i += NT) {
    row[i] = -1;
    if (row_scores) row_scores[i] = -__int_as_float(0x7f800000);
  }
  return m;
}

// Write the indices (and optionally scores) of the entries of buf[0..n) that are >= th
// (th >= 1, so zero pads never qualify) to row[0..) in arbitrary order and pad the rest
// of row[0..width) with -1.  Each warp appends its qualifying entries with one shared
// atomic per 32 entries (no group-wide prefix passes); *count is shared scratch.
template <int NT>
__device__ uint32_t emit_ge_warps(const uint64_t* buf, uint32_t n, uint64_t th, int32_t* row, float* row_scores,
                                  uint32_t width, uint32_t* count, const Group<NT>& G) {
  if (G.tid == 0) *count = 0u;
  G.sync();
  const uint32_t lane = G.tid & 31, lt = lanemask_lt();
  for (uint32_t i0 = G.tid & ~31u; i0 < n; i0 += NT) {
    const uint32_t i = i0 + lane;
    const uint64_t x = i < n ? buf[i] : 0ull;
    const bool take = x >= th;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
    if (m == 0u) continue;
    const int leader = __ffs(m) - 1;
    uint32_t base = 0;
    if ((int)lane == leader) base = atomicAdd(count, (uint32_t)__popc(m));
    base = __shfl_sync(0xFFFFFFFFu, base, leader);
    if (take) {
      const uint32_t pos = base + __popc(m & lt);
      if (pos < width) {
        row[pos] = (int32_t)entry_idx(x);
        if (row_scores) row_scores[pos] = entry_score(x);
      }
    }
  }
  G.sync();
  const uint32_t got = *count < width ? *count : width;
  for (uint32_t p = got + G.tid; p < width; p += NT) {
    row[p] = -1;
    if (row_scores) row_scores[p] = -__int_as_float(0x7f800000);
  }
  return got;
}

// Eq. (6) emit for one group after its exact top-(k+g-1) sits in buf[0..m):
// member t keeps the k best of { entries with index <= t }.  Removing the
// r <= g-1 entries above t leaves at least k; the ones to drop beyond the
// k best are the lowest eligible entries, all among the m-k lowest of buf.
// One counting pass (each entry's first eligible member) and one emission
// pass that writes every entry to each member row it belongs to (row order
// is free; rows are padded with -1 to width topk).  nmem <= 16.
template <int NT>
__device__ void emit_reuse(uint64_t* buf, uint32_t m, int topk, int64_t t_first, int nmem, int64_t out_row0,
                           int32_t* out_idx, float* out_sc, SelSmem& S, uint64_t* bot, const Group<NT>& G) {
  // bottom entries (the m - topk lowest, at most 15), ascending: one group-wide
  // minimum per entry (packed entries are distinct)
  uint32_t nb = 0;
  if (m > (uint32_t)topk) {
    nb = m - (uint32_t)topk;
    if (nb > 16u) nb = 16u;
    static_assert(NT / 32 <= 16, "one minimum per warp in hist[128..159]");
    uint64_t* wmin = reinterpret_cast<uint64_t*>(&S.hist[128]);
    uint64_t last = 0ull;
    for (uint32_t r = 0; r < nb; ++r) {
      uint64_t mn = ~0ull;
      for (uint32_t i = G.tid; i < m; i += NT) {
        const uint64_t x = buf[i];
        if ((r == 0 || x > last) && x < mn) mn = x;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
        mn = y < mn ? y : mn;
      }
      if ((G.tid & 31) == 0) wmin[G.tid >> 5] = mn;
      G.sync();
      mn = wmin[0];
      for (int x = 1; x < NT / 32; ++x) mn = wmin[x] < mn ? wmin[x] : mn;
      if (G.tid == 0) bot[r] = mn;
      last = mn;
      G.sync();  // every warp has read wmin before the next round rewrites it
    }
  }
  // eligible count of every member: entry i is eligible for members r >= first(i)
  for (int i = G.tid; i < 16; i += NT) S.hist[i] = 0u;
  G.sync();
  for (uint32_t i0 = 0; i0 < m; i0 += NT) {
    const uint32_t i = i0 + G.tid;
    uint32_t r0 = 16u;
    if (i < m) {
      const int64_t s = entry_idx(buf[i]);
      r0 = (uint32_t)(s <= t_first ? 0 : (s - t_first));
    }
    hist_add(S.hist, r0 < 16u ? r0 : 256u);
  }
  G.sync();
  // per member: its cut (drop the lowest eligible beyond k) and its row counter
  uint64_t* cut = reinterpret_cast<uint64_t*>(&S.hist[32]);  // 16 x uint64 after the 16 counts
  uint32_t* rowc = &S.hist[64];
  if (G.tid < nmem) {
    const int r = G.tid;
    uint32_t elig = 0;
    for (int u = 0; u <= r; ++u) elig += S.hist[u];
    uint64_t c = 0;
    if (nb > 0 && elig > (uint32_t)topk) {
      const uint32_t mdrop = elig - topk;
      const int64_t t = t_first + r;
      uint32_t cc = 0;
      for (uint32_t u = 0; u < nb && u < 16; ++u)
        if ((int64_t)entry_idx(bot[u]) <= t && ++cc == mdrop) {
          c = bot[u];
          break;
        }
    }
    cut[r] = c;
    rowc[r] = 0u;
  }
  G.sync();
  const uint32_t lt = lanemask_lt();
  for (uint32_t i0 = 0; i0 < m; i0 += NT) {
    const uint32_t i = i0 + G.tid;
    uint64_t x = 0;
    int64_t s = 0;
    if (i < m) {
      x = buf[i];
      s = entry_idx(x);
    }
    for (int r = 0; r < nmem; ++r) {
      const bool in = (i < m) && s <= t_first + r && x > cut[r];
      const uint32_t msk = __ballot_sync(0xFFFFFFFFu, in);
      if (msk == 0u) continue;
      const int leader = __ffs(msk) - 1;
      uint32_t base = 0;
      if ((int)lane_id() == leader) base = atomicAdd(&rowc[r], (uint32_t)__popc(msk));
      base = __shfl_sync(0xFFFFFFFFu, base, leader);
      if (in) {
        const uint32_t pos = base + __popc(msk & lt);
        if (pos < (uint32_t)topk) {
          const int64_t row = out_row0 + r;
          out_idx[row * topk + pos] = (int32_t)s;
          if (out_sc) out_sc[row * topk + pos] = entry_score(x);
        }
      }
    }
  }
  G.sync();
  for (int r = 0; r < nmem; ++r) {  // pad
    const uint32_t cnt = rowc[r] < (uint32_t)topk ? rowc[r] : (uint32_t)topk;
    const int64_t row = out_row0 + r;
    for (uint32_t p = cnt + G.tid; p < (uint32_t)topk; p += NT) {
      out_idx[row * topk + p] = -1;
      if (out_sc) out_sc[row * topk + p] = -__int_as_float(0x7f800000);
    }
  }
  G.sync();
}

}  // namespace pivot
