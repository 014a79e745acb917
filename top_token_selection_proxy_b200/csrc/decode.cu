// decode.cu -- MTP decode groups (PIVOT, picx.dev summary of the paper,
// Methodology, Eq. 3): sequence b holds P_b cached keys and one group of g
// draft positions at the end of its prefix, so each sequence is one group
// with one proxy (Eq. 4) scanned over its whole prefix (Eq. 5), followed by
// the group's exact top-(k+g-1) (Reuse, Eq. 6) or top-c (Refine, Eq. 7).
//
// With one group per sequence the whole proxy-score vector of the batch is
// small (4 bytes per cached key, against 2*d bytes of key read to make it),
// so the selection runs on stored scores instead of inside the scan:
//   1. prep: pool the proxies (bf16, row-major, read by TMA) and w-bar, and
//      plan the scan (512-key sets, a block scan over the sequences);
//   2. scan: persistent CTAs over equal shares of the batch's sets.  One set
//      is 4 key tiles of one sequence; each tile is an M=128, N=64 MMA
//      against the sequence's proxy into its own 64-column slot of a TMEM
//      accumulator, so the 16 epilogue warps read (tile, lane quarter)
//      blocks exactly as the prefill scan reads (group, lane quarter).  The
//      epilogue writes each key's order key and counts its top 11 bits in a
//      per-sequence histogram;
//   3. select + emit (one thread-block cluster per sequence, one launch): the
//      histogram's threshold bin, then the next 11 bits inside that bin, counted
//      in the CTAs' shared memory and summed through distributed shared memory;
//      the best of the last bin's keys by the full (score, index) order complete
//      the exact selection, and the candidate row (Refine) or the g member rows
//      (Reuse) are written from it.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <cstddef>

#include "headsum.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

namespace {

constexpr int kDH = 64;          // heads (the tensor-core shape)
constexpr int kSetTiles = kDecodeSetKeys / 128;  // key tiles per accumulator: one per 64-column slot

template <int D>
struct DScanCfg {
  static constexpr int KB = D / 64;            // 128-byte k-blocks per row
  static constexpr int BM = 128;               // keys per tile (MMA M)
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * D * 2;   // one key tile
  static constexpr int P_BYTES = kDH * D * 2;  // one proxy (MMA B, N = 64)
  static constexpr int NEPI = 512;             // 16 epilogue warps: (tile slot, lane quarter)
  static constexpr int THREADS = 64 + NEPI;    // warp 0 TMA, warp 1 MMA
};

struct DScanTail {
  uint64_t full[4], empty[4], accf[2], acce[2], pfull[2], pempty[2];
  uint32_t tmem_slot;
  volatile int abort_flag;
  uint32_t hist[kHist11Words];  // this CTA's counts of the current sequence's top-11-bit digits
};

template <int D>
constexpr size_t dscan_smem() {
  using C = DScanCfg<D>;
  return 1024 + C::STAGES * C::A_BYTES + 2 * C::P_BYTES + sizeof(DScanTail);
}

// Sequence holding set `s`: the largest b with set_off[b] <= s.
__device__ __forceinline__ int seq_of_set(const int32_t* set_off, int B, int64_t s) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)set_off[mid] <= s) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

}  // namespace

// ------------------------------------------------------------------ 1. prep
// Blocks per sequence: one 16-byte chunk of the proxy per thread.
__host__ __device__ constexpr int prep_blocks_per_seq(int D) { return (kDH * (D / 8) + 255) / 256; }

// Blocks b*PB .. b*PB+PB-1: sequence b's proxy (Eq. 4: the fp32 mean of its g
// query rows, summed in member order, rounded to bf16), w-bar (written in the
// epilogue's permuted layout) and its zeroed digit histogram.  Last block:
// set_off[b] = sum over b' < b of ceil(P_b' / kDecodeSetKeys).
__global__ void __launch_bounds__(256) dprep_kernel(const DecodeArgs a) {
  const int tid = threadIdx.x;
  const int PB = prep_blocks_per_seq(a.D);
  if ((int64_t)blockIdx.x == (int64_t)a.B * PB) {
    __shared__ int32_t wsum[8];
    __shared__ int32_t carry;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < a.B; base += 256) {
      const int b = base + tid;
      const int32_t v =
          b < a.B ? (int32_t)((a.key_off[b + 1] - a.key_off[b] + kDecodeSetKeys - 1) / kDecodeSetKeys) : 0;
      const int32_t incl = (int32_t)warp_incl_scan((uint32_t)v);
      if ((tid & 31) == 31) wsum[tid >> 5] = incl;
      __syncthreads();
      int32_t before = carry;
      for (int u = 0; u < (tid >> 5); ++u) before += wsum[u];
      if (b < a.B) a.set_off[b + 1] = before + incl;
      __syncthreads();
      if (tid == 255) carry = before + incl;
      __syncthreads();
    }
    if (tid == 0) a.set_off[0] = 0;
    return;
  }
  const int b = blockIdx.x / PB, part = blockIdx.x % PB;
  for (int i = part * 256 + tid; i < 2048; i += PB * 256) a.hist1[(int64_t)b * 2048 + i] = 0u;
  const int XC = a.D / 8;  // 16-byte chunks per row
  const int g = a.g;       // <= 16
  const int64_t r0 = (int64_t)b * g;
  const int u = part * 256 + tid;
  if (u < kDH * XC) {
    const int hj = u / XC, xc = u % XC;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int m0 = 0; m0 < g; m0 += 8) {  // 8 members' loads in flight, summed in member order
      uint4 vv[8];
#pragma unroll
      for (int x = 0; x < 8; ++x)
        vv[x] = (m0 + x < g) ? __ldg(reinterpret_cast<const uint4*>(a.q + ((r0 + m0 + x) * kDH + hj) * (int64_t)a.D) + xc)
                             : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        if (m0 + x < g) {
          const uint32_t wv[4] = {vv[x].x, vv[x].y, vv[x].z, vv[x].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(wv[i] << 16);
            acc[2 * i + 1] += __uint_as_float(wv[i] & 0xFFFF0000u);
          }
        }
      }
    }
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float lo = acc[2 * i], hi = acc[2 * i + 1];
      if (g > 1) {
        lo = __fdiv_rn(lo, (float)g);
        hi = __fdiv_rn(hi, (float)g);
      }
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
      pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(a.proxy + ((int64_t)b * kDH + hj) * a.D + xc * 8) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  if (part == 0 && tid < kDH) {
    const int hj = tid;
    float wl[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) wl[x] = (x < g) ? __ldg(a.w + (r0 + x) * kDH + hj) : 0.f;
    float sw = 0.f;
#pragma unroll
    for (int x = 0; x < 16; ++x)
      if (x < g) sw += wl[x];
    a.wbar[(int64_t)b * kWbarStride + wperm_index(0, hj)] = g > 1 ? __fdiv_rn(sw, (float)g) : sw;
  }
}

// ------------------------------------------------------------------ 2. scan
template <int D>
__global__ void __launch_bounds__(576, 1) dscan_kernel(const __grid_constant__ CUtensorMap kmap,
                                                       const __grid_constant__ CUtensorMap pmap, const DecodeArgs a) {
  using C = DScanCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sP = smem + C::STAGES * C::A_BYTES;
  DScanTail& T = *reinterpret_cast<DScanTail*>(sP + 2 * C::P_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&T.full[s], 1);
      mbar_init(&T.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&T.accf[x], 1);
      mbar_init(&T.acce[x], C::NEPI);
      mbar_init(&T.pfull[x], 1);
      mbar_init(&T.pempty[x], 1);
    }
    T.abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&kmap);
    prefetch_tmap(&pmap);
  }
  for (int i = tid; i < kHist11Words; i += C::THREADS) T.hist[i] = 0u;
  if (warp == 1) {
    tmem_alloc(&T.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T.tmem_slot;

  // this CTA's share of the batch's sets
  const int64_t set0 = a.n_sets * (int64_t)blockIdx.x / gridDim.x;
  const int64_t set1 = a.n_sets * (int64_t)(blockIdx.x + 1) / gridDim.x;
  int b = set0 < set1 ? seq_of_set(a.set_off, a.B, set0) : 0;
  auto fail = [&]() {
    T.abort_flag = 1;
    atomicOr(a.status, DEV_ERR_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t st = 0, ph = 0, ps = 0, pph = 0;
      int cur = -1;
      for (int64_t sg = set0; sg < set1; ++sg) {
        while (sg >= (int64_t)a.set_off[b + 1]) ++b;
        if (b != cur) {  // the sequence's proxy into the next proxy slot
          if (cur >= 0 && ++ps == 2) {
            ps = 0;
            pph ^= 1u;
          }
          if (!mbar_wait(&T.pempty[ps], pph ^ 1u, a.timeout_ns, &T.abort_flag)) {
            fail();
            break;
          }
          mbar_arrive_expect_tx(&T.pfull[ps], C::P_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sP + ps * C::P_BYTES + kb * (kDH * 128), &pmap, &T.pfull[ps], kb * 64, b * kDH);
          cur = b;
        }
        const int64_t P = a.key_off[b + 1] - a.key_off[b];
        const int64_t t0 = (sg - a.set_off[b]) * kSetTiles;
        const int nt = (int)min64(kSetTiles, (P + C::BM - 1) / C::BM - t0);
        bool ok = true;
        for (int t = 0; t < nt; ++t) {
          if (!mbar_wait(&T.empty[st], ph ^ 1u, a.timeout_ns, &T.abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&T.full[st], C::A_BYTES);
          const int row = (int)(a.key_off[b] + (t0 + t) * C::BM);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sA + st * C::A_BYTES + kb * (C::BM * 128), &kmap, &T.full[st], kb * 64, row);
          if (++st == C::STAGES) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          fail();
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(C::BM, kDH);
      uint32_t st = 0, ph = 0, ab = 0, aph = 0, ps = 0, pph = 0;
      int cur = -1;
      for (int64_t sg = set0; sg < set1; ++sg) {
        while (sg >= (int64_t)a.set_off[b + 1]) ++b;
        const int64_t P = a.key_off[b + 1] - a.key_off[b];
        const int64_t t0 = (sg - a.set_off[b]) * kSetTiles;
        const int nt = (int)min64(kSetTiles, (P + C::BM - 1) / C::BM - t0);
        if (!mbar_wait(&T.acce[ab], aph ^ 1u, a.timeout_ns, &T.abort_flag)) {
          fail();
          break;
        }
        if (b != cur) {
          if (cur >= 0 && ++ps == 2) {
            ps = 0;
            pph ^= 1u;
          }
          if (!mbar_wait(&T.pfull[ps], pph, a.timeout_ns, &T.abort_flag)) {
            fail();
            break;
          }
          cur = b;
        }
        const uint32_t baddr = smem_u32(sP + ps * C::P_BYTES);
        bool ok = true;
        for (int t = 0; t < nt; ++t) {
          if (!mbar_wait(&T.full[st], ph, a.timeout_ns, &T.abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aaddr = smem_u32(sA + st * C::A_BYTES);
          const uint32_t dtm = tmem + ab * 256u + (uint32_t)(t * kDH);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(aaddr + kb * (C::BM * 128) + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(baddr + kb * (kDH * 128) + kk * 32);
              umma_bf16(dtm, ad, bd, idesc, (kb | kk) ? 1u : 0u);
            }
          umma_commit(&T.empty[st]);
          if (++st == C::STAGES) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          fail();
          break;
        }
        umma_commit(&T.accf[ab]);
        if (sg + 1 == set1 || sg + 1 >= (int64_t)a.set_off[b + 1]) umma_commit(&T.pempty[ps]);  // proxy slot free
        if (++ab == 2) {
          ab = 0;
          aph ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w reads TMEM lanes 32*(w%4).. of tile slot (w-2)/4: Eq. (5) for 32 keys
    const int q4 = warp & 3;
    const int slot = (warp - 2) >> 2;
    const int etid = tid - 64;
    const int my_lane = quad_key_lane(lane);
    uint32_t eab = 0, eaph = 0;
    int cur = -1;
    int64_t P = 0, kbase = 0;
    auto flush = [&](int seq) {  // this CTA's digit counts of sequence seq -> its global histogram
      named_bar_sync(1, C::NEPI);
      for (int i = etid; i < 2048; i += C::NEPI) {
        const uint32_t v = T.hist[h11(i)];
        if (v) {
          atomicAdd(&a.hist1[(int64_t)seq * 2048 + i], v);
          T.hist[h11(i)] = 0u;
        }
      }
      named_bar_sync(1, C::NEPI);
    };
    for (int64_t sg = set0; sg < set1; ++sg) {
      while (sg >= (int64_t)a.set_off[b + 1]) ++b;
      if (b != cur) {
        if (cur >= 0) flush(cur);
        cur = b;
        P = a.key_off[b + 1] - a.key_off[b];
        kbase = a.key_off[b];
      }
      const int64_t t0 = (sg - a.set_off[b]) * kSetTiles;
      const int nt = (int)min64(kSetTiles, (P + C::BM - 1) / C::BM - t0);
      const bool ok = mbar_wait(&T.accf[eab], eaph, a.timeout_ns, &T.abort_flag);
      if (!ok) fail();
      if (ok) {
        tc_fence_after();
        if (slot < nt) {
          float2 w2[8];
          load_w2(a.wbar + (int64_t)b * kWbarStride, 0, lane, w2);
          float v[4];
#pragma unroll
          for (int slab = 0; slab < 2; ++slab) {
            uint32_t r[32];
            tmem_ld16x256b_x8(tmem + ((uint32_t)(q4 * 32 + slab * 16) << 16) + eab * 256u + (uint32_t)(slot * kDH),
                              r);
            tmem_wait_ld();
            if (slab == 1) {
              tc_fence_before();
              mbar_arrive(&T.acce[eab]);
            }
            slab_head_sums(r, w2, v[2 * slab], v[2 * slab + 1]);
          }
          const float sc = quad_reduce_scatter(v, lane);
          const int64_t s = (t0 + slot) * C::BM + q4 * 32 + my_lane;
          const bool valid = s < P;
          const uint32_t u = score_key(sc);
          if (valid) a.scores[kbase + s] = u;
          const uint32_t bin = valid ? (u >> 21) : 0xFFFFFFFFu;
          const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
          if (valid && lane == __ffs(peers) - 1) atomicAdd(&T.hist[h11(bin)], (uint32_t)__popc(peers));
        } else {  // no tile in this slot (the sequence's last set)
          tc_fence_before();
          mbar_arrive(&T.acce[eab]);
        }
      }
      if (++eab == 2) {
        eab = 0;
        eaph ^= 1u;
      }
    }
    if (cur >= 0) flush(cur);
  }

  __syncthreads();
  if (T.abort_flag) {  // let in-flight async copies / MMAs drain before releasing TMEM
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ 3. select + emit
// One thread-block cluster of kSelCl CTAs per sequence, one launch for the exact
// selection of n = min(n_sel, P) keys by the order (score desc, index asc):
//   level 1  T1 = the bin of the scan's top-11-bit histogram where the count from the
//            top reaches n.  Each CTA reads its share of the sequence's order keys once
//            (16-byte loads): keys above T1 are selected, keys in T1 are listed as
//            level-1 ties and their next 11 bits are counted in the CTA's histogram;
//   level 2  the CTAs' histograms are summed through distributed shared memory; T2 is
//            the bin where the count reaches the rest of n; the level-1 ties are split
//            over the CTAs: above T2 selected, in T2 listed as level-2 ties;
//   final    CTA 0 takes the best of the level-2 ties by the full (score, index) order
//            and writes the candidate row (Refine), the g member rows (Reuse), or, for
//            one key shard of a prefix split over GPUs, the selection itself as packed
//            entries with prefix positions (merged after the exchange, dmerge_kernel).
// The list counters sit in CTA 0's shared memory (one remote atomic per warp and chunk).
// Selected entries go straight into CTA 0's shared memory when n_sel fits its stage
// (kSelStage entries), else to the workspace; the ties lists have room for every key
// of the sequence, so no list can overflow.
namespace {

struct BinThr {
  int T;           // threshold bin (-1: every entry is selected)
  uint32_t above;  // entries in bins above T
  uint32_t at;     // entries in bin T
};

// Over 2048 counts read by ld(bin) with `total` entries: the bin T where the count from
// the top first reaches need (need <= total).  All NT threads of the block call it.
template <int NT, typename Ld>
__device__ BinThr bin_threshold(Ld&& ld, uint32_t need, uint32_t total, uint32_t* wtot, int* scal) {
  constexpr int BPT = 2048 / NT;
  BinThr r{-1, total, 0u};
  if (need >= total) return r;
  const int t = threadIdx.x;
  if (t == 0) {  // kept only if the counts do not reach `need` (an aborted scan): select everything
    scal[0] = -1;
    scal[1] = (int)total;
    scal[2] = 0;
  }
  uint32_t loc[BPT], sum = 0;
#pragma unroll
  for (int u = 0; u < BPT; ++u) {
    loc[u] = ld(2047 - BPT * t - u);
    sum += loc[u];
  }
  const uint32_t incl = warp_incl_scan(sum);
  if ((t & 31) == 31) wtot[t >> 5] = incl;
  __syncthreads();
  uint32_t excl = incl - sum;
  for (int w = 0; w < (t >> 5); ++w) excl += wtot[w];
  if (excl < need && need <= excl + sum) {
    uint32_t c = excl;
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
      if (c + loc[u] >= need) {
        scal[0] = 2047 - BPT * t - u;
        scal[1] = (int)c;
        scal[2] = (int)loc[u];
        break;
      }
      c += loc[u];
    }
  }
  __syncthreads();
  r.T = scal[0];
  r.above = (uint32_t)scal[1];
  r.at = (uint32_t)scal[2];
  __syncthreads();
  return r;
}

constexpr int kSelV4 = 4;  // 16-byte loads of order keys per thread and level-1 chunk (16 keys)

struct SelClSmem {
  uint4 keys[kSelV4][kSelClThreads];  // each thread's keys of the current chunk (read back only by it)
  uint32_t h2[kHist11Words];     // this CTA's counts of the second digit of its level-1 ties
  uint32_t comb[2048 / kSelCl];  // cluster sums of this CTA's slice of the second-digit bins
  uint32_t ctr[4];               // (CTA 0) list lengths: selected, level-1 ties, level-2 ties
  uint32_t wtot[kSelClThreads / 32];
  int scal[4];
  SelSmem S;
  uint64_t bot[16];
};

// Warp-aggregated append of each thread's candidates (bit u of win / tie; entry(u) is the
// packed entry) to the selected list sl (counter cs) and a ties list tl (counter ct); the
// counters may be another CTA's shared memory.  Positions at or past cap_s / cap_t are
// dropped and reported.  The whole warp calls.
template <int U, typename E>
__device__ __forceinline__ bool append2(E&& entry, uint32_t win, uint32_t tie, uint64_t* sl, uint32_t* cs,
                                        uint32_t cap_s, uint64_t* tl, uint32_t* ct, uint32_t cap_t) {
  const int lane = threadIdx.x & 31;
  const uint32_t nw = __popc(win), nt = __popc(tie);
  const uint32_t iw = warp_incl_scan(nw), it = warp_incl_scan(nt);
  const uint32_t tw = __shfl_sync(0xFFFFFFFFu, iw, 31), tt = __shfl_sync(0xFFFFFFFFu, it, 31);
  if (tw == 0u && tt == 0u) return false;
  uint32_t bw = 0, bt = 0;
  if (lane == 31) {
    if (tw) bw = atomicAdd(cs, tw);
    if (tt) bt = atomicAdd(ct, tt);
  }
  bw = __shfl_sync(0xFFFFFFFFu, bw, 31);
  bt = __shfl_sync(0xFFFFFFFFu, bt, 31);
  uint32_t pw = bw + iw - nw, pt = bt + it - nt;
  bool over = false;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (win & (1u << u)) {
      if (pw < cap_s) sl[pw] = entry(u);
      else over = true;
      ++pw;
    }
    if (tie & (1u << u)) {
      if (pt < cap_t) tl[pt] = entry(u);
      else over = true;
      ++pt;
    }
  }
  return over;
}

}  // namespace

__global__ void __launch_bounds__(kSelClThreads) dselect_cluster_kernel(const DecodeArgs a) {
  namespace cg = cooperative_groups;
  constexpr int NT = kSelClThreads, SL = 2048 / kSelCl;
  constexpr int V4 = kSelV4;
  __shared__ SelClSmem sm;
  extern __shared__ uint64_t stage[];  // kSelStage entries; CTA 0's holds the selected entries
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = (int)(blockIdx.x / kSelCl);
  const int tid = threadIdx.x;
  const int64_t kbase = a.key_off[b];
  const int64_t P = a.key_off[b + 1] - kbase;
  const uint32_t need = (uint32_t)min64(a.n_sel, P);
  uint64_t* X = a.ties + kbase;   // level-1 ties
  uint64_t* Y = a.ties2 + kbase;  // level-2 ties
  const bool staged = a.n_sel <= kSelStage;
  uint64_t* sel = staged ? cluster.map_shared_rank(stage, 0) : a.sel + (int64_t)b * a.n_sel;
  uint32_t* ctr = cluster.map_shared_rank(sm.ctr, 0);

  // this CTA's share [s0, s1) of the order keys: up to 3 keys on each side by plain loads,
  // the 16-byte-aligned middle [a0, a1) by vector loads; its first chunk is prefetched
  // into L2 while the level-1 threshold is found
  const int64_t s0 = P * rank / kSelCl, s1 = P * (rank + 1) / kSelCl;
  const uint32_t* keys = a.scores + kbase;
  const int64_t a0 = min64(s1, s0 + ((4 - ((kbase + s0) & 3)) & 3));
  const int64_t a1 = max64(a0, s1 - ((kbase + s1) & 3));
  const int64_t nvec = (a1 - a0) >> 2;
  const uint4* kv = reinterpret_cast<const uint4*>(keys + a0);
#pragma unroll
  for (int j = 0; j < V4; ++j)
    if (j * NT + tid < nvec) prefetch_l2(kv + j * NT + tid);

  for (int i = tid; i < kHist11Words; i += NT) sm.h2[i] = 0u;
  if (tid < 4) sm.ctr[tid] = 0u;
  const uint32_t* hg1 = a.hist1 + (int64_t)b * 2048;
  const BinThr t1 = bin_threshold<NT>([&](int i) { return hg1[i]; }, need, (uint32_t)P, sm.wtot, sm.scal);
  __syncthreads();
  cluster.sync();  // (0) CTA 0's counters are zero before any append
  bool over = false;

  // ---- level 1: a key is selected when its top 11 bits exceed T1 (every key when T1 < 0),
  // a level-1 tie when they equal T1
  const bool all1 = t1.T < 0;
  const uint32_t top1 = all1 ? 0u : (((uint32_t)t1.T << 21) | 0x1FFFFFu);  // selected: key > top1
  // append the candidates (bits of win | tie) of each thread: warp-aggregated positions, one
  // remote counter update per warp and list; each thread then writes only its own few entries
  auto place = [&](uint32_t win, uint32_t tie, auto&& key_of, auto&& pos_of) {
    const int lane = tid & 31;
    const uint32_t nw = __popc(win), nt = __popc(tie);
    const uint32_t iw = warp_incl_scan(nw), it = warp_incl_scan(nt);
    const uint32_t tw = __shfl_sync(0xFFFFFFFFu, iw, 31), tt = __shfl_sync(0xFFFFFFFFu, it, 31);
    if (tw == 0u && tt == 0u) return;
    uint32_t bw = 0, bt = 0;
    if (lane == 31) {
      if (tw) bw = atomicAdd(&ctr[0], tw);
      if (tt) bt = atomicAdd(&ctr[1], tt);
    }
    uint32_t pw = __shfl_sync(0xFFFFFFFFu, bw, 31) + iw - nw, pt = __shfl_sync(0xFFFFFFFFu, bt, 31) + it - nt;
    for (uint32_t c = win | tie; c; c &= c - 1u) {
      const int u = __ffs(c) - 1;
      const uint32_t v = key_of(u);
      const uint64_t e = pack_entry(v, (uint32_t)pos_of(u));
      if ((win >> u) & 1u) {
        if (pw < need) sel[pw] = e;
        else over = true;
        ++pw;
      } else {
        if (pt < (uint32_t)P) X[pt] = e;
        else over = true;
        ++pt;
        atomicAdd(&sm.h2[h11((v >> 10) & 2047u)], 1u);  // second digit of the tie
      }
    }
  };
  {
    const int nh = (int)(a0 - s0);
    const int64_t s = tid < nh ? s0 + tid : a1 + (tid - nh);
    const bool valid = tid < 8 && (tid < nh || s < s1);
    const uint32_t v = valid ? keys[s] : 0u;
    const uint32_t win = (valid && (all1 || v > top1)) ? 1u : 0u;
    const uint32_t tie = (valid && (int)(v >> 21) == t1.T) ? 1u : 0u;
    place(win, tie, [&](int) { return v; }, [&](int) { return s; });
  }
  uint32_t* kst = reinterpret_cast<uint32_t*>(&sm.keys[0][0]);
  for (int64_t v0 = 0; v0 < nvec; v0 += (int64_t)NT * V4) {
    uint4 x[V4];
#pragma unroll
    for (int j = 0; j < V4; ++j) {
      const int64_t vi = v0 + j * NT + tid;
      x[j] = vi < nvec ? kv[vi] : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t win = 0u, tie = 0u;
#pragma unroll
    for (int j = 0; j < V4; ++j) {
      const bool valid = v0 + j * NT + tid < nvec;
      const uint32_t c4[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (valid && (all1 || c4[e] > top1)) win |= 1u << (4 * j + e);
        if (valid && (int)(c4[e] >> 21) == t1.T) tie |= 1u << (4 * j + e);
      }
    }
    if (win | tie) {
#pragma unroll
      for (int j = 0; j < V4; ++j) sm.keys[j][tid] = x[j];
    }
    place(win, tie, [&](int u) { return kst[((u >> 2) * NT + tid) * 4 + (u & 3)]; },
          [&](int u) { return a0 + 4 * (v0 + (u >> 2) * NT + tid) + (u & 3); });
  }
  __syncthreads();
  cluster.sync();  // (1) the level-1 lists and every CTA's second-digit histogram are complete

  if (tid < SL) {
    uint32_t c = 0;
    for (int r = 0; r < kSelCl; ++r) c += cluster.map_shared_rank(sm.h2, r)[h11((uint32_t)(rank * SL + tid))];
    sm.comb[tid] = c;
  }
  const uint32_t NW1 = ctr[0], at1 = min(ctr[1], (uint32_t)P);
  cluster.sync();  // (2) the combined second-digit histogram is complete; the counts are read
  BinThr t2{-1, 0u, 0u};
  if (t1.T >= 0 && NW1 < need)
    t2 = bin_threshold<NT>([&](int i) { return cluster.map_shared_rank(sm.comb, i / SL)[i % SL]; }, need - NW1, at1,
                           sm.wtot, sm.scal);

  // ---- level 2 over this CTA's portion [q0, q1) of the level-1 ties
  {
    constexpr int U = 8;
    const uint32_t q0 = (uint32_t)((uint64_t)at1 * rank / kSelCl),
                   q1 = (uint32_t)((uint64_t)at1 * (rank + 1) / kSelCl);
    for (uint32_t c0 = q0; c0 < q1; c0 += NT * U) {
      uint64_t x[U];
      uint32_t win = 0u, tie = 0u;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t i = c0 + u * NT + tid;
        x[u] = i < q1 ? X[i] : 0ull;
        const int d2 = (int)((x[u] >> 42) & 2047u);
        if (i < q1 && d2 > t2.T) win |= 1u << u;
        if (i < q1 && d2 == t2.T) tie |= 1u << u;
      }
      over |= append2<U>([&](int u) { return x[u]; }, win, tie, sel, &ctr[0], need, Y, &ctr[2], (uint32_t)P);
    }
  }
  if (over) atomicOr(a.status, DEV_ERR_BOUNDS);
  __syncthreads();
  cluster.sync();  // (3) the selected list and the level-2 ties are complete
  if (rank != 0) return;

  const Group<NT> G{tid, 0};
  uint64_t* buf = staged ? stage : sel;
  const uint32_t nw = min(sm.ctr[0], need);
  uint32_t m = nw;
  if (nw < need) {  // the best (need - nw) level-2 ties by the full (score, index) order
    const uint32_t nt = min(sm.ctr[2], (uint32_t)P), need3 = need - nw;
    const uint64_t th = radix_threshold<NT>(Y, nt, need3, need3, sm.S, G);
    m += compact_ge<NT>(Y, buf + nw, nt, th, sm.S, G);
  }
  G.sync();
  if (a.mode == EMIT_CAND) {
    emit_row<NT>(buf, m, 0xFFFFFFFFu, 0ull, a.cand + (int64_t)b * a.n_sel,
                 a.cand_scores ? a.cand_scores + (int64_t)b * a.n_sel : nullptr, (uint32_t)a.n_sel, sm.S, G);
  } else if (a.mode == EMIT_REUSE) {
    emit_reuse<NT>(buf, m, a.topk, P - a.g, a.g, (int64_t)b * a.g, a.out_idx, a.out_scores, sm.S, sm.bot, G);
  } else {  // EMIT_ENTRIES: this key shard's selection, positions made global, 0 pads
    const uint32_t base = a.pos_base ? (uint32_t)a.pos_base[b] : 0u;
    uint64_t* e = a.entries + (int64_t)b * a.n_sel;
    for (uint32_t i = tid; i < (uint32_t)a.n_sel; i += NT)
      e[i] = i < m ? pack_entry((uint32_t)(buf[i] >> 32), entry_idx(buf[i]) + base) : 0ull;
  }
}

// ------------------------------------------------------------------ decode split: merge
// One CTA per sequence: the ranks' shard selections (each the exact top-n of its keys, so
// their union holds the exact top-n of the whole prefix) are gathered, the top n = min(n_sel,
// P_b) are selected by the full (score, index) order, and the candidate row (Refine) or the
// g member rows (Reuse, members at positions P_b - g .. P_b - 1) are written.
__global__ void __launch_bounds__(512) dmerge_kernel(const MergeArgs a) {
  constexpr int NT = 512;
  __shared__ SelSmem S;
  __shared__ uint32_t hist11[kHist11Words];
  __shared__ uint64_t bot[16];
  const Group<NT> G{(int)threadIdx.x, 0};
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    const int64_t P = a.plen_off[b + 1] - a.plen_off[b];
    const uint32_t need = (uint32_t)min64(a.n_sel, P);
    const uint32_t n = (uint32_t)a.R * (uint32_t)a.n_sel;
    uint64_t* buf = a.gather + (int64_t)b * n;
    for (int r = 0; r < a.R; ++r) {  // (n_sel may be odd: plain 8-byte copies)
      const uint64_t* src = a.entries + ((int64_t)r * a.B + b) * a.n_sel;
      for (int i = G.tid; i < a.n_sel; i += NT) buf[(int64_t)r * a.n_sel + i] = src[i];
    }
    G.sync();
    // the need-th largest; zero pads never pass (a threshold of 0 means "every entry")
    uint64_t th = radix11_threshold<NT>(buf, n, need, need, hist11, S, G);
    if (th == 0ull) th = 1ull;
    uint64_t* sel = a.sel + (int64_t)b * a.n_sel;
    const uint32_t m = compact_ge<NT>(buf, sel, n, th, S, G);
    G.sync();
    if (a.mode == EMIT_CAND) {
      int32_t* row = a.cand + (int64_t)b * a.n_sel;
      emit_row<NT>(sel, m, 0xFFFFFFFFu, 0ull, row, a.cand_scores ? a.cand_scores + (int64_t)b * a.n_sel : nullptr,
                   (uint32_t)a.n_sel, S, G);
      G.sync();
      if (a.cand_local) {  // C in the rows of this rank's key shard, -1 where another rank holds the key
        const int64_t base = a.pos_base[b], len = a.shard_off[b + 1] - a.shard_off[b];
        for (int i = G.tid; i < a.n_sel; i += NT) {
          const int64_t v = row[i];
          a.cand_local[(int64_t)b * a.n_sel + i] = (v >= base && v < base + len) ? (int32_t)(v - base) : -1;
        }
      }
    } else {
      emit_reuse<NT>(sel, m, a.topk, P - a.g, a.g, (int64_t)b * a.g, a.out_idx, a.out_scores, S, bot, G);
    }
    G.sync();
  }
}

// ------------------------------------------------------------------ launchers
size_t decode_scan_smem_bytes(int D) {
  if (D == 128) return dscan_smem<128>();
  if (D == 64) return dscan_smem<64>();
  return 0;
}

cudaError_t launch_decode_scan(const DecodeArgs& a, const CUtensorMap* kmap, const CUtensorMap* pmap, int scan_grid,
                               cudaStream_t s) {
  if (a.H != kDH || (a.D != 64 && a.D != 128)) return cudaErrorInvalidValue;
  const int64_t prep_grid = (int64_t)a.B * prep_blocks_per_seq(a.D) + 1;
  if (prep_grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  dprep_kernel<<<(unsigned)prep_grid, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = decode_scan_smem_bytes(a.D);
  if (a.D == 128) {
    auto k = dscan_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<scan_grid, DScanCfg<128>::THREADS, smem, s>>>(*kmap, *pmap, a);
  } else {
    auto k = dscan_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<scan_grid, DScanCfg<64>::THREADS, smem, s>>>(*kmap, *pmap, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_merge(const MergeArgs& a, cudaStream_t s) {
  dmerge_kernel<<<a.B < 1184 ? a.B : 1184, 512, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_select(const DecodeArgs& a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.B * kSelCl);
  cfg.blockDim = dim3(kSelClThreads);
  cfg.dynamicSmemBytes = kSelStage * sizeof(uint64_t);
  cudaFuncSetAttribute(dselect_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)cfg.dynamicSmemBytes);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kSelCl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dselect_cluster_kernel, a);
}

}  // namespace pivot
