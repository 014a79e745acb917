// scan.cu -- K1: fused proxy pooling + proxy scan + streaming exact select.
//
// PIVOT (picx.dev summary of the paper, Methodology):
//   Eq. (4)  q-bar_j = mean of q_{t,j} over the group, w-bar_j = mean of w_{t,j}
//            (or the first / last member's q and w: the aggregation variants of
//            the paper's ablation, Proxy aggregation, Table 2)
//   Eq. (5)  I-bar_s = sum_j w-bar_j ReLU(q-bar_j . k_s),  s <= group end
//   Eq. (6)/(7) the group's top-(k+g-1) (Reuse) or top-c (Refine) by I-bar
//   Eq. (1)  the dense indexer is the same scan with g = 1 and n_sel = k.
//
// One persistent CTA per SM.  A work item is a block of NB = 256/H groups
// (consecutive, so their prefixes are nearly equal), scheduled longest
// prefix first from an atomic counter.  Per item:
//   * all threads pool the NB proxies (fp32 sum, divide by |G|, round to
//     bf16) straight into the MMA's B operand in shared memory (K-major,
//     128-byte swizzle) and w-bar into shared memory;
//   * warp 0 streams 128-key tiles of k_I with TMA (4-stage ring);
//   * warp 1 issues tcgen05.mma  D[128 keys x N] = K_tile . Proxy^T  into one
//     of two 256-column TMEM accumulators (double buffered);
//   * warps 2-5 (one thread per key / TMEM lane) load the accumulator row,
//     apply ReLU, weight by w-bar and sum the H heads of each group in
//     registers, mask s > group end, and feed the scores to a per-group
//     streaming exact selection: packed (score, index) entries above the
//     group's running threshold are appended to an L2-resident buffer; when a
//     buffer fills it is cut back (radix threshold + compaction) and the
//     threshold rises.  No score matrix ever reaches HBM.
//   * at the end of the item the epilogue warps run the exact top-n_sel and
//     emit rows (dense / Reuse) or the candidate set C_i (Refine).
#include <cuda_bf16.h>

#include <cstddef>

#include "headsum.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

template <int H, int D>
struct ScanCfg {
  static constexpr int NB = 256 / H;  // groups per work item
  static constexpr int N = NB * H;    // MMA N (256)
  static constexpr int KB = D / 64;   // 128-byte k-blocks per row
  static constexpr int BM = 128;      // keys per tile (MMA M)
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * D * 2;
  static constexpr int B_BYTES = N * D * 2;
  static constexpr int THREADS = 64 + 128 * NB;  // warp 0 TMA, warp 1 MMA, 4 epilogue warps per group
  static constexpr int NEPI = 128 * NB;          // one warp per (group, TMEM lane quarter)
  static constexpr int SMEM_CAP = STAGES * A_BYTES / 8;  // packed entries the freed stage ring can hold
  static_assert(NB == 4, "four groups per item (H = 64)");
};

// Sample-first tile order: on the first attempt at a long item the tiles
// 0, S, 2S, ... are scanned first (every entry admitted), the groups are cut
// back to the best ~1.5 * n_sel * (sample share) of that sample, and the
// remaining tiles are scanned with the resulting threshold.  The selection
// stays exact: if fewer than n_sel entries end above the estimate, the item
// is scanned again in natural order from an empty threshold.
constexpr int kSampleStride = 32;

// Key tile visited at step j of an item of ntiles tiles with ns sample tiles (ns = 0: natural order).
__device__ __forceinline__ int tile_of(int j, int ns) {
  if (ns == 0 || j < ns) return ns == 0 ? j : j * kSampleStride;
  const int r = j - ns;  // the r-th tile that is not a sample tile
  return (r / (kSampleStride - 1)) * kSampleStride + 1 + r % (kSampleStride - 1);
}

struct ScanTail {
  uint64_t full[4], empty[4], accf[2], acce[2];
  uint64_t never;  // a barrier nothing arrives on (forced-timeout test hook)
  uint32_t tmem_slot;
  int item, nb_act, ntiles;
  volatile int abort_flag;
  int64_t row_base, s_begin, s_end, grp0;
  int64_t e[16];      // last member position of each group (causal mask of the proxy)
  int64_t mrow0[16];  // first q row of each group's members
  int nmem[16];
  uint64_t tau[16];         // running admission threshold of each group (admit packed > tau)
  uint32_t qcnt[8][4];      // per group, entries in each lane quarter's sub-buffer (published on demand)
  uint32_t cflags;          // groups whose sub-buffers need a cut-back
  int est[4];               // group got a sampled threshold estimate in this attempt
  int retry;                // the attempt's estimate was too high: scan the item again
  uint32_t hist11[kHist11Words];    // radix-select histogram (11-bit digits)
  // sample-tile histogram of each group's scores: 2048 bins of bits 30..20 of the order key
  // (exponent and 3 mantissa bits of a positive score; every other key in bin 0), two
  // 16-bit counts per word
  uint32_t esth[4][1024];
  uint32_t escan[4][4];     // per group, per warp partial sums of the bin search
  int ebin[4];              // per group, the bin where the running count reaches r0
  uint64_t bot[16];
  uint32_t ecount;          // final selection: entries written so far
  SelSmem sel;
  // w-bar of the item's groups, permuted for the epilogue: row (b, m) holds heads
  // 8j + 2m, 8j + 2m + 1 (j = 0..7) of group b in 16 floats, rows 20 floats apart
  // so the 4 rows a warp reads sit in distinct banks
  alignas(16) float wperm[16 * 20];
};
static_assert(offsetof(ScanTail, wperm) % 16 == 0, "wperm must be 16-byte aligned");

template <int H, int D>
constexpr size_t scan_smem() {
  using C = ScanCfg<H, D>;
  return 1024 + C::B_BYTES + C::STAGES * C::A_BYTES + sizeof(ScanTail);
}
static_assert(scan_smem<64, 128>() <= 232448, "227 KB of dynamic shared memory per CTA");

template <int H, int D>
__global__ void __launch_bounds__(576, 1) scan_kernel(const __grid_constant__ CUtensorMap kmap, const ScanArgs a) {
  using C = ScanCfg<H, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  uint8_t* sA = smem + C::B_BYTES;
  ScanTail& T = *reinterpret_cast<ScanTail*>(smem + C::B_BYTES + C::STAGES * C::A_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&T.full[s], 1);
      mbar_init(&T.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&T.accf[b], 1);
      mbar_init(&T.acce[b], C::NEPI);
    }
    mbar_init(&T.never, 1);
    T.abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(&T.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T.tmem_slot;

  uint32_t p_st = 0, p_ph = 0;                          // producer ring position
  uint32_t m_st = 0, m_ph = 0, m_ab = 0, m_aph = 0;     // MMA: ring + accumulator
  uint32_t e_ab = 0, e_aph = 0;                         // epilogue: accumulator
  uint64_t* selbase = a.selbuf + (uint64_t)blockIdx.x * C::NB * (uint64_t)a.cap;
  const Group<C::NEPI> EG{tid - 64, 1};

  for (;;) {
    // ---------------------------------------------------------------- item geometry
    if (tid == 0) {
      const int item = (int)atomicAdd(a.counter, 1u);
      T.item = item;
      if (item < a.n_items) {
        const int64_t blk = (int64_t)a.n_items - 1 - item;  // longest prefix first
        const int64_t g0 = a.grp_base + blk * C::NB;
        const int nb_act = (int)min64(C::NB, a.n_groups - g0);
        T.grp0 = g0;
        T.nb_act = nb_act;
        for (int b = 0; b < C::NB; ++b) {
          const int64_t grp = g0 + b;
          if (b < nb_act) {
            const int64_t t0 = grp * a.g;
            const int64_t t1 = min64(t0 + a.g, a.L);
            T.mrow0[b] = t0;
            T.nmem[b] = (int)(t1 - t0);
            T.e[b] = t1 - 1;
          } else {
            T.mrow0[b] = 0;
            T.nmem[b] = 0;
            T.e[b] = -1;
          }
        }
        T.row_base = 0;
        T.s_begin = 0;
        T.s_end = T.e[nb_act - 1] + 1;
        T.ntiles = (int)((T.s_end - T.s_begin + C::BM - 1) / C::BM);
        for (int b = 0; b < C::NB; ++b) {
          T.tau[b] = 0;
          T.est[b] = 0;
        }
        T.cflags = 0;
        T.retry = 0;
      }
    }
    __syncthreads();
    const int item = T.item;
    if (item >= a.n_items || T.abort_flag) break;
    const int nb_act = T.nb_act;
    const int ntiles = T.ntiles;

    // ---------------------------------------------------------------- Eq. (4): pool proxies into B
    // the members' q rows are read once: evict-first in L2, so they do not push the groups'
    // selection sub-buffers out to DRAM
    {
      const uint64_t qpol = l2_policy_evict_first();
      constexpr int XC = D / 8;  // 16-byte chunks per row
      for (int u = tid; u < C::NB * H * XC; u += C::THREADS) {
        const int xc = u % XC;
        const int hj = (u / XC) % H;
        const int b = u / (XC * H);
        const int n = b * H + hj;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        int nm = T.nmem[b];
        int64_t r0 = T.mrow0[b];
        if (a.agg != 0 && nm > 0) {  // first- / last-query proxy: pool that one member
          if (a.agg == 2) r0 += nm - 1;
          nm = 1;
        }
        for (int m0 = 0; m0 < nm; m0 += 8) {  // 8 members' loads in flight, summed in member order
          uint4 vv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            vv[u] = (m0 + u < nm)
                        ? ldg_hint(reinterpret_cast<const uint4*>(a.q + ((r0 + m0 + u) * H + hj) * (int64_t)D) + xc, qpol)
                        : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (m0 + u < nm) {
              const uint32_t wv[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
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
          if (nm > 1) {
            lo = __fdiv_rn(lo, (float)nm);
            hi = __fdiv_rn(hi, (float)nm);
          }
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        const int kb = xc >> 3, ch = xc & 7;
        uint8_t* dst = sB + kb * (C::N * 128) + n * 128 + ((ch ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      for (int u = tid; u < 4 * 1024; u += C::THREADS) (&T.esth[0][0])[u] = 0u;
      for (int u = tid; u < C::NB * H; u += C::THREADS) {
        const int b = u / H, hj = u % H;
        int nm = T.nmem[b];
        int64_t r0 = T.mrow0[b];
        if (a.agg != 0 && nm > 0) {
          if (a.agg == 2) r0 += nm - 1;
          nm = 1;
        }
        float wl[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) wl[u] = (u < nm) ? __ldg(a.w + (r0 + u) * H + hj) : 0.f;
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (u < nm) s += wl[u];
        T.wperm[wperm_index(b, hj)] = nm > 1 ? __fdiv_rn(s, (float)nm) : s;
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    for (int attempt = 0;; ++attempt) {
    const int ns = (attempt == 0 && !(a.debug_flags & 2) && (int64_t)ntiles * C::BM >= 8 * (int64_t)a.n_sel)
                       ? (ntiles + kSampleStride - 1) / kSampleStride
                       : 0;
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        const int64_t row0 = T.row_base + T.s_begin;
        for (int j = 0; j < ntiles; ++j) {
          if (!mbar_wait(&T.empty[p_st], p_ph ^ 1u, a.timeout_ns, &T.abort_flag)) {
            T.abort_flag = 1;
            atomicOr(a.status, DEV_ERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&T.full[p_st], C::A_BYTES);
          uint8_t* dst = sA + p_st * C::A_BYTES;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(dst + kb * (C::BM * 128), &kmap, &T.full[p_st], kb * 64,
                        (int)(row0 + (int64_t)tile_of(j, ns) * C::BM));
          if (++p_st == C::STAGES) {
            p_st = 0;
            p_ph ^= 1u;
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(C::BM, C::N);
        const uint32_t baddr = smem_u32(sB);
        for (int j = 0; j < ntiles; ++j) {
          if (!mbar_wait(&T.full[m_st], m_ph, a.timeout_ns, &T.abort_flag) ||
              !mbar_wait(&T.acce[m_ab], m_aph ^ 1u, a.timeout_ns, &T.abort_flag)) {
            T.abort_flag = 1;
            atomicOr(a.status, DEV_ERR_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint32_t aaddr = smem_u32(sA + m_st * C::A_BYTES);
          const uint32_t dtm = tmem + m_ab * 256u;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(aaddr + kb * (C::BM * 128) + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(baddr + kb * (C::N * 128) + kk * 32);
              umma_bf16(dtm, ad, bd, idesc, (kb | kk) ? 1u : 0u);
            }
          umma_commit(&T.empty[m_st]);
          umma_commit(&T.accf[m_ab]);
          if (++m_st == C::STAGES) {
            m_st = 0;
            m_ph ^= 1u;
          }
          if (++m_ab == 2) {
            m_ab = 0;
            m_aph ^= 1u;
          }
        }
      }
    } else {
      // ------------------------------------------------------------ epilogue + select
      // warp w reads TMEM lanes 32*(w%4).. (its keys) and handles one group: warps
      // 2-5 group 0, 6-9 group 1, ...  Each (group, lane quarter) owns a sub-buffer of
      // sub_cap entries that only its warp appends to, with the count in a register.
      const int q4 = warp & 3;
      const int grp_w = (warp - 2) >> 2;  // this warp's group within the item
      // the key (TMEM lane within the quarter) whose score this thread ends up with
      const int my_lane = quad_key_lane(lane);

      const uint32_t need = (uint32_t)a.n_sel;
      const uint32_t gstride = (uint32_t)a.cap;    // 4 sub-buffers per group
      const uint32_t scap = (uint32_t)a.sub_cap;
      uint32_t qcnt = 0;
      uint64_t tau_r = 0;
      const int64_t e_r = T.e[grp_w];  // causal bound of this warp's group
      // the estimate comes from the sample histogram when its 16-bit counts cannot overflow
      const bool hist_est = ns > 0 && (int64_t)ns * C::BM < 65536;
      const int64_t s_begin = T.s_begin, s_end = T.s_end;
      auto seg_of = [&](int b, int q) { return selbase + (uint64_t)b * gstride + (uint64_t)q * scap; };
      auto publish_counts = [&]() {
        if (lane == 0) T.qcnt[grp_w][q4] = qcnt;
        EG.sync();
      };
      // cut group b back to a superset of its best `need` (keep <= maxk), every warp
      // of the group compacting its own sub-buffer in place
      auto cut_back = [&](int b, uint32_t nd, uint32_t maxk) -> uint64_t {
        Segs sg;
        sg.cnt = 4;
        for (int q = 0; q < 4; ++q) {
          sg.p[q] = seg_of(b, q);
          sg.n[q] = T.qcnt[b][q];
        }
        const uint64_t th = radix11_threshold<C::NEPI>(sg, nd, maxk, T.hist11, T.sel, EG);
        if (grp_w == b) {
          qcnt = warp_compact_ge(seg_of(b, q4), qcnt, th);
          if (th > 0) tau_r = th - 1ull;  // admit x >= th from now on
        }
        EG.sync();
        return th;
      };
      for (int j = 0; j < ntiles; ++j) {
        bool ok;
        if ((a.debug_flags & 1) && j == 0)
          ok = mbar_wait(&T.never, 0u, a.timeout_ns, &T.abort_flag);  // runs out by design
        else
          ok = mbar_wait(&T.accf[e_ab], e_aph, a.timeout_ns, &T.abort_flag);
        if (!ok) {
          T.abort_flag = 1;
          atomicOr(a.status, DEV_ERR_TIMEOUT);
        }
        float sc = 0.f;
        if (ok) {
          tc_fence_after();
          // Eq. (5) for 4 keys x 16 heads per thread (two 16-lane slabs, 16x256b shape),
          // then a reduce-scatter over the 4 threads of the quad: thread m ends with the
          // full 64-head score of key m (slab m >> 1, lane kq + 8 (m & 1))
          float2 w2[8];
          load_w2(T.wperm, grp_w, lane, w2);
          float v[4];
#pragma unroll
          for (int slab = 0; slab < 2; ++slab) {
            uint32_t r[32];
            tmem_ld16x256b_x8(tmem + ((uint32_t)(q4 * 32 + slab * 16) << 16) + e_ab * 256u + (uint32_t)(grp_w * H), r);
            tmem_wait_ld();
            if (slab == 1) {
              tc_fence_before();
              mbar_arrive(&T.acce[e_ab]);  // this warp's columns are in registers: the MMA may refill
            }
            slab_head_sums(r, w2, v[2 * slab], v[2 * slab + 1]);
          }
          sc = quad_reduce_scatter(v, lane);
        }
        if (++e_ab == 2) {
          e_ab = 0;
          e_aph ^= 1u;
        }
        // streaming selection: append entries above the group's threshold
        bool near_full = false;
        if (ok && grp_w < nb_act) {
          const int64_t s = s_begin + (int64_t)tile_of(j, ns) * C::BM + q4 * 32 + my_lane;
          const bool valid = (s < s_end) && (s <= e_r);
          const uint32_t key = score_key(sc);
          const uint64_t p = pack_entry(key, (uint32_t)s);
          if (hist_est && j < ns && valid) {  // sample tile: count the score for the estimate
            const uint32_t bin = key >= 0x80000000u ? (key >> 20) - 0x800u : 0u;
            atomicAdd(&T.esth[grp_w][bin >> 1], (bin & 1u) ? 0x10000u : 1u);
          }
          const bool pass = valid && p > tau_r;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, pass);
          if (pass) seg_of(grp_w, q4)[qcnt + __popc(m & lanemask_lt())] = p;
          qcnt += __popc(m);
          if (qcnt > scap - 8u * 32u) {  // the next 8 tiles could overflow this sub-buffer
            near_full = true;
            if (lane == 0) atomicOr(&T.cflags, 1u << grp_w);
          }
        }
        // consensus every 8 tiles (the same tiles for every epilogue thread, so all of them
        // execute the same barriers; a thread whose wait ran out fails its next waits fast
        // and reports the abort here): a warp adds at most 32 entries per tile to a sub-buffer
        const bool est_now = (j + 1 == ns);  // the sample is complete
        if (((j & 7) == 7 || j + 1 == ntiles || est_now) &&
            named_bar_or(1, C::NEPI, near_full || est_now || T.abort_flag != 0)) {  // rare
          if (named_bar_or(1, C::NEPI, T.abort_flag != 0)) break;                   // uniform decision
          const uint32_t flags = T.cflags;
          publish_counts();
          // keep the sample's best r0 (the sample's expected share of 1.5 * need, plus a
          // margin); the threshold admits about 1.5 * need of the remaining keys
          uint32_t r0 = (uint32_t)((3 * (int64_t)need * ns) / (2 * (int64_t)ntiles)) + 64u;
          if (a.debug_flags & 4) r0 = 1;  // test hook: an estimate that is always too high
          if (est_now && hist_est) {
            // from the sample histogram: each group's 4 warps find the bin (from the top) where
            // the count reaches r0; its lower edge is the estimate, below the r0-th best of the
            // sample (so at least r0 sample entries stay), and each warp compacts its own
            // sub-buffer against it -- no pass over the sub-buffers
            const int gt = q4 * 32 + lane;  // thread within the group
            uint32_t loc[16], sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {  // bins 2047 - 16 gt - 2u - {0, 1}, descending
              const uint32_t wv = T.esth[grp_w][1023 - 8 * gt - u];
              loc[2 * u] = wv >> 16;
              loc[2 * u + 1] = wv & 0xFFFFu;
              sum += loc[2 * u] + loc[2 * u + 1];
            }
            uint32_t incl = warp_incl_scan(sum);
            if (lane == 31) T.escan[grp_w][q4] = incl;
            if (EG.tid < 4) T.ebin[EG.tid] = 0;
            EG.sync();
            for (int w = 0; w < q4; ++w) incl += T.escan[grp_w][w];
            const uint32_t excl = incl - sum;
            if (excl < r0 && r0 <= incl) {
              uint32_t c = excl;
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                if (c + loc[u] >= r0) {
                  T.ebin[grp_w] = 2047 - 16 * gt - u;
                  break;
                }
                c += loc[u];
              }
            }
            EG.sync();
            const int eb = T.ebin[grp_w];  // 0 when the sample holds fewer than r0 scores above bin 0
            const uint64_t th = eb > 0 ? (uint64_t)(((uint32_t)eb + 0x800u) << 20) << 32 : 0ull;
            if (grp_w < nb_act && th > 0) {
              qcnt = warp_compact_ge(seg_of(grp_w, q4), qcnt, th);
              if (th - 1ull > tau_r) tau_r = th - 1ull;  // admit x >= th from now on
            }
            if (EG.tid < 4) T.est[EG.tid] = (EG.tid < nb_act && T.ebin[EG.tid] > 0) ? 1 : 0;
            publish_counts();
          }
          for (int b = 0; b < nb_act; ++b) {
            const uint32_t tot = T.qcnt[b][0] + T.qcnt[b][1] + T.qcnt[b][2] + T.qcnt[b][3];
            const bool over = T.qcnt[b][0] > scap - 256u || T.qcnt[b][1] > scap - 256u ||
                              T.qcnt[b][2] > scap - 256u || T.qcnt[b][3] > scap - 256u;
            if (est_now && !hist_est) {
              const uint64_t th = cut_back(b, r0, r0 + r0 / 4u);
              if (EG.tid == 0) T.est[b] = th > 0 ? 1 : 0;
            } else if ((flags & (1u << b)) || (est_now && over && tot > need)) {
              // keep at most sub_cap - 128 in total (>= need + 128 since sub_cap >= need + 256):
              // then every sub-buffer has room for the 4 tiles until the next consensus
              cut_back(b, need, scap - 256u);
            }
          }
          if (EG.tid == 0) T.cflags = 0;
          EG.sync();
        }
      }
      // ---------------------------------------------------------------- final exact selection + emit
      if (EG.tid == 0) T.retry = 0;
      if (!named_bar_or(1, C::NEPI, T.abort_flag != 0)) {
        // each group's entries are >= tau + 1: tau is the group's admission threshold (entries
        // kept by a cut-back are >= the new tau + 1, later ones are above it)
        if (lane == 0 && q4 == 0) T.tau[grp_w] = tau_r;
        publish_counts();
        // every entry left lies above the group's estimate (if it has one): with fewer
        // than `need` of them the estimate was too high and the top-need is not complete
        bool redo = false;
        for (int b = 0; b < nb_act; ++b)
          redo |= T.est[b] && (T.qcnt[b][0] + T.qcnt[b][1] + T.qcnt[b][2] + T.qcnt[b][3] < need);
        if (redo && EG.tid == 0) {
          T.retry = 1;
          for (int b = 0; b < C::NB; ++b) T.est[b] = 0;
        }
        uint64_t* sbuf = reinterpret_cast<uint64_t*>(sA);  // the stage ring is idle now
        for (int b = 0; b < (redo ? 0 : nb_act); ++b) {
          uint32_t n = T.qcnt[b][0] + T.qcnt[b][1] + T.qcnt[b][2] + T.qcnt[b][3];
          if (n > (uint32_t)C::SMEM_CAP) {  // rare: cut back to exactly `need` first
            cut_back(b, need, need);
            publish_counts();
            n = T.qcnt[b][0] + T.qcnt[b][1] + T.qcnt[b][2] + T.qcnt[b][3];
          }
          // gather the four sub-buffers into shared memory (each segment starts 16-byte aligned),
          // keeping the largest entry for the selection's range
          uint32_t off = 0;
          uint64_t hi = 0ull;
          for (int q = 0; q < 4; ++q) {
            const uint32_t nq = T.qcnt[b][q];
            hi = group_copy_max<C::NEPI>(sbuf + off, seg_of(b, q), nq, hi, EG);
            off += (nq + 1u) & ~1u;
            if (nq & 1u) {  // pad to keep the next segment aligned: a zero entry sorts below everything
              if (EG.tid == 0) sbuf[off - 1] = 0ull;
            }
          }
          const uint32_t n_real = n;
          n = off;
          EG.sync();
          uint64_t* buf = sbuf;
          // keep-all is th = 1, so the zero pads never survive; otherwise the need-th
          // largest is a real entry (n_real > need), found within the entries' range
          uint64_t th = 1ull;
          if (n_real > need) {
            uint64_t lo = T.tau[b] + 1ull;
            group_minmax64<C::NEPI>(lo, hi, T.sel, EG);  // (lo is the same in every thread)
            th = radix11_threshold<C::NEPI>(buf, n, need, need, T.hist11, T.sel, EG, lo, hi);
          }
          const int64_t grp = T.grp0 + b;
          // dense rows and candidate sets are written straight from the entries >= th (exactly
          // `need` of them, or all when fewer); Reuse emission works on the compacted set
          if (a.mode == EMIT_DENSE) {
            emit_ge_warps<C::NEPI>(buf, n, th, a.out_idx + grp * a.topk,
                                   a.out_scores ? a.out_scores + grp * a.topk : nullptr, (uint32_t)a.topk, &T.ecount,
                                   EG);
          } else if (a.mode == EMIT_CAND) {
            emit_ge_warps<C::NEPI>(buf, n, th, a.cand + grp * a.n_sel,
                                   a.cand_scores ? a.cand_scores + grp * a.n_sel : nullptr, need, &T.ecount, EG);
          } else {  // EMIT_REUSE
            const uint32_t m = compact_ge<C::NEPI>(buf, buf, n, th, T.sel, EG);
            emit_reuse<C::NEPI>(buf, m, a.topk, T.mrow0[b], T.nmem[b], T.mrow0[b], a.out_idx, a.out_scores, T.sel,
                            T.bot, EG);
          }
          EG.sync();
        }
      }
    }
    __syncthreads();  // attempt done: the stage ring and the select state are free
    const bool again = T.retry != 0 && T.abort_flag == 0;
    __syncthreads();
    if (!again) break;
    }  // attempts
  }

  __syncthreads();
  if (T.abort_flag) {  // let in-flight async copies / MMAs drain before releasing TMEM
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t scan_smem_bytes(int H, int D) {
  if (H == 64 && D == 128) return scan_smem<64, 128>();
  if (H == 64 && D == 64) return scan_smem<64, 64>();
  return 0;
}

cudaError_t launch_scan(const ScanArgs& a, const CUtensorMap* kmap, int grid, cudaStream_t s) {
  const size_t smem = scan_smem_bytes(a.H, a.D);
  if (a.H == 64 && a.D == 128) {
    auto k = scan_kernel<64, 128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, ScanCfg<64, 128>::THREADS, smem, s>>>(*kmap, a);
  } else if (a.H == 64 && a.D == 64) {
    auto k = scan_kernel<64, 64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, ScanCfg<64, 64>::THREADS, smem, s>>>(*kmap, a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pivot
