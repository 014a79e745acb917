// refine.cu -- K2: PIVOT-Refine candidate re-scoring on tcgen05.
//
// PIVOT (picx.dev summary of the paper, Methodology, "Two Variants"):
//   Eq. (8)  I_{t,s} = sum_j w_{t,j} ReLU(q_{t,j} . k_s)   for s in C (the
//            group's proxy top-c) and every member t of the group.
// The causal mask s <= t is applied per member.  This kernel produces the
// per-member scores of all c candidates as order-preserving 32-bit keys
// (0 = masked / no candidate); the member top-k (Eq. 9) is taken by the
// row-select kernel.
//
// One persistent CTA per SM; a work item is (group, chunk of MC = 512/H
// members, part of the candidate tiles: one part for prefill, several when
// there are few groups, as in a decode batch).  Per item the members' query rows (MC*H rows x D, bf16) are the
// MMA's B operand in shared memory (K-major, 128-byte swizzle), loaded by TMA.
// Each 128-candidate A tile (3-stage ring) is gathered in two halves that
// complete on the same barrier: rows 0-63 by TMA 4-row gathers (warp 17),
// rows 64-127 by 16-byte cp.async into the same swizzled layout (warps 18-19,
// one row per thread), so both the TMA and the load/store path have requests
// in flight.  Warp 16 issues
//     D[128 candidates x (members*H)] = K_gathered . Q_members^T
// as up to two N=256 MMAs into two TMEM accumulators.  Warps 0-15 (one per
// TMEM lane quarter and member of an accumulator half) read their member's 64
// columns in the 16x256b shape, apply ReLU, weight each head by the member's
// own w (16 weights per thread) and sum the heads across the thread quad, then
// write the member's key row.
#include <cuda_bf16.h>

#include <cstddef>

#include "headsum.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

template <int H, int D>
struct RefCfg {
  static constexpr int NROW = 512;      // B rows (members * H) per item
  static constexpr int MC = NROW / H;   // members per item
  static constexpr int KB = D / 64;
  static constexpr int BM = 128;
  static constexpr int STAGES = 3;
  static constexpr int A_BYTES = BM * D * 2;
  static constexpr int B_BYTES = NROW * D * 2;
  // warps 0-15 epilogue (one per TMEM lane quarter and member of an accumulator
  // half), 16 MMA, 17 TMA gather, 18-19 cp.async gather
  static constexpr int THREADS = 640;
  static constexpr int W_MMA = 16, W_TMA = 17, W_CPA = 18;
  static constexpr int TMA_ROWS = 64;   // rows 0..63 of a tile by TMA gather, the rest by cp.async
  static constexpr int NEPI = 512;
  static constexpr int MPH = 256 / H;   // members per accumulator half
  static_assert(MPH * 4 * 32 == NEPI, "one epilogue warp per (lane quarter, member of a half)");
  static_assert(H == 64, "the epilogue reads 64 heads per member in the 16x256b.x8 shape");
};

// Geometry of one work item, written by the conductor (the MMA thread) into a two-slot ring.
struct RefItem {
  int item, nm, ntiles, nhalf, n_c, tile0;
  int64_t grp, key_base, qrow0, t0, orow0;
};

struct RefTail {
  uint64_t full[3], empty[3], accf[2], acce[2];
  uint64_t bfull[2], bfree[2];      // per half of B (members 0-3 / 4-7): landed / its last MMA done
  uint64_t itfull[2], itempty[2];   // item ring: geometry written / every consumer warp done with it
  uint32_t tmem_slot;
  volatile int abort_flag;
  RefItem it[2];
  alignas(16) float wperm[8 * 4 * 20];  // members' w in the row-permuted layout of wperm_index
};
static_assert(offsetof(RefTail, wperm) % 16 == 0, "wperm must be 16-byte aligned");

template <int H, int D>
constexpr size_t refine_smem() {
  using C = RefCfg<H, D>;
  return C::B_BYTES + C::STAGES * C::A_BYTES + sizeof(RefTail);  // base must be 1024-aligned (checked)
}
static_assert(refine_smem<64, 128>() <= 232448, "227 KB of dynamic shared memory per CTA");

// The roles run their own item loops (no block-wide barrier between items): the conductor
// (MMA thread) claims items and publishes their geometry one item ahead; the gather warps
// run ahead into the next item as ring stages free up; each half of the members' q rows
// (B) is reloaded as soon as the previous item's last MMA on that half has completed, so
// an item's first MMAs overlap the previous item's last ones.
template <int H, int D>
__global__ void __launch_bounds__(640, 1) refine_kernel(const __grid_constant__ CUtensorMap kmap,
                                                              const __grid_constant__ CUtensorMap qmap, const RefineArgs a,
                                                              uint32_t* __restrict__ out_keys) {
  using C = RefCfg<H, D>;
  constexpr int kConsumers = 16 + 1 + 2;  // epilogue, TMA-gather and cp.async warps: one arrive per item each
  constexpr uint32_t kHalfBytes = C::KB * 256 * 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte-swizzled operands need a 1024-byte aligned base; there is no
  // room for alignment slack next to a 3-stage ring, so refuse to run otherwise
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(a.status, DEV_ERR_BOUNDS);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sB = smem;
  uint8_t* sA = smem + C::B_BYTES;
  RefTail& T = *reinterpret_cast<RefTail*>(smem + C::B_BYTES + C::STAGES * C::A_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&T.full[s], 1 + (C::BM - C::TMA_ROWS));  // TMA expect-tx arrive + one per cp.async row
      mbar_init(&T.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&T.accf[b], 1);
      mbar_init(&T.acce[b], C::NEPI);
      mbar_init(&T.bfull[b], 1);
      mbar_init(&T.bfree[b], 1);
      mbar_init(&T.itfull[b], 1);
      mbar_init(&T.itempty[b], kConsumers);
    }
    T.abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&kmap);
    prefetch_tmap(&qmap);
  }
  if (warp == C::W_MMA) {
    tmem_alloc(&T.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T.tmem_slot;
  const int chunks = (a.g + C::MC - 1) / C::MC;
  const bool decode = (a.key_off != nullptr);
  auto fail = [&]() {
    T.abort_flag = 1;
    atomicOr(a.status, DEV_ERR_TIMEOUT);
  };

  if (warp == C::W_MMA) {
    // ------------------------------------------------------------ conductor + MMA issuer
    if (lane == 0) {
      // claim the next item and publish its geometry in ring slot I
      auto claim = [&](RefItem& I) {
        const int item = (int)atomicAdd(a.counter, 1u);
        I.item = item;
        if (item < a.n_items) {
          // longest prefix first: prefill groups in descending order; an item is
          // (group, member chunk, candidate part)
          const int cp = item % a.cparts, gi = item / a.cparts;
          const int64_t grp = decode ? (int64_t)(gi / chunks) : (a.n_groups - 1 - gi / chunks);
          const int mc = gi % chunks;
          const int r0 = mc * C::MC;
          int64_t P, nmem_g;
          if (decode) {
            // a key shard (pos_base / plen_off): the candidate ids are rows of this shard, the
            // members' positions and the candidate count follow the full prefix
            P = a.plen_off ? a.plen_off[grp + 1] - a.plen_off[grp] : a.key_off[grp + 1] - a.key_off[grp];
            nmem_g = a.g;
            I.key_base = a.key_off[grp];
            I.qrow0 = grp * a.g + r0;
            I.t0 = P - a.g + r0;
            I.orow0 = grp * a.g + r0;
          } else {
            const int64_t first = grp * a.g;
            const int64_t last = min64(first + a.g, a.L) - 1;
            P = last + 1;
            nmem_g = last - first + 1;
            I.key_base = 0;
            I.qrow0 = first + r0;
            I.t0 = first + r0;
            I.orow0 = first + r0;
          }
          I.grp = grp;
          I.nm = (int)max64(0, min64(C::MC, nmem_g - r0));
          I.n_c = (int)min64(a.c, P);
          const int tiles = (I.n_c + C::BM - 1) / C::BM, tpp = (tiles + a.cparts - 1) / a.cparts;
          I.tile0 = min(tiles, cp * tpp);
          I.ntiles = min(tiles, I.tile0 + tpp) - I.tile0;
          I.nhalf = (I.nm * H + 255) / 256;
        }
      };
      uint32_t m_st = 0, m_ph = 0, m_ab = 0, m_aph = 0;
      uint32_t lb[2] = {0u, 0u}, cb[2] = {0u, 0u};  // loads issued / releases committed, per half of B
      bool held[2] = {false, false};                 // an earlier item's MMAs may still read this half
      const uint32_t baddr = smem_u32(sB);
      claim(T.it[0]);
      mbar_arrive(&T.itfull[0]);
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int s = n & 1;
        const RefItem I = T.it[s];
        if (I.item >= a.n_items || T.abort_flag) break;
        bool fetched = false;
        // the next item goes into the other slot once every consumer is done with item n-1
        auto fetch_next = [&]() {
          if (n >= 1 && !mbar_wait(&T.itempty[s ^ 1], (uint32_t)((n - 1) >> 1) & 1u, a.timeout_ns, &T.abort_flag)) {
            fail();
            return false;
          }
          claim(T.it[s ^ 1]);
          mbar_arrive(&T.itfull[s ^ 1]);
          return true;
        };
        if (I.nm == 0 || I.ntiles == 0) {
          ok = fetch_next();
          continue;
        }
        for (int j = 0; j < I.ntiles && ok; ++j) {
          if (!mbar_wait(&T.full[m_st], m_ph, a.timeout_ns, &T.abort_flag)) {
            fail();
            ok = false;
            break;
          }
          const uint32_t aaddr = smem_u32(sA + m_st * C::A_BYTES);
          for (int h = 0; h < I.nhalf; ++h) {
            if (j == 0) {
              // this item's half h of B: once the last MMA of the previous user of the half has
              // completed, load this item's members' q rows for it (rows past the members are
              // loaded too, not multiplied)
              if (held[h] && !mbar_wait(&T.bfree[h], (cb[h] - 1u) & 1u, a.timeout_ns, &T.abort_flag)) {
                fail();
                ok = false;
                break;
              }
              held[h] = false;
              mbar_arrive_expect_tx(&T.bfull[h], kHalfBytes);
              for (int kb = 0; kb < C::KB; ++kb)
                tma_load_2d(sB + kb * (C::NROW * 128) + h * 256 * 128, &qmap, &T.bfull[h], kb * 64,
                            (int)(I.qrow0 * H + h * 256));
              ++lb[h];
              if (!mbar_wait(&T.bfull[h], (lb[h] - 1u) & 1u, a.timeout_ns, &T.abort_flag)) {
                fail();
                ok = false;
                break;
              }
            }
            if (!mbar_wait(&T.acce[m_ab], m_aph ^ 1u, a.timeout_ns, &T.abort_flag)) {
              fail();
              ok = false;
              break;
            }
            tc_fence_after();
            const int nh = min(256, I.nm * H - 256 * h);
            const uint32_t idesc = idesc_bf16_f32(C::BM, nh);
            const uint32_t dtm = tmem + m_ab * 256u;
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = sw128_kmajor_desc(aaddr + kb * (C::BM * 128) + kk * 32);
                const uint64_t bd = sw128_kmajor_desc(baddr + kb * (C::NROW * 128) + h * 256 * 128 + kk * 32);
                umma_bf16(dtm, ad, bd, idesc, (kb | kk) ? 1u : 0u);
              }
            umma_commit(&T.accf[m_ab]);
            if (j + 1 == I.ntiles) {  // the item's last MMA on this half: the half may be reloaded after it
              umma_commit(&T.bfree[h]);
              ++cb[h];
              held[h] = true;
            }
            if (++m_ab == 2) {
              m_ab = 0;
              m_aph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(&T.empty[m_st]);
          if (++m_st == C::STAGES) {
            m_st = 0;
            m_ph ^= 1u;
          }
          if (!fetched) {  // after the item's first tile: the epilogue has finished item n-1 by now
            fetched = true;
            ok = fetch_next();
          }
        }
      }
      if (!ok) {  // unblock the consumers: publish an empty item in both slots
        T.it[0].item = a.n_items;
        T.it[1].item = a.n_items;
        mbar_arrive(&T.itfull[0]);
        mbar_arrive(&T.itfull[1]);
      }
    }
  } else if (warp == C::W_TMA) {
    // ------------------------------------------------------------ TMA gather producer
    // lane l gathers candidate rows 4l..4l+3 of each 128-row tile: one 16-byte load of
    // their ids, then one 4-row gather per 64-column k-block (ids past n_c read row 0;
    // those slots are masked by the epilogue)
    uint32_t p_st = 0, p_ph = 0;
    for (int n = 0;; ++n) {
      const int s = n & 1;
      int okw = 1;
      if (lane == 0) okw = mbar_wait(&T.itfull[s], (uint32_t)(n >> 1) & 1u, a.timeout_ns, &T.abort_flag) ? 1 : 0;
      okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
      if (!okw) {
        if (lane == 0) fail();
        break;
      }
      const RefItem I = T.it[s];
      if (I.item >= a.n_items || T.abort_flag) break;
      const int32_t* cand = a.cand + I.grp * (int64_t)a.c;
      const int n_c = I.n_c, tile0 = I.tile0, ntiles = I.nm > 0 ? I.ntiles : 0;
      auto load_ids = [&](int j, int (&id)[4]) {
        const int slot0 = (tile0 + j) * C::BM + 4 * lane;
        if (slot0 + 3 < n_c && (reinterpret_cast<uintptr_t>(cand + slot0) & 15u) == 0) {
          const int4 v = __ldg(reinterpret_cast<const int4*>(cand + slot0));
          id[0] = v.x;
          id[1] = v.y;
          id[2] = v.z;
          id[3] = v.w;
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) id[u] = (slot0 + u < n_c) ? __ldg(cand + slot0 + u) : -1;
        }
      };
      int idn[4] = {-1, -1, -1, -1};
      if (ntiles > 0) load_ids(0, idn);  // ids of the next tile are loaded one tile ahead
      bool okt = true;
      for (int j = 0; j < ntiles; ++j) {
        int id[4] = {idn[0], idn[1], idn[2], idn[3]};
        if (j + 1 < ntiles) load_ids(j + 1, idn);
        if (lane == 0) okw = mbar_wait(&T.empty[p_st], p_ph ^ 1u, a.timeout_ns, &T.abort_flag) ? 1 : 0;
        okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
        if (!okw) {
          if (lane == 0) fail();
          okt = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&T.full[p_st], (uint32_t)(C::TMA_ROWS * D * 2));
        __syncwarp();
        int row[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) row[u] = (int)(I.key_base + (id[u] >= 0 ? id[u] : 0));
        uint8_t* dst = sA + p_st * C::A_BYTES + (4 * lane) * 128;
        if (4 * lane < C::TMA_ROWS) {
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_gather4(dst + kb * (C::BM * 128), &kmap, &T.full[p_st], kb * 64, row[0], row[1], row[2], row[3]);
        }
        if (++p_st == C::STAGES) {
          p_st = 0;
          p_ph ^= 1u;
        }
      }
      if (!okt) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&T.itempty[s]);
    }
  } else if (warp >= C::W_CPA) {
    // ------------------------------------------------------------ cp.async gather producer
    // thread u copies candidate row TMA_ROWS + u of each tile (16-byte chunks into the
    // 128-byte-swizzled layout the TMA would produce); tile j's copies are committed as
    // one group, and once the group of tile j-1 has landed the thread makes it visible
    // to the tensor core (proxy fence) and arrives on that stage's full barrier
    const int row = C::TMA_ROWS + (tid - 32 * C::W_CPA);
    uint32_t p_st = 0, p_ph = 0;
    uint32_t prev_st = 0;
    bool pending = false;
    auto drain = [&]() {
      if (pending) {
        cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&T.full[prev_st]);
        pending = false;
      }
    };
    for (int n = 0;; ++n) {
      const int s = n & 1;
      int okw = 1;
      if (lane == 0) okw = mbar_wait(&T.itfull[s], (uint32_t)(n >> 1) & 1u, a.timeout_ns, &T.abort_flag) ? 1 : 0;
      okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
      if (!okw) {
        if (lane == 0) fail();
        break;
      }
      const RefItem I = T.it[s];
      if (I.item >= a.n_items || T.abort_flag) break;
      const int32_t* cand = a.cand + I.grp * (int64_t)a.c;
      const int n_c = I.n_c, tile0 = I.tile0, ntiles = I.nm > 0 ? I.ntiles : 0;
      auto id_of = [&](int j) {
        const int slot = (tile0 + j) * C::BM + row;
        const int id = (slot < n_c) ? __ldg(cand + slot) : -1;
        return id >= 0 ? id : 0;  // slots without a candidate copy row 0 (masked later)
      };
      int idn = ntiles > 0 ? id_of(0) : 0;
      bool okt = true;
      for (int j = 0; j < ntiles; ++j) {
        const int id = idn;
        if (j + 1 < ntiles) idn = id_of(j + 1);
        if (!mbar_wait(&T.empty[p_st], p_ph ^ 1u, a.timeout_ns, &T.abort_flag)) {
          fail();
          okt = false;
          break;
        }
        const uint16_t* src = a.k + (I.key_base + id) * (int64_t)D;
        uint8_t* dst = sA + p_st * C::A_BYTES + row * 128;
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            cp_async_16(dst + kb * (C::BM * 128) + ((ch ^ (row & 7)) << 4), src + kb * 64 + ch * 8);
        cp_async_commit();
        if (pending) {
          cp_async_wait<1>();
          fence_proxy_async_smem();
          mbar_arrive(&T.full[prev_st]);
        }
        pending = true;
        prev_st = p_st;
        if (++p_st == C::STAGES) {
          p_st = 0;
          p_ph ^= 1u;
        }
      }
      drain();  // the item's last tile: its rows land and its full barrier is armed before moving on
      if (!okt) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&T.itempty[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-15)
    // warp w reads TMEM lanes 32*(w%4).. (its candidates) and handles member w/4 of
    // each accumulator half; 16x256b loads, 16 heads per thread, then the quad
    // reduce-scatter leaves each thread with one candidate's score (lane my_lane)
    const int q4 = warp & 3;
    const int ml = warp >> 2;
    const int my_lane = quad_key_lane(lane);
    uint32_t e_ab = 0, e_aph = 0;
    for (int n = 0;; ++n) {
      const int s = n & 1;
      const bool got = mbar_wait(&T.itfull[s], (uint32_t)(n >> 1) & 1u, a.timeout_ns, &T.abort_flag);
      if (!got) fail();
      const RefItem I = T.it[s];
      const bool valid = got && I.item < a.n_items;
      const int nm = valid ? I.nm : 0;
      // the members' w (one value per thread), read before the barrier that waits for every
      // epilogue warp to be done with the previous item's table; the barrier also makes the
      // decision to stop uniform (a warp whose wait ran out arrives late but does arrive)
      const float wv = tid < nm * H ? __ldg(a.w + I.qrow0 * H + tid) : 0.f;
      if (named_bar_or(2, C::NEPI, !valid || T.abort_flag != 0)) break;
      const int32_t* cand = a.cand + I.grp * (int64_t)a.c;
      const int ntiles = nm > 0 ? I.ntiles : 0, nhalf = I.nhalf, tile0 = I.tile0, n_c = I.n_c;
      const int64_t pos0 = (valid && a.pos_base) ? a.pos_base[I.grp] : 0;  // global position of key row 0 here
      if (tid < nm * H) T.wperm[wperm_index(tid / H, tid % H)] = wv;
      named_bar_sync(2, C::NEPI);
      bool stop = false;
      for (int j = 0; j < ntiles && !stop; ++j) {
        const int slot = (tile0 + j) * C::BM + q4 * 32 + my_lane;
        const int sidx = (slot < n_c) ? __ldg(cand + slot) : -1;
        for (int h = 0; h < nhalf; ++h) {
          const bool ok = mbar_wait(&T.accf[e_ab], e_aph, a.timeout_ns, &T.abort_flag);
          const int r = h * C::MPH + ml;  // member within the item
          const bool mv = r < nm;          // uniform across the warp
          float sc = 0.f;
          if (ok) {
            tc_fence_after();
            float2 w2[8];
            if (mv) load_w2(T.wperm, r, lane, w2);
            float v[4];
#pragma unroll
            for (int slab = 0; slab < 2; ++slab) {
              uint32_t rr[32];
              tmem_ld16x256b_x8(tmem + ((uint32_t)(q4 * 32 + slab * 16) << 16) + e_ab * 256u + (uint32_t)(ml * H), rr);
              tmem_wait_ld();
              if (slab == 1) {
                tc_fence_before();
                mbar_arrive(&T.acce[e_ab]);  // accumulator copied: the MMA may refill it
              }
              if (mv) slab_head_sums(rr, w2, v[2 * slab], v[2 * slab + 1]);
            }
            if (mv) sc = quad_reduce_scatter(v, lane);
          } else {
            fail();
          }
          if (++e_ab == 2) {
            e_ab = 0;
            e_aph ^= 1u;
          }
          if (!ok) {
            stop = true;
            break;
          }
          // Eq. (8) with the member's causal mask s <= t; key 0 marks "not eligible"
          if (mv && slot < a.c) {
            const int64_t t = I.t0 + r;
            const bool valid = (sidx >= 0) && ((int64_t)sidx + pos0 <= t);
            out_keys[(I.orow0 + r) * (int64_t)a.c + slot] = valid ? score_key(sc) : 0u;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&T.itempty[s]);  // (after a failure the abort flag is set: the next round stops)
    }
  }

  __syncthreads();
  if (T.abort_flag) {  // let in-flight async copies / MMAs drain before releasing TMEM
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  if (warp == C::W_MMA) tmem_dealloc(tmem, 512);
}

size_t refine_smem_bytes(int H, int D, int /*mc*/) {
  if (H == 64 && D == 128) return refine_smem<64, 128>();
  if (H == 64 && D == 64) return refine_smem<64, 64>();
  return 0;
}

cudaError_t launch_refine(const RefineArgs& a, const CUtensorMap* kmap, const CUtensorMap* qmap, int grid,
                          cudaStream_t s) {
  const size_t smem = refine_smem_bytes(a.H, a.D, a.mc);
  uint32_t* keys = a.keys;
  if (a.H == 64 && a.D == 128) {
    auto k = refine_kernel<64, 128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, RefCfg<64, 128>::THREADS, smem, s>>>(*kmap, *qmap, a, keys);
  } else if (a.H == 64 && a.D == 64) {
    auto k = refine_kernel<64, 64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, RefCfg<64, 64>::THREADS, smem, s>>>(*kmap, *qmap, a, keys);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pivot
