// aux.cu -- the non-tensor-core kernels of the library:
//   * rowselect_kernel  Eq. (9): per member row, the top-k of its candidates'
//                       re-scored keys (written by the refine kernel);
//   * simt_kernel       portable CUDA-core path (fp32 inputs, or shapes the
//                       tensor-core kernels do not take): Eq. (1)/(4)-(9) per
//                       group with the same exact selection.
// PIVOT: picx.dev summary of the paper, Methodology, Eq. (1)-(9).
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

// ------------------------------------------------------------------ Eq. (9)
__global__ void __launch_bounds__(256) rowselect_kernel(const RowSelArgs a) {
  extern __shared__ uint64_t sbuf[];  // c packed entries of the row
  __shared__ SelSmem S;
  __shared__ uint32_t hist11[kHist11Words];
  const Group<256> G{(int)threadIdx.x, 0};
  for (int64_t row = a.row_base + blockIdx.x; row < a.n_rows; row += gridDim.x) {
    const int64_t grp = row / a.g;
    int64_t P;
    if (a.key_off)
      P = a.key_off[grp + 1] - a.key_off[grp];
    else
      P = min64(grp * a.g + a.g, a.L);
    const uint32_t n_c = (uint32_t)min64(a.c, P);
    const uint32_t* kr = a.keys + row * (int64_t)a.c;
    const int32_t* cr = a.cand + grp * (int64_t)a.c;
    uint32_t nv = 0;
    for (uint32_t i = G.tid; i < n_c; i += 256) {
      const uint32_t key = __ldg(kr + i);
      const int32_t id = __ldg(cr + i);
      const bool ok = key != 0u && id >= 0;
      sbuf[i] = ok ? pack_entry(key, (uint32_t)id) : 0ull;
      nv += ok ? 1u : 0u;
    }
    uint32_t total;
    group_offsets<256>(nv, &total, S, G);
    G.sync();
    const uint64_t th =
        (total <= (uint32_t)a.topk) ? 1ull : radix11_threshold<256>(sbuf, n_c, a.topk, a.topk, hist11, S, G);
    emit_row<256>(sbuf, n_c, 0xFFFFFFFFu, th - 1ull, a.out_idx + row * a.topk,
                  a.out_scores ? a.out_scores + row * a.topk : nullptr, (uint32_t)a.topk, S, G);
    G.sync();
  }
}

cudaError_t launch_rowselect(const RowSelArgs& a, int grid, cudaStream_t s) {
  const size_t smem = (size_t)a.c * sizeof(uint64_t);
  cudaFuncSetAttribute(rowselect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  rowselect_kernel<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ portable path
__device__ __forceinline__ float ld_elem(const void* p, int is_bf16, int64_t i) {
  if (is_bf16) return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t*>(p)[i]) << 16);
  return reinterpret_cast<const float*>(p)[i];
}

// sum_j w_j ReLU(q_j . k_s) with q/w in fp32 shared/global scratch
__device__ __forceinline__ float simt_score(const float* qv, const float* wv, int H, int D, const void* k,
                                            int is_bf16, int64_t krow) {
  float total = 0.f;
  for (int j = 0; j < H; ++j) {
    float dot = 0.f;
    for (int x = 0; x < D; ++x) dot = fmaf(qv[j * D + x], ld_elem(k, is_bf16, krow * D + x), dot);
    total = fmaf(wv[j], fmaxf(dot, 0.f), total);
  }
  return total;
}

__global__ void __launch_bounds__(256) simt_kernel(const SimtArgs a) {
  __shared__ SelSmem S;
  __shared__ uint64_t bot[16];
  __shared__ uint32_t cnt2;
  const Group<256> G{(int)threadIdx.x, 0};
  const int H = a.H, D = a.D;
  float* qv = a.fscratch + (int64_t)blockIdx.x * (H * D + H);
  float* wv = qv + H * D;
  uint64_t* buf = a.scratch + (int64_t)blockIdx.x * a.scratch_per_block;
  uint64_t* mb = buf + a.member_off;  // member entries (Refine)
  for (int64_t grp = a.grp_base + blockIdx.x; grp < a.n_groups; grp += gridDim.x) {
    int64_t kbase, P, mrow0, t_first, orow0;
    int nm;
    if (a.key_off) {
      kbase = a.key_off[grp];
      P = a.key_off[grp + 1] - kbase;
      mrow0 = grp * a.g;
      nm = a.g;
      t_first = P - a.g;
      orow0 = grp * a.g;
    } else {
      kbase = 0;
      mrow0 = grp * a.g;
      nm = (int)min64(a.g, a.L - mrow0);
      P = mrow0 + nm;
      t_first = mrow0;
      orow0 = mrow0;
    }
    // Eq. (4): proxy = per-head mean, rounded to the input dtype (one member: the query
    // itself); the first- / last-query aggregation pools that one member
    const int pn = a.agg != 0 ? 1 : nm;
    const int64_t prow0 = a.agg == 2 ? mrow0 + nm - 1 : mrow0;
    for (int i = G.tid; i < H * D; i += 256) {
      float s = 0.f;
      for (int m = 0; m < pn; ++m) s += ld_elem(a.q, a.is_bf16, (prow0 + m) * (int64_t)H * D + i);
      float v = pn > 1 ? __fdiv_rn(s, (float)pn) : s;
      if (a.is_bf16) v = __bfloat162float(__float2bfloat16_rn(v));
      qv[i] = v;
    }
    for (int j = G.tid; j < H; j += 256) {
      float s = 0.f;
      for (int m = 0; m < pn; ++m) s += a.w[(prow0 + m) * H + j];
      wv[j] = pn > 1 ? __fdiv_rn(s, (float)pn) : s;
    }
    G.sync();
    // Eq. (5) (Eq. (1) when g == 1) over the causal prefix s <= group end
    for (int64_t s = G.tid; s < P; s += 256)
      buf[s] = pack_entry(score_key(simt_score(qv, wv, H, D, a.k, a.is_bf16, kbase + s)), (uint32_t)s);
    G.sync();
    const uint32_t n = (uint32_t)P;
    if (a.variant == 0) {
      const uint64_t th = radix_threshold<256>(buf, n, a.topk, a.topk, S, G);
      const uint32_t m = compact_ge<256>(buf, buf, n, th, S, G);
      emit_row<256>(buf, m, 0xFFFFFFFFu, 0ull, a.out_idx + orow0 * a.topk,
                    a.out_scores ? a.out_scores + orow0 * a.topk : nullptr, (uint32_t)a.topk, S, G);
    } else if (a.variant == 1) {
      const uint32_t nsel = (uint32_t)(a.topk + a.g - 1);
      const uint64_t th = radix_threshold<256>(buf, n, nsel, nsel, S, G);
      const uint32_t m = compact_ge<256>(buf, buf, n, th, S, G);
      emit_reuse<256>(buf, m, a.topk, t_first, nm, orow0, a.out_idx, a.out_scores, S, bot, G);
    } else {
      const uint64_t th = radix_threshold<256>(buf, n, a.c, a.c, S, G);  // Eq. (7)
      const uint32_t m = compact_ge<256>(buf, buf, n, th, S, G);
      if (a.cand_out)
        emit_row<256>(buf, m, 0xFFFFFFFFu, 0ull, a.cand_out + grp * a.c,
                      a.cand_scores ? a.cand_scores + grp * a.c : nullptr, (uint32_t)a.c, S, G);
      for (int r = 0; r < nm; ++r) {
        const int64_t t = t_first + r;
        const int64_t qrow = mrow0 + r;
        G.sync();
        for (int i = G.tid; i < H * D; i += 256) qv[i] = ld_elem(a.q, a.is_bf16, qrow * (int64_t)H * D + i);
        for (int j = G.tid; j < H; j += 256) wv[j] = a.w[qrow * H + j];
        if (G.tid == 0) cnt2 = 0;
        G.sync();
        for (uint32_t i0 = 0; i0 < m; i0 += 256) {  // Eq. (8) over s in C, s <= t
          const uint32_t i = i0 + G.tid;
          bool pass = false;
          uint64_t val = 0;
          if (i < m) {
            const uint32_t s = entry_idx(buf[i]);
            if ((int64_t)s <= t) {
              val = pack_entry(score_key(simt_score(qv, wv, H, D, a.k, a.is_bf16, kbase + s)), s);
              pass = true;
            }
          }
          warp_append(pass, val, mb, &cnt2);
        }
        G.sync();
        const uint32_t n2 = cnt2;
        const uint64_t th2 = radix_threshold<256>(mb, n2, a.topk, a.topk, S, G);  // Eq. (9)
        const uint32_t m2 = compact_ge<256>(mb, mb, n2, th2, S, G);
        emit_row<256>(mb, m2, 0xFFFFFFFFu, 0ull, a.out_idx + (orow0 + r) * a.topk,
                      a.out_scores ? a.out_scores + (orow0 + r) * a.topk : nullptr, (uint32_t)a.topk, S, G);
      }
    }
    G.sync();
  }
}

cudaError_t launch_simt(const SimtArgs& a, int grid, cudaStream_t s) {
  simt_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pivot
