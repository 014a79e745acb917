// headsum.cuh -- the ReLU-weighted head sum of Eq. (5) / Eq. (8) on accumulator
// rows read from TMEM in the 16x256b shape (see tmem_ld16x256b_x8).
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace pivot {

// Partial sums of one 16x256b.x8 slab: sum over this thread's 16 heads
// (8j + 2(t%4) + {0,1}, j = 0..7) of w_h * ReLU(x_h) for its two keys (lanes
// t/4 and t/4 + 8 of the slab); w2[j] holds the weights of heads 8j + 2(t%4) + {0,1}.
__device__ __forceinline__ void slab_head_sums(const uint32_t (&r)[32], const float2 (&w2)[8], float& ka,
                                               float& kb) {
  float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
  for (int jj = 0; jj < 8; jj += 2) {
    a0 = __ffma2_rn(w2[jj], make_float2(fmaxf(__uint_as_float(r[4 * jj + 0]), 0.f),
                                        fmaxf(__uint_as_float(r[4 * jj + 1]), 0.f)), a0);
    b0 = __ffma2_rn(w2[jj], make_float2(fmaxf(__uint_as_float(r[4 * jj + 2]), 0.f),
                                        fmaxf(__uint_as_float(r[4 * jj + 3]), 0.f)), b0);
    a1 = __ffma2_rn(w2[jj + 1], make_float2(fmaxf(__uint_as_float(r[4 * jj + 4]), 0.f),
                                            fmaxf(__uint_as_float(r[4 * jj + 5]), 0.f)), a1);
    b1 = __ffma2_rn(w2[jj + 1], make_float2(fmaxf(__uint_as_float(r[4 * jj + 6]), 0.f),
                                            fmaxf(__uint_as_float(r[4 * jj + 7]), 0.f)), b1);
  }
  ka = (a0.x + a0.y) + (a1.x + a1.y);
  kb = (b0.x + b0.y) + (b1.x + b1.y);
}

// Reduce-scatter over the 4 threads of a quad: v[i] is this thread's partial sum
// for key i (slab i >> 1, lane t/4 + 8 (i & 1)); thread t%4 = m returns the full
// sum of key m.  The whole warp calls.
__device__ __forceinline__ float quad_reduce_scatter(const float (&v)[4], int lane) {
  const bool x1 = (lane & 1) != 0, x2 = (lane & 2) != 0;
  float k0 = x1 ? v[1] : v[0], k1 = x1 ? v[3] : v[2];  // keys with bit 0 == lane bit 0
  k0 += __shfl_xor_sync(0xFFFFFFFFu, x1 ? v[0] : v[1], 1);
  k1 += __shfl_xor_sync(0xFFFFFFFFu, x1 ? v[2] : v[3], 1);
  return (x2 ? k1 : k0) + __shfl_xor_sync(0xFFFFFFFFu, x2 ? k0 : k1, 2);
}

// The TMEM lane (within the warp's 32-lane quarter) whose key thread `lane` ends
// up with after quad_reduce_scatter.
__device__ __forceinline__ int quad_key_lane(int lane) { return (lane >> 2) + 8 * (lane & 1) + 16 * ((lane >> 1) & 1); }

// Row-permuted weight table: row (b, m) of 20 floats holds heads 8j + 2m + {0,1},
// j = 0..7, of weight vector b (16 floats used; the stride keeps the 4 rows a warp
// reads in distinct banks).  Index of head hj of vector b:
__device__ __forceinline__ int wperm_index(int b, int hj) {
  return (b * 4 + ((hj >> 1) & 3)) * 20 + 2 * (hj >> 3) + (hj & 1);
}
// This thread's 16 weights of vector b (4 16-byte loads).
__device__ __forceinline__ void load_w2(const float* wperm, int b, int lane, float2 (&w2)[8]) {
#pragma unroll
  for (int jj = 0; jj < 8; jj += 2) {
    const float4 w4 = *reinterpret_cast<const float4*>(&wperm[(b * 4 + (lane & 3)) * 20 + 2 * jj]);
    w2[jj] = make_float2(w4.x, w4.y);
    w2[jj + 1] = make_float2(w4.z, w4.w);
  }
}

}  // namespace pivot
