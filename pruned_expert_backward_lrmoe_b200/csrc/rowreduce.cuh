// Warp-level row reductions shared by the score and the routing-weight gradient.
//
// One fixed order makes every result bit-reproducible: for a row of V 16-byte
// vectors, lane l sums vectors l, l+32, ... element by element as
// fl(acc + fl(x*y)) (x*x for norms), then a butterfly fl(acc[l] + acc[l^o]) for
// o = 16, 8, 4, 2, 1; lane 0 (every lane) then holds the result.
#pragma once

#include <atomic>

#include "common.cuh"
#include "launch.h"

namespace lrmoe {
namespace rowred {

template <lrmoe_dtype DT>
__device__ __forceinline__ float acc_vec(float acc, const uint4& v) {
  if constexpr (DT == LRMOE_BF16) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = bf16_bits_to_f32(w[i] & 0xffffu);
      const float hi = bf16_bits_to_f32(w[i] >> 16);
      acc = __fadd_rn(acc, __fmul_rn(lo, lo));
      acc = __fadd_rn(acc, __fmul_rn(hi, hi));
    }
  } else {
    const float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                        __uint_as_float(v.w)};
#pragma unroll
    for (int i = 0; i < 4; ++i) acc = __fadd_rn(acc, __fmul_rn(f[i], f[i]));
  }
  return acc;
}

__device__ __forceinline__ float butterfly(float acc) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, o));
  return acc;
}

template <lrmoe_dtype DT>
__device__ __forceinline__ float dot_vec(float acc, const uint4& a, const uint4& b) {
  if constexpr (DT == LRMOE_BF16) {
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = __fadd_rn(acc, __fmul_rn(bf16_bits_to_f32(wa[i] & 0xffffu),
                                     bf16_bits_to_f32(wb[i] & 0xffffu)));
      acc = __fadd_rn(acc, __fmul_rn(bf16_bits_to_f32(wa[i] >> 16), bf16_bits_to_f32(wb[i] >> 16)));
    }
  } else {
    acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(a.x), __uint_as_float(b.x)));
    acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(a.y), __uint_as_float(b.y)));
    acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(a.z), __uint_as_float(b.z)));
    acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(a.w), __uint_as_float(b.w)));
  }
  return acc;
}

// Squared norms of rows [0, nrows) (nrows <= RPW) of V vectors each, row stride V.
// Chunks of 32*VL vectors per row; all RPW*VL loads of a chunk are issued first.
template <lrmoe_dtype DT, int VL, int RPW>
__device__ __forceinline__ void warp_row_norms(const uint4* __restrict__ base, int V, int nrows,
                                               int lane, float (&nrm)[RPW]) {
  float acc[RPW];
#pragma unroll
  for (int i = 0; i < RPW; ++i) acc[i] = 0.0f;
  for (int c0 = 0; c0 < V; c0 += 32 * VL) {
    uint4 v[RPW][VL];
#pragma unroll
    for (int i = 0; i < RPW; ++i)
#pragma unroll
      for (int j = 0; j < VL; ++j) {
        const int c = c0 + lane + 32 * j;
        v[i][j] = (i < nrows && c < V) ? __ldg(base + (size_t)i * V + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
    for (int i = 0; i < RPW; ++i)
#pragma unroll
      for (int j = 0; j < VL; ++j)
        if (c0 + lane + 32 * j < V) acc[i] = acc_vec<DT>(acc[i], v[i][j]);
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) nrm[i] = butterfly(acc[i]);
}

// RPW keeps RPW*VL <= 24 live vectors per lane.
template <int VL>
constexpr int rpw_of() {
  return 24 / VL < 8 ? 24 / VL : 8;
}

// Grid: enough 8-warp blocks for the work, at most what is resident at once.
// The occupancy is looked up once per kernel (the template argument) and device.
template <auto Kern>
int grid_for(long long warps_needed) {
  static std::atomic<int> per_sm[64];  // resident 256-thread blocks per SM; 0 = not known yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  int occ = dev >= 0 ? per_sm[dev].load(std::memory_order_relaxed) : 0;
  if (occ == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kern, 256, 0) != cudaSuccess || n < 1)
      n = 1;
    occ = n;
    if (dev >= 0) per_sm[dev].store(n, std::memory_order_relaxed);
  }
  const long long need = (warps_needed + 7) / 8;
  const long long cap = (long long)num_sms() * occ;
  return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

// Vectors per lane per chunk for rows of V vectors: 1, 2, 3, 4, 6 or 8.
template <lrmoe_dtype DT, template <lrmoe_dtype, int> class F, typename... Args>
cudaError_t by_vl(int V, Args... args) {
  if (V <= 32) return F<DT, 1>::run(args...);
  if (V <= 64) return F<DT, 2>::run(args...);
  if (V <= 96) return F<DT, 3>::run(args...);
  if (V <= 128) return F<DT, 4>::run(args...);
  if (V <= 192) return F<DT, 6>::run(args...);
  return F<DT, 8>::run(args...);
}

}  // namespace rowred
}  // namespace lrmoe
