// a1  LRM score: w^2 * ||dY_t||^2 * ||a_p||^2 per routed pair.
//
// Follows "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE",
// bullet 3: the squared norm of a pair's outer-product contribution factorises,
// so each pair needs two row norms and three multiplies, never the H x I matrix.
//
// One warp per token: it reads dY_t once and the k saved rows a_p, 16 bytes
// per lane per load (HBM-bound: T*H + T*k*I elements + 8 bytes per pair).
// The reduction order is fixed so that the result is bit-reproducible:
// lane l sums vectors l, l+32, ... element by element as fl(acc + fl(x*x)),
// then a butterfly fl(acc[l] + acc[l^o]) for o = 16, 8, 4, 2, 1.
#include "common.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

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

// Squared norm of one row of V 16-byte vectors in the canonical order.
template <lrmoe_dtype DT>
__device__ __forceinline__ float row_sqnorm(const uint4* __restrict__ row, int V, int lane) {
  float acc = 0.0f;
  int c = lane;
  // four vectors in flight per lane, accumulated in ascending order
  for (; c + 96 < V; c += 128) {
    const uint4 v0 = __ldg(row + c);
    const uint4 v1 = __ldg(row + c + 32);
    const uint4 v2 = __ldg(row + c + 64);
    const uint4 v3 = __ldg(row + c + 96);
    acc = acc_vec<DT>(acc, v0);
    acc = acc_vec<DT>(acc, v1);
    acc = acc_vec<DT>(acc, v2);
    acc = acc_vec<DT>(acc, v3);
  }
  for (; c < V; c += 32) acc = acc_vec<DT>(acc, __ldg(row + c));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, o));
  return acc;
}

template <lrmoe_dtype DT>
__global__ void __launch_bounds__(256) score_kernel(const int32_t* __restrict__ idx,
                                                    const float* __restrict__ w, int T, int k,
                                                    int E, const uint4* __restrict__ dY, int VH,
                                                    const uint4* __restrict__ a, int VD,
                                                    float* __restrict__ score,
                                                    uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
       t += gridDim.x * warps_per_block) {
    const float ny = row_sqnorm<DT>(dY + (size_t)t * VH, VH, lane);
    for (int j = 0; j < k; ++j) {
      const size_t p = (size_t)t * k + j;
      const int e = __ldg(idx + p);
      float s = 0.0f;
      if (e >= 0 && e < E) {
        const float na = row_sqnorm<DT>(a + p * VD, VD, lane);
        const float wp = __ldg(w + p);
        s = __fmul_rn(__fmul_rn(__fmul_rn(wp, wp), ny), na);
        if (!isfinite(s)) {
          if (lane == 0) raise_status(status, LRMOE_ST_NONFINITE);
          if (isnan(s)) s = __uint_as_float(0x7fffffffu);
        }
      } else if (e >= E && lane == 0) {
        raise_status(status, LRMOE_ST_BAD_EXPERT);
      }
      if (lane == 0) score[p] = s;
    }
  }
}

}  // namespace

cudaError_t launch_score(const int32_t* idx, const float* w, int T, int k, int E, const void* dY,
                         int H, const void* a, int D, lrmoe_dtype dt, float* score,
                         uint32_t* status, cudaStream_t s) {
  const int per_vec = dt == LRMOE_BF16 ? 8 : 4;
  const int VH = H / per_vec, VD = D / per_vec;
  const int threads = 256, wpb = threads / 32;
  const int blocks_needed = (T + wpb - 1) / wpb;
  const int max_blocks = num_sms() * (2048 / threads);
  const int blocks = blocks_needed < max_blocks ? blocks_needed : max_blocks;
  if (dt == LRMOE_BF16)
    score_kernel<LRMOE_BF16><<<blocks, threads, 0, s>>>(
        idx, w, T, k, E, static_cast<const uint4*>(dY), VH, static_cast<const uint4*>(a), VD,
        score, status);
  else
    score_kernel<LRMOE_F32><<<blocks, threads, 0, s>>>(
        idx, w, T, k, E, static_cast<const uint4*>(dY), VH, static_cast<const uint4*>(a), VD,
        score, status);
  return cudaGetLastError();
}

}  // namespace lrmoe
