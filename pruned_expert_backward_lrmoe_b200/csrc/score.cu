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

// Vectors a lane keeps in registers per row chunk (rows longer than 32 * kMaxV
// vectors are processed chunk by chunk, which keeps the same order).
constexpr int kMaxV = 8;

// Load this lane's vectors c = base + lane + 32 i (i < kMaxV) of a row.
__device__ __forceinline__ void load_chunk(uint4 (&v)[kMaxV], const uint4* __restrict__ row,
                                           int base, int V, int lane) {
#pragma unroll
  for (int i = 0; i < kMaxV; ++i) {
    const int c = base + lane + 32 * i;
    v[i] = c < V ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
  }
}

// Accumulate a loaded chunk in ascending vector order (padding vectors are zero).
template <lrmoe_dtype DT>
__device__ __forceinline__ float acc_chunk(float acc, const uint4 (&v)[kMaxV], int base, int V,
                                           int lane) {
#pragma unroll
  for (int i = 0; i < kMaxV; ++i)
    if (base + lane + 32 * i < V) acc = acc_vec<DT>(acc, v[i]);
  return acc;
}

__device__ __forceinline__ float butterfly(float acc) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, o));
  return acc;
}

// Squared norm of a row whose first chunk is already in `v`.
template <lrmoe_dtype DT>
__device__ __forceinline__ float row_sqnorm_from(uint4 (&v)[kMaxV],
                                                 const uint4* __restrict__ row, int V, int lane) {
  float acc = acc_chunk<DT>(0.0f, v, 0, V, lane);
  for (int base = 32 * kMaxV; base < V; base += 32 * kMaxV) {
    load_chunk(v, row, base, V, lane);
    acc = acc_chunk<DT>(acc, v, base, V, lane);
  }
  return butterfly(acc);
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
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
       t += gridDim.x * warps_per_block) {
    // routing slots of this token: lane j holds slot j (k <= 32)
    const size_t p0 = (size_t)t * k;
    const int e_l = lane < k ? __ldg(idx + p0 + lane) : -1;
    const float w_l = lane < k ? __ldg(w + p0 + lane) : 0.0f;
    const unsigned routed = __ballot_sync(kFull, lane < k && e_l >= 0 && e_l < E);
    if (__any_sync(kFull, lane < k && e_l >= E) && lane == 0)
      raise_status(status, LRMOE_ST_BAD_EXPERT);

    uint4 vy[kMaxV], va[kMaxV], vn[kMaxV];
    load_chunk(vy, dY + (size_t)t * VH, 0, VH, lane);
    int j = routed ? __ffs(routed) - 1 : -1;
    if (j >= 0) load_chunk(va, a + (p0 + j) * VD, 0, VD, lane);
    const float ny = row_sqnorm_from<DT>(vy, dY + (size_t)t * VH, VH, lane);

    float s_mine = 0.0f;  // lane j ends up holding slot j's score
    unsigned todo = routed;
    while (todo) {
      j = __ffs(todo) - 1;
      todo &= todo - 1;
      const int jn = todo ? __ffs(todo) - 1 : -1;
      if (jn >= 0) load_chunk(vn, a + (p0 + jn) * VD, 0, VD, lane);  // next row in flight
      const float na = row_sqnorm_from<DT>(va, a + (p0 + j) * VD, VD, lane);
      const float wp = __shfl_sync(kFull, w_l, j);
      float s = __fmul_rn(__fmul_rn(__fmul_rn(wp, wp), ny), na);
      if (!isfinite(s)) {
        if (lane == 0) raise_status(status, LRMOE_ST_NONFINITE);
        if (isnan(s)) s = __uint_as_float(0x7fffffffu);
      }
      if (lane == j) s_mine = s;
      if (jn >= 0) {
#pragma unroll
        for (int i = 0; i < kMaxV; ++i) va[i] = vn[i];
      }
    }
    if (lane < k) score[p0 + lane] = s_mine;
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
  auto kern = dt == LRMOE_BF16 ? score_kernel<LRMOE_BF16> : score_kernel<LRMOE_F32>;
  return launch_pdl(kern, dim3(blocks), dim3(threads), 0, s, idx, w, T, k, E,
                    static_cast<const uint4*>(dY), VH, static_cast<const uint4*>(a), VD, score,
                    status);
}

}  // namespace lrmoe
