// a1  LRM score: w^2 * ||dY_t||^2 * ||a_p||^2 per routed pair.
//
// Follows "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE",
// bullet 3: the squared norm of a pair's outer-product contribution factorises,
// so each pair needs two row norms and three multiplies, never the H x I matrix.
//
// Three HBM-bound kernels:
//   score_fused       lrmoe_score: per token ||dY_t||^2, then its k rows' ||a_p||^2,
//                     then w^2 * ||dY_t||^2 * ||a_p||^2 per slot, in one pass;
//   row_sqnorm        ||row||^2 of every row of a matrix (the forward can save
//                     ||a_p||^2 with it while it owns a);
//   score_from_norms  ||dY_t||^2 per token, then the product with a saved ||a_p||^2,
//                     so that a is not read at all.
// Every row norm takes the same order whichever kernel computes it, so the two
// routes give the same bits.
//
// A warp reduces RPW rows at once with every 16-byte load of a row chunk in
// flight together.  The order is fixed so that results are bit-reproducible:
// lane l sums vectors l, l+32, ... element by element as fl(acc + fl(x*x)),
// then a butterfly fl(acc[l] + acc[l^o]) for o = 16, 8, 4, 2, 1.
#include "common.cuh"
#include "launch.h"
#include "rowreduce.cuh"

namespace lrmoe {
namespace {

using namespace rowred;

template <lrmoe_dtype DT, int VL, int RPW>
__global__ void __launch_bounds__(256) row_sqnorm_kernel(const uint4* __restrict__ rows, int n,
                                                         int V, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  for (long long r0 = (long long)gw * RPW; r0 < n; r0 += (long long)nw * RPW) {
    const int here = (int)(n - r0 < RPW ? n - r0 : RPW);
    float nrm[RPW];
    warp_row_norms<DT, VL, RPW>(rows + r0 * V, V, here, lane, nrm);
    float mine = 0.0f;
#pragma unroll
    for (int i = 0; i < RPW; ++i)
      if (lane == i) mine = nrm[i];
    if (lane < here) out[r0 + lane] = mine;
  }
}

// score[p] = fl(fl(fl(w*w) * ||dY_t||^2) * na[p]) for routed slots, +0 otherwise.
// `na` may be the score buffer itself: each slot is read before it is written,
// by the same thread.
template <lrmoe_dtype DT, int VL, int RPW>
__global__ void __launch_bounds__(256) score_norms_kernel(const int32_t* __restrict__ idx,
                                                          const float* __restrict__ w, int T,
                                                          int k, int E,
                                                          const uint4* __restrict__ dY, int VH,
                                                          const float* na, float* score,
                                                          uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  for (long long t0 = (long long)gw * RPW; t0 < T; t0 += (long long)nw * RPW) {
    const int here = (int)(T - t0 < RPW ? T - t0 : RPW);
    // routing slots of the RPW tokens (lane j holds slot j, k <= 32), in flight
    // together with the dY rows
    int e_l[RPW];
    float w_l[RPW], a_l[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const bool ok = i < here && lane < k;
      const size_t p = (size_t)(t0 + i) * k + lane;
      e_l[i] = ok ? __ldg(idx + p) : -1;
      w_l[i] = ok ? __ldg(w + p) : 0.0f;
      a_l[i] = ok ? na[p] : 0.0f;
    }
    float ny[RPW];
    warp_row_norms<DT, VL, RPW>(dY + t0 * VH, VH, here, lane, ny);
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      if (i >= here) break;
      if (__any_sync(kFull, lane < k && e_l[i] >= E) && lane == 0)
        raise_status(status, LRMOE_ST_BAD_EXPERT);
      const bool routed = lane < k && e_l[i] >= 0 && e_l[i] < E;
      float s = 0.0f;
      if (routed) {
        s = __fmul_rn(__fmul_rn(__fmul_rn(w_l[i], w_l[i]), ny[i]), a_l[i]);
        if (!isfinite(s)) {
          raise_status(status, LRMOE_ST_NONFINITE);
          if (isnan(s)) s = __uint_as_float(0x7fffffffu);
        }
      }
      if (lane < k) score[(size_t)(t0 + i) * k + lane] = s;
    }
  }
}

// One warp per token: ||dY_t||^2 (8 vectors per lane per chunk), then the token's
// k saved rows a_p, RA at a time (RA * VLI <= 24 vectors per lane in flight),
// lane j keeping ||a_{t,j}||^2; then the product as in score_norms_kernel.
template <lrmoe_dtype DT, int VLI, int RA>
__global__ void __launch_bounds__(256) score_fused_kernel(const int32_t* __restrict__ idx,
                                                          const float* __restrict__ w, int T,
                                                          int k, int E,
                                                          const uint4* __restrict__ dY, int VH,
                                                          const uint4* __restrict__ a, int VI,
                                                          float* __restrict__ score,
                                                          uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  for (long long t = gw; t < T; t += nw) {
    const bool slot = lane < k;
    const size_t p = (size_t)t * k + lane;
    const int e = slot ? __ldg(idx + p) : -1;
    const float wv = slot ? __ldg(w + p) : 0.0f;
    float ny[1];
    warp_row_norms<DT, 8, 1>(dY + t * VH, VH, 1, lane, ny);
    float na = 0.0f;
    for (int j0 = 0; j0 < k; j0 += RA) {
      const int here = k - j0 < RA ? k - j0 : RA;
      float nrm[RA];
      warp_row_norms<DT, VLI, RA>(a + ((size_t)t * k + j0) * VI, VI, here, lane, nrm);
#pragma unroll
      for (int i = 0; i < RA; ++i)
        if (lane == j0 + i) na = nrm[i];
    }
    if (__any_sync(kFull, slot && e >= E) && lane == 0) raise_status(status, LRMOE_ST_BAD_EXPERT);
    float sc = 0.0f;
    if (slot && e >= 0 && e < E) {
      sc = __fmul_rn(__fmul_rn(__fmul_rn(wv, wv), ny[0]), na);
      if (!isfinite(sc)) {
        raise_status(status, LRMOE_ST_NONFINITE);
        if (isnan(sc)) sc = __uint_as_float(0x7fffffffu);
      }
    }
    if (slot) score[p] = sc;
  }
}

template <lrmoe_dtype DT, int VLI>
struct FusedF {
  static cudaError_t run(const int32_t* idx, const float* w, int T, int k, int E, const void* dY,
                         int VH, const void* a, int VI, float* score, uint32_t* status,
                         cudaStream_t s) {
    constexpr int RA = rpw_of<VLI>();
    constexpr auto kern = score_fused_kernel<DT, VLI, RA>;
    const int grid = grid_for<kern>(T);
    return launch_pdl(kern, dim3(grid), dim3(256), 0, s, idx, w, T, k, E,
                      static_cast<const uint4*>(dY), VH, static_cast<const uint4*>(a), VI, score,
                      status);
  }
};

template <lrmoe_dtype DT, int VL>
struct NormsF {
  static cudaError_t run(const void* rows, int n, int V, float* out, cudaStream_t s) {
    constexpr int RPW = rpw_of<VL>();
    constexpr auto kern = row_sqnorm_kernel<DT, VL, RPW>;
    const int grid = grid_for<kern>(((long long)n + RPW - 1) / RPW);
    return launch_pdl(kern, dim3(grid), dim3(256), 0, s, static_cast<const uint4*>(rows), n, V,
                      out);
  }
};

template <lrmoe_dtype DT, int VL>
struct ScoreF {
  static cudaError_t run(const int32_t* idx, const float* w, int T, int k, int E, const void* dY,
                         int VH, const float* na, float* score, uint32_t* status, cudaStream_t s) {
    constexpr int RPW = rpw_of<VL>();
    constexpr auto kern = score_norms_kernel<DT, VL, RPW>;
    const int grid = grid_for<kern>(((long long)T + RPW - 1) / RPW);
    return launch_pdl(kern, dim3(grid), dim3(256), 0, s, idx, w, T, k, E,
                      static_cast<const uint4*>(dY), VH, na, score, status);
  }
};

}  // namespace

cudaError_t launch_row_sqnorm(const void* rows, int n, int D, lrmoe_dtype dt, float* out,
                              cudaStream_t s) {
  const int V = D / (dt == LRMOE_BF16 ? 8 : 4);
  if (dt == LRMOE_BF16) return by_vl<LRMOE_BF16, NormsF>(V, rows, n, V, out, s);
  return by_vl<LRMOE_F32, NormsF>(V, rows, n, V, out, s);
}

cudaError_t launch_score_from_norms(const int32_t* idx, const float* w, int T, int k, int E,
                                    const void* dY, int H, const float* a_sqnorm, lrmoe_dtype dt,
                                    float* score, uint32_t* status, cudaStream_t s) {
  const int VH = H / (dt == LRMOE_BF16 ? 8 : 4);
  if (dt == LRMOE_BF16)
    return by_vl<LRMOE_BF16, ScoreF>(VH, idx, w, T, k, E, dY, VH, a_sqnorm, score, status, s);
  return by_vl<LRMOE_F32, ScoreF>(VH, idx, w, T, k, E, dY, VH, a_sqnorm, score, status, s);
}

cudaError_t launch_score(const int32_t* idx, const float* w, int T, int k, int E, const void* dY,
                         int H, const void* a, int D, lrmoe_dtype dt, float* score,
                         uint32_t* status, cudaStream_t s) {
  const int per = dt == LRMOE_BF16 ? 8 : 4;
  const int VH = H / per, VI = D / per;
  if (dt == LRMOE_BF16)
    return by_vl<LRMOE_BF16, FusedF>(VI, idx, w, T, k, E, dY, VH, a, VI, score, status, s);
  return by_vl<LRMOE_F32, FusedF>(VI, idx, w, T, k, E, dY, VH, a, VI, score, status, s);
}

}  // namespace lrmoe
