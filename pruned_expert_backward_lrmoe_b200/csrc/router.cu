// Routing-weight gradient dL/dw_p = <dY_t, y_p> (y_p = W_down[e] a_p, the pair's
// expert output saved by the forward; the layer output is sum_j w_tj y_tj).
//
// The pages ("LRMoE урезает обратный проход MoE ...", section "Что делает
// LRMoE") prune only the expert weight-gradient contributions and say nothing of
// the router; this kernel serves either reading: every routed pair, or (given
// pos) the retained pairs only, dropped pairs getting 0.
//
// HBM-bound: the saved y rows of the pairs it computes (P*H or M*H elements)
// plus dY (T*H, re-read from L1/L2 by the token's k pairs).  All loads of RPW
// pairs' row chunks are in flight together; the dot uses the canonical order of
// the score (lane partials, fl(acc + fl(x*y)), butterfly).
#include "common.cuh"
#include "launch.h"
#include "rowreduce.cuh"

namespace lrmoe {
namespace {

using namespace rowred;

// A warp takes windows of 32 consecutive pairs (lane i owns pair p0 + i), ballots
// the pairs to compute and walks only those, RPW at a time, so dropped pairs cost
// no loads.
template <lrmoe_dtype DT, int VL, int RPW>
__global__ void __launch_bounds__(256) router_grad_kernel(
    const int32_t* __restrict__ idx, int P, int k, int E, const uint4* __restrict__ dY, int VH,
    const uint4* __restrict__ y, const int32_t* __restrict__ pos, float* __restrict__ dw,
    uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  for (long long p0 = (long long)gw * 32; p0 < P; p0 += (long long)nw * 32) {
    const long long pl = p0 + lane;
    bool want = false;
    if (pl < P) {
      const int e = __ldg(idx + pl);
      if (e >= E) raise_status(status, LRMOE_ST_BAD_EXPERT);
      want = e >= 0 && e < E && (pos == nullptr || __ldg(pos + pl) >= 0);
    }
    unsigned todo = __ballot_sync(kFull, want);
    float res = 0.0f;  // this lane's pair
    while (todo) {
      int q[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        q[i] = todo ? __ffs(todo) - 1 : -1;
        if (todo) todo &= todo - 1;
      }
      float acc[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) acc[i] = 0.0f;
      for (int c0 = 0; c0 < VH; c0 += 32 * VL) {
        uint4 va[RPW][VL], vb[RPW][VL];
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const long long p = p0 + (q[i] >= 0 ? q[i] : 0);
          const uint4* yr = y + p * VH;
          const uint4* dr = dY + (p / k) * VH;
#pragma unroll
          for (int j = 0; j < VL; ++j) {
            const int c = c0 + lane + 32 * j;
            const bool ok = q[i] >= 0 && c < VH;
            va[i][j] = ok ? __ldg(dr + c) : make_uint4(0, 0, 0, 0);
            vb[i][j] = ok ? __ldg(yr + c) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int i = 0; i < RPW; ++i)
#pragma unroll
          for (int j = 0; j < VL; ++j)
            if (c0 + lane + 32 * j < VH) acc[i] = dot_vec<DT>(acc[i], va[i][j], vb[i][j]);
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const float d = butterfly(acc[i]);
        if (lane == q[i]) res = d;
      }
    }
    if (pl < P) dw[pl] = res;
  }
}

template <lrmoe_dtype DT, int VL>
struct RouterF {
  static cudaError_t run(const int32_t* idx, int P, int k, int E, const void* dY, int VH,
                         const void* y, const int32_t* pos, float* dw, uint32_t* status,
                         cudaStream_t s) {
    // two rows (dY, y) per pair in flight: RPW*VL*2 <= 24 vectors per lane
    constexpr int RPW = rpw_of<2 * VL>();
    constexpr auto kern = router_grad_kernel<DT, VL, RPW>;
    const int grid = grid_for<kern>(((long long)P + 31) / 32);
    return launch_pdl(kern, dim3(grid), dim3(256), 0, s, idx, P, k, E,
                      static_cast<const uint4*>(dY), VH, static_cast<const uint4*>(y), pos, dw,
                      status);
  }
};

}  // namespace

cudaError_t launch_router_grad(const int32_t* idx, int T, int k, int E, const void* dY, int H,
                               const void* y, lrmoe_dtype dt, const int32_t* pos, float* dw,
                               uint32_t* status, cudaStream_t s) {
  const int VH = H / (dt == LRMOE_BF16 ? 8 : 4);
  const int P = T * k;
  if (dt == LRMOE_BF16)
    return by_vl<LRMOE_BF16, RouterF>(VH, idx, P, k, E, dY, VH, y, pos, dw, status, s);
  return by_vl<LRMOE_F32, RouterF>(VH, idx, P, k, E, dY, VH, y, pos, dw, status, s);
}

}  // namespace lrmoe
