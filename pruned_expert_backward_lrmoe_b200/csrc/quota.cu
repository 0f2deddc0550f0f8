// Quota controller (before the backward).
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 2:
// before the backward a controller sees how many tokens came to each expert and,
// within the memory limit, decides how many pairs of each expert stay; the quota
// is fixed for the whole layer call.  Reading used here (water-filling):
//   q_e = min(c_e, cap, tau),  tau = the largest integer level with sum_e q_e <= budget,
// so the most loaded experts lose pairs first.  cap <= 0: no per-expert cap;
// budget < 0: no budget.  Everything stays on the device (no host round trip).
//
// One CTA: expert histogram in shared memory (16-byte loads, eight in flight per
// thread), then a binary search over tau with block reductions.
#include "common.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

constexpr int kQuotaThreads = 1024;

__device__ long long block_sum_ll(long long v, long long* ws) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (lane == 0) ws[wid] = v;
  __syncthreads();
  long long t = 0;
  if (wid == 0) {
    t = lane < nw ? ws[lane] : 0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
    if (lane == 0) ws[32] = t;
  }
  __syncthreads();
  t = ws[32];
  __syncthreads();
  return t;
}

__global__ void __launch_bounds__(kQuotaThreads) quota_kernel(const int32_t* __restrict__ idx, int P,
                                                              int E, int cap, long long budget,
                                                              int32_t* __restrict__ quota,
                                                              int32_t* __restrict__ counts,
                                                              uint32_t* __restrict__ status) {
  extern __shared__ int hist[];  // [E]
  __shared__ long long ws[33];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  bool bad = false;
  const int P4 = P & ~3;
  for (int base = 4 * threadIdx.x; base < P4; base += 4 * 8 * blockDim.x) {
    int4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int p = base + u * 4 * blockDim.x;
      v[u] = p < P4 ? __ldg(reinterpret_cast<const int4*>(idx + p)) : make_int4(-1, -1, -1, -1);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int ev[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (ev[i] >= 0 && ev[i] < E) atomicAdd(&hist[ev[i]], 1);
        bad |= ev[i] >= E;
      }
    }
  }
  for (int p = P4 + threadIdx.x; p < P; p += blockDim.x) {
    const int e = __ldg(idx + p);
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    bad |= e >= E;
  }
  if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) raise_status(status, LRMOE_ST_BAD_EXPERT);
  __syncthreads();

  // per-expert cap, then the largest level tau whose total fits the budget
  long long total = 0;
  int cmax = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = hist[e];
    const int cc = cap > 0 ? min(c, cap) : c;
    total += cc;
    cmax = max(cmax, cc);
  }
  total = block_sum_ll(total, ws);
  __shared__ int smax;  // largest capped count: the top of the search range for tau
  if (threadIdx.x == 0) smax = 0;
  __syncthreads();
  atomicMax(&smax, cmax);
  __syncthreads();
  int tau = smax;  // no budget cut: every expert keeps min(c, cap)
  if (budget >= 0 && total > budget) {
    int lo = 0, hi = smax;  // sum(level lo) <= budget < sum(level hi)
    while (hi - lo > 1) {
      const int mid = lo + (hi - lo) / 2;
      long long s = 0;
      for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int c = hist[e];
        s += min(cap > 0 ? min(c, cap) : c, mid);
      }
      s = block_sum_ll(s, ws);
      if (s <= budget) lo = mid; else hi = mid;
    }
    tau = lo;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = hist[e];
    const int cc = cap > 0 ? min(c, cap) : c;
    counts[e] = c;
    quota[e] = min(cc, tau);
  }
}

}  // namespace

cudaError_t launch_quota(const int32_t* idx, int P, int E, int cap, long long budget,
                         int32_t* quota, int32_t* counts, uint32_t* status, cudaStream_t s) {
  return launch_pdl(quota_kernel, dim3(1), dim3(kQuotaThreads), (size_t)E * 4, s, idx, P, E, cap,
                    budget, quota, counts, status);
}

}  // namespace lrmoe
