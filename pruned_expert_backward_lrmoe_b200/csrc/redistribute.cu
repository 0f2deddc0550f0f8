// Integer redistribution of retained pairs over expert copies, and the split of
// the packed rows by destination GPU.
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 4:
// the remaining pairs are spread over the admissible copies of their expert by
// an integer algorithm whose goal is the smallest peak load on one GPU; no new
// copies appear in the backward.  Bullet 5: the remaining rows are grouped by
// receiver and expert, so the all-to-all moves compact blocks.
//
// Planner (host): binary search on the peak L, each probe one max-flow (Dinic)
// on source -> expert (m_e) -> its copies -> GPU (L) -> sink; L is feasible iff
// the flow saturates every expert.  Integral capacities give an integral plan.
//
// Split (device): expert e's local rows have global indices start_e + i; copy g
// serves the global run [C[e][g], C[e][g+1]) (C = prefix sum of the plan over g).
// One CTA computes the (destination, expert) block sizes and offsets; a second
// kernel places every row.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "grouped.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

struct MaxFlow {
  struct Edge {
    int to;
    long long cap;
  };
  std::vector<Edge> edges;
  std::vector<std::vector<int>> adj;
  std::vector<int> level, it;
  explicit MaxFlow(int n) : adj(n), level(n), it(n) {}
  int add(int u, int v, long long c) {
    adj[u].push_back((int)edges.size());
    edges.push_back({v, c});
    adj[v].push_back((int)edges.size());
    edges.push_back({u, 0});
    return (int)edges.size() - 2;
  }
  bool bfs(int s, int t) {
    std::fill(level.begin(), level.end(), -1);
    std::vector<int> q{s};
    level[s] = 0;
    for (size_t h = 0; h < q.size(); ++h)
      for (int id : adj[q[h]])
        if (edges[id].cap > 0 && level[edges[id].to] < 0) {
          level[edges[id].to] = level[q[h]] + 1;
          q.push_back(edges[id].to);
        }
    return level[t] >= 0;
  }
  long long dfs(int u, int t, long long f) {
    if (u == t) return f;
    for (int& i = it[u]; i < (int)adj[u].size(); ++i) {
      Edge& e = edges[adj[u][i]];
      if (e.cap > 0 && level[e.to] == level[u] + 1) {
        const long long d = dfs(e.to, t, std::min(f, e.cap));
        if (d > 0) {
          e.cap -= d;
          edges[adj[u][i] ^ 1].cap += d;
          return d;
        }
      }
    }
    return 0;
  }
  long long run(int s, int t) {
    long long total = 0;
    while (bfs(s, t)) {
      std::fill(it.begin(), it.end(), 0);
      while (long long f = dfs(s, t, (long long)1 << 62)) total += f;
    }
    return total;
  }
};

// Max-flow at peak L; fills x (row-major [E][G]) when every expert is saturated.
bool plan_at(const int64_t* m, const uint8_t* adm, int E, int G, long long L, int64_t* x) {
  MaxFlow f(E + G + 2);
  const int s = E + G, t = E + G + 1;
  long long need = 0;
  std::vector<int> eid((size_t)E * G, -1);
  for (int e = 0; e < E; ++e) {
    if (m[e] == 0) continue;
    need += m[e];
    f.add(s, e, m[e]);
    for (int g = 0; g < G; ++g)
      if (adm[(size_t)e * G + g]) eid[(size_t)e * G + g] = f.add(e, E + g, m[e]);
  }
  for (int g = 0; g < G; ++g) f.add(E + g, t, L);
  if (f.run(s, t) != need) return false;
  if (x)
    for (size_t i = 0; i < (size_t)E * G; ++i)
      x[i] = eid[i] < 0 ? 0 : f.edges[eid[i] ^ 1].cap;  // reverse capacity = flow
  return true;
}

// Per (destination g, expert e): this rank's rows of e that copy g serves.
__device__ __forceinline__ int run_count(const int32_t* plan, int G, int e, int g, long long a,
                                         long long b) {
  long long lo = 0;
  for (int h = 0; h < g; ++h) lo += plan[(size_t)e * G + h];
  const long long hi = lo + plan[(size_t)e * G + g];
  const long long l = a > lo ? a : lo, r = b < hi ? b : hi;
  return r > l ? (int)(r - l) : 0;
}

// One CTA: block sizes, their offsets, and the coverage check.
__global__ void __launch_bounds__(1024) dest_plan_kernel(
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ plan,
    const int32_t* __restrict__ start, int E, int G, int32_t* __restrict__ dest_offsets,
    int32_t* __restrict__ dest_expert_offsets, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int cnt[];  // [G][E]
  for (int i = threadIdx.x; i < E * G; i += blockDim.x) {
    if (plan[i] < 0) raise_status(status, LRMOE_ST_BAD_INDEX);  // a negative run length
    const int g = i / E, e = i - g * E;
    const long long a = (start ? start[e] : 0), b = a + offsets[e + 1] - offsets[e];
    cnt[i] = run_count(plan, G, e, g, a, b);
  }
  __syncthreads();
  // rows that no copy covers (the plan is too short for this rank's range)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int covered = 0;
    for (int g = 0; g < G; ++g) covered += cnt[g * E + e];
    if (covered != offsets[e + 1] - offsets[e]) raise_status(status, LRMOE_ST_BAD_INDEX);
  }
  if (threadIdx.x == 0) {  // E*G is small: one sequential scan in destination-major order
    int run = 0;
    for (int g = 0; g < G; ++g) {
      dest_offsets[g] = run;
      int inner = 0;
      for (int e = 0; e < E; ++e) {
        dest_expert_offsets[(size_t)g * (E + 1) + e] = inner;
        inner += cnt[g * E + e];
      }
      dest_expert_offsets[(size_t)g * (E + 1) + E] = inner;
      run += inner;
    }
    dest_offsets[G] = run;
  }
}

// Every local packed row to its slot in destination-major order.
__global__ void __launch_bounds__(256) dest_scatter_kernel(
    const int32_t* __restrict__ perm, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ plan, const int32_t* __restrict__ start, int E, int G,
    int rows_cap, const int32_t* __restrict__ dest_offsets,
    const int32_t* __restrict__ dest_expert_offsets, int32_t* __restrict__ perm_dest,
    int32_t* __restrict__ row_dest, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  int M = offsets[E];
  if (M > rows_cap) M = rows_cap;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < M; r += gridDim.x * blockDim.x) {
    int lo = 0, hi = E - 1;  // expert of row r: largest e with offsets[e] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const long long base = start ? start[e] : 0;
    const long long gi = base + (r - offsets[e]);
    long long c = 0;
    for (int g = 0; g < G; ++g) {
      const long long next = c + plan[(size_t)e * G + g];
      if (gi < next) {
        // first global index of this rank's rows inside copy g's run
        const long long first = base > c ? base : c;
        const long long slot = dest_offsets[g] + dest_expert_offsets[(size_t)g * (E + 1) + e] +
                               (gi - first);
        if (slot >= 0 && slot < rows_cap) {
          perm_dest[slot] = perm[r];
          if (row_dest) row_dest[r] = (int32_t)slot;
        } else if (kChecked) {
          raise_status(status, LRMOE_ST_BAD_INDEX);
        }
        break;
      }
      c = next;
    }
  }
}

// Received rows (source-major blocks) regrouped expert-major.  Every CTA builds
// the start of each (expert, source) block in grouped order in shared memory
// (E * G entries, one block-wide scan), then places its share of the rows.
__global__ void __launch_bounds__(1024) group_received_kernel(
    const int32_t* __restrict__ tab /* [G][E+1] */, int G, int E, int rows_cap,
    int32_t* __restrict__ order, int32_t* __restrict__ inv, int32_t* __restrict__ offsets,
    uint32_t* __restrict__ status) {
  extern __shared__ int sm[];  // gstart [E*G] (expert-major), base [G+1], scan scratch [33]
  int* gstart = sm;
  int* base = sm + (size_t)E * G;
  int* scratch = base + G + 1;
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < E * G; i += blockDim.x) {
    const int e = i / G, q = i - e * G;
    const int32_t* row = tab + (size_t)q * (E + 1);
    const int c = row[e + 1] - row[e];
    if (c < 0 && blockIdx.x == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
    gstart[i] = c > 0 ? c : 0;
  }
  __syncthreads();
  const int total = block_scan_inplace(gstart, E * G, scratch);
  if (threadIdx.x == 0) {
    int run = 0;
    for (int q = 0; q < G; ++q) {
      base[q] = run;
      run += tab[(size_t)q * (E + 1) + E];
    }
    base[G] = run;
    if (run != total && blockIdx.x == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = gstart[e * G];
    if (threadIdx.x == 0) offsets[E] = total;
  }
  int R = base[G];
  if (R > rows_cap || R > total) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
    R = min(min(R, rows_cap), total);
  }
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < R; j += gridDim.x * blockDim.x) {
    int lo = 0, hi = G - 1;  // source of row j: largest q with base[q] <= j
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (base[mid] <= j) lo = mid; else hi = mid - 1;
    }
    const int q = lo;
    const int l = j - base[q];
    const int32_t* row = tab + (size_t)q * (E + 1);
    int a = 0, b = E - 1;  // expert: largest e with row[e] <= l
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (row[mid] <= l) a = mid; else b = mid - 1;
    }
    const int i = gstart[a * G + q] + (l - row[a]);
    if (i < 0 || i >= R) {
      raise_status(status, LRMOE_ST_BAD_INDEX);
      continue;
    }
    order[i] = j;
    inv[j] = i;
  }
}

}  // namespace

int redistribute_plan(const int64_t* m, const uint8_t* adm, int E, int G, int64_t* x,
                      int64_t* peak) {
  long long total = 0, lo = 0, hi = 0;
  for (int e = 0; e < E; ++e) {
    total += m[e];
    hi = std::max<long long>(hi, m[e]);
  }
  if (total == 0) {
    std::fill(x, x + (size_t)E * G, 0);
    *peak = 0;
    return 0;
  }
  lo = (total + G - 1) / G;  // nobody can do better than an even split
  hi = std::max(hi, lo);
  // widen hi until feasible: a peak of `total` always is when every loaded
  // expert has a copy
  while (!plan_at(m, adm, E, G, hi, nullptr)) {
    if (hi >= total) return -1;
    hi = std::min(total, hi * 2);
  }
  while (lo < hi) {
    const long long mid = lo + (hi - lo) / 2;
    if (plan_at(m, adm, E, G, mid, nullptr)) hi = mid; else lo = mid + 1;
  }
  plan_at(m, adm, E, G, lo, x);
  *peak = lo;
  return 0;
}

cudaError_t launch_split_by_destination(const int32_t* perm, const int32_t* offsets,
                                        const int32_t* plan, const int32_t* start, int E, int G,
                                        int rows_cap, int32_t* perm_dest, int32_t* dest_offsets,
                                        int32_t* dest_expert_offsets, int32_t* row_dest,
                                        uint32_t* status, cudaStream_t s) {
  const size_t smem = (size_t)E * G * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(dest_plan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_pdl(dest_plan_kernel, dim3(1), dim3(1024), smem, s, offsets, plan, start,
                             E, G, dest_offsets, dest_expert_offsets, status);
  if (e != cudaSuccess) return e;
  const int blocks = num_sms() * 4;
  return launch_pdl(dest_scatter_kernel, dim3(blocks), dim3(256), 0, s, perm, offsets, plan, start,
                    E, G, rows_cap, (const int32_t*)dest_offsets,
                    (const int32_t*)dest_expert_offsets, perm_dest, row_dest, status);
}

cudaError_t launch_group_received(const int32_t* tab, int G, int E, int rows_cap, int32_t* order,
                                  int32_t* inv, int32_t* offsets, uint32_t* status,
                                  cudaStream_t s) {
  const size_t smem = ((size_t)E * G + G + 1 + 33) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(group_received_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int blocks = (rows_cap + 1023) / 1024;
  if (blocks > num_sms()) blocks = num_sms();
  if (blocks < 1) blocks = 1;
  return launch_pdl(group_received_kernel, dim3(blocks), dim3(1024), smem, s, tab, G, E, rows_cap,
                    order, inv, offsets, status);
}

}  // namespace lrmoe
