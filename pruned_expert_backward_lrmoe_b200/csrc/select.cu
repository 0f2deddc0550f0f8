// a2  Per-expert top-quota selection.
//
// Follows "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE",
// bullets 2-3: the quota of every expert is fixed for the layer call, and
// within it the pairs with the highest score stay.  Key: score bit pattern as
// uint32 descending, then pair index ascending (scores are >= +0, so the bit
// order is the numeric order; NaN sorts above +Inf).
//
// Three kernels, integer work only, deterministic (no order-dependent atomics):
//   1. chunk_count : per chunk of pairs, an expert histogram (+ pos = -1 for
//                    empty/invalid slots)
//   2. chunk_scatter: per expert, the scan over chunks (counts, the segment
//                    starts, m_e = min(max(q_e,0), c_e), offsets), then a stable
//                    counting sort of the chunk's pairs by expert (ascending p
//                    inside each expert) into seg_p / seg_key
//   3. expert_topk : one CTA per expert: 3-pass (11, 11, 10-bit) radix select
//                    of the m_e-th largest key, then an ordered compaction that
//                    keeps keys above the threshold and the first (m_e - #above)
//                    equal keys in ascending p; writes perm and pos.
#include "common.cuh"
#include "grouped.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

constexpr int kCountThreads = 256;
constexpr int kScatterWarps = 8;
constexpr int kTopkThreads = 1024;
constexpr int kScanSmemInts = 32768;  // bound on E * nchunks (every scatter CTA reads it all)
constexpr int kTopkSmemKeys = 53248;  // segments up to this length are staged in smem (keys)

__global__ void __launch_bounds__(kCountThreads) chunk_count(const int32_t* __restrict__ idx,
                                                              int P, int E, int chunk,
                                                              int nchunks, int32_t* __restrict__ cc,
                                                              int32_t* __restrict__ pos,
                                                              uint32_t* __restrict__ status) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x;
  const int begin = c * chunk;
  const int end = min(P, begin + chunk);
  bool bad = false;
  // four consecutive pairs per thread and pass, one 16-byte load when in range
  for (int p0 = begin + 4 * threadIdx.x; p0 < end; p0 += 4 * blockDim.x) {
    int ev[4];
    if (p0 + 3 < end) {
      const int4 v = __ldg(reinterpret_cast<const int4*>(idx + p0));
      ev[0] = v.x, ev[1] = v.y, ev[2] = v.z, ev[3] = v.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) ev[i] = p0 + i < end ? __ldg(idx + p0 + i) : -1;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = ev[i];
      if (p0 + i >= end) break;
      if (e >= 0 && e < E) {
        atomicAdd(&hist[e], 1);
      } else {
        pos[p0 + i] = -1;
        bad |= (e >= E);
      }
    }
  }
  if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) raise_status(status, LRMOE_ST_BAD_EXPERT);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cc[(size_t)e * nchunks + c] = hist[e];
}

// Stable counting sort of the pairs by expert, with the scan over chunks folded
// in.  CTA c handles chunk c.  First every CTA reads the whole per-(expert,
// chunk) count matrix (one warp per expert, 32 chunks per load): the expert's
// total and the count of the chunks before c.  An exclusive scan of the totals
// gives the segment starts; CTA 0 also writes counts, kept (m_e = min(max(q_e,
// 0), c_e)), offsets (scan of kept) and seg_start.  Then the chunk's pairs are
// placed in ascending pair order (per-warp ranks by match_any).
__global__ void __launch_bounds__(kScatterWarps * 32) chunk_scatter(
    const int32_t* __restrict__ idx, const uint32_t* __restrict__ score_bits, int P, int E,
    int chunk, int nchunks, const int32_t* __restrict__ cc, const int32_t* __restrict__ quota,
    int32_t* __restrict__ counts, int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
    int32_t* __restrict__ seg_start, int32_t* __restrict__ seg_p, uint32_t* __restrict__ seg_key,
    uint32_t* __restrict__ status) {
  extern __shared__ int sm_sc[];  // wbase [kScatterWarps][E], tot [E], pre [E], scratch [33]
  int* wbase = sm_sc;
  int* tot = wbase + kScatterWarps * E;
  int* pre = tot + E;
  int* scratch = pre + E;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int c = blockIdx.x;
  const int begin = c * chunk;
  const int end = min(P, begin + chunk);
  const int sub = (chunk + kScatterWarps - 1) / kScatterWarps;
  const int wbeg = min(end, begin + wid * sub);
  const int wend = min(end, wbeg + sub);
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) wbase[i] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  // per expert: total over chunks and the part before this chunk.  A warp takes
  // kExpertsInFlight experts at a time with all their loads in flight (one
  // round trip per group instead of one per expert).
  constexpr int kExpertsInFlight = 8;
  for (int e0 = wid * kExpertsInFlight; e0 < E; e0 += kScatterWarps * kExpertsInFlight) {
    int t_all[kExpertsInFlight], t_pre[kExpertsInFlight];
#pragma unroll
    for (int u = 0; u < kExpertsInFlight; ++u) t_all[u] = t_pre[u] = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 32) {
      const int ci = c0 + lane;
      int v[kExpertsInFlight];
#pragma unroll
      for (int u = 0; u < kExpertsInFlight; ++u) {
        const int e = e0 + u;
        v[u] = (e < E && ci < nchunks) ? __ldcg(cc + (size_t)e * nchunks + ci) : 0;
      }
#pragma unroll
      for (int u = 0; u < kExpertsInFlight; ++u) {
        t_all[u] += __reduce_add_sync(kFull, v[u]);
        t_pre[u] += __reduce_add_sync(kFull, ci < c ? v[u] : 0);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < kExpertsInFlight; ++u)
        if (e0 + u < E) {
          tot[e0 + u] = t_all[u];
          pre[e0 + u] = t_pre[u];
        }
    }
  }
  __syncthreads();
  if (c == 0) {
    bool badq = false;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const int q = quota[e];
      badq |= q < 0;
      const int m = min(max(q, 0), tot[e]);
      counts[e] = tot[e];
      kept[e] = m;
      wbase[e] = m;  // scratch for the scan of kept (wbase is rebuilt below)
    }
    if (__any_sync(kFull, badq) && lane == 0) raise_status(status, LRMOE_ST_BAD_QUOTA);
    __syncthreads();
    const int ktot = block_scan_inplace(wbase, E, scratch);
    for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = wbase[e];
    if (threadIdx.x == 0) offsets[E] = ktot;
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) wbase[i] = 0;
  }
  // segment starts: exclusive scan of the totals (tot becomes the start)
  const int ctot = block_scan_inplace(tot, E, scratch);
  if (c == 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) seg_start[e] = tot[e];
    if (threadIdx.x == 0) seg_start[E] = ctot;
  }
  int* mine = wbase + wid * E;
  constexpr int kSteps = 4;  // 32-pair steps whose loads are in flight together
  for (int q0 = wbeg; q0 < wend; q0 += 32 * kSteps) {
    int ev[kSteps];
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
      const int p = q0 + 32 * s + lane;
      ev[s] = p < wend ? __ldg(idx + p) : -1;
    }
#pragma unroll
    for (int s = 0; s < kSteps; ++s)
      if (ev[s] >= 0 && ev[s] < E) atomicAdd(&mine[ev[s]], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = tot[e] + pre[e];
#pragma unroll
    for (int w = 0; w < kScatterWarps; ++w) {
      const int v = wbase[w * E + e];
      wbase[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int q0 = wbeg; q0 < wend; q0 += 32 * kSteps) {
    int ev[kSteps];
    uint32_t sv[kSteps];
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
      const int p = q0 + 32 * s + lane;
      ev[s] = p < wend ? __ldg(idx + p) : -1;
      sv[s] = p < wend ? __ldg(score_bits + p) : 0u;
    }
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {  // steps in ascending pair order
      const int p = q0 + 32 * s + lane;
      const int e = ev[s];
      const bool valid = e >= 0 && e < E;
      const unsigned m = __match_any_sync(kFull, valid ? e : -1);
      int base = 0;
      if (valid) {
        base = mine[e];
        const int dst = base + __popc(m & lt);
        if (idx_ok(dst, P, status)) {
          seg_p[dst] = p;
          seg_key[dst] = sv[s];
        }
      }
      __syncwarp();
      if (valid && lane == __ffs(m) - 1) mine[e] = base + __popc(m);
      __syncwarp();
    }
  }
}

// Digits of the radix select, most significant first: 11 + 11 + 10 bits.
__device__ __forceinline__ int digit_shift(int d) { return d == 0 ? 21 : (d == 1 ? 10 : 0); }
__device__ __forceinline__ int digit_bins(int d) { return d == 2 ? 1024 : 2048; }

// One CTA per expert.  The expert's keys (its segment of seg_key, pairs in
// ascending p) are staged in shared memory when they fit.  A 3-pass radix
// select (11, 11, 10 bits) finds tau, the m-th largest key, and how many keys
// equal to tau stay (the first ones in segment order, i.e. ascending p).  The
// compaction is warp-contiguous: warp w owns a contiguous run of the segment,
// walked 32 keys at a time; ballots give each kept key its rank inside the step,
// one block scan of the warps' (above, equal) counts gives each warp's start.
__global__ void __launch_bounds__(kTopkThreads) expert_topk(
    const int32_t* __restrict__ counts, const int32_t* __restrict__ kept,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ seg_start,
    const int32_t* __restrict__ seg_p, const uint32_t* __restrict__ seg_key,
    int32_t* __restrict__ perm, int32_t* __restrict__ pos, int P, uint32_t* __restrict__ status) {
  extern __shared__ uint32_t sm_keys[];  // [kTopkSmemKeys]
  __shared__ int hist[2048];
  __shared__ int warp_gt[kTopkThreads / 32], warp_eq[kTopkThreads / 32];
  __shared__ int warp_sum[kTopkThreads / 32];
  __shared__ int found_bin, found_above;
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const int c = counts[e];
  const int m = kept[e];
  const int s0 = seg_start[e];
  const int out0 = offsets[e];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nt = blockDim.x, nw = nt >> 5;
  const int32_t* sp = seg_p + s0;
  const uint32_t* sk = seg_key + s0;
  if (kChecked && !(c >= 0 && m >= 0 && m <= c && idx_ok(s0, P - c + 1, status) &&
                    idx_ok(out0, P - m + 1, status))) {
    if (tid == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
    return;
  }

  if (m == c) {  // everything stays, already in ascending p
    for (int i = tid; i < c; i += nt) {
      const int p = sp[i];
      perm[out0 + i] = p;
      if (idx_ok(p, P, status)) pos[p] = out0 + i;
    }
    return;
  }
  if (m == 0) {
    for (int i = tid; i < c; i += nt)
      if (idx_ok(sp[i], P, status)) pos[sp[i]] = -1;
    return;
  }

  // stage the keys (eight loads in flight per thread)
  const bool in_smem = c <= kTopkSmemKeys;
  const uint32_t* K = sk;
  if (in_smem) {
    for (int i0 = 0; i0 < c; i0 += 8 * nt) {
      uint32_t kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nt + tid;
        kv[u] = i < c ? __ldcg(sk + i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nt + tid;
        if (i < c) sm_keys[i] = kv[u];
      }
    }
    K = sm_keys;
  }
  __syncthreads();

  // radix select of the m-th largest key
  uint32_t prefix = 0, pmask = 0;
  int need = m;
  for (int d = 0; d < 3; ++d) {
    const int shift = digit_shift(d), nb = digit_bins(d);
    for (int i = tid; i < nb; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < c; i0 += nt) {
      const int i = i0 + tid;
      int digit = -1;
      if (i < c) {
        const uint32_t key = K[i];
        if ((key & pmask) == prefix) digit = (int)((key >> shift) & (uint32_t)(nb - 1));
      }
      if (__any_sync(kFull, digit >= 0)) {  // later passes: most warps hold no candidate
        const unsigned grp = __match_any_sync(kFull, digit);
        if (digit >= 0 && lane == __ffs(grp) - 1) atomicAdd(&hist[digit], __popc(grp));
      }
    }
    __syncthreads();
    {
      // thread t owns the nb/1024 bins just below nb - 1 - t*nb/1024 (descending
      // key order); one block-wide scan of the per-thread sums finds the bin
      const int per = nb / kTopkThreads;
      const int top = nb - 1 - tid * per;
      int lsum = 0;
      for (int b = 0; b < per; ++b) lsum += hist[top - b];
      const int incl_w = warp_incl_scan(lsum);
      if (lane == 31) warp_sum[wid] = incl_w;
      __syncthreads();
      if (wid == 0) {
        const int x = lane < nw ? warp_sum[lane] : 0;
        const int xi = warp_incl_scan(x);
        if (lane < nw) warp_sum[lane] = xi - x;
      }
      __syncthreads();
      const int incl = warp_sum[wid] + incl_w;
      const int excl = incl - lsum;
      if (excl < need && need <= incl) {
        int cum = excl;
        for (int b = 0; b < per; ++b) {
          const int v = hist[top - b];
          if (cum + v >= need) {
            found_bin = top - b;
            found_above = cum;
            break;
          }
          cum += v;
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)found_bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    need -= found_above;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need_eq = need;  // keys equal to tau that stay, first ones in ascending p

  // warp-contiguous compaction
  const int run = ((c + nw - 1) / nw + 31) & ~31;  // keys per warp, whole steps
  const int w0 = min(c, wid * run), w1 = min(c, w0 + run);
  int ngt = 0, neq = 0;
  for (int i = w0 + lane; i < w1; i += 32) {
    const uint32_t key = K[i];
    ngt += key > tau;
    neq += key == tau;
  }
  ngt = __reduce_add_sync(kFull, ngt);
  neq = __reduce_add_sync(kFull, neq);
  if (lane == 0) {
    warp_gt[wid] = ngt;
    warp_eq[wid] = neq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;  // exclusive prefix over the warps before this one
  {
    const int g = lane < nw && lane < wid ? warp_gt[lane] : 0;
    const int q = lane < nw && lane < wid ? warp_eq[lane] : 0;
    gt_before = __reduce_add_sync(kFull, g);
    eq_before = __reduce_add_sync(kFull, q);
  }
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const bool in = i < w1;
    const uint32_t key = in ? K[i] : 0u;
    const int p = in ? __ldg(sp + i) : 0;
    const bool gt = in && key > tau, eq = in && key == tau;
    const unsigned mgt = __ballot_sync(kFull, gt), meq = __ballot_sync(kFull, eq);
    const int eq_rank = eq_before + __popc(meq & lt);
    const bool keep = gt || (eq && eq_rank < need_eq);
    if (keep) {
      const int kept_eq_before = min(eq_rank, need_eq);
      const int row = out0 + gt_before + __popc(mgt & lt) + kept_eq_before;
      perm[row] = p;
      if (idx_ok(p, P, status)) pos[p] = row;
    } else if (in && idx_ok(p, P, status)) {
      pos[p] = -1;
    }
    gt_before += __popc(mgt);
    eq_before += __popc(meq);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for lrmoe_select_quota_noalloc: a fixed device array owned by the
// library, so callers that may not allocate device memory can still select.
// Every GPU that loads this module holds these bytes until the process exits.
// All calls on a device share it; calls that overlap on the GPU race on it.
// No byte of it needs to start at zero: each kernel writes what it reads.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_select_scratch[LRMOE_NOALLOC_SCRATCH_BYTES];

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The four selection kernels on `s` (workspace pieces already carved out).
static cudaError_t enqueue_select(const SelectWs& L, const int32_t* idx, const float* score, int P,
                                  int E, const int32_t* quota, int32_t* counts, int32_t* kept,
                                  int32_t* offsets, int32_t* perm, int32_t* pos, int32_t* cc,
                                  int32_t* seg_start, int32_t* seg_p, uint32_t* seg_key,
                                  uint32_t* status, cudaStream_t s) {
  // Shared-memory limits are set on every call (host-side calls, no device
  // work), so that they hold in whatever context is current, also after a
  // context reset, and no host-side flag is shared between threads.
  const size_t scatter_smem = ((size_t)kScatterWarps * E + 2 * (size_t)E + 33) * 4;
  cudaError_t e = cudaFuncSetAttribute(chunk_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)((kScatterWarps + 2) * 4096 + 33) * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(expert_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTopkSmemKeys * 4);
  if (e != cudaSuccess) return e;
  e = launch_pdl(chunk_count, dim3(L.nchunks), dim3(kCountThreads), (size_t)E * 4, s, idx, P, E,
                 L.chunk, L.nchunks, cc, pos, status);
  if (e != cudaSuccess) return e;
  e = launch_pdl(chunk_scatter, dim3(L.nchunks), dim3(kScatterWarps * 32), scatter_smem, s, idx,
                 reinterpret_cast<const uint32_t*>(score), P, E, L.chunk, L.nchunks,
                 static_cast<const int32_t*>(cc), quota, counts, kept, offsets, seg_start, seg_p,
                 seg_key, status);
  if (e != cudaSuccess) return e;
  return launch_pdl(expert_topk, dim3(E), dim3(kTopkThreads), (size_t)kTopkSmemKeys * 4, s,
                    static_cast<const int32_t*>(counts), static_cast<const int32_t*>(kept),
                    static_cast<const int32_t*>(offsets), static_cast<const int32_t*>(seg_start),
                    static_cast<const int32_t*>(seg_p), static_cast<const uint32_t*>(seg_key),
                    perm, pos, P, status);
}

SelectWs select_ws_layout(int T, int k, int E) {
  SelectWs L;
  const long long P = (long long)T * k;
  long long chunk = 1024;  // one 16-byte load per count thread; 4 steps per scatter warp
  const long long max_chunks = kScanSmemInts / (E > 0 ? E : 1);
  if (max_chunks > 0 && (P + chunk - 1) / chunk > max_chunks) {
    chunk = (P + max_chunks - 1) / max_chunks;
    chunk = (chunk + 255) / 256 * 256;
  }
  L.chunk = (int)chunk;
  L.nchunks = (int)((P + chunk - 1) / chunk);
  if (L.nchunks < 1) L.nchunks = 1;
  size_t off = 0;
  L.off_cc = off;
  off += align256((size_t)E * L.nchunks * 4);
  L.off_seg_start = off;
  off += align256((size_t)(E + 1) * 4);
  L.off_seg_p = off;
  off += align256((size_t)P * 4);
  L.off_seg_key = off;
  off += align256((size_t)P * 4);
  L.total = off;
  return L;
}

cudaError_t launch_select(const int32_t* idx, const float* score, int T, int k, int E,
                          const int32_t* quota, int32_t* counts, int32_t* kept, int32_t* offsets,
                          int32_t* perm, int32_t* pos, void* ws, uint32_t* status,
                          cudaStream_t s) {
  const SelectWs L = select_ws_layout(T, k, E);
  const int P = T * k;
  char* base = static_cast<char*>(ws);
  int32_t* cc = reinterpret_cast<int32_t*>(base + L.off_cc);
  int32_t* seg_start = reinterpret_cast<int32_t*>(base + L.off_seg_start);
  int32_t* seg_p = reinterpret_cast<int32_t*>(base + L.off_seg_p);
  uint32_t* seg_key = reinterpret_cast<uint32_t*>(base + L.off_seg_key);

  return enqueue_select(L, idx, score, P, E, quota, counts, kept, offsets, perm, pos, cc,
                        seg_start, seg_p, seg_key, status, s);
}

// Device address of the built-in scratch array in the context current on this
// thread.  In host code `g_select_scratch` names only a host-side stand-in,
// never device memory; the real address comes from the runtime.  It is looked
// up on every call (a host-side query that allocates nothing), so that it
// stays right when the device's context is reset and the module is loaded
// again at another address.  The first lookup in a context loads the module.
static cudaError_t select_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

size_t select_noalloc_scratch_bytes() { return sizeof(g_select_scratch); }

// Same kernels and launch sequence as launch_select, with the built-in array
// as the workspace.  The caller has checked that the layout fits in it.
cudaError_t launch_select_noalloc(const int32_t* idx, const float* score, int T, int k, int E,
                                  const int32_t* quota, int32_t* counts, int32_t* kept,
                                  int32_t* offsets, int32_t* perm, int32_t* pos, uint32_t* status,
                                  cudaStream_t s) {
  const SelectWs L = select_ws_layout(T, k, E);
  if (L.total > sizeof(g_select_scratch)) return cudaErrorInvalidValue;
  void* ws = nullptr;
  cudaError_t err = select_scratch_address(&ws);
  if (err != cudaSuccess) return err;
  const int P = T * k;
  char* base = static_cast<char*>(ws);
  int32_t* cc = reinterpret_cast<int32_t*>(base + L.off_cc);
  int32_t* seg_start = reinterpret_cast<int32_t*>(base + L.off_seg_start);
  int32_t* seg_p = reinterpret_cast<int32_t*>(base + L.off_seg_p);
  uint32_t* seg_key = reinterpret_cast<uint32_t*>(base + L.off_seg_key);

  return enqueue_select(L, idx, score, P, E, quota, counts, kept, offsets, perm, pos, cc,
                        seg_start, seg_p, seg_key, status, s);
}

}  // namespace lrmoe
