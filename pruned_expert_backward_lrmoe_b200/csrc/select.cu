// a2  Per-expert top-quota selection.
//
// Follows "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE",
// bullets 2-3: the quota of every expert is fixed for the layer call, and
// within it the pairs with the highest score stay.  Key: score bit pattern as
// uint32 descending, then pair index ascending (scores are >= +0, so the bit
// order is the numeric order; NaN sorts above +Inf).
//
// Four kernels, integer work only, deterministic (no order-dependent atomics):
//   1. chunk_count : per chunk of pairs, an expert histogram (+ pos = -1 for
//                    empty/invalid slots)
//   2. chunk_scan  : per expert, exclusive scan over chunks; counts, the
//                    segment starts, m_e = min(max(q_e,0), c_e), offsets
//   3. chunk_scatter: stable counting sort of the pairs by expert (ascending p
//                    inside each expert) into seg_p / seg_key
//   4. expert_topk : one CTA per expert: 4 x 8-bit radix select of the m_e-th
//                    largest key, then an ordered compaction that keeps keys
//                    above the threshold and the first (m_e - #above) equal
//                    keys in ascending p; writes perm and pos.
#include "common.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kCountThreads = 256;
constexpr int kScatterWarps = 8;
constexpr int kTopkThreads = 1024;
constexpr int kScanSmemInts = 32768;  // E * nchunks kept in shared memory by chunk_scan
constexpr int kTopkSmemKeys = 24576;  // segments up to this length are staged in smem

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

// Exclusive scan of n ints held one per thread (n <= blockDim.x * items); returns
// per-thread exclusive prefix of the thread's item sum, and the total.
__device__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int incl = warp_incl_scan(v);
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? warp_sums[lane] : 0;
    int si = warp_incl_scan(s);
    if (lane < nw) warp_sums[lane] = si - s;
    if (lane == 31) warp_sums[32] = si;
  }
  __syncthreads();
  const int r = warp_sums[wid] + incl - v;
  *total = warp_sums[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kScanThreads) chunk_scan(int32_t* __restrict__ cc, int E,
                                                           int nchunks,
                                                           const int32_t* __restrict__ quota,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ kept,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ seg_start,
                                                           uint32_t* __restrict__ status) {
  extern __shared__ int sm[];  // [33] warp sums, then [E] counts, then cc copy if it fits
  int* warp_sums = sm;
  int* cnt = sm + 33;
  int* ccs = cnt + E;
  const bool in_smem = (size_t)E * nchunks <= (size_t)kScanSmemInts;
  int* mat = in_smem ? ccs : cc;
  const int n = E * nchunks;
  pdl_wait();
  pdl_trigger();
  if (in_smem) {
    // eight loads in flight per thread, then the stores
    for (int i0 = 0; i0 < n; i0 += 8 * blockDim.x) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x + threadIdx.x;
        v[u] = i < n ? __ldcg(cc + i) : 0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x + threadIdx.x;
        if (i < n) ccs[i] = v[u];
      }
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int e = wid; e < E; e += nw) {
    int carry = 0;
    int* row = mat + (size_t)e * nchunks;
    for (int c0 = 0; c0 < nchunks; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < nchunks ? row[c] : 0;
      const int incl = warp_incl_scan(v);
      if (c < nchunks) row[c] = carry + incl - v;
      carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) cnt[e] = carry;
  }
  __syncthreads();
  if (in_smem)
    for (int i = threadIdx.x; i < n; i += blockDim.x) cc[i] = ccs[i];
  // segment starts (exclusive scan of counts) and offsets (exclusive scan of kept)
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int csum = 0, ksum = 0;
  bool badq = false;
  for (int i = 0; i < per; ++i) {
    const int e = e0 + i;
    if (e < E) {
      const int c = cnt[e];
      const int q = quota[e];
      badq |= q < 0;
      csum += c;
      ksum += min(max(q, 0), c);
    }
  }
  if (__any_sync(kFull, badq) && lane == 0) raise_status(status, LRMOE_ST_BAD_QUOTA);
  int ctot, ktot;
  int cex = block_excl_scan(csum, warp_sums, &ctot);
  int kex = block_excl_scan(ksum, warp_sums, &ktot);
  for (int i = 0; i < per; ++i) {
    const int e = e0 + i;
    if (e < E) {
      const int c = cnt[e];
      const int m = min(max(quota[e], 0), c);
      counts[e] = c;
      kept[e] = m;
      seg_start[e] = cex;
      offsets[e] = kex;
      cex += c;
      kex += m;
    }
  }
  if (threadIdx.x == 0) {
    seg_start[E] = ctot;
    offsets[E] = ktot;
  }
}

__global__ void __launch_bounds__(kScatterWarps * 32) chunk_scatter(
    const int32_t* __restrict__ idx, const uint32_t* __restrict__ score_bits, int P, int E,
    int chunk, int nchunks, const int32_t* __restrict__ cc, const int32_t* __restrict__ seg_start,
    int32_t* __restrict__ seg_p, uint32_t* __restrict__ seg_key) {
  extern __shared__ int wbase[];  // [kScatterWarps][E]
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
    int run = seg_start[e] + cc[(size_t)e * nchunks + c];
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
        seg_p[dst] = p;
        seg_key[dst] = sv[s];
      }
      __syncwarp();
      if (valid && lane == __ffs(m) - 1) mine[e] = base + __popc(m);
      __syncwarp();
    }
  }
}

// Block-wide exclusive scan of 64-bit values (two 32-bit counters packed in one
// word, low and high halves); returns the total too.  blockDim.x <= 1024.
__device__ __forceinline__ unsigned long long block_excl_scan_u64(unsigned long long v,
                                                                  unsigned long long* ws,
                                                                  unsigned long long* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ws[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const unsigned long long x = lane < nw ? ws[lane] : 0ull;
    unsigned long long xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long n = __shfl_up_sync(kFull, xi, o);
      if (lane >= o) xi += n;
    }
    if (lane < nw) ws[lane] = xi - x;
    if (lane == 31) ws[32] = xi;
  }
  __syncthreads();
  const unsigned long long r = ws[wid] + incl - v;
  *total = ws[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kTopkThreads) expert_topk(
    const int32_t* __restrict__ counts, const int32_t* __restrict__ kept,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ seg_start,
    const int32_t* __restrict__ seg_p, const uint32_t* __restrict__ seg_key,
    int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
  extern __shared__ uint32_t sm_keys[];  // [kTopkSmemKeys] keys, then [kTopkSmemKeys] pairs
  __shared__ int hist[256];
  __shared__ unsigned long long scan_ws[33];
  __shared__ int found_bin, found_above;
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const int c = counts[e];
  const int m = kept[e];
  const int s0 = seg_start[e];
  const int out0 = offsets[e];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nt = blockDim.x;
  const int32_t* sp = seg_p + s0;
  const uint32_t* sk = seg_key + s0;

  if (m == c) {  // everything stays, already in ascending p
    for (int i = tid; i < c; i += nt) {
      const int p = sp[i];
      perm[out0 + i] = p;
      pos[p] = out0 + i;
    }
    return;
  }
  if (m == 0) {
    for (int i = tid; i < c; i += nt) pos[sp[i]] = -1;
    return;
  }

  // stage the segment in shared memory (four loads in flight per thread)
  const bool in_smem = c <= kTopkSmemKeys;
  const uint32_t* K = sk;
  const int32_t* PP = sp;
  if (in_smem) {
    uint32_t* ks = sm_keys;
    int32_t* ps = reinterpret_cast<int32_t*>(sm_keys + kTopkSmemKeys);
    for (int i0 = 0; i0 < c; i0 += 4 * nt) {
      uint32_t kv[4];
      int pv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * nt + tid;
        if (i < c) {
          kv[u] = sk[i];
          pv[u] = sp[i];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * nt + tid;
        if (i < c) {
          ks[i] = kv[u];
          ps[i] = pv[u];
        }
      }
    }
    K = ks;
    PP = ps;
  }
  __syncthreads();

  // radix select of the m-th largest key, most significant byte first
  uint32_t prefix = 0;
  int need = m;
  for (int d = 3; d >= 0; --d) {
    const int shift = 8 * d;
    const uint32_t hmask = d == 3 ? 0u : (0xffffffffu << (shift + 8));
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < c; i0 += nt) {
      const int i = i0 + tid;
      int digit = -1;
      if (i < c) {
        const uint32_t key = K[i];
        if ((key & hmask) == prefix) digit = (int)((key >> shift) & 255u);
      }
      if (__any_sync(kFull, digit >= 0)) {  // later passes: most warps hold no candidate
        const unsigned grp = __match_any_sync(kFull, digit);
        if (digit >= 0 && lane == __ffs(grp) - 1) atomicAdd(&hist[digit], __popc(grp));
      }
    }
    __syncthreads();
    if (wid == 0) {
      // lane l owns bins 255-8l down to 248-8l (descending key order)
      int cnt8[8];
      int lsum = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        cnt8[b] = hist[255 - 8 * lane - b];
        lsum += cnt8[b];
      }
      const int incl = warp_incl_scan(lsum);
      const int excl = incl - lsum;
      if (excl < need && need <= incl) {
        int cum = excl;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (cum + cnt8[b] >= need) {
            found_bin = 255 - 8 * lane - b;
            found_above = cum;
            break;
          }
          cum += cnt8[b];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)found_bin << shift;
    need -= found_above;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const unsigned long long need_eq = (unsigned long long)need;  // equal keys kept, in ascending p

  // ordered compaction: thread t owns the contiguous run [t*R, t*R + R); one scan
  // of (above, equal) counts gives every run its starting row.
  const int R = (c + nt - 1) / nt;
  const int b0 = min(c, tid * R), b1 = min(c, b0 + R);
  unsigned long long ngt = 0, neq = 0;
  for (int i = b0; i < b1; ++i) {
    const uint32_t key = K[i];
    ngt += key > tau;
    neq += key == tau;
  }
  unsigned long long tot;
  const unsigned long long ex = block_excl_scan_u64(ngt | (neq << 32), scan_ws, &tot);
  unsigned long long gt_before = ex & 0xffffffffull, eq_before = ex >> 32;
  for (int i = b0; i < b1; ++i) {
    const uint32_t key = K[i];
    const int p = PP[i];
    const bool gt = key > tau, eq = key == tau;
    if (gt || (eq && eq_before < need_eq)) {
      const int row = out0 + (int)(gt_before + (eq_before < need_eq ? eq_before : need_eq));
      perm[row] = p;
      pos[p] = row;
    } else {
      pos[p] = -1;
    }
    gt_before += gt;
    eq_before += eq;
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
  cudaError_t e = cudaFuncSetAttribute(chunk_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (33 + 4096 + kScanSmemInts) * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chunk_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kScatterWarps * 4096 * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(expert_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTopkSmemKeys * 8);
  if (e != cudaSuccess) return e;
  e = launch_pdl(chunk_count, dim3(L.nchunks), dim3(kCountThreads), (size_t)E * 4, s,
                             idx, P, E, L.chunk, L.nchunks, cc, pos, status);
  if (e != cudaSuccess) return e;
  const bool fits = (size_t)E * L.nchunks <= (size_t)kScanSmemInts;
  const size_t scan_smem = (33 + (size_t)E + (fits ? (size_t)E * L.nchunks : 0)) * 4;
  e = launch_pdl(chunk_scan, dim3(1), dim3(kScanThreads), scan_smem, s, cc, E, L.nchunks, quota,
                 counts, kept, offsets, seg_start, status);
  if (e != cudaSuccess) return e;
  e = launch_pdl(chunk_scatter, dim3(L.nchunks), dim3(kScatterWarps * 32),
                 (size_t)kScatterWarps * E * 4, s, idx, reinterpret_cast<const uint32_t*>(score),
                 P, E, L.chunk, L.nchunks, static_cast<const int32_t*>(cc),
                 static_cast<const int32_t*>(seg_start), seg_p, seg_key);
  if (e != cudaSuccess) return e;
  return launch_pdl(expert_topk, dim3(E), dim3(kTopkThreads), (size_t)kTopkSmemKeys * 8, s,
                    static_cast<const int32_t*>(counts), static_cast<const int32_t*>(kept),
                    static_cast<const int32_t*>(offsets), static_cast<const int32_t*>(seg_start),
                    static_cast<const int32_t*>(seg_p), static_cast<const uint32_t*>(seg_key),
                    perm, pos);
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
