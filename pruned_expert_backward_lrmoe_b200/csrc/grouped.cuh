// Device-side tile bookkeeping of the variable-size grouped GEMMs.
//
// Expert e owns packed rows [offsets[e], offsets[e+1]).  The group sizes stay
// on the device, so every persistent CTA rebuilds the tile table from
// `offsets` in shared memory at start-up (E <= kMaxExperts) and walks the
// same tile sequence; no host synchronisation and no zero padding.
#pragma once

#include "common.cuh"
#include "launch.h"

namespace lrmoe {

constexpr int kMaxExperts = kMaxGroupedExperts;

// Exclusive scan of v[0..n) in place (shared memory), block-wide; returns total.
__device__ __forceinline__ int block_scan_inplace(int* v, int n, int* scratch /*[33]*/) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b = tid * per;
  int s = 0;
  for (int i = 0; i < per; ++i)
    if (b + i < n) s += v[b + i];
  const int incl = warp_incl_scan(s);
  if (lane == 31) scratch[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int x = lane < nw ? scratch[lane] : 0;
    const int xi = warp_incl_scan(x);
    if (lane < nw) scratch[lane] = xi - x;
    if (lane == 31) scratch[32] = xi;
  }
  __syncthreads();
  int run = scratch[wid] + incl - s;
  for (int i = 0; i < per; ++i)
    if (b + i < n) {
      const int t = v[b + i];
      v[b + i] = run;
      run += t;
    }
  const int total = scratch[32];
  __syncthreads();
  return total;
}

// Checked-index build: offsets must rise from offsets[0] >= 0 to offsets[E] <=
// rows_cap.  Block-wide; true (and LRMOE_ST_BAD_INDEX raised) when they do not,
// in which case the launch computes no tile.  Always false in the normal build.
__device__ __forceinline__ bool offsets_invalid(const int32_t* offs, int E, int rows_cap,
                                                uint32_t* status) {
  if constexpr (!kChecked) {
    return false;
  } else {
    bool bad = false;
    for (int i = threadIdx.x; i < E; i += blockDim.x) bad |= offs[i] > offs[i + 1];
    if (threadIdx.x == 0) bad |= offs[0] < 0 || offs[E] > rows_cap;
    const bool any = __syncthreads_or(bad);
    if (any && blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
    return any;
  }
}

// Which rows of each expert a dgrad launch covers (variable M).
//   kRowsAll   : every row, in tiles of BM rows
//   kRowsPairs : the 256-row tiles of a two-SM launch, without a last tile of at
//                most 128 rows (m_e / 256 tiles, plus one if m_e % 256 > 128)
//   kRowsTails : that last tile of at most 128 rows (m_e % 256 in (0, 128]), for a
//                one-SM launch of 128-row tiles
enum RowPart : int { kRowsAll = 0, kRowsPairs = 1, kRowsTails = 2 };

__device__ __forceinline__ int dgrad_row_tiles(int m, int BM, int part) {
  if (m <= 0) return 0;
  if (part == kRowsPairs) return m / 256 + (m % 256 > 128 ? 1 : 0);
  if (part == kRowsTails) return (m % 256 > 0 && m % 256 <= 128) ? 1 : 0;
  return (m + BM - 1) / BM;
}

// First packed row of row tile j of expert e (rows [first, first + BM) clipped
// to the expert's end).
__device__ __forceinline__ int dgrad_tile_row0(int e_first, int m, int BM, int part, int j) {
  if (part == kRowsTails) return e_first + m - m % 256;
  return e_first + j * BM;
}

// dgrad (variable M): tiles of expert e = row tiles(m_e) * n_tiles, experts in order.
// tstart[0..E] receives the exclusive prefix; returns the total tile count.
__device__ __forceinline__ int build_dgrad_tiles(const int32_t* __restrict__ offsets, int E,
                                                 int BM, int n_tiles, int* tstart,
                                                 int* scratch, int part = kRowsAll) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int m = offsets[e + 1] - offsets[e];
    tstart[e] = dgrad_row_tiles(m, BM, part) * n_tiles;
  }
  __syncthreads();
  const int total = block_scan_inplace(tstart, E, scratch);
  if (threadIdx.x == 0) tstart[E] = total;
  __syncthreads();
  return total;
}

// Largest e with tstart[e] <= t (tstart non-decreasing, tstart[0] = 0).
__device__ __forceinline__ int find_group(const int* tstart, int E, int t) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tstart[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// wgrad (variable K): every expert has the same tiles; experts are visited in
// descending m_e (ties by ascending e) so that the longest K loops start first.
// order[0..E) receives the expert sequence.
__device__ __forceinline__ void build_wgrad_order(const int32_t* __restrict__ offsets, int E,
                                                  int* order, int* msz) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) msz[e] = offsets[e + 1] - offsets[e];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int me = msz[e];
    int rank = 0;
    for (int f = 0; f < E; ++f) {
      const int mf = msz[f];
      rank += (mf > me) || (mf == me && f < e);
    }
    order[rank] = e;
  }
  __syncthreads();
}

}  // namespace lrmoe
