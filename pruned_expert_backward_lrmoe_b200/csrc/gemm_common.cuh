// Pieces shared by the grouped-GEMM kernels of gemm_tc.cu (one CTA per tile)
// and gemm_pair.cu (a two-CTA cluster per tile): tile constants, launch
// parameters, tile decoding, the epilogue helpers (bf16 store, SwiGLU backward)
// and the host-side tensor-map encoding.  Each including file gets its own copy
// (anonymous namespace), including its own tile-scheduler counters.
#pragma once

#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "grouped.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

constexpr int BM = 128;        // tile rows = TMEM lanes
constexpr int BK = 64;         // 64 bf16 = one 128-byte swizzle row
constexpr int UK = 16;         // K of one kind::f16 MMA
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;  // TMA warp, MMA warp, 8 epilogue warps
constexpr int kEpiThreads = 32 * kEpiWarps;

// kFused*: one launch runs a dgrad (store or SwiGLU epilogue) and a wgrad that
// share their packed gradient rows.
// kWgradGather: wgrad whose B rows are gathered from an unpacked tensor.
enum Mode : int { kDgradStore = 0, kDgradSwiglu = 1, kWgrad = 2, kFusedStore = 3, kFusedSwiglu = 4,
                  kWgradGather = 5 };
constexpr int kBNT = 256;  // tile N (TMEM columns per accumulator)

// Dynamic tile scheduling.  Each CTA's producer takes the next tile index from a
// global counter and hands it to the MMA and epilogue warps through a ring of
// kRing shared-memory slots, so faster SMs take more tiles.  The counters live
// here, one pair (next tile, CTAs done) per slot; launches rotate over
// kSchedSlots slots, and the last CTA of a launch to finish puts its pair back
// to zero.  Up to kSchedSlots grouped-GEMM launches may run at once per device.
constexpr int kRing = 4;
constexpr int kSchedSlots = 64;
__device__ unsigned int g_sched[kSchedSlots][2];

// Shared-memory layout.  OUTBUFS = fp32 staging buffers per epilogue warp (wgrad
// only).  The tables at the end are sized by the launch's expert count E.
template <int BN, int STAGES, int OUTBUFS>
struct Layout {
  static constexpr int kABytes = BM * BK * 2;                 // 16 KB
  static constexpr int kBBytes = BN * BK * 2;                 // 32 KB at BN = 256
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTilesBytes = STAGES * kStageBytes;
  // fp32 output staging: per epilogue warp OUTBUFS 32 x 32 fp32 sub-tiles (4 KB each)
  static constexpr int kOutBufBytes = 32 * 32 * 4;
  static constexpr int kOutOff = kTilesBytes;
  static constexpr int kOutBytes = kEpiWarps * OUTBUFS * kOutBufBytes;
  static constexpr int kBarOff = kOutOff + kOutBytes;         // 8-byte barriers
  static constexpr int kNumBars = 2 * STAGES + 5 + 2 * kRing;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;     // tmem base, abort flag, tile ring
  static constexpr int kTableOff = kMiscOff + 16 + 4 * kRing;
  // tile table, expert order / sizes (E + 1 each), scan scratch, offsets[0..E]
  __host__ __device__ static constexpr int table_ints(int E) { return 3 * (E + 1) + 33; }
  __host__ __device__ static constexpr int alloc(int E) {
    return kTableOff + table_ints(E) * 4 + 1024;  // + slack for 1024-B alignment
  }
};
constexpr int kSmemLimit = 232448;  // per-block dynamic shared memory on sm_100

// Scalars of one launch.  dgrad: out_d[R_e] = rows[R_e] . W[e] (K x Nd); wgrad:
// dW[e] = grad[R_e]^T . in[R_e] (N1 x N2, fp32).  A fused launch runs both over
// the same packed gradient rows (dgrad K = wgrad N1).
struct GemmParams {
  const int32_t* offsets;
  int E;
  int Kd, Nd;           // dgrad
  int N1, N2;           // wgrad
  const uint16_t* Gp;   // SwiGLU epilogue: saved g, u [rows][Nd] (packed), or [gu_rows][Nd]
  const uint16_t* Up;   // read at row perm[r] when perm is given
  const int32_t* perm;
  int gu_rows;
  void* out_d;          // dgrad output [rows][Nd] (SwiGLU: [rows][2 Nd])
  int accumulate;       // wgrad: add into dW
  // kWgradGather: B row of packed row r = gsrc[perm[r] / gdiv] ([*][N2]); perm
  // entries must lie in [0, gperm_max)
  const uint16_t* gsrc;
  int gdiv, gperm_max;
  uint32_t* status;
  int sched_slot;
  // diagnostics (zero in normal launches): wait_ns > 0 replaces the limit of
  // every bounded wait; stall != 0 makes the producers withhold the first K
  // block of their first tile, so that the MMA issuer's wait runs out
  unsigned long long wait_ns;
  int stall;
  int part;             // dgrad: which row tiles of each expert (RowPart)
  int late_wait;        // launched after another dgrad over other rows of the same
                        // output: run first, wait for the preceding kernel at the end
  int rows_cap;         // rows of the packed operands (the tensor maps' row extent)
};

template <int MODE>
struct Traits {
  static constexpr bool kHasD = MODE != kWgrad && MODE != kWgradGather;
  static constexpr bool kHasW =
      MODE == kWgrad || MODE == kFusedStore || MODE == kFusedSwiglu || MODE == kWgradGather;
  static constexpr bool kSwiglu = MODE == kDgradSwiglu || MODE == kFusedSwiglu;
  static constexpr bool kGatherB = MODE == kWgradGather;
};

struct TileInfo {
  int kind;    // 0: dgrad tile, 1: wgrad tile
  int e;       // expert
  int row0;    // dgrad: first packed row of the tile; wgrad: first packed row of the expert
  int row_end; // end of the expert's rows
  int m0, n0;  // output tile origin (dgrad: m0 unused)
  int nk;      // number of K blocks
};

// Tile counts of a launch: dgrad (variable M) and wgrad (fixed per expert).
struct TileCounts {
  int td, tw, total;
  int nt_d;        // dgrad N tiles
  int mt_w, nt_w;  // wgrad M and N tiles
};

// Tile t of the launch.  A fused launch spreads its td dgrad tiles evenly over
// the tw wgrad tiles (position t is a dgrad tile when floor((t+1) td / T) steps),
// so that every SM alternates the read-bound and the write-bound kind.
template <int MODE>
__device__ __forceinline__ TileInfo decode_tile(int t, const GemmParams& p, const int* offs,
                                                const int* tab_d, const int* tab_w,
                                                const TileCounts& tc) {
  using Tr = Traits<MODE>;
  TileInfo ti;
  int idx;
  if constexpr (Tr::kHasD && Tr::kHasW) {
    const long long before = (long long)t * tc.td / tc.total;
    const long long upto = ((long long)t + 1) * tc.td / tc.total;
    ti.kind = upto > before ? 0 : 1;
    idx = ti.kind == 0 ? (int)before : t - (int)upto;
  } else {
    ti.kind = Tr::kHasW ? 1 : 0;
    idx = t;
  }
  if (ti.kind == 1) {
    const int per_e = tc.mt_w * tc.nt_w;
    const int oi = idx / per_e, local = idx - oi * per_e;
    ti.e = tab_w[oi];
    ti.m0 = (local / tc.nt_w) * BM;
    ti.n0 = (local % tc.nt_w) * kBNT;
    ti.row0 = offs[ti.e];
    ti.row_end = offs[ti.e + 1];
    ti.nk = (ti.row_end - ti.row0 + BK - 1) / BK;
  } else {
    const int e = find_group(tab_d, p.E, idx);
    const int local = idx - tab_d[e];
    ti.e = e;
    ti.m0 = 0;
    ti.n0 = (local % tc.nt_d) * kBNT;
    ti.row0 = dgrad_tile_row0(offs[e], offs[e + 1] - offs[e], BM, p.part, local / tc.nt_d);
    ti.row_end = offs[e + 1];
    ti.nk = (p.Kd + BK - 1) / BK;
  }
  return ti;
}

__device__ __forceinline__ float sigmoid_fast(float x) { return 1.0f / (1.0f + __expf(-x)); }

// Make later uses of `r` depend on the preceding tcgen05.wait::ld.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i])::"memory");
}

// bf16 row segment [nb, nb + 32) of `orow`, columns >= N skipped (N % 8 == 0).
__device__ __forceinline__ void epi_store_bf16(const uint32_t (&r)[32], uint16_t* orow, int nb,
                                               int N) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (nb + v * 8 < N) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
      w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
      w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
      w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
      *reinterpret_cast<uint4*>(orow + nb + v * 8) = w;
    }
  }
}

// saved g, u of one row, columns [nb, nb + 32)
__device__ __forceinline__ void load_gu(uint4 (&gv)[4], uint4 (&uv)[4],
                                        const uint16_t* __restrict__ Gp,
                                        const uint16_t* __restrict__ Up, int row, int nb, int N) {
  const uint16_t* gp = Gp + (size_t)row * N + nb;
  const uint16_t* up = Up + (size_t)row * N + nb;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (nb + v * 8 < N) {
      gv[v] = __ldg(reinterpret_cast<const uint4*>(gp + v * 8));
      uv[v] = __ldg(reinterpret_cast<const uint4*>(up + v * 8));
    }
  }
}

// SwiGLU backward of one row segment: with s = sigmoid(g),
// dG = dA u s (1 + g (1 - s)), dU = dA g s; stored as bf16.
__device__ __forceinline__ void epi_swiglu(const uint32_t (&r)[32], const uint4 (&gv)[4],
                                           const uint4 (&uv)[4], uint16_t* og, uint16_t* ou, int nb,
                                           int N) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (nb + v * 8 < N) {
      const uint32_t gw[4] = {gv[v].x, gv[v].y, gv[v].z, gv[v].w};
      const uint32_t uw[4] = {uv[v].x, uv[v].y, uv[v].z, uv[v].w};
      uint32_t dg[4], du[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float res_g[2], res_u[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float da = __uint_as_float(r[8 * v + 2 * i + h]);
          const float g = bf16_bits_to_f32(h ? (gw[i] >> 16) : (gw[i] & 0xffffu));
          const float u = bf16_bits_to_f32(h ? (uw[i] >> 16) : (uw[i] & 0xffffu));
          const float s = sigmoid_fast(g);
          res_g[h] = da * u * s * (1.0f + g * (1.0f - s));
          res_u[h] = da * g * s;
        }
        dg[i] = pack_bf16x2(res_g[0], res_g[1]);
        du[i] = pack_bf16x2(res_u[0], res_u[1]);
      }
      *reinterpret_cast<uint4*>(og + nb + v * 8) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
      *reinterpret_cast<uint4*>(ou + nb + v * 8) = make_uint4(du[0], du[1], du[2], du[3]);
    }
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process.  The lookup runs
// inside the initialiser of a function-local static, which C++ runs exactly
// once even when several host threads make their first GEMM call together.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// 2D bf16 map over a row-major [rows][cols] matrix, box = box_cols x box_rows, 128-B swizzle.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-window map over a [rows][cols] bf16 matrix, for K-tail blocks that must end at
// an arbitrary row: dims (cols, 64, rows - 63) with both outer dims stepping one row
// (the same stride).  A 64 x 64 box loaded at coordinates (c, 64 - v, e - 64) holds
// rows e-v .. e-1 of columns c .. c+63 and then 64 - v rows of zeros: element i of
// the box sits at window coordinate 64 - v + i, past the window's extent for i >= v.
// Needs e >= 64 (a smaller end is a negative, out-of-range coordinate: zeros only);
// an element inside all extents is row (64 - v + i) + (e - 64) <= rows - 1, so
// nothing outside the matrix is read.  128-B swizzle, like the 2D maps.
bool make_map_rows_window(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, 64, rows > 64 ? rows - 63 : 1};
  cuuint64_t strides[2] = {cols * 2, cols * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map over [E][K][N], box = 64 (N) x 64 (K) x 1, 128-B swizzle.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {N, K, E};
  cuuint64_t strides[2] = {N * 2, K * N * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D fp32 map over dW [E][N1][N2], box = 32 (N2) x 32 (N1) x 1, 128-B swizzle (store side).
bool make_map_out_f32(CUtensorMap* m, void* base, uint64_t E, uint64_t N1, uint64_t N2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {N2, N1, E};
  cuuint64_t strides[2] = {N2 * 4, N1 * N2 * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace lrmoe
