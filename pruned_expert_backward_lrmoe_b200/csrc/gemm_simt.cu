// a4 for fp32 storage: variable-size grouped GEMMs in fp32 FFMA.
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 5:
// grouped GEMMs of variable size over the compacted per-expert blocks, with
// no zero padding.  The tensor cores have no fp32 x fp32 kind that meets a
// 1e-5 relative error, so fp32 layers use this CUDA-core path (64x64 tiles,
// 16-deep K slices, 4x4 outputs per thread, persistent grid over a tile table
// built on the device from `offsets`).
#include "common.cuh"
#include "grouped.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// D[r][n] = sum_k rows[r][k] W[e][k][n] for r in R_e; epilogue STORE or SWIGLU_BWD.
__global__ void __launch_bounds__(NT) dgrad_simt_kernel(
    const float* __restrict__ rows, const float* __restrict__ W,
    const int32_t* __restrict__ offsets, int E, int K, int N, int epi,
    const float* __restrict__ Gp, const float* __restrict__ Up, float* __restrict__ out,
    int rows_cap, uint32_t* __restrict__ status) {
  __shared__ int tstart[kMaxExperts + 1];
  __shared__ int scratch[33];
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN];
  pdl_wait();
  pdl_trigger();
  const int n_tiles = (N + BN - 1) / BN;
  const int total = offsets_invalid(offsets, E, rows_cap, status)
                        ? 0 : build_dgrad_tiles(offsets, E, BM, n_tiles, tstart, scratch);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    const int e = find_group(tstart, E, t);
    const int local = t - tstart[e];
    const int mt = local / n_tiles, nt = local % n_tiles;
    const int row_beg = offsets[e] + mt * BM;
    const int row_end = offsets[e + 1];
    const int n0 = nt * BN;
    const float* We = W + (size_t)e * K * N;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += BK) {
      // A: 64 rows x 16 k, thread loads 4 (kk fastest)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = tid + i * NT;
        const int r = idx >> 4, kk = idx & 15;
        const int gr = row_beg + r, gk = k0 + kk;
        As[kk][r] = (gr < row_end && gk < K) ? rows[(size_t)gr * K + gk] : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = tid + i * NT;
        const int kk = idx >> 6, n = idx & 63;
        const int gk = k0 + kk, gn = n0 + n;
        Bs[kk][n] = (gk < K && gn < N) ? We[(size_t)gk * N + gn] : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gr = row_beg + ty * 4 + i;
      if (gr >= row_end) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gn = n0 + tx * 4 + j;
        if (gn >= N) continue;
        const float d = acc[i][j];
        if (epi == LRMOE_EPI_SWIGLU_BWD) {
          const float g = Gp[(size_t)gr * N + gn];
          const float u = Up[(size_t)gr * N + gn];
          const float s = sigmoidf_(g);
          out[(size_t)gr * 2 * N + gn] = d * u * s * (1.0f + g * (1.0f - s));
          out[(size_t)gr * 2 * N + N + gn] = d * g * s;
        } else {
          out[(size_t)gr * N + gn] = d;
        }
      }
    }
  }
}

// dW[e][m][n] = sum_{r in R_e} grad[r][m] in[r][n]
__global__ void __launch_bounds__(NT) wgrad_simt_kernel(
    const float* __restrict__ grad, const float* __restrict__ in,
    const int32_t* __restrict__ offsets, int E, int N1, int N2, float* __restrict__ dW,
    int accumulate, int rows_cap, uint32_t* __restrict__ status) {
  __shared__ float As[BK][BM];
  __shared__ float Bs[BK][BN];
  pdl_wait();
  pdl_trigger();
  const int m_tiles = (N1 + BM - 1) / BM, n_tiles = (N2 + BN - 1) / BN;
  const int per_e = m_tiles * n_tiles;
  const int total = offsets_invalid(offsets, E, rows_cap, status) ? 0 : per_e * E;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    const int e = t / per_e;
    const int local = t % per_e;
    const int m0 = (local / n_tiles) * BM, n0 = (local % n_tiles) * BN;
    const int r_beg = offsets[e], r_end = offsets[e + 1];
    float acc[4][4] = {};
    for (int r0 = r_beg; r0 < r_end; r0 += BK) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = tid + i * NT;
        const int kk = idx >> 6, c = idx & 63;
        const int r = r0 + kk;
        As[kk][c] = (r < r_end && m0 + c < N1) ? grad[(size_t)r * N1 + m0 + c] : 0.0f;
        Bs[kk][c] = (r < r_end && n0 + c < N2) ? in[(size_t)r * N2 + n0 + c] : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
    float* dWe = dW + (size_t)e * N1 * N2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty * 4 + i;
      if (m >= N1) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n >= N2) continue;
        float* dst = dWe + (size_t)m * N2 + n;
        *dst = accumulate ? *dst + acc[i][j] : acc[i][j];
      }
    }
  }
}

}  // namespace

cudaError_t launch_dgrad_simt(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                              lrmoe_epilogue epi, const void* Gp, const void* Up, void* out,
                              uint32_t* status, cudaStream_t s) {
  (void)dt;
  return launch_pdl(dgrad_simt_kernel, dim3(num_sms() * 4), dim3(NT), 0, s,
                    static_cast<const float*>(rows), static_cast<const float*>(W), offsets, E, K,
                    N, (int)epi, static_cast<const float*>(Gp), static_cast<const float*>(Up),
                    static_cast<float*>(out), rows_cap, status);
}

cudaError_t launch_wgrad_simt(const void* grad_rows, const void* in_rows, int rows_cap,
                              const int32_t* offsets, int E, int N1, int N2, lrmoe_dtype dt,
                              float* dW, int accumulate, uint32_t* status, cudaStream_t s) {
  (void)dt;
  return launch_pdl(wgrad_simt_kernel, dim3(num_sms() * 4), dim3(NT), 0, s,
                    static_cast<const float*>(grad_rows), static_cast<const float*>(in_rows),
                    offsets, E, N1, N2, dW, accumulate, rows_cap, status);
}

}  // namespace lrmoe
