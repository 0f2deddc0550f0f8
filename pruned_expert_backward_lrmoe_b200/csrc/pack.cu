// a3  Physical compaction and a5  return to the token layout.
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 5
// and the note after it: retained gradient and activation rows are gathered
// into dense per-expert blocks (masking rows inside full-size tensors would
// save nothing), and the result then goes back to the original layout.
//
// Both are HBM-bound row gathers.  One warp per row, 16 bytes per lane per
// access; persistent grid-stride loops, since the retained-row count M lives
// on the device (offsets[E]) and is never read back by the host.
#include "common.cuh"
#include "launch.h"
#include "rowreduce.cuh"

namespace lrmoe {
namespace {

constexpr int kUnpackLoads = 8;  // a token's (column chunk, row) loads in flight together

__device__ __forceinline__ void copy_row(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                         int V, int lane) {
  int c = lane;
  for (; c + 96 < V; c += 128) {
    const uint4 v0 = __ldg(src + c), v1 = __ldg(src + c + 32), v2 = __ldg(src + c + 64),
                v3 = __ldg(src + c + 96);
    dst[c] = v0;
    dst[c + 32] = v1;
    dst[c + 64] = v2;
    dst[c + 96] = v3;
  }
  for (; c < V; c += 32) dst[c] = __ldg(src + c);
}

template <lrmoe_dtype DT>
__device__ __forceinline__ uint4 scale_vec(uint4 v, float w) {
  if constexpr (DT == LRMOE_BF16) {
    uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = f32_to_bf16_bits_rne(__fmul_rn(w, bf16_bits_to_f32(in[i] & 0xffffu)));
      const uint32_t hi = f32_to_bf16_bits_rne(__fmul_rn(w, bf16_bits_to_f32(in[i] >> 16)));
      out[i] = lo | (hi << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
  } else {
    return make_uint4(__float_as_uint(__fmul_rn(w, __uint_as_float(v.x))),
                      __float_as_uint(__fmul_rn(w, __uint_as_float(v.y))),
                      __float_as_uint(__fmul_rn(w, __uint_as_float(v.z))),
                      __float_as_uint(__fmul_rn(w, __uint_as_float(v.w))));
  }
}

template <lrmoe_dtype DT>
__device__ __forceinline__ void scale_row(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                          int V, float w, int lane) {
  int c = lane;
  for (; c + 96 < V; c += 128) {
    const uint4 v0 = __ldg(src + c), v1 = __ldg(src + c + 32), v2 = __ldg(src + c + 64),
                v3 = __ldg(src + c + 96);
    dst[c] = scale_vec<DT>(v0, w);
    dst[c + 32] = scale_vec<DT>(v1, w);
    dst[c + 64] = scale_vec<DT>(v2, w);
    dst[c + 96] = scale_vec<DT>(v3, w);
  }
  for (; c < V; c += 32) dst[c] = scale_vec<DT>(__ldg(src + c), w);
}

template <lrmoe_dtype DT>
__global__ void __launch_bounds__(256) pack_kernel(
    const int32_t* __restrict__ perm, const int32_t* __restrict__ offsets, int E,
    const float* __restrict__ w, int P, int k, const uint4* __restrict__ x,
    const uint4* __restrict__ dY, int VH, const uint4* __restrict__ a,
    const uint4* __restrict__ g, const uint4* __restrict__ u, int VI, uint4* __restrict__ Xp,
    uint4* __restrict__ DYp, uint4* __restrict__ Ap, uint4* __restrict__ Gp,
    uint4* __restrict__ Up, int ldH, int ldI, int rows_cap, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  pdl_wait();
  pdl_trigger();
  int M = offsets[E];
  if (M > rows_cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
    M = rows_cap;
  }
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < M; r += gridDim.x * wpb) {
    const int p = perm[r];
    if (p < 0 || p >= P) {
      if (lane == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
      continue;
    }
    const int t = p / k;
    const float wp = __ldg(w + p);
    const size_t rr = (size_t)r;
    // output row strides: ldH for X_p, DY_p and ldI for A_p, G_p, U_p (16-byte
    // vectors); VH and VI for dense blocks, the wide-row width for exchange rows
    if (Xp) copy_row(Xp + rr * ldH, x + (size_t)t * VH, VH, lane);  // X_p, A_p optional: the
    scale_row<DT>(DYp + rr * ldH, dY + (size_t)t * VH, VH, wp, lane);
    if (Ap) copy_row(Ap + rr * ldI, a + (size_t)p * VI, VI, lane);  // wgrad can gather them
    if (Gp) copy_row(Gp + rr * ldI, g + (size_t)p * VI, VI, lane);  // optional: the SwiGLU
    if (Up) copy_row(Up + rr * ldI, u + (size_t)p * VI, VI, lane);  // epilogue can gather g, u
  }
}

// acc += the 16-byte vector v (fp32 adds, element by element)
template <lrmoe_dtype DT>
__device__ __forceinline__ void add_vec(float (&acc)[DT == LRMOE_BF16 ? 8 : 4], const uint4& v) {
  if constexpr (DT == LRMOE_BF16) {
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] = __fadd_rn(acc[2 * q], bf16_bits_to_f32(ww[q] & 0xffffu));
      acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], bf16_bits_to_f32(ww[q] >> 16));
    }
  } else {
    acc[0] = __fadd_rn(acc[0], __uint_as_float(v.x));
    acc[1] = __fadd_rn(acc[1], __uint_as_float(v.y));
    acc[2] = __fadd_rn(acc[2], __uint_as_float(v.z));
    acc[3] = __fadd_rn(acc[3], __uint_as_float(v.w));
  }
}

// the sums rounded once to the storage type
template <lrmoe_dtype DT>
__device__ __forceinline__ uint4 to_vec(const float (&acc)[DT == LRMOE_BF16 ? 8 : 4]) {
  if constexpr (DT == LRMOE_BF16) {
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  } else {
    return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                      __float_as_uint(acc[3]));
  }
}

// dX[t] = sum over retained slots j (ascending) of dXp[pos[t*k+j]], fp32, rounded once.
// A token's loads form one list, column chunk by column chunk (32 vectors each),
// retained rows in ascending slot order inside a chunk; the warp issues
// kUnpackLoads of them at once, so a token with n retained rows needs about
// ceil(n * chunks / kUnpackLoads) memory round trips rather than one per chunk.
template <lrmoe_dtype DT>
__global__ void __launch_bounds__(256) unpack_kernel(const uint4* __restrict__ dXp, int rows_cap,
                                                     const int32_t* __restrict__ pos, int T,
                                                     int k, int VH, uint4* __restrict__ dX,
                                                     uint32_t* __restrict__ status) {
  constexpr int PER = DT == LRMOE_BF16 ? 8 : 4;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int stride = gridDim.x * wpb;
  int t = blockIdx.x * wpb + (threadIdx.x >> 5);
  // the next token's slots are loaded while this token's rows are in flight
  int r_next = (t < T && lane < k) ? __ldg(pos + (size_t)t * k + lane) : -1;
  for (; t < T; t += stride) {
    // retained rows of this token, in ascending slot order (k <= 32)
    int r = r_next;
    {
      const int tn = t + stride;
      r_next = (tn < T && lane < k) ? __ldg(pos + (size_t)tn * k + lane) : -1;
    }
    if (r >= rows_cap) {
      raise_status(status, LRMOE_ST_BAD_INDEX);
      r = -1;
    }
    const unsigned have = __ballot_sync(kFull, r >= 0);
    const int nrows = __popc(have);
    int comp = 0;  // lane i: packed row of the i-th retained slot (ascending slot order)
    {
      unsigned todo = have;
      for (int i = 0; todo; ++i) {
        const int rj = __shfl_sync(kFull, r, __ffs(todo) - 1);
        if (lane == i) comp = rj;
        todo &= todo - 1;
      }
    }
    uint4* __restrict__ out = dX + (size_t)t * VH;
    if (nrows == 0) {
      for (int c = lane; c < VH; c += 32) out[c] = make_uint4(0, 0, 0, 0);
      continue;
    }
    // item i = (chunk i / nrows, row i % nrows); nrows, items, ch and ri are warp-uniform
    const int items = ((VH + 31) >> 5) * nrows;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    int ch = 0, ri = 0;  // chunk and row of item i0
    for (int i0 = 0; i0 < items; i0 += kUnpackLoads) {
      uint4 v[kUnpackLoads];
      {
        int c2 = ch, r2 = ri;
#pragma unroll
        for (int q = 0; q < kUnpackLoads; ++q) {
          const int row = __shfl_sync(kFull, comp, r2);
          const int c = (c2 << 5) + lane;
          v[q] = (i0 + q < items && c < VH) ? __ldg(dXp + (size_t)row * VH + c)
                                            : make_uint4(0, 0, 0, 0);
          if (++r2 == nrows) {
            r2 = 0;
            ++c2;
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kUnpackLoads; ++q) {
        if (i0 + q >= items) break;
        add_vec<DT>(acc, v[q]);
        if (++ri == nrows) {  // the chunk's last retained row: store, start the next chunk
          const int c = (ch << 5) + lane;
          if (c < VH) out[c] = to_vec<DT>(acc);
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
          ri = 0;
          ++ch;
        }
      }
    }
  }
}

// dst[i] = src[idx[i]] (rows of V 16-byte vectors); bad indices flagged, row skipped.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src, int n_src,
                                                          const int32_t* __restrict__ idx, int n,
                                                          int V, uint4* __restrict__ dst,
                                                          uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  pdl_wait();
  pdl_trigger();
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const int r = idx[i];
    if (r < 0 || r >= n_src) {
      if (lane == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
      continue;
    }
    copy_row(dst + (size_t)i * V, src + (size_t)r * V, V, lane);
  }
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx,
                               int n, void* dst, uint32_t* status, cudaStream_t s) {
  const int V = row_bytes / 16;
  int blocks = (n + 7) / 8;
  const int maxb = num_sms() * 8;
  if (blocks > maxb) blocks = maxb;
  if (blocks < 1) blocks = 1;
  return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, s,
                    static_cast<const uint4*>(src), n_src, idx, n, V, static_cast<uint4*>(dst),
                    status);
}

cudaError_t launch_pack(const int32_t* perm, const int32_t* offsets, const float* w, int T,
                        int k, int E, const void* x, const void* dY, int H, const void* a,
                        const void* g, const void* u, int I, lrmoe_dtype dt, void* Xp, void* DYp,
                        void* Ap, void* Gp, void* Up, int rows_cap, uint32_t* status,
                        cudaStream_t s) {
  const int per = dt == LRMOE_BF16 ? 8 : 4;
  const int VH = H / per, VI = I / per;
  auto X = static_cast<const uint4*>(x);
  auto D = static_cast<const uint4*>(dY);
  auto A = static_cast<const uint4*>(a);
  auto G = static_cast<const uint4*>(g);
  auto U = static_cast<const uint4*>(u);
  // one resident wave (the row count lives on the device; a grid-stride loop)
  const int blocks = dt == LRMOE_BF16 ? rowred::grid_for<pack_kernel<LRMOE_BF16>>(rows_cap)
                                      : rowred::grid_for<pack_kernel<LRMOE_F32>>(rows_cap);
  auto kern = dt == LRMOE_BF16 ? pack_kernel<LRMOE_BF16> : pack_kernel<LRMOE_F32>;
  return launch_pdl(kern, dim3(blocks), dim3(256), 0, s, perm, offsets, E, w, T * k, k, X, D, VH,
                    A, G, U, VI, static_cast<uint4*>(Xp), static_cast<uint4*>(DYp),
                    static_cast<uint4*>(Ap), static_cast<uint4*>(Gp), static_cast<uint4*>(Up), VH,
                    VI, rows_cap, status);
}

// Exchange rows: packed row r = [x_t | RNE(w_p dY_t) | a_p | g_p | u_p] side by side
// (2H + 3I elements), so that one all-to-all moves every operand of a pair.
cudaError_t launch_pack_wide(const int32_t* perm, const int32_t* offsets, const float* w, int T,
                             int k, int E, const void* x, const void* dY, int H, const void* a,
                             const void* g, const void* u, int I, lrmoe_dtype dt, void* rows,
                             int rows_cap, uint32_t* status, cudaStream_t s) {
  const int per = dt == LRMOE_BF16 ? 8 : 4;
  const int VH = H / per, VI = I / per;
  const int W = 2 * VH + 3 * VI;
  uint4* base = static_cast<uint4*>(rows);
  const int blocks = dt == LRMOE_BF16 ? rowred::grid_for<pack_kernel<LRMOE_BF16>>(rows_cap)
                                      : rowred::grid_for<pack_kernel<LRMOE_F32>>(rows_cap);
  auto kern = dt == LRMOE_BF16 ? pack_kernel<LRMOE_BF16> : pack_kernel<LRMOE_F32>;
  return launch_pdl(kern, dim3(blocks), dim3(256), 0, s, perm, offsets, E, w, T * k, k,
                    static_cast<const uint4*>(x), static_cast<const uint4*>(dY), VH,
                    static_cast<const uint4*>(a), static_cast<const uint4*>(g),
                    static_cast<const uint4*>(u), VI, base, base + VH, base + 2 * VH,
                    base + 2 * VH + VI, base + 2 * VH + 2 * VI, W, W, rows_cap, status);
}

// dst operand rows i = the column blocks of exchange row idx[i] (bad indices
// flagged, row skipped).
__global__ void __launch_bounds__(256) split_wide_kernel(const uint4* __restrict__ rows, int n_src,
                                                         const int32_t* __restrict__ idx, int n,
                                                         int VH, int VI, uint4* __restrict__ Xp,
                                                         uint4* __restrict__ DYp,
                                                         uint4* __restrict__ Ap,
                                                         uint4* __restrict__ Gp,
                                                         uint4* __restrict__ Up,
                                                         uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int W = 2 * VH + 3 * VI;
  pdl_wait();
  pdl_trigger();
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const int r = idx[i];
    if (r < 0 || r >= n_src) {
      if (lane == 0) raise_status(status, LRMOE_ST_BAD_INDEX);
      continue;
    }
    const uint4* src = rows + (size_t)r * W;
    const size_t ii = (size_t)i;
    copy_row(Xp + ii * VH, src, VH, lane);
    copy_row(DYp + ii * VH, src + VH, VH, lane);
    copy_row(Ap + ii * VI, src + 2 * VH, VI, lane);
    copy_row(Gp + ii * VI, src + 2 * VH + VI, VI, lane);
    copy_row(Up + ii * VI, src + 2 * VH + 2 * VI, VI, lane);
  }
}

cudaError_t launch_split_wide(const void* rows, int n_src, const int32_t* idx, int n, int H, int I,
                              lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
                              uint32_t* status, cudaStream_t s) {
  const int per = dt == LRMOE_BF16 ? 8 : 4;
  int blocks = (n + 7) / 8;
  const int maxb = num_sms() * 8;
  if (blocks > maxb) blocks = maxb;
  if (blocks < 1) blocks = 1;
  return launch_pdl(split_wide_kernel, dim3(blocks), dim3(256), 0, s,
                    static_cast<const uint4*>(rows), n_src, idx, n, H / per, I / per,
                    static_cast<uint4*>(Xp), static_cast<uint4*>(DYp), static_cast<uint4*>(Ap),
                    static_cast<uint4*>(Gp), static_cast<uint4*>(Up), status);
}

cudaError_t launch_unpack(const void* dXp, int rows_cap, const int32_t* pos, int T, int k, int H,
                          lrmoe_dtype dt, void* dX, uint32_t* status, cudaStream_t s) {
  const int per = dt == LRMOE_BF16 ? 8 : 4;
  const int VH = H / per;
  // a warp per token (up to eight blocks per SM, then a grid-stride loop); one
  // resident wave with two tokens per warp measured slower
  const int wpb = 8;
  int blocks = (T + wpb - 1) / wpb;
  const int maxb = num_sms() * 8;
  if (blocks > maxb) blocks = maxb;
  auto kern = dt == LRMOE_BF16 ? unpack_kernel<LRMOE_BF16> : unpack_kernel<LRMOE_F32>;
  return launch_pdl(kern, dim3(blocks), dim3(256), 0, s, static_cast<const uint4*>(dXp), rows_cap,
                    pos, T, k, VH, static_cast<uint4*>(dX), status);
}

}  // namespace lrmoe
