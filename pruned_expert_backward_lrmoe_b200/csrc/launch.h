// Internal launchers behind the C ABI (host side).  Arguments are already
// validated by abi.cu; each launcher only enqueues kernels on `s`.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/lrmoe.h"

namespace lrmoe {

// Largest expert count the grouped GEMMs build their tile table for.
constexpr int kMaxGroupedExperts = 1024;

// Launch `kernel` on `s` with programmatic stream serialization allowed, so
// that it may start while the previous kernel in the stream drains (the
// kernels order themselves with griddepcontrol.wait / launch_dependents).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int num_sms();

cudaError_t launch_score(const int32_t* idx, const float* w, int T, int k, int E, const void* dY,
                         int H, const void* a, int D, lrmoe_dtype dt, float* score,
                         uint32_t* status, cudaStream_t s);
cudaError_t launch_router_grad(const int32_t* idx, int T, int k, int E, const void* dY, int H,
                               const void* y, lrmoe_dtype dt, const int32_t* pos, float* dw,
                               uint32_t* status, cudaStream_t s);
int redistribute_plan(const int64_t* m, const uint8_t* adm, int E, int G, int64_t* x,
                      int64_t* peak);
cudaError_t launch_split_by_destination(const int32_t* perm, const int32_t* offsets,
                                        const int32_t* plan, const int32_t* start, int E, int G,
                                        int rows_cap, int32_t* perm_dest, int32_t* dest_offsets,
                                        int32_t* dest_expert_offsets, int32_t* row_dest,
                                        uint32_t* status, cudaStream_t s);
cudaError_t launch_group_received(const int32_t* tab, int G, int E, int rows_cap, int32_t* order,
                                  int32_t* inv, int32_t* offsets, uint32_t* status,
                                  cudaStream_t s);
cudaError_t launch_pack_wide(const int32_t* perm, const int32_t* offsets, const float* w, int T,
                             int k, int E, const void* x, const void* dY, int H, const void* a,
                             const void* g, const void* u, int I, lrmoe_dtype dt, void* rows,
                             int rows_cap, uint32_t* status, cudaStream_t s);
cudaError_t launch_split_wide(const void* rows, int n_src, const int32_t* idx, int n, int H, int I,
                              lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
                              uint32_t* status, cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx,
                               int n, void* dst, uint32_t* status, cudaStream_t s);
cudaError_t launch_row_sqnorm(const void* rows, int n, int D, lrmoe_dtype dt, float* out,
                              cudaStream_t s);
cudaError_t launch_score_from_norms(const int32_t* idx, const float* w, int T, int k, int E,
                                    const void* dY, int H, const float* a_sqnorm, lrmoe_dtype dt,
                                    float* score, uint32_t* status, cudaStream_t s);

struct SelectWs {
  int chunk;        // pairs per chunk
  int nchunks;
  size_t off_cc, off_seg_start, off_seg_p, off_seg_key, total;
};
SelectWs select_ws_layout(int T, int k, int E);

cudaError_t launch_select(const int32_t* idx, const float* score, int T, int k, int E,
                          const int32_t* quota, int32_t* counts, int32_t* kept, int32_t* offsets,
                          int32_t* perm, int32_t* pos, void* ws, uint32_t* status,
                          cudaStream_t s);

// Selection with the library's built-in scratch array (no caller workspace).
size_t select_noalloc_scratch_bytes();
cudaError_t launch_select_noalloc(const int32_t* idx, const float* score, int T, int k, int E,
                                  const int32_t* quota, int32_t* counts, int32_t* kept,
                                  int32_t* offsets, int32_t* perm, int32_t* pos, uint32_t* status,
                                  cudaStream_t s);

cudaError_t launch_pack(const int32_t* perm, const int32_t* offsets, const float* w, int T,
                        int k, int E, const void* x, const void* dY, int H, const void* a,
                        const void* g, const void* u, int I, lrmoe_dtype dt, void* Xp, void* DYp,
                        void* Ap, void* Gp, void* Up, int rows_cap, uint32_t* status,
                        cudaStream_t s);

cudaError_t launch_unpack(const void* dXp, int rows_cap, const int32_t* pos, int T, int k, int H,
                          lrmoe_dtype dt, void* dX, uint32_t* status, cudaStream_t s);

// fp32 FFMA grouped GEMMs (fp32 storage)
cudaError_t launch_dgrad_simt(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                              lrmoe_epilogue epi, const void* Gp, const void* Up, void* out,
                              uint32_t* status, cudaStream_t s);
cudaError_t launch_wgrad_simt(const void* grad_rows, const void* in_rows, int rows_cap,
                              const int32_t* offsets, int E, int N1, int N2, lrmoe_dtype dt,
                              float* dW, int accumulate, uint32_t* status, cudaStream_t s);

// quota controller: water-filling of per-expert quotas under a cap and a pair budget
cudaError_t launch_quota(const int32_t* idx, int P, int E, int cap, long long budget,
                         int32_t* quota, int32_t* counts, uint32_t* status, cudaStream_t s);

// diagnostic: a bounded wait that must time out
cudaError_t launch_selftest_wait(uint32_t limit_us, uint32_t* status, cudaStream_t s);
// diagnostic: a grouped dgrad whose first K block never arrives (one-SM / two-SM tiles)
cudaError_t launch_dgrad_stall_tc(const void* rows, int rows_cap, const void* W,
                                  const int32_t* offsets, int E, int K, int N, void* out,
                                  unsigned long long wait_ns, uint32_t* status, cudaStream_t s);
cudaError_t launch_dgrad_stall_pair(const void* rows, int rows_cap, const void* W,
                                    const int32_t* offsets, int E, int K, int N, void* out,
                                    unsigned long long wait_ns, uint32_t* status, cudaStream_t s);

// tcgen05 grouped GEMMs (bf16 storage)
// perm != nullptr: the SwiGLU epilogue reads g, u ([gu_rows][N]) at row perm[r]
cudaError_t launch_dgrad_tc(const void* rows, int rows_cap, const void* W,
                            const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                            const void* Gp, const void* Up, void* out, uint32_t* status,
                            cudaStream_t s, const char** why, const int32_t* perm = nullptr,
                            int gu_rows = 0);
cudaError_t launch_wgrad_tc(const void* grad_rows, const void* in_rows, int rows_cap,
                            const int32_t* offsets, int E, int N1, int N2, float* dW,
                            int accumulate, uint32_t* status, cudaStream_t s, const char** why);
// the same GEMMs with one MMA per pair of SMs (two-CTA clusters, 256 x 256 tiles)
cudaError_t launch_dgrad_pair(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                              const void* Gp, const void* Up, void* out, uint32_t* status,
                              cudaStream_t s, const char** why, const int32_t* perm, int gu_rows,
                              int part);
cudaError_t launch_wgrad_pair(const void* grad_rows, const void* in_rows, int rows_cap,
                              const int32_t* offsets, int E, int N1, int N2, float* dW,
                              int accumulate, uint32_t* status, cudaStream_t s, const char** why);
cudaError_t launch_wgrad_gather_tc(const void* grad_rows, int rows_cap, const int32_t* perm,
                                   const void* src, int src_div, int perm_max,
                                   const int32_t* offsets, int E, int N1, int N2, float* dW,
                                   int accumulate, uint32_t* status, cudaStream_t s,
                                   const char** why);
cudaError_t launch_dgrad_wgrad_tc(const void* grad_rows, int rows_cap, const void* W,
                                  const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                                  const void* Gp, const void* Up, void* out, const void* in_rows,
                                  int N2, float* dW, int accumulate, uint32_t* status,
                                  cudaStream_t s, const char** why);

}  // namespace lrmoe
