// extern "C" entry points of liblrmoe.so: argument checks, then the launchers.
// Host-visible problems return a status code before anything is enqueued.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "../../include/lrmoe.h"
#include "launch.h"

namespace lrmoe {

static thread_local char g_last_error[512] = "";

static int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

static int cuda_fail(cudaError_t e, const char* where) {
  return fail(LRMOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// SM count of the current device, looked up once per device ordinal (it does
// not change while the process runs); safe to call from several host threads.
int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) dev = 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int elem_multiple(lrmoe_dtype dt) { return dt == LRMOE_BF16 ? 8 : 4; }

static bool valid_dtype(lrmoe_dtype dt) { return dt == LRMOE_F32 || dt == LRMOE_BF16; }

#define REQUIRE(cond, ...)                                 \
  do {                                                     \
    if (!(cond)) return fail(LRMOE_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p) REQUIRE((p) != nullptr && aligned16(p), "%s is null or not 16-byte aligned", #p)

static int check_feature(int n, lrmoe_dtype dt, const char* name) {
  if (n <= 0 || n % elem_multiple(dt))
    return fail(LRMOE_ERR_INVALID_ARG, "%s=%d must be a positive multiple of %d", name, n,
                elem_multiple(dt));
  return LRMOE_OK;
}

static int check_pairs(int T, int k, int E) {
  REQUIRE(T > 0 && k > 0 && E > 0, "T, k, E must be positive (T=%d k=%d E=%d)", T, k, E);
  REQUIRE(k <= 32, "k=%d > 32 is not supported", k);
  REQUIRE((long long)T * k < (1LL << 31) - 1, "T*k overflows int32");
  return LRMOE_OK;
}

}  // namespace lrmoe

using namespace lrmoe;

extern "C" {

int lrmoe_version(void) { return (1 << 16) | 0; }

const char* lrmoe_status_string(int code) {
  switch (code) {
    case LRMOE_OK: return "ok";
    case LRMOE_ERR_INVALID_ARG: return "invalid argument";
    case LRMOE_ERR_UNSUPPORTED: return "unsupported";
    case LRMOE_ERR_CUDA: return "CUDA error";
    case LRMOE_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

const char* lrmoe_last_error(void) { return g_last_error; }

int lrmoe_score(const int32_t* topk_idx, const float* topk_w, int T, int k, int E,
                const void* dY, int H, const void* a_saved, int D, lrmoe_dtype dt,
                float* score, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (int r = check_pairs(T, k, E)) return r;
  if (int r = check_feature(H, dt, "H")) return r;
  if (int r = check_feature(D, dt, "D")) return r;
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(topk_w);
  REQUIRE_PTR(dY);
  REQUIRE_PTR(a_saved);
  REQUIRE_PTR(score);
  cudaError_t e = launch_score(topk_idx, topk_w, T, k, E, dY, H, a_saved, D, dt, score, status,
                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_score launch");
}

int lrmoe_row_sqnorm(const void* rows, int n_rows, int D, lrmoe_dtype dt, float* out,
                     void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  REQUIRE(n_rows > 0, "n_rows=%d must be positive", n_rows);
  if (int r = check_feature(D, dt, "D")) return r;
  REQUIRE_PTR(rows);
  REQUIRE_PTR(out);
  cudaError_t e = launch_row_sqnorm(rows, n_rows, D, dt, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_row_sqnorm launch");
}

int lrmoe_score_from_norms(const int32_t* topk_idx, const float* topk_w, int T, int k, int E,
                           const void* dY, int H, const float* a_sqnorm, lrmoe_dtype dt,
                           float* score, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (int r = check_pairs(T, k, E)) return r;
  if (int r = check_feature(H, dt, "H")) return r;
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(topk_w);
  REQUIRE_PTR(dY);
  REQUIRE_PTR(a_sqnorm);
  REQUIRE_PTR(score);
  cudaError_t e = launch_score_from_norms(topk_idx, topk_w, T, k, E, dY, H, a_sqnorm, dt, score,
                                          status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_score_from_norms launch");
}

int lrmoe_router_grad(const int32_t* topk_idx, int T, int k, int E, const void* dY, int H,
                      const void* y_saved, lrmoe_dtype dt, const int32_t* pos, float* dw,
                      uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (int r = check_pairs(T, k, E)) return r;
  if (int r = check_feature(H, dt, "H")) return r;
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(dY);
  REQUIRE_PTR(y_saved);
  REQUIRE_PTR(dw);
  REQUIRE(pos == nullptr || aligned16(pos), "pos is not 16-byte aligned");
  cudaError_t e = launch_router_grad(topk_idx, T, k, E, dY, H, y_saved, dt, pos, dw, status,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_router_grad launch");
}

int lrmoe_redistribute(const int64_t* m, const uint8_t* admissible, int E, int G, int64_t* plan,
                       int64_t* peak) {
  g_last_error[0] = 0;
  REQUIRE(E > 0 && G > 0, "E=%d and G=%d must be positive", E, G);
  REQUIRE(E <= 65536 && G <= 4096, "E=%d or G=%d too large for the planner", E, G);
  REQUIRE(m != nullptr && admissible != nullptr && plan != nullptr && peak != nullptr,
          "m, admissible, plan and peak must be non-null host pointers");
  for (int e = 0; e < E; ++e) {
    REQUIRE(m[e] >= 0, "m[%d]=%lld is negative", e, (long long)m[e]);
    bool any = false;
    for (int g = 0; g < G; ++g) any = any || admissible[(size_t)e * G + g] != 0;
    REQUIRE(any || m[e] == 0, "expert %d has %lld retained pairs but no copy", e,
            (long long)m[e]);
  }
  if (redistribute_plan(m, admissible, E, G, plan, peak) != 0)
    return fail(LRMOE_ERR_INVALID_ARG, "no plan exists (an expert without a copy)");
  return LRMOE_OK;
}

int lrmoe_split_by_destination(const int32_t* perm, const int32_t* offsets, const int32_t* plan,
                               const int32_t* global_start, int E, int G, int rows_cap,
                               int32_t* perm_dest, int32_t* dest_offsets,
                               int32_t* dest_expert_offsets, int32_t* row_dest, uint32_t* status,
                               void* stream) {
  g_last_error[0] = 0;
  REQUIRE(E > 0 && E <= kMaxGroupedExperts, "E=%d must be in [1, %d]", E, kMaxGroupedExperts);
  REQUIRE(G > 0 && (size_t)E * G * sizeof(int) <= 200 * 1024, "G=%d out of range for E=%d", G, E);
  REQUIRE(rows_cap > 0, "rows_cap=%d must be positive", rows_cap);
  REQUIRE_PTR(perm);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(plan);
  REQUIRE_PTR(perm_dest);
  REQUIRE_PTR(dest_offsets);
  REQUIRE_PTR(dest_expert_offsets);
  REQUIRE(global_start == nullptr || aligned16(global_start), "global_start is not 16-byte aligned");
  REQUIRE(row_dest == nullptr || aligned16(row_dest), "row_dest is not 16-byte aligned");
  cudaError_t e = launch_split_by_destination(perm, offsets, plan, global_start, E, G, rows_cap,
                                              perm_dest, dest_offsets, dest_expert_offsets,
                                              row_dest, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_split_by_destination launch");
}

int lrmoe_group_received(const int32_t* src_expert_offsets, int G, int E, int rows_cap,
                         int32_t* order, int32_t* inv, int32_t* offsets, uint32_t* status,
                         void* stream) {
  g_last_error[0] = 0;
  REQUIRE(E > 0 && E <= kMaxGroupedExperts, "E=%d must be in [1, %d]", E, kMaxGroupedExperts);
  REQUIRE(G > 0 && (size_t)E * G * sizeof(int) <= 200 * 1024, "G=%d out of range for E=%d", G, E);
  REQUIRE(rows_cap > 0, "rows_cap=%d must be positive", rows_cap);
  REQUIRE_PTR(src_expert_offsets);
  REQUIRE_PTR(order);
  REQUIRE_PTR(inv);
  REQUIRE_PTR(offsets);
  cudaError_t e = launch_group_received(src_expert_offsets, G, E, rows_cap, order, inv, offsets,
                                        status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_group_received launch");
}

int lrmoe_pack_wide(const int32_t* perm, const int32_t* offsets, const float* topk_w, int T, int k,
                    int E, const void* x, const void* dY, int H, const void* a, const void* g,
                    const void* u, int I, lrmoe_dtype dt, void* rows, int rows_cap,
                    uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (int r = check_pairs(T, k, E)) return r;
  if (int r = check_feature(H, dt, "H")) return r;
  if (int r = check_feature(I, dt, "I")) return r;
  REQUIRE(rows_cap > 0, "rows_cap must be positive");
  REQUIRE_PTR(perm);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(topk_w);
  REQUIRE_PTR(x);
  REQUIRE_PTR(dY);
  REQUIRE_PTR(a);
  REQUIRE_PTR(g);
  REQUIRE_PTR(u);
  REQUIRE_PTR(rows);
  cudaError_t e = launch_pack_wide(perm, offsets, topk_w, T, k, E, x, dY, H, a, g, u, I, dt, rows,
                                   rows_cap, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_pack_wide launch");
}

int lrmoe_split_wide(const void* rows, int n_src, const int32_t* idx, int n, int H, int I,
                     lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
                     uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  REQUIRE(n >= 0 && n_src > 0, "n=%d must be >= 0 and n_src=%d positive", n, n_src);
  if (int r = check_feature(H, dt, "H")) return r;
  if (int r = check_feature(I, dt, "I")) return r;
  REQUIRE_PTR(rows);
  REQUIRE_PTR(idx);
  REQUIRE_PTR(Xp);
  REQUIRE_PTR(DYp);
  REQUIRE_PTR(Ap);
  REQUIRE_PTR(Gp);
  REQUIRE_PTR(Up);
  if (n == 0) return LRMOE_OK;
  cudaError_t e = launch_split_wide(rows, n_src, idx, n, H, I, dt, Xp, DYp, Ap, Gp, Up, status,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_split_wide launch");
}

size_t lrmoe_select_workspace_bytes(int T, int k, int E) {
  if (T <= 0 || k <= 0 || E <= 0) return 0;
  return select_ws_layout(T, k, E).total;
}

int lrmoe_select_quota(const int32_t* topk_idx, const float* score, int T, int k, int E,
                       const int32_t* quota, int32_t* counts, int32_t* kept, int32_t* offsets,
                       int32_t* perm, int32_t* pos, void* workspace, size_t workspace_bytes,
                       uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  if (int r = check_pairs(T, k, E)) return r;
  if (E > 4096) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > 4096", E);
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(score);
  REQUIRE_PTR(quota);
  REQUIRE_PTR(counts);
  REQUIRE_PTR(kept);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(perm);
  REQUIRE_PTR(pos);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(LRMOE_ERR_WORKSPACE, "workspace is null or not 256-byte aligned");
  const size_t need = select_ws_layout(T, k, E).total;
  if (workspace_bytes < need)
    return fail(LRMOE_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  cudaError_t e = launch_select(topk_idx, score, T, k, E, quota, counts, kept, offsets, perm, pos,
                                workspace, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_select_quota launch");
}

int lrmoe_quota_controller(const int32_t* topk_idx, int T, int k, int E, int32_t cap,
                           int64_t max_pairs, int32_t* quota, int32_t* counts, uint32_t* status,
                           void* stream) {
  g_last_error[0] = 0;
  if (int r = check_pairs(T, k, E)) return r;
  if (E > 4096) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > 4096", E);
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(quota);
  REQUIRE_PTR(counts);
  cudaError_t e = launch_quota(topk_idx, T * k, E, cap, (long long)max_pairs, quota, counts,
                               status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_quota_controller launch");
}

// Selection for callers that cannot provide device scratch: the kernels use a
// fixed array inside the library instead (see select.cu).  Nothing here or
// below allocates.
int lrmoe_select_quota_noalloc(const int32_t* topk_idx, const float* score, int T, int k, int E,
                               const int32_t* quota, int32_t* counts, int32_t* kept,
                               int32_t* offsets, int32_t* perm, int32_t* pos, uint32_t* status,
                               void* stream) {
  g_last_error[0] = 0;
  if (int r = check_pairs(T, k, E)) return r;
  if (E > 4096) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > 4096", E);
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(score);
  REQUIRE_PTR(quota);
  REQUIRE_PTR(counts);
  REQUIRE_PTR(kept);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(perm);
  REQUIRE_PTR(pos);
  const size_t need = select_ws_layout(T, k, E).total;
  const size_t have = select_noalloc_scratch_bytes();
  if (need > have)
    return fail(LRMOE_ERR_WORKSPACE,
                "T*k=%lld pairs need %zu bytes of scratch, more than the %zu-byte built-in "
                "array; call lrmoe_select_quota with a workspace instead",
                (long long)T * k, need, have);
  cudaError_t e = launch_select_noalloc(topk_idx, score, T, k, E, quota, counts, kept, offsets,
                                        perm, pos, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_select_quota_noalloc");
}

int lrmoe_pack(const int32_t* perm, const int32_t* offsets, const float* topk_w, int T, int k, int E,
               const void* x, const void* dY, int H, const void* a, const void* g, const void* u,
               int I, lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
               int rows_cap, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (int r = check_pairs(T, k, E)) return r;
  if (int r = check_feature(H, dt, "H")) return r;
  if (int r = check_feature(I, dt, "I")) return r;
  REQUIRE(rows_cap > 0, "rows_cap must be positive");
  REQUIRE_PTR(perm);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(topk_w);
  REQUIRE_PTR(dY);
  REQUIRE_PTR(DYp);
  if (Xp) {  // X_p and A_p are optional too (the gathering wgrad reads x, a in place)
    REQUIRE_PTR(x);
    REQUIRE_PTR(Xp);
  }
  if (Ap) {
    REQUIRE_PTR(a);
    REQUIRE_PTR(Ap);
  }
  REQUIRE((Gp == nullptr) == (Up == nullptr), "Gp and Up must both be given or both be NULL");
  if (Gp) {  // G_p, U_p are optional (the gathering SwiGLU epilogue reads g, u in place)
    REQUIRE_PTR(g);
    REQUIRE_PTR(u);
    REQUIRE_PTR(Gp);
    REQUIRE_PTR(Up);
  }
  cudaError_t e = launch_pack(perm, offsets, topk_w, T, k, E, x, dY, H, a, g, u, I, dt, Xp, DYp, Ap,
                              Gp, Up, rows_cap, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_pack launch");
}

int lrmoe_grouped_dgrad(const void* rows, int rows_cap, const void* W, const int32_t* offsets,
                        int E, int K, int N, lrmoe_dtype dt, lrmoe_epilogue epi,
                        const void* Gp, const void* Up, void* out, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  REQUIRE(epi == LRMOE_EPI_STORE || epi == LRMOE_EPI_SWIGLU_BWD, "unknown epilogue %d", (int)epi);
  REQUIRE(E > 0 && rows_cap > 0, "E and rows_cap must be positive");
  if (E > kMaxGroupedExperts) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > %d", E, kMaxGroupedExperts);
  if (int r = check_feature(K, dt, "K")) return r;
  if (int r = check_feature(N, dt, "N")) return r;
  REQUIRE_PTR(rows);
  REQUIRE_PTR(W);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(out);
  if (epi == LRMOE_EPI_SWIGLU_BWD) {
    REQUIRE_PTR(Gp);
    REQUIRE_PTR(Up);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dt == LRMOE_BF16) {
    const char* why = "launch failed";
    e = launch_dgrad_tc(rows, rows_cap, W, offsets, E, K, N, epi, Gp, Up, out, status, s, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
  } else {
    e = launch_dgrad_simt(rows, rows_cap, W, offsets, E, K, N, dt, epi, Gp, Up, out, status, s);
    if (e != cudaSuccess) return cuda_fail(e, "lrmoe_grouped_dgrad launch");
  }
  return LRMOE_OK;
}

int lrmoe_grouped_dgrad_swiglu_gather(const void* rows, int rows_cap, const void* W,
                                      const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                                      const int32_t* perm, const void* g, const void* u, int gu_rows,
                                      void* out, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (dt != LRMOE_BF16)
    return fail(LRMOE_ERR_UNSUPPORTED, "the gathering epilogue is bf16 only; pack G_p, U_p");
  REQUIRE(E > 0 && rows_cap > 0 && gu_rows > 0, "E, rows_cap and gu_rows must be positive");
  if (E > kMaxGroupedExperts) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > %d", E, kMaxGroupedExperts);
  if (int r = check_feature(K, dt, "K")) return r;
  if (int r = check_feature(N, dt, "N")) return r;
  REQUIRE_PTR(rows);
  REQUIRE_PTR(W);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(perm);
  REQUIRE_PTR(g);
  REQUIRE_PTR(u);
  REQUIRE_PTR(out);
  const char* why = "launch failed";
  cudaError_t e = launch_dgrad_tc(rows, rows_cap, W, offsets, E, K, N, LRMOE_EPI_SWIGLU_BWD, g, u,
                                  out, status, static_cast<cudaStream_t>(stream), &why, perm,
                                  gu_rows);
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, why);
}

int lrmoe_grouped_wgrad_gather(const void* grad_rows, int rows_cap, const int32_t* perm,
                               const void* src, int src_div, int n_pairs, const int32_t* offsets,
                               int E, int N1, int N2, lrmoe_dtype dt, float* dW, int accumulate,
                               uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (dt != LRMOE_BF16)
    return fail(LRMOE_ERR_UNSUPPORTED, "the gathering wgrad is bf16 only; pack the rows");
  REQUIRE(E > 0 && rows_cap > 0 && n_pairs > 0, "E, rows_cap and n_pairs must be positive");
  REQUIRE(src_div > 0 && n_pairs % src_div == 0, "src_div=%d must divide n_pairs=%d", src_div,
          n_pairs);
  if (E > kMaxGroupedExperts) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > %d", E, kMaxGroupedExperts);
  if (int r = check_feature(N1, dt, "N1")) return r;
  if (int r = check_feature(N2, dt, "N2")) return r;
  REQUIRE_PTR(grad_rows);
  REQUIRE_PTR(perm);
  REQUIRE_PTR(src);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(dW);
  const char* why = "launch failed";
  cudaError_t e = launch_wgrad_gather_tc(grad_rows, rows_cap, perm, src, src_div, n_pairs, offsets,
                                         E, N1, N2, dW, accumulate, status,
                                         static_cast<cudaStream_t>(stream), &why);
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, why);
}

int lrmoe_grouped_wgrad(const void* grad_rows, const void* in_rows, int rows_cap,
                        const int32_t* offsets, int E, int N1, int N2, lrmoe_dtype dt, float* dW,
                        int accumulate, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  REQUIRE(E > 0 && rows_cap > 0, "E and rows_cap must be positive");
  if (E > kMaxGroupedExperts) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > %d", E, kMaxGroupedExperts);
  if (int r = check_feature(N1, dt, "N1")) return r;
  if (int r = check_feature(N2, dt, "N2")) return r;
  REQUIRE_PTR(grad_rows);
  REQUIRE_PTR(in_rows);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(dW);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dt == LRMOE_BF16) {
    const char* why = "launch failed";
    e = launch_wgrad_tc(grad_rows, in_rows, rows_cap, offsets, E, N1, N2, dW, accumulate, status, s,
                        &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
  } else {
    e = launch_wgrad_simt(grad_rows, in_rows, rows_cap, offsets, E, N1, N2, dt, dW, accumulate,
                          status, s);
    if (e != cudaSuccess) return cuda_fail(e, "lrmoe_grouped_wgrad launch");
  }
  return LRMOE_OK;
}

int lrmoe_grouped_dgrad_wgrad(const void* grad_rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                              lrmoe_epilogue epi, const void* Gp, const void* Up, void* out,
                              const void* in_rows, int N2, float* dW, int accumulate,
                              uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  if (dt != LRMOE_BF16)
    return fail(LRMOE_ERR_UNSUPPORTED, "the fused launch is bf16 only; use the two calls");
  REQUIRE(epi == LRMOE_EPI_STORE || epi == LRMOE_EPI_SWIGLU_BWD, "unknown epilogue %d", (int)epi);
  REQUIRE(E > 0 && rows_cap > 0, "E and rows_cap must be positive");
  if (E > kMaxGroupedExperts) return fail(LRMOE_ERR_UNSUPPORTED, "E=%d > %d", E, kMaxGroupedExperts);
  if (int r = check_feature(K, dt, "K")) return r;
  if (int r = check_feature(N, dt, "N")) return r;
  if (int r = check_feature(N2, dt, "N2")) return r;
  REQUIRE_PTR(grad_rows);
  REQUIRE_PTR(W);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(out);
  REQUIRE_PTR(in_rows);
  REQUIRE_PTR(dW);
  if (epi == LRMOE_EPI_SWIGLU_BWD) {
    REQUIRE_PTR(Gp);
    REQUIRE_PTR(Up);
  }
  const char* why = "launch failed";
  cudaError_t e = launch_dgrad_wgrad_tc(grad_rows, rows_cap, W, offsets, E, K, N, epi, Gp, Up, out,
                                        in_rows, N2, dW, accumulate, status,
                                        static_cast<cudaStream_t>(stream), &why);
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, why);
}

int lrmoe_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx, int n,
                      void* dst, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(n >= 0 && n_src > 0, "n=%d must be >= 0 and n_src=%d positive", n, n_src);
  REQUIRE(row_bytes > 0 && row_bytes % 16 == 0, "row_bytes=%d must be a positive multiple of 16",
          row_bytes);
  REQUIRE_PTR(src);
  REQUIRE_PTR(idx);
  REQUIRE_PTR(dst);
  if (n == 0) return LRMOE_OK;
  cudaError_t e = launch_gather_rows(src, n_src, row_bytes, idx, n, dst, status,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_gather_rows launch");
}

int lrmoe_unpack(const void* dXp, int rows_cap, const int32_t* pos, int T, int k, int H,
                 lrmoe_dtype dt, void* dX, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  REQUIRE(T > 0 && k > 0 && rows_cap > 0, "T, k, rows_cap must be positive");
  REQUIRE(k <= 32, "k=%d > 32 is not supported", k);
  if (int r = check_feature(H, dt, "H")) return r;
  REQUIRE_PTR(dXp);
  REQUIRE_PTR(pos);
  REQUIRE_PTR(dX);
  cudaError_t e = launch_unpack(dXp, rows_cap, pos, T, k, H, dt, dX, status,
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_unpack launch");
}

int lrmoe_selftest_bounded_wait(uint32_t limit_us, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) == 0,
          "status is null or misaligned");
  REQUIRE(limit_us >= 1 && limit_us <= 1000000u, "limit_us=%u outside [1, 1000000]", limit_us);
  cudaError_t e = launch_selftest_wait(limit_us, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_selftest_bounded_wait launch");
}

int lrmoe_selftest_gemm_stall(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, void* out, int two_sm,
                              uint32_t limit_us, uint32_t* status, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) == 0,
          "status is null or misaligned");
  REQUIRE(limit_us >= 1 && limit_us <= 1000000u, "limit_us=%u outside [1, 1000000]", limit_us);
  REQUIRE(E > 0 && E <= kMaxGroupedExperts && rows_cap > 0, "E or rows_cap out of range");
  if (int r = check_feature(K, LRMOE_BF16, "K")) return r;
  if (int r = check_feature(N, LRMOE_BF16, "N")) return r;
  REQUIRE_PTR(rows);
  REQUIRE_PTR(W);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned long long ns = 1000ull * limit_us;
  cudaError_t e = two_sm ? launch_dgrad_stall_pair(rows, rows_cap, W, offsets, E, K, N, out, ns,
                                                   status, s)
                         : launch_dgrad_stall_tc(rows, rows_cap, W, offsets, E, K, N, out, ns,
                                                 status, s);
  return e == cudaSuccess ? LRMOE_OK : cuda_fail(e, "lrmoe_selftest_gemm_stall launch");
}

int lrmoe_pruned_backward(const lrmoe_buffers* b, int T, int k, int E, int H, int I,
                          int rows_cap, lrmoe_dtype dt, void* stream) {
  g_last_error[0] = 0;
  REQUIRE(b != nullptr, "buffers is null");
  REQUIRE(rows_cap > 0, "rows_cap must be positive");
  int r;
  if ((r = lrmoe_score(b->topk_idx, b->topk_w, T, k, E, b->dY, H, b->a, I, dt, b->score, b->status,
                       stream)))
    return r;
  if ((r = lrmoe_select_quota(b->topk_idx, b->score, T, k, E, b->quota, b->counts, b->kept,
                              b->offsets, b->perm, b->pos, b->workspace, b->workspace_bytes,
                              b->status, stream)))
    return r;
  if (dt == LRMOE_BF16) {
    // g, u are read in place by the SwiGLU epilogue (row perm[r]); only the
    // operands the tensor cores load with TMA are packed
    if ((r = lrmoe_pack(b->perm, b->offsets, b->topk_w, T, k, E, b->x, b->dY, H, b->a, nullptr,
                        nullptr, I, dt, b->Xp, b->DYp, b->Ap, nullptr, nullptr, rows_cap, b->status,
                        stream)))
      return r;
    if ((r = lrmoe_grouped_dgrad_swiglu_gather(b->DYp, rows_cap, b->W_down, b->offsets, E, H, I, dt,
                                               b->perm, b->g, b->u, T * k, b->dGUp, b->status,
                                               stream)))
      return r;
  } else {
    if ((r = lrmoe_pack(b->perm, b->offsets, b->topk_w, T, k, E, b->x, b->dY, H, b->a, b->g, b->u,
                        I, dt, b->Xp, b->DYp, b->Ap, b->Gp, b->Up, rows_cap, b->status, stream)))
      return r;
    // dA -> [dG | dU]  (m_e x H) . (H x I), SwiGLU backward in the epilogue
    if ((r = lrmoe_grouped_dgrad(b->DYp, rows_cap, b->W_down, b->offsets, E, H, I, dt,
                                 LRMOE_EPI_SWIGLU_BWD, b->Gp, b->Up, b->dGUp, b->status, stream)))
      return r;
  }
  // dW_down = DY_p^T A_p
  if ((r = lrmoe_grouped_wgrad(b->DYp, b->Ap, rows_cap, b->offsets, E, H, I, dt, b->dW_down, 0,
                               b->status, stream)))
    return r;
  // dW_gu = dGU_p^T X_p
  if ((r = lrmoe_grouped_wgrad(b->dGUp, b->Xp, rows_cap, b->offsets, E, 2 * I, H, dt, b->dW_gu, 0,
                               b->status, stream)))
    return r;
  // dX_p = dGU_p W_gu
  if ((r = lrmoe_grouped_dgrad(b->dGUp, rows_cap, b->W_gu, b->offsets, E, 2 * I, H, dt,
                               LRMOE_EPI_STORE, nullptr, nullptr, b->dXp, b->status, stream)))
    return r;
  return lrmoe_unpack(b->dXp, rows_cap, b->pos, T, k, H, dt, b->dX, b->status, stream);
}

}  // extern "C"
