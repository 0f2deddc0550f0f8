/*
 * lrmoe.h -- C ABI of the B200 (sm_100a) pruned MoE expert backward (LRMoE).
 *
 * The method (three news pages on LRMoE; sections cited per entry point):
 *   RU-B  = "LRMoE урезает обратный проход MoE и ускоряет обучение на 21–45%",
 *           section "Что делает LRMoE: полный прямой проход, обрезанный обратный"
 *   FR-B  = "LRMoE élague la passe arrière des MoE ...", section
 *           "Ce que fait LRMoE : passe avant complète, passe arrière élaguée"
 *   DE    = "LRMoE führt eine Nachkalibrierung der Last auf der Nachfrageseite ...",
 *           paragraphs 3 and 4
 *
 * Notation: T tokens, E experts, k routed experts per token, H hidden size,
 * I SwiGLU intermediate size.  Pair p = t*k + j is slot j of token t
 * (token-major).  c_e = routed count of expert e, q_e = quota,
 * m_e = min(max(q_e, 0), c_e) retained pairs, M = sum m_e.
 * Expert FFN: g = x W_gate^T, u = x W_up^T, a = silu(g) * u, y = a W_down^T,
 * layer output Y_t = sum_j w_tj y_{e(t,j)}.  Weights are stored row-major as
 * W_gu[E][2I][H] (gate rows 0..I-1, up rows I..2I-1) and W_down[E][H][I].
 *
 * Conventions shared by every entry point
 *   - Every data pointer is a DEVICE pointer, 16-byte aligned, rows contiguous
 *     and row-major.  `stream` is a cudaStream_t passed as void* (NULL = the
 *     legacy default stream).
 *   - The caller owns all memory.  The library allocates nothing.  Its only
 *     device-side state is fixed and internal: 64 pairs of tile counters that
 *     the grouped GEMMs use for dynamic tile scheduling (each launch takes the
 *     next pair and leaves it zeroed, so up to 64 grouped-GEMM launches may be
 *     in flight at once on one device), and the scratch array of
 *     lrmoe_select_quota_noalloc.  Calls are thread-safe on the host.
 *   - Calls only enqueue work on `stream` and never synchronise the host.
 *     Counts and offsets stay on the device; later kernels read them there.
 *   - Errors a host can see (null pointer, size <= 0, feature size not a
 *     multiple of 8 elements for bf16 or 4 for fp32, too small workspace, a
 *     failed launch) return a nonzero lrmoe_status before or instead of
 *     launching; nothing is written then.  lrmoe_last_error() describes it.
 *   - Errors that depend on data set bits in the optional device status word
 *     (`status`, uint32, may be NULL) with atomicOr; kernels then continue
 *     safely: an expert id >= E is skipped as a pair, a negative quota counts
 *     as 0.  The caller clears the word and reads it after its own sync.
 *   - topk_idx < 0 marks an empty slot (no pair).
 *   - Feature sizes H, I (and the GEMM sizes K, N, N1, N2) are multiples of 8
 *     elements for bf16 and of 4 for fp32.
 *   - Checked-index debug build (liblrmoe_checked.so, the same ABI compiled
 *     with -DLRMOE_CHECKED): indices the kernels derive from their inputs or
 *     from their own scans are also bounds-checked before use, including the
 *     grouped GEMMs' offsets (offsets[0] >= 0, rising, offsets[E] <= rows_cap;
 *     otherwise the launch computes nothing).  A failed check skips the access
 *     and sets LRMOE_ST_BAD_INDEX.  The normal build trusts those contracts.
 */
#ifndef LRMOE_H
#define LRMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LRMOE_OK = 0,
  LRMOE_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or enum */
  LRMOE_ERR_UNSUPPORTED = 2,  /* valid but outside what this build handles (e.g. E > 1024) */
  LRMOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a launch failed */
  LRMOE_ERR_WORKSPACE = 4     /* workspace pointer NULL or smaller than required */
} lrmoe_status;

/* Storage type of activations, gradients and weights.  Arithmetic is fp32
 * (score, pack, unpack, fp32 GEMMs) or bf16 x bf16 -> fp32 (tensor-core GEMMs). */
typedef enum { LRMOE_F32 = 0, LRMOE_BF16 = 1 } lrmoe_dtype;

/* Epilogue of lrmoe_grouped_dgrad. */
typedef enum {
  LRMOE_EPI_STORE = 0,       /* out = rows . W[e], stored in the storage dtype */
  LRMOE_EPI_SWIGLU_BWD = 1   /* out = [dG | dU] from dA = rows . W[e] and saved g, u */
} lrmoe_epilogue;

/* Device status word bits. */
#define LRMOE_ST_BAD_EXPERT 1u /* some topk_idx >= E (that pair was skipped) */
#define LRMOE_ST_BAD_QUOTA  2u /* some quota < 0 (treated as 0) */
#define LRMOE_ST_NONFINITE  4u /* some score was +Inf or NaN */
#define LRMOE_ST_TIMEOUT    8u /* a bounded device-side wait gave up; outputs invalid */
#define LRMOE_ST_BAD_INDEX 16u /* an index (perm/pos entry; checked build: any) was out of range; skipped */

/* Library version, (major << 16) | minor. */
int lrmoe_version(void);

/* Static text for a status code. */
const char* lrmoe_status_string(int code);

/* Message of the last failing call on this host thread ("" if none). */
const char* lrmoe_last_error(void);

/* ---------------------------------------------------------------------------
 * a1  LRM score.  RU-B bullet 3, FR-B bullet 3, DE paragraph 3: a pair's
 * contribution to its expert's weight update is the outer product of the
 * incoming gradient and the projection's saved input, so the squared norm of
 * that contribution factorises into routing weight^2 * ||gradient||^2 *
 * ||saved input||^2 and no gradient matrix is formed.
 *
 *   score[p] = w_p^2 * ||dY_t||^2 * ||a_p||^2     (p = t*k + j, e = topk_idx[p] in [0,E))
 *
 * topk_idx [T*k] int32, topk_w [T*k] fp32, dY [T][H] and a_saved [T*k][D] in
 * dtype `dt` (a_saved is the saved input of the down projection, D = I; any
 * other [T*k][D] saved input may be passed).  Output score [T*k] fp32; slots
 * with topk_idx < 0 or >= E get +0.
 * Arithmetic (bit-reproducible): each squared norm uses 32 fp32 partials, lane
 * l summing 16-byte vectors l, l+32, ... element by element as
 * fl(acc + fl(x*x)), then a butterfly fl(acc[l] + acc[l^o]) for o = 16..1;
 * score = fl(fl(fl(w*w) * n_dY) * n_a).  NaN scores are written as 0x7FFFFFFF
 * and, like +Inf, set LRMOE_ST_NONFINITE.  No fused multiply-add, no FTZ.
 * ------------------------------------------------------------------------- */
int lrmoe_score(const int32_t* topk_idx, const float* topk_w, int T, int k, int E,
                const void* dY, int H, const void* a_saved, int D, lrmoe_dtype dt,
                float* score, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a1 split at the factorisation (same passage as lrmoe_score): ||a_p||^2 does
 * not depend on the backward, so the forward, which writes a, can save it, and
 * the backward's score then reads dY and the saved norms instead of all of a
 * (T*H + 4*T*k bytes instead of T*H + T*k*I elements).  The pages describe no
 * such split; it changes no value: the two calls below give, bit for bit,
 * what lrmoe_score gives (every row norm takes the same order in each kernel).
 *
 * lrmoe_row_sqnorm: out[r] = ||rows[r]||^2 for r < n_rows, rows [n_rows][D] in
 *   dtype dt, out [n_rows] fp32, in the canonical order of lrmoe_score.
 *   No status word: a non-finite row gives a non-finite norm (a NaN of
 *   unspecified payload for NaN input), which the score call then flags.
 * lrmoe_score_from_norms: score[p] = fl(fl(fl(w_p*w_p) * ||dY_t||^2) *
 *   a_sqnorm[p]) for routed slots, +0 otherwise; status bits, NaN handling and
 *   layouts as lrmoe_score.  a_sqnorm [T*k] fp32 may be the score buffer
 *   itself (each slot is read before it is overwritten).
 * ------------------------------------------------------------------------- */
int lrmoe_row_sqnorm(const void* rows, int n_rows, int D, lrmoe_dtype dt, float* out,
                     void* stream);

int lrmoe_score_from_norms(const int32_t* topk_idx, const float* topk_w, int T, int k, int E,
                           const void* dY, int H, const float* a_sqnorm, lrmoe_dtype dt,
                           float* score, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Routing-weight gradient.  The pages (RU-B, FR-B, DE) prune the expert
 * weight-gradient contributions and do not treat the router; this call gives
 * what the layer output sum_j w_tj y_tj implies:
 *
 *   dw[p] = <dY_t, y_p>            (p = t*k + j, e = topk_idx[p] in [0,E))
 *
 * y_saved [T*k][H] in dtype dt is the pair's expert output y_p = W_down[e] a_p,
 * saved by the forward (rows of empty or invalid slots are not read).  With
 * pos == NULL every routed pair is computed; with pos (the [T*k] int32 output
 * of lrmoe_select_quota) only retained pairs (pos[p] >= 0) are, and dropped
 * pairs get +0 -- the pages are silent on which reading LRMoE uses.  Empty and
 * invalid slots get +0; invalid ids set LRMOE_ST_BAD_EXPERT.
 * Arithmetic: the canonical order of lrmoe_score with x*x replaced by dY*y:
 * 32 lane partials, fl(acc + fl(dY*y)) element by element, butterfly.
 * Output dw [T*k] fp32.
 * ------------------------------------------------------------------------- */
int lrmoe_router_grad(const int32_t* topk_idx, int T, int k, int E, const void* dY, int H,
                      const void* y_saved, lrmoe_dtype dt, const int32_t* pos, float* dw,
                      uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a2  Per-expert top-quota selection.  RU-B bullets 2-3, FR-B bullets 2-3,
 * DE paragraph 3: a quota per expert is fixed for the layer call before the
 * backward, and within it the pairs with the highest score stay.
 *
 * For each expert e keep the m_e = min(max(q_e,0), c_e) pairs that are
 * largest under the key (score bit pattern as uint32 descending, p ascending).
 * Outputs (int32, device):
 *   counts[E]   = c_e            kept[E] = m_e
 *   offsets[E+1]= exclusive prefix sum of m_e (offsets[E] = M)
 *   perm[T*k]   = first M entries: packed row r holds pair perm[r]; expert
 *                 blocks in ascending e, pairs ascending inside a block
 *   pos[T*k]    = packed row of pair p, or -1 (dropped, empty or invalid slot)
 * quota [E] int32 on the device.  Deterministic: integer/bitwise work only.
 * workspace: device scratch of at least lrmoe_select_workspace_bytes(T,k,E)
 * bytes, 256-byte aligned; its contents on entry do not matter.
 * E <= 4096 (else LRMOE_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------- */
size_t lrmoe_select_workspace_bytes(int T, int k, int E);

int lrmoe_select_quota(const int32_t* topk_idx, const float* score, int T, int k, int E,
                       const int32_t* quota, int32_t* counts, int32_t* kept, int32_t* offsets,
                       int32_t* perm, int32_t* pos, void* workspace, size_t workspace_bytes,
                       uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Redistribution over expert copies.  RU-B bullet 4, FR-B bullet 4: the
 * remaining pairs are spread over the admissible copies of their expert by an
 * integer algorithm that minimises the peak load of one GPU; no new copies
 * appear in the backward.
 *
 * lrmoe_redistribute (HOST pointers, no CUDA call): m [E] int64 retained pairs
 * per expert (all ranks together), admissible [E][G] uint8 (nonzero: GPU g
 * holds a copy of expert e).  Writes plan [E][G] int64 with sum_g plan[e][g] =
 * m_e, plan[e][g] = 0 where there is no copy, and the smallest possible peak
 * max_g sum_e plan[e][g] into *peak (binary search on the peak, each probe a
 * max-flow; the load of a GPU is its number of pairs).  The plan is one of
 * possibly several optimal ones.  Errors: sizes <= 0, m_e < 0, or m_e > 0 for
 * an expert with no copy -> LRMOE_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------- */
int lrmoe_redistribute(const int64_t* m, const uint8_t* admissible, int E, int G, int64_t* plan,
                       int64_t* peak);

/* ---------------------------------------------------------------------------
 * Split by destination.  RU-B bullet 5, FR-B bullet 5: the remaining rows are
 * grouped by receiver and expert, so the all-to-all moves compact blocks.
 *
 * This rank's packed rows (perm, offsets [E+1] from lrmoe_select_quota) are
 * cut by plan [E][G] int32 (device; the redistribute plan): expert e's local
 * rows have global indices global_start[e] + (r - offsets[e]) (global_start
 * [E] int32 device = the rows of e on lower ranks; NULL = 0, one rank), and
 * GPU g serves the global run [C[e][g], C[e][g+1]), C = prefix sum of
 * plan[e] over g.  Outputs (device, int32):
 *   perm_dest [rows_cap]         the pair ids regrouped destination-major, then
 *                                expert, then in packed order
 *   dest_offsets [G+1]           start of each destination's block (last = M)
 *   dest_expert_offsets [G][E+1] expert offsets inside each block (the
 *                                receiver's grouped-GEMM offsets for this source)
 *   row_dest [rows_cap]          (optional, NULL = not written) the send slot
 *                                of each local packed row r < offsets[E]:
 *                                perm_dest[row_dest[r]] = perm[r]; rows that come
 *                                back in send order return to the packed layout
 *                                with lrmoe_gather_rows(back, row_dest, ...)
 * lrmoe_pack(perm_dest, dest_offsets, ..., E = G, ...) or lrmoe_pack_wide then
 * gathers the send buffer (pack reads only offsets[E], the row count).  Rows
 * that the plan does not cover, and negative plan entries, set
 * LRMOE_ST_BAD_INDEX; such rows are left out.
 * ------------------------------------------------------------------------- */
int lrmoe_split_by_destination(const int32_t* perm, const int32_t* offsets, const int32_t* plan,
                               const int32_t* global_start, int E, int G, int rows_cap,
                               int32_t* perm_dest, int32_t* dest_offsets,
                               int32_t* dest_expert_offsets, int32_t* row_dest, uint32_t* status,
                               void* stream);

/* ---------------------------------------------------------------------------
 * Receiver's grouping.  RU-B bullet 5, FR-B bullet 5: the copy that receives
 * rows from every source runs the grouped GEMMs on dense per-expert blocks.
 *
 * src_expert_offsets [G][E+1] int32 device: row q is source q's
 * dest_expert_offsets row for this receiver (as exchanged by an all-to-all);
 * the received rows are source-major (source q's block after those of
 * sources < q, expert e's rows at [T[q][e], T[q][e+1]) inside it).  Writes
 * (device, int32):
 *   order [rows_cap]  grouped position i holds received row order[i]; grouped
 *                     order = experts ascending, then sources in rank order,
 *                     then arrival order
 *   inv [rows_cap]    its inverse: received row j sits at grouped position inv[j]
 *   offsets [E+1]     the grouped blocks' offsets (the receiver's GEMM offsets)
 * for the R = sum_q T[q][E] received rows (R <= rows_cap; more, or a
 * decreasing row of T, sets LRMOE_ST_BAD_INDEX).  E*G*4 <= 200 KB.
 * ------------------------------------------------------------------------- */
int lrmoe_group_received(const int32_t* src_expert_offsets, int G, int E, int rows_cap,
                         int32_t* order, int32_t* inv, int32_t* offsets, uint32_t* status,
                         void* stream);

/* ---------------------------------------------------------------------------
 * Exchange rows.  RU-B bullet 5: the retained rows move in compact blocks.  One
 * wide row per retained pair holds all five operands the receiver needs side by
 * side, [x_t | RNE(w_p dY_t) | a_p | g_p | u_p] (2H + 3I elements, the same
 * values lrmoe_pack writes), so that a single all-to-all moves them.
 *
 * lrmoe_pack_wide: like lrmoe_pack with every output present, into
 * rows [rows_cap][2H+3I] (usually in the order of lrmoe_split_by_destination).
 * lrmoe_split_wide: the receiver's gather and split: for i < n, the five
 * column blocks of rows[idx[i]] go to X_p[i], DY_p[i] [.][H] and A_p[i],
 * G_p[i], U_p[i] [.][I] (dense blocks for the grouped GEMMs; idx = order of
 * lrmoe_group_received).  idx outside [0, n_src) sets LRMOE_ST_BAD_INDEX and
 * leaves that row unwritten; n = 0 is a no-op.
 * ------------------------------------------------------------------------- */
int lrmoe_pack_wide(const int32_t* perm, const int32_t* offsets, const float* topk_w, int T, int k,
                    int E, const void* x, const void* dY, int H, const void* a, const void* g,
                    const void* u, int I, lrmoe_dtype dt, void* rows, int rows_cap,
                    uint32_t* status, void* stream);
int lrmoe_split_wide(const void* rows, int n_src, const int32_t* idx, int n, int H, int I,
                     lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
                     uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Row gather for the exchange of retained rows (RU-B bullet 5: rows move in
 * compact blocks and come back to their original layout): dst[i] = src[idx[i]]
 * for i < n, rows of row_bytes bytes (a multiple of 16), src [n_src][.],
 * dst [n][.], idx [n] int32 device.  idx outside [0, n_src) sets
 * LRMOE_ST_BAD_INDEX and leaves that dst row unwritten.  n = 0 is a no-op.
 * ------------------------------------------------------------------------- */
int lrmoe_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx, int n,
                      void* dst, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Quota controller.  RU-B bullet 2, FR-B bullet 2, DE paragraph 3: before the
 * backward a controller sees how many tokens came to each expert and, within
 * the memory limit, fixes how many pairs of each expert stay for the layer
 * call.  Reading implemented (water-filling):
 *
 *   c_e = #{p : topk_idx[p] == e},  q_e = min(c_e, cap, tau),
 *   tau = the largest integer level with sum_e q_e <= max_pairs,
 *
 * so the most loaded experts are cut first.  cap <= 0 disables the per-expert
 * cap; max_pairs < 0 disables the budget (then q_e = min(c_e, cap); with
 * cap = T*k/E this is the "capacity" quota of the configs).  Outputs quota[E]
 * and counts[E] (int32, device); nothing goes back to the host, so the result
 * can feed lrmoe_select_quota on the same stream.  ids >= E are skipped and set
 * LRMOE_ST_BAD_EXPERT.  E <= 4096.
 * ------------------------------------------------------------------------- */
int lrmoe_quota_controller(const int32_t* topk_idx, int T, int k, int E, int32_t cap,
                           int64_t max_pairs, int32_t* quota, int32_t* counts, uint32_t* status,
                           void* stream);

/* ---------------------------------------------------------------------------
 * Selection that allocates nothing.  The LRMoE pages have no counterpart of
 * this entry point; it exists for callers of this library that cannot hand
 * it device scratch: a host framework or plugin host that owns every byte of
 * device memory and gives its extensions no allocator, or a latency-critical
 * caller that must not call cudaMalloc/cudaFree because those calls can
 * synchronise the device and stall work on other streams.
 *
 * Same arguments (minus the workspace), same outputs and the same guarantees
 * as lrmoe_select_quota.  The scratch is a fixed array of
 * LRMOE_NOALLOC_SCRATCH_BYTES that the library keeps in device memory: every
 * GPU that loads the library holds it until the process exits.  Every call
 * asks the runtime for that array's device address in the context current on
 * the calling thread (a host-side query that allocates nothing), so the
 * address stays right across a reset of the device's context.  The first
 * such query in a context also loads the library's device code, so make the
 * first call on each device before any stream capture.  The call itself
 * allocates nothing and calls no allocating routine.  All calls on one device share the array: two calls whose kernels
 * overlap on the GPU (different streams, no ordering between them) race and
 * give undefined results; calls on one stream are safe.  Nothing in the
 * array has to start at zero and its stale contents never affect a result.
 * Returns LRMOE_ERR_WORKSPACE, writing nothing, when the problem needs more
 * scratch than the array holds (lrmoe_select_workspace_bytes(T,k,E) >
 * LRMOE_NOALLOC_SCRATCH_BYTES, roughly T*k > 500 000 pairs at E = 128).
 * ------------------------------------------------------------------------- */
#define LRMOE_NOALLOC_SCRATCH_BYTES (4u << 20)

int lrmoe_select_quota_noalloc(const int32_t* topk_idx, const float* score, int T, int k, int E,
                               const int32_t* quota, int32_t* counts, int32_t* kept,
                               int32_t* offsets, int32_t* perm, int32_t* pos, uint32_t* status,
                               void* stream);

/* ---------------------------------------------------------------------------
 * a3  Physical compaction.  RU-B bullet 5 and the note after it, FR-B bullet
 * 5, DE paragraph 4: the retained gradient and activation rows are gathered
 * into dense blocks per expert; masking rows inside full-size tensors would
 * save neither time nor memory.
 *
 * For packed rows r < offsets[E] (read on the device), p = perm[r], t = p / k:
 *   Xp[r] = x[t] (H)      DYp[r] = RNE_dt(fl(topk_w[p] * dY[t])) (H)
 *   Ap[r] = a[p] (I)      Gp[r] = g[p] (I)       Up[r] = u[p] (I)
 * x, dY [T][H]; a, g, u [T*k][I]; outputs [rows_cap][.] with rows_cap >= M
 * (T*k always suffices).  Rows >= M are not touched.  A perm entry outside
 * [0, T*k) is skipped and sets LRMOE_ST_BAD_INDEX.  Only DYp is required:
 * Gp and Up may both be NULL (then g, u may be NULL too), and Xp or Ap may be
 * NULL (then x or a may be NULL), for the kernels that read those rows in
 * place (lrmoe_grouped_dgrad_swiglu_gather, lrmoe_grouped_wgrad_gather).
 * ------------------------------------------------------------------------- */
int lrmoe_pack(const int32_t* perm, const int32_t* offsets, const float* topk_w, int T, int k, int E,
               const void* x, const void* dY, int H, const void* a, const void* g, const void* u,
               int I, lrmoe_dtype dt, void* Xp, void* DYp, void* Ap, void* Gp, void* Up,
               int rows_cap, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a4  Variable-size grouped GEMMs without zero padding.  RU-B bullet 5, FR-B
 * bullet 5, DE paragraph 4 ("gruppierte GEMMs variabler Größe").  Expert e
 * owns packed rows R_e = [offsets[e], offsets[e+1]) (offsets read on the
 * device; m_e may be 0).
 *
 * lrmoe_grouped_dgrad: for each e, D = rows[R_e] (m_e x K) . W[e] (K x N)
 *   rows [rows_cap][K], W [E][K][N] row-major, accumulate fp32.
 *   LRMOE_EPI_STORE:      out[R_e] = D                  out [rows_cap][N]
 *   LRMOE_EPI_SWIGLU_BWD: with s = sigmoid(g), g = Gp[R_e], u = Up[R_e] ([rows_cap][N]):
 *       dG = D * u * s * (1 + g (1 - s)),   dU = D * g * s,
 *       out[R_e] = [dG | dU]                            out [rows_cap][2N]
 *   (D = dA, the gradient of the down projection's input, is never stored.)
 *   Rows outside every R_e are not written.
 *
 * lrmoe_grouped_wgrad: for each e, dW[e] (N1 x N2) = grad_rows[R_e]^T . in_rows[R_e]
 *   grad_rows [rows_cap][N1], in_rows [rows_cap][N2], dW [E][N1][N2] fp32.
 *   accumulate = 0 overwrites dW (zeros for m_e = 0); 1 adds to it.
 *
 * Uses: dA/dGU  = dgrad(DYp, W_down, K=H, N=I, SWIGLU_BWD)
 *       dW_down = wgrad(DYp, Ap, N1=H, N2=I)
 *       dW_gu   = wgrad(dGUp, Xp, N1=2I, N2=H)
 *       dXp     = dgrad(dGUp, W_gu, K=2I, N=H, STORE)
 * bf16 runs on the tensor cores (bf16 operands, fp32 accumulation, bf16
 * outputs for dgrad); fp32 runs in fp32 FFMA.  E <= 1024.
 * ------------------------------------------------------------------------- */
int lrmoe_grouped_dgrad(const void* rows, int rows_cap, const void* W, const int32_t* offsets,
                        int E, int K, int N, lrmoe_dtype dt, lrmoe_epilogue epi,
                        const void* Gp, const void* Up, void* out, uint32_t* status, void* stream);

int lrmoe_grouped_wgrad(const void* grad_rows, const void* in_rows, int rows_cap,
                        const int32_t* offsets, int E, int N1, int N2, lrmoe_dtype dt,
                        float* dW, int accumulate, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a4 wgrad gathering its second operand in place (same passages as
 * lrmoe_grouped_wgrad): dW[e] = grad[R_e]^T . B[R_e] with the row of B for
 * packed row r being src[perm[r] / src_div], src [n_pairs / src_div][N2]:
 *   dW_down: grad = DY_p, src = a [T*k][I], src_div = 1
 *   dW_gu:   grad = dGU_p, src = x [T][H],  src_div = k
 * Bit-identical to lrmoe_grouped_wgrad on the packed rows.  perm entries
 * outside [0, n_pairs) set LRMOE_ST_BAD_INDEX and read as zero rows.  bf16 only
 * (fp32: LRMOE_ERR_UNSUPPORTED).  The rows come in through 16-byte cp.async
 * copies issued by one producer warp, which on a B200 is about half as fast as
 * the TMA loads of packed rows, so lrmoe_pruned_backward packs X_p and A_p.
 * ------------------------------------------------------------------------- */
int lrmoe_grouped_wgrad_gather(const void* grad_rows, int rows_cap, const int32_t* perm,
                               const void* src, int src_div, int n_pairs, const int32_t* offsets,
                               int E, int N1, int N2, lrmoe_dtype dt, float* dW, int accumulate,
                               uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a4 dgrad with the SwiGLU-backward epilogue, gathering g and u in place (the
 * pages' dense per-expert blocks are what the tensor cores read; the
 * epilogue's per-row operands need no copy).  As lrmoe_grouped_dgrad with
 * epi = LRMOE_EPI_SWIGLU_BWD, except that packed row r reads g, u [gu_rows][N]
 * at row perm[r] (perm from lrmoe_select_quota, gu_rows = T*k) instead of
 * Gp[r], Up[r]; bit-identical results.  perm entries outside [0, gu_rows) set
 * LRMOE_ST_BAD_INDEX and leave that output row unwritten.  bf16 only (fp32:
 * LRMOE_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------- */
int lrmoe_grouped_dgrad_swiglu_gather(const void* rows, int rows_cap, const void* W,
                                      const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                                      const int32_t* perm, const void* g, const void* u, int gu_rows,
                                      void* out, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a4, two GEMMs that share their gradient rows in one launch (same passages).
 * Exactly lrmoe_grouped_dgrad(grad_rows, rows_cap, W, offsets, E, K, N, dt,
 * epi, Gp, Up, out) plus lrmoe_grouped_wgrad(grad_rows, in_rows, rows_cap,
 * offsets, E, N1 = K, N2, dt, dW, accumulate) in one persistent launch whose
 * tile queue interleaves the two kinds evenly (dgrad reads W, wgrad writes dW).
 * lrmoe_pruned_backward does not use it: on a B200 the two separate launches
 * are faster for the shapes measured.  The two pairs of the path are:
 *   (DYp; W_down, SWIGLU -> dGUp; Ap -> dW_down)   K = H, N = I, N2 = I
 *   (dGUp; W_gu, STORE -> dXp;  Xp -> dW_gu)       K = 2I, N = H, N2 = H
 * Layouts, outputs and errors as the two calls.  bf16 only (fp32 returns
 * LRMOE_ERR_UNSUPPORTED: use the two calls).
 * ------------------------------------------------------------------------- */
int lrmoe_grouped_dgrad_wgrad(const void* grad_rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_dtype dt,
                              lrmoe_epilogue epi, const void* Gp, const void* Up, void* out,
                              const void* in_rows, int N2, float* dW, int accumulate,
                              uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * a5  Back to the original layout.  RU-B bullet 5, last sentence; FR-B
 * bullet 5, last sentence.
 *
 *   dX[t] = RNE_dt( sum_{j ascending, pos[t*k+j] >= 0} dXp[pos[t*k+j]] )
 * summed in fp32 and rounded once; a token with no retained pair gets 0.
 * dXp [rows_cap][H], pos [T*k], dX [T][H].  A gather: no atomics,
 * deterministic.  pos >= rows_cap is skipped and sets LRMOE_ST_BAD_INDEX.
 * ------------------------------------------------------------------------- */
int lrmoe_unpack(const void* dXp, int rows_cap, const int32_t* pos, int T, int k, int H,
                 lrmoe_dtype dt, void* dX, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * The whole path a1..a5 on one stream (RU-B bullets 3-5): score, selection,
 * compaction, the four grouped GEMMs and the return to the token layout, as
 * one enqueue with no host synchronisation.  All buffers are caller-owned
 * device memory; rows_cap >= M (T*k always suffices).  For bf16 the SwiGLU
 * epilogue reads g, u in place, so Gp and Up are neither written nor needed
 * (they may be NULL); fp32 packs them.
 * ------------------------------------------------------------------------- */
typedef struct {
  /* inputs */
  const int32_t* topk_idx;  /* [T*k] */
  const float* topk_w;      /* [T*k] */
  const int32_t* quota;     /* [E] */
  const void* x;            /* [T][H] */
  const void* dY;           /* [T][H] */
  const void* g;            /* [T*k][I] saved gate pre-activation */
  const void* u;            /* [T*k][I] saved up projection */
  const void* a;            /* [T*k][I] saved down-projection input */
  const void* W_gu;         /* [E][2I][H] */
  const void* W_down;       /* [E][H][I] */
  /* selection outputs */
  float* score;             /* [T*k] */
  int32_t* counts;          /* [E] */
  int32_t* kept;            /* [E] */
  int32_t* offsets;         /* [E+1] */
  int32_t* perm;            /* [T*k] */
  int32_t* pos;             /* [T*k] */
  /* packed blocks and intermediates, rows_cap rows each */
  void* Xp;                 /* [rows_cap][H] */
  void* DYp;                /* [rows_cap][H] */
  void* Ap;                 /* [rows_cap][I] */
  void* Gp;                 /* [rows_cap][I] */
  void* Up;                 /* [rows_cap][I] */
  void* dGUp;               /* [rows_cap][2I] */
  void* dXp;                /* [rows_cap][H] */
  /* gradients */
  float* dW_gu;             /* [E][2I][H] fp32 */
  float* dW_down;           /* [E][H][I] fp32 */
  void* dX;                 /* [T][H] */
  /* scratch and status */
  void* workspace;          /* >= lrmoe_select_workspace_bytes(T,k,E) */
  size_t workspace_bytes;
  uint32_t* status;         /* may be NULL */
} lrmoe_buffers;

int lrmoe_pruned_backward(const lrmoe_buffers* b, int T, int k, int E, int H, int I,
                          int rows_cap, lrmoe_dtype dt, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostic (no counterpart in the pages): run one bounded device-side wait
 * on a barrier that nothing ever completes, with a limit of `limit_us`
 * microseconds (1 .. 1 000 000).  The kernel gives up, sets LRMOE_ST_TIMEOUT
 * in *status (device memory) and returns; the context stays usable.  It
 * checks the mechanism that every pipeline wait of the grouped GEMMs uses
 * (their limit is 2 s) without hanging or faulting the GPU.
 * ------------------------------------------------------------------------- */
int lrmoe_selftest_bounded_wait(uint32_t limit_us, uint32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostic (no counterpart in the pages): the grouped dgrad (bf16, store
 * epilogue; the same operands as lrmoe_grouped_dgrad with E, K, N) launched so
 * that its producers withhold the first K block of their first tile, with every
 * device-side wait limited to limit_us microseconds (1 .. 1 000 000).  The
 * MMA issuer's wait for that block runs out, the kernel raises
 * LRMOE_ST_TIMEOUT, lets the copies and tensor-core work already in flight
 * finish, releases its tensor memory and returns; the output is then invalid,
 * and the context stays usable.  two_sm selects the two-SM tiles (else the
 * one-SM tiles).  status is required.
 * ------------------------------------------------------------------------- */
int lrmoe_selftest_gemm_stall(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, void* out, int two_sm,
                              uint32_t limit_us, uint32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LRMOE_H */
