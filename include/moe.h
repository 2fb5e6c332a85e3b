/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE layer hot path.
 *
 * The layer, in the order the pages give it ("A Survey on Mixture of Experts",
 * section 5 System Design: gate routing, input encode, expert computation,
 * output decode; the All-to-All steps between them are the identity on one
 * GPU):
 *
 *   moe_gate               router logits = x . Wg^T                     (a0)
 *   moe_route              top-k softmax gate with expert capacity      (a1)
 *   moe_dispatch           input encode: group each expert's tokens     (a2)
 *   moe_expert_ffn         per-expert FC -> ReLU -> FC                  (a3)
 *   moe_combine            output decode: gate-weighted un-permute      (a4)
 *   moe_popularity_update  per-expert popularity, sliding-window mean   (a5)
 *
 * and the backward of each step (moe_combine_backward, moe_expert_ffn_backward,
 * moe_dispatch_backward, moe_route_backward, moe_gate_backward).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers to memory the caller owns.  The
 *    library allocates nothing; the only scratch (moe_route's) is a caller
 *    buffer sized by moe_route_workspace_size().
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and returns an int status: MOE_OK (0) or a negative
 *    MOE_ERR_* code.  Arguments are validated on the host before anything is
 *    launched; a call that returns an error has launched nothing.
 *  - Row-major tensors, no padding between rows.  `dtype` is MOE_DTYPE_F32 or
 *    MOE_DTYPE_BF16 (bf16 = the upper 16 bits of an IEEE binary32).
 *  - Vector paths need every tensor base 16-byte aligned and every row a
 *    multiple of 16 bytes (d, F multiples of 8 for bf16, of 4 for fp32);
 *    anything else is rejected with MOE_ERR_UNSUPPORTED.
 *  - Index tensors produced by moe_route are validated again on the device:
 *    an out-of-range row index is skipped (never dereferenced) and recorded in
 *    the per-device error word read by moe_device_error().
 *  - Limits: 1 <= E <= 1024, 1 <= k <= min(E, 32), T*k < 2^31.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* null pointer, size out of range, k > E, ...   */
    MOE_ERR_UNSUPPORTED = -2, /* dtype or alignment the kernels do not handle */
    MOE_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required   */
    MOE_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed          */
    MOE_ERR_DEVICE = -5       /* device-side check failed (moe_device_error)   */
};

enum moe_dtype { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };

/* Device-side error bits (moe_device_error). */
enum moe_device_error_bits {
    MOE_DEVERR_ROW_INDEX = 1, /* a slot_row / row_slot entry outside [0, R_max) */
    MOE_DEVERR_OFFSETS = 2,   /* offsets not non-decreasing or beyond R_max      */
    MOE_DEVERR_TIMEOUT = 4,   /* a pipeline wait inside a kernel ran past its
                                 time limit; the kernel gave up and returned     */
    MOE_DEVERR_EXPERT_INDEX = 8 /* an expert id outside [0, E) was skipped       */
};

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(int status);

/* Library ABI version: 100 * major + minor. */
MOE_API int moe_version(void);

/* Reads the device error word of the CURRENT device (synchronous: waits for
 * all work on the device) into *bits, then clears it if `clear` != 0.
 * Returns MOE_OK or MOE_ERR_CUDA. */
MOE_API int moe_device_error(int32_t* bits, int clear);

/* ---------------------------------------------------------------- a0 ----
 * Router logits.  PopFetcher, section 2.1.2: the gate network scores each
 * token against every expert.
 *   x       [T, d]  dtype     tokens
 *   Wg      [E, d]  dtype     one row per expert (out x in)
 *   logits  [T, E]  fp32      logits[t][e] = sum_c x[t][c] * Wg[e][c],
 *                             accumulated in fp32 (bf16 products are exact)
 * T >= 0 (T = 0 launches nothing).  d >= 1.
 */
MOE_API int moe_gate(const void* x, const void* Wg, int dtype, int T, int d, int E, float* logits,
             moe_stream_t stream);

/* ---------------------------------------------------------------- a1 ----
 * Top-k softmax gate with GShard expert capacity.  "A Survey on Mixture of
 * Experts", section 5 (gate routing; capacity-limited dispatch) and PopFetcher,
 * section 2.1.2 (top-k gate); MoE-MPMC, problem statement (softmax router).
 *
 *   z[t][e] = logits[t][e] + bias[e]                (one fp32 addition)
 *   ids[t][0..k-1]  the k largest z, larger first; equal z: lower index first.
 *                   +0.0 and -0.0 are equal.  A NaN z ranks above every number
 *                   (NaNs among themselves by index), so a diverged row still
 *                   gets k distinct ids in [0, E); its weights are NaN.
 *   w[t][j]         = exp(z_j - z_0) / sum_{i<k} exp(z_i - z_0)  (fp32): the
 *                     k softmax probabilities renormalised to sum to 1
 *   counts[e]       tokens that chose e (demand, before drops)
 *   kept[e]         min(counts[e], capacity)     (capacity <= 0: unlimited)
 *   offsets[0..E]   exclusive prefix sum of kept; offsets[E] = R
 *   slot_row[t][j]  row of slot (t, j) in the grouped layout, or -1 if dropped.
 *                   Inside an expert, slots are ranked in token order; the
 *                   first `capacity` are kept.
 *   row_slot[r]     t*k + j of the slot stored in row r, for r < R.  The buffer
 *                   must hold T*k entries; entries r >= R are not written.
 *   n_dropped[0]    T*k - R
 *
 *   logits [T,E] fp32; bias [E] fp32 or NULL; ids, slot_row [T,k] int32;
 *   w [T,k] fp32; counts, kept [E] int32; offsets [E+1] int32;
 *   row_slot [T*k] int32; n_dropped [1] int32.
 *   workspace: device buffer of at least moe_route_workspace_size(T, E, k)
 *   bytes, 256-byte aligned; its contents need no initialisation.
 * Results are bit-identical run to run (no atomics whose order is visible).
 * T = 0 writes zeros to counts, kept, offsets and n_dropped.
 */
MOE_API size_t moe_route_workspace_size(int T, int E, int k);

MOE_API int moe_route(const float* logits, const float* bias, int T, int E, int k, int capacity,
              int32_t* ids, float* w, int32_t* counts, int32_t* kept, int32_t* offsets,
              int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped, void* workspace,
              size_t workspace_bytes, moe_stream_t stream);

/* moe_route without a caller workspace (the pages have no counterpart; this
 * is an integration convenience).  For callers that may not allocate device
 * memory where they run the layer (fixed memory plans in serving loops,
 * plugins whose host framework owns all allocations, code that must avoid
 * the device-wide synchronisation an allocation can trigger).  Same arguments,
 * results and errors as moe_route, minus the workspace: the scratch is a
 * 4 MiB device array built into the library (held on every device that loads
 * it until the process exits).
 *  - Size limit: the router's two per-chunk tables for chunks of 128 tokens,
 *    2 * ceil(T / 128) * E int32 (each table rounded up to 256 bytes), plus
 *    256 bytes must fit 4 MiB (e.g. E = 256 up to T = 262016 tokens, E = 1024
 *    up to T = 65408); larger problems return MOE_ERR_WORKSPACE and launch
 *    nothing.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - All calls share the one array: calls whose kernels may overlap on a
 *    device (several streams or host threads) race and must be serialised by
 *    the caller.  Nothing in it needs clearing between calls.
 *  - Allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 */
MOE_API int moe_route_noalloc(const float* logits, const float* bias, int T, int E, int k, int capacity,
                      int32_t* ids, float* w, int32_t* counts, int32_t* kept, int32_t* offsets,
                      int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped,
                      moe_stream_t stream);

/* ---------------------------------------------------------------- a2 ----
 * Input encode.  "A Survey on Mixture of Experts", section 5: the tokens
 * routed to one expert are gathered into one contiguous block of rows.
 *   Xp[slot_row[t][j]] = x[t]   for every kept slot (slot_row >= 0)
 *   x [T, d] dtype; slot_row [T, k] from moe_route; Xp [R_max, d] dtype with
 *   R_max >= R (T*k always suffices).  Rows of Xp that no slot names are left
 *   untouched.  A slot_row entry >= R_max is skipped and flagged on the device.
 */
MOE_API int moe_dispatch(const void* x, int dtype, int T, int d, int k, const int32_t* slot_row,
                 void* Xp, int R_max, moe_stream_t stream);

/* ---------------------------------------------------------------- a3 ----
 * Expert computation.  PopFetcher, section 5.1: each expert is FC(d -> F),
 * ReLU, FC(F -> d) (two weight matrices, no bias terms).
 *   for each expert e, rows r in [offsets[e], offsets[e+1]):
 *     H[r][f]  = max(0, sum_c Xp[r][c] * W1[e][f][c])   stored in dtype
 *     Yp[r][o] = sum_f H[r][f] * W2[e][o][f]             stored in dtype
 *   Accumulation in fp32.  bf16 runs on the tcgen05 tensor cores; fp32 runs
 *   on the CUDA cores (no TF32).
 *   Xp [R_max, d]; W1 [E, F, d]; W2 [E, d, F]; offsets [E+1] (device, from
 *   moe_route); H [R_max, F] caller scratch for the hidden activation;
 *   Yp [R_max, d].  Rows >= offsets[E] of H and Yp are not written.
 *   Offsets that decrease or exceed R_max are flagged on the device and the
 *   offending expert is skipped.
 */
MOE_API int moe_expert_ffn(const void* Xp, const void* W1, const void* W2, int dtype, int E, int d,
                   int F, const int32_t* offsets, int R_max, void* H, void* Yp,
                   moe_stream_t stream);

/* Expert computation fused with input encode and the gate weights (ScatterMoE
 * style; "A Survey on Mixture of Experts", section 5 names the encode/decode
 * memory traffic as MoE overhead).  bf16 only, tcgen05 tensor cores:
 *   H[r][f]  = max(0, sum_c x[t(r)][c] * W1[e][f][c]),  t(r) = row_slot[r] / k
 *              (the A tiles are gathered from x directly: no Xp is written)
 *   Yp[r][o] = s(r) * sum_f H[r][f] * W2[e][o][f],  s(r) = w[row_slot[r]]
 *              (w = NULL: s = 1, i.e. moe_expert_ffn's Yp)
 * for the rows r of each group e.  Output decode is then a plain sum of each
 * token's rows: moe_combine with w = NULL.  x [T, d]; row_slot [R_max] and
 * offsets [E+1] from moe_route; w [T, k] from moe_route or NULL; H [R_max, F];
 * Yp [R_max, d].  Rounding: the scaled fp32 sum is rounded once to bf16.
 * row_slot entries outside [0, T*k) are flagged (MOE_DEVERR_ROW_INDEX) and
 * read as zero rows.  fp32 layers: MOE_ERR_UNSUPPORTED.
 */
MOE_API int moe_expert_ffn_gather(const void* x, int T, int k, const int32_t* row_slot,
                                  const float* w, const void* W1, const void* W2, int dtype, int E,
                                  int d, int F, const int32_t* offsets, int R_max, void* H,
                                  void* Yp, moe_stream_t stream);

/* ---------------------------------------------------------------- a4 ----
 * Output decode.  "A Survey on Mixture of Experts", section 5: the inverse of
 * input encode restores token order by the gating indices; each token's
 * output is the gate-weighted sum of its experts' outputs:
 *   y[t] = sum_{j < k, slot_row[t][j] >= 0} w[t][j] * Yp[slot_row[t][j]]
 *   accumulated in fp32 with j ascending, rounded once to dtype.  A token
 *   whose slots were all dropped gets zeros.  w = NULL: unit weights (the
 *   rows already carry them, as moe_expert_ffn_gather writes them).
 *   Yp [R_max, d] dtype; slot_row, w [T, k]; y [T, d] dtype.
 */
MOE_API int moe_combine(const void* Yp, int dtype, int T, int d, int k, const int32_t* slot_row,
                const float* w, void* y, int R_max, moe_stream_t stream);

/* ---------------------------------------------------------------- a5 ----
 * Expert popularity over a sliding window.  PopFetcher, section 3.1 (the
 * routing information collector counts the tokens routed to each expert) and
 * section 4.2 (Eq. 1, a window over recent iterations; read here as the
 * arithmetic mean of the last n = min(step + 1, W) count vectors).
 *   hist [W, E] int32   caller-owned ring; step `step` writes row step % W.
 *                       Start from any contents at step 0: rows not yet
 *                       written are never read.
 *   mean [E] fp32       (float)window_sum / (float)n, correctly rounded
 *   hot  [P] int32      the P experts with the largest window sum, larger
 *                       first, equal sums to the lower index
 *   counts [E] int32 (e.g. moe_route's); 0 <= P <= E; W >= 1; step >= 0.
 *   The state across steps is hist plus the caller's step counter: copying
 *   hist out and back resumes the sequence exactly.
 */
MOE_API int moe_popularity_update(const int32_t* counts, int E, int32_t* hist, int W, int64_t step,
                          float* mean, int P, int32_t* hot, moe_stream_t stream);

/* The same update with the step counter in device memory: reads *step
 * (int64, 8-byte aligned device pointer), updates as above, then stores
 * *step + 1.  A captured CUDA graph that replays the layer therefore advances
 * the window on every replay.  A negative *step makes the call a no-op. */
MOE_API int moe_popularity_update_dev(const int32_t* counts, int E, int32_t* hist, int W, int64_t* step,
                              float* mean, int P, int32_t* hot, moe_stream_t stream);

/* ------------------------------------------------------------- next ----
 * Cross-layer expert correlation.  PopFetcher, section 4.1 (Fig. 6): a
 * token's expert choices at two consecutive MoE layers form a correlated pair.
 * Adds, for every token t, one to C[i][h] for each i in ids_prev[t][0..k_prev)
 * and each h in ids_next[t][0..k_next).
 *   ids_prev [T, k_prev], ids_next [T, k_next] int32 (e.g. moe_route's ids of
 *   layers j and j+1 for the same tokens); C [E, E] int32, accumulated into
 *   (clear it to start a new window).  Ids outside [0, E) are skipped and
 *   flagged (MOE_DEVERR_EXPERT_INDEX).  Deterministic (integer sums).
 */
MOE_API int moe_correlation_update(const int32_t* ids_prev, int k_prev, const int32_t* ids_next,
                                   int k_next, int T, int E, int32_t* C, moe_stream_t stream);

/* Correlation-based popularity forecast of the next layer.  PopFetcher,
 * section 4.2 (Eq. 2-3, lost in extraction; read as below):
 *   P(h|i)  = C[i][h] / n_i,  n_i = (sum_h C[i][h]) / k_next
 *   pred[h] = sum_i pop_prev[i] * P(h|i) / k_prev
 * evaluated in IEEE double as q_i = (pop_prev[i] * k_next) / (S_i * k_prev)
 * (S_i = sum_h C[i][h]; q_i = 0 when S_i = 0), pred[h] = sum_i q_i * C[i][h]
 * with i ascending, each operation rounded separately, rounded once to fp32.
 * hot [P]: the P largest forecasts, equal values to the lower index.
 *   pop_prev [E] fp32 (e.g. moe_popularity_update's window mean of layer j);
 *   C [E, E] from moe_correlation_update; pred [E] fp32; 0 <= P <= E.
 * With pop_prev = layer j's counts and C from the same batch, pred equals
 * layer j+1's counts.
 */
MOE_API int moe_popularity_forecast(const float* pop_prev, const int32_t* C, int E, int k_prev,
                                    int k_next, float* pred, int P, int32_t* hot,
                                    moe_stream_t stream);

/* GShard load-balancing loss of one routing call.  PopFetcher, section 2.3.1
 * names it (it evens out the workload across workers); the formula is not on
 * the pages and is read as the GShard / Switch form:
 *   f_e = counts[e] / (T k),  P_e = mean_t softmax(logits[t] + bias)_e,
 *   loss = E * sum_e f_e P_e   (1 for a uniform router, E for a collapsed one)
 *   logits [T,E] fp32, bias [E] or NULL (the same keys moe_route ranked);
 *   counts [E] from moe_route; loss [1] fp32; prob_mean [E] fp32 or NULL.
 *   workspace: at least moe_route_workspace_size(T, E, k) bytes (the router's
 *   workspace can be reused once moe_route's kernels are done).
 * fp32 softmax per token, sums in a fixed order (deterministic).
 */
MOE_API int moe_aux_loss(const float* logits, const float* bias, int T, int E, int k,
                         const int32_t* counts, float* loss, float* prob_mean, void* workspace,
                         size_t workspace_bytes, moe_stream_t stream);

/* ------------------------------------------------------------ backward --
 * Gradients of the layer above.  PopFetcher, section 5.2.1: each expert GEMM
 * of the forward pass has two in the backward pass, one for its input and one
 * for its weights.  The other steps are the adjoints of the forward gathers
 * and of the gate's softmax.  The forward values they need (Yp, H, Xp, w,
 * ids, slot_row, offsets) are the ones the forward calls wrote.
 */

/* Output decode, backward.  For every kept slot (row = slot_row[t][j] >= 0):
 *   dw[t][j] = <dy[t], Yp[row]>     fp32 (lanes in fp32, fixed-order sum)
 *   dYp[row] = w[t][j] * dy[t]      the exact product rounded once to dtype
 * and dw[t][j] = 0 for a dropped slot.  dy [T, d], Yp and dYp [R_max, d]
 * dtype; slot_row, w, dw [T, k].  Rows of dYp no slot names are not written.
 */
MOE_API int moe_combine_backward(const void* dy, const void* Yp, int dtype, int T, int d, int k,
                                 const int32_t* slot_row, const float* w, float* dw, void* dYp,
                                 int R_max, moe_stream_t stream);

/* Expert computation, backward, for the rows r of each group e
 * (offsets[e] <= r < offsets[e+1]):
 *   dH[r][f]     = H[r][f] > 0 ? sum_o dYp[r][o] W2[e][o][f] : 0   (ReLU)
 *   dXp[r][c]    = sum_f dH[r][f] W1[e][f][c]
 *   dW2[e][o][f] = sum_r dYp[r][o] H[r][f]
 *   dW1[e][f][c] = sum_r dH[r][f] Xp[r][c]
 * dH and dXp [R_max, F] / [R_max, d] in dtype (the stored dH feeds dXp and
 * dW1); dW1 [E, F, d] and dW2 [E, d, F] fp32, either may be NULL; an expert
 * with no rows gets zero weight gradients.  Accumulation in fp32: bf16 on the
 * tcgen05 tensor cores (weights read in their forward layout as N-major
 * operands), fp32 on the CUDA cores.  Same alignment rules as moe_expert_ffn.
 */
MOE_API int moe_expert_ffn_backward(const void* Xp, const void* H, const void* dYp, const void* W1,
                                    const void* W2, int dtype, int E, int d, int F,
                                    const int32_t* offsets, int R_max, void* dH, void* dXp,
                                    float* dW1, float* dW2, moe_stream_t stream);

/* Input encode, backward: dx[t] = sum of dXp[slot_row[t][j]] over the token's
 * kept slots, j ascending, accumulated in fp32 and rounded once to dtype
 * (zeros for a token whose slots were all dropped).  dXp [R_max, d], dx [T, d].
 */
MOE_API int moe_dispatch_backward(const void* dXp, int dtype, int T, int d, int k,
                                  const int32_t* slot_row, void* dx, int R_max,
                                  moe_stream_t stream);

/* Gate routing, backward.  The gate weights are the softmax renormalised over
 * the token's selected experts S_t, so for e in S_t
 *   dlogits[t][e] = w_e (dw_e - sum_{i in S_t} w_i dw_i)
 * taken in double (each operation rounded, i ascending) and rounded to fp32;
 * dlogits [T, E] fp32 is dense, zero off S_t (the selection passes no
 * gradient).  dbias [E] fp32 = sum_t dlogits[t][e] (NULL: skipped); it needs
 * a workspace of moe_route_workspace_size(T, E, k) bytes (the router's may be
 * reused).  ids, w [T, k] from moe_route; dw [T, k] from moe_combine_backward.
 * Deterministic.
 */
MOE_API int moe_route_backward(const int32_t* ids, const float* w, const float* dw, int T, int E,
                               int k, float* dlogits, float* dbias, void* workspace,
                               size_t workspace_bytes, moe_stream_t stream);

/* Gate projection, backward (logits = x . Wg^T):
 *   dx[t][c] += sum_e dlogits[t][e] Wg[e][c]   added to dx in place, rounded
 *                                              once to dtype
 *   dWg[e][c] = sum_t dlogits[t][e] x[t][c]    fp32 (NULL: skipped)
 * x, dx [T, d] and Wg [E, d] in dtype; dlogits [T, E] fp32, and the router
 * gradient keeps its fp32 precision on both paths:
 *  - bf16 with d and E multiples of 8: tcgen05 tensor cores; dlogits is split
 *    exactly into three bf16 planes (hi + mid + lo = dlogits), so every
 *    product with the bf16 x or Wg is exact and accumulates in fp32;
 *  - otherwise fp32 products on the CUDA cores.
 * dWg sums the tokens in consecutive slices whose fp32 partial products are
 * then added in slice order; the slicing depends on (T, d, E) only, so the
 * result is the same on every run and every device.  workspace: at least
 * moe_gate_backward_workspace_size(T, d, E, dtype) bytes (0: NULL accepted).
 */
MOE_API size_t moe_gate_backward_workspace_size(int T, int d, int E, int dtype);

MOE_API int moe_gate_backward(const void* x, const void* Wg, int dtype, int T, int d, int E,
                              const float* dlogits, void* dx, float* dWg, void* workspace,
                              size_t workspace_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
