/*
 * moe_oracle.c -- plain, slow, obviously correct CPU oracle of the MoE layer
 * hot path: gate projection, top-k routing with expert capacity, input encode
 * (dispatch), expert FC-ReLU-FC, output decode (combine) and the per-expert
 * popularity window.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file.  Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library: every conversion and loop below is written out here.
 *
 * Sources (each function names the passage it follows):
 *   [Survey-5]  "A Survey on Mixture of Experts", section 5 System Design:
 *               expert parallelism is gate routing -> input encode -> (All-to-All
 *               dispatch) -> expert computation -> (All-to-All combine) -> output
 *               decode; input encode gathers the tokens of one expert into
 *               contiguous memory; output decode restores the original layout
 *               by the gating indices; GShard bounds each expert's load by an
 *               expert capacity.
 *   [Pop-2.1.2] PopFetcher (ATC'25), section 2.1.2: each token is routed by the
 *               gate network to one or more experts by top-k selection.
 *   [Pop-5.1]   PopFetcher, section 5.1: an expert is two FC layers H x aH and
 *               aH x H with a ReLU between them (4H^2 parameters at a = 2).
 *   [Pop-3.1]   PopFetcher, section 3.1: the routing information collector
 *               counts the tokens routed to each expert (expert popularity).
 *   [Pop-4.2]   PopFetcher, section 4.2, Eq. 1 (lost in extraction): the token
 *               distribution of recent iterations over a sliding window of s
 *               iterations.  Reading taken: the arithmetic mean of the last
 *               n = min(steps seen, W) per-expert count vectors.
 *   [Pop-4.1]   PopFetcher, section 4.1 (Fig. 6): a token's expert choices at two
 *               consecutive layers form a correlated pair; the next layer's hot
 *               experts follow from the previous layer's choices.
 *   [Pop-4.2b]  PopFetcher, section 4.2, Eq. 2-3 (lost): the conditional
 *               probability of the next-layer expert given the previous-layer
 *               one, and the correlation-based popularity forecast.
 *   [Pop-2.3.1] PopFetcher, section 2.3.1: GShard adds a load-balancing loss to
 *               spread the workload evenly (formula not on the pages).
 *   [MPMC]      MoE-MPMC summary, problem statement item 3: routing is softmax
 *               based.
 *
 * Precision: routing keys are fp32 (logit + bias is one fp32 add, as the router
 * is stated to be fp32); everything else accumulates in double and rounds once
 * to the storage type (bf16 or fp32) of the tensor it writes.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * A second build adds -fopenmp: the loops over tokens and rows marked
 * "omp parallel for" below are independent (each iteration writes its own
 * output row and reads nothing another iteration writes), so the threaded
 * build computes every value with the same operations in the same order as
 * the single-threaded one; only which core computes a row changes.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

/* ---------------------------------------------------------------- numbers -- */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits, binary32 exponent
 * range), ties to even, in ONE rounding step (no detour through float, which
 * would round twice).  Finite inputs only; overflow gives infinity. */
static uint16_t double_to_bf16_bits(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0x0000u;
    int neg = v < 0.0;
    double a = fabs(v);
    int ex;
    (void)frexp(a, &ex);           /* a = m * 2^ex, m in [0.5, 1) */
    int q = ex - 8;                /* quantum exponent for 8 significant bits */
    if (q < -133) q = -133;        /* bf16 subnormal quantum is 2^-133 */
    double r = rint(ldexp(a, -q)); /* default rounding mode: nearest, ties even */
    double rounded = ldexp(r, q);
    if (rounded >= 0x1p128) return neg ? 0xFF80u : 0x7F80u; /* +-infinity */
    float f = (float)rounded;      /* exact: at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    return neg ? (uint16_t)(b | 0x8000u) : b;
}

static double load_elem(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_BF16) return bf16_bits_to_double(((const uint16_t*)base)[i]);
    return (double)((const float*)base)[i];
}

static void store_elem(void* base, int dtype, int64_t i, double v) {
    if (dtype == ORC_BF16)
        ((uint16_t*)base)[i] = double_to_bf16_bits(v);
    else
        ((float*)base)[i] = (float)v; /* one rounding, nearest even */
}

static size_t elem_size(int dtype) { return dtype == ORC_BF16 ? 2u : 4u; }

/* Exposed so the tests can pin the rounding against numpy's float32 path. */
uint16_t oracle_round_bf16(double v) { return double_to_bf16_bits(v); }

/* Threads the marked loops may use (1 in the single-threaded build). */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------ gate (a0) ---- */

/* Router logits of each token: logits[t][e] = sum_c x[t][c] * Wg[e][c].
 * [Pop-2.1.2] the gate network scores every expert for every token.  Wg is
 * stored one row per expert (the nn.Linear out x in layout).  Accumulated in
 * double over c ascending, rounded once to fp32. */
void oracle_gate(const void* x, const void* Wg, int dtype, int T, int d, int E,
                 float* logits) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += load_elem(x, dtype, (int64_t)t * d + c) *
                       load_elem(Wg, dtype, (int64_t)e * d + c);
            logits[(int64_t)t * E + e] = (float)acc;
        }
}

/* ----------------------------------------------------------- route (a1) ---- */

/* Strict order of routing keys: a NaN ranks above every number (and no NaN
 * above another NaN), numbers by value (+0 and -0 equal).  The pages assume
 * finite scores; this reading gives a diverged row (NaN logits) a defined
 * top-k of valid expert indices, and its weights come out NaN. */
static int ranks_above(float a, float b) {
    if (isnan(b)) return 0;
    if (isnan(a)) return 1;
    return a > b;
}

/* Gate routing with expert capacity.
 *
 * [Pop-2.1.2] top-k selection; [MPMC] softmax router; [Survey-5] GShard expert
 * capacity.  Steps, in order:
 *  1. z[t][e] = logits[t][e] + bias[e], one fp32 addition.
 *  2. k times, pick the not-yet-chosen expert with the largest z; on equal z
 *     the lower expert index wins (strict '>' while scanning e upward).  A NaN
 *     z counts as larger than every number (ranks_above).
 *     Softmax is strictly increasing, so this is the top-k of the softmax.
 *  3. The k chosen softmax probabilities renormalised to sum to one:
 *     w_j = exp(z_j - z_0) / sum_i exp(z_i - z_0)  (the full softmax
 *     denominator cancels), in double, rounded to fp32.
 *  4. counts[e] = number of (t, j) with ids[t][j] == e (demand before drops).
 *  5. kept[e] = min(counts[e], capacity) (capacity <= 0: unlimited);
 *     offsets = exclusive prefix sum of kept, offsets[E] = R.
 *  6. Slot positions inside each expert.  Token-major (default): slots are
 *     visited t = 0..T-1, j = 0..k-1 and the p-th visitor of expert e gets
 *     position p.  Rank-major (GShard's own order, flag set): all j = 0 slots
 *     of every token first, then all j = 1 slots, and so on.
 *     A slot at position p < capacity goes to row offsets[e] + p and
 *     row_slot[row] = t*k + j; a later slot is dropped: slot_row = -1.
 *  7. n_dropped = T*k - sum(kept).
 * Returns 0, or -1 on invalid sizes. */
int oracle_route(const float* logits, const float* bias, int T, int E, int k,
                 int capacity, int rank_major, int32_t* ids, float* w,
                 int32_t* counts, int32_t* kept, int32_t* offsets,
                 int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped) {
    if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
    float* z = (float*)malloc(sizeof(float) * (size_t)(E > 0 ? E : 1));
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    if (!z || !taken) { free(z); free(taken); return -1; }

    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            float b = bias ? bias[e] : 0.0f;
            z[e] = logits[(int64_t)t * E + e] + b; /* fp32 + fp32 -> fp32 */
            taken[e] = 0;
        }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || ranks_above(z[e], z[best])) best = e;
            }
            taken[best] = 1;
            ids[(int64_t)t * k + j] = best;
            counts[best] += 1;
        }
        double zmax = (double)z[ids[(int64_t)t * k + 0]];
        double denom = 0.0;
        for (int i = 0; i < k; ++i) denom += exp((double)z[ids[(int64_t)t * k + i]] - zmax);
        for (int j = 0; j < k; ++j)
            w[(int64_t)t * k + j] =
                (float)(exp((double)z[ids[(int64_t)t * k + j]] - zmax) / denom);
    }

    int32_t total = 0;
    for (int e = 0; e < E; ++e) {
        int32_t c = counts[e];
        kept[e] = (capacity > 0 && c > capacity) ? capacity : c;
        offsets[e] = total;
        total += kept[e];
    }
    offsets[E] = total;

    int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    if (!seen) { free(z); free(taken); return -1; }
    int outer = rank_major ? k : T, inner = rank_major ? T : k;
    for (int a = 0; a < outer; ++a)
        for (int b = 0; b < inner; ++b) {
            int t = rank_major ? b : a, j = rank_major ? a : b;
            int64_t s = (int64_t)t * k + j;
            int e = ids[s];
            int32_t p = seen[e]++;
            if (capacity <= 0 || p < capacity) {
                int32_t row = offsets[e] + p;
                slot_row[s] = row;
                row_slot[row] = (int32_t)s;
            } else {
                slot_row[s] = -1;
            }
        }
    *n_dropped = (int32_t)((int64_t)T * k - total);
    free(seen);
    free(z);
    free(taken);
    return 0;
}

/* -------------------------------------------------------- dispatch (a2) ---- */

/* Input encode.  [Survey-5] the tokens of each expert are gathered into one
 * contiguous block, as the token-expert mapping of gate routing dictates:
 * Xp[row] = x[row_slot[row] / k] for every kept row 0 <= row < R. */
void oracle_dispatch(const void* x, int dtype, int T, int d, int k,
                     const int32_t* row_slot, int R, void* Xp) {
    size_t rowbytes = elem_size(dtype) * (size_t)d;
    (void)T;
#pragma omp parallel for schedule(static)
    for (int row = 0; row < R; ++row) {
        int t = row_slot[row] / k;
        memcpy((char*)Xp + (size_t)row * rowbytes, (const char*)x + (size_t)t * rowbytes,
               rowbytes);
    }
}

/* ----------------------------------------------------- expert FFN (a3) ---- */

/* One row through expert e.  [Pop-5.1] FC(d -> F), ReLU, FC(F -> d), no bias
 * terms (4H^2 parameters leave no room for them).  W1 is [E][F][d] and W2 is
 * [E][d][F] (out x in).  h[f] = max(0, sum_c xrow[c] W1[e][f][c]) is rounded to
 * the storage dtype (the intermediate activation is a tensor of that type);
 * y[o] = sum_f h[f] W2[e][o][f] is rounded to the storage dtype.  Sums in
 * double, c and f ascending.  hrow may be NULL. */
void oracle_expert_ffn_row(const void* xrow, const void* W1, const void* W2,
                           int dtype, int e, int d, int F, void* hrow, void* yrow) {
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    if (!h) return;
    const int64_t w1base = (int64_t)e * F * d, w2base = (int64_t)e * d * F;
    for (int f = 0; f < F; ++f) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += load_elem(xrow, dtype, c) * load_elem(W1, dtype, w1base + (int64_t)f * d + c);
        double r = acc > 0.0 ? acc : 0.0;
        /* round to storage precision, then use the stored value downstream */
        if (dtype == ORC_BF16)
            h[f] = bf16_bits_to_double(double_to_bf16_bits(r));
        else
            h[f] = (double)(float)r;
        if (hrow) store_elem(hrow, dtype, f, h[f]);
    }
    for (int o = 0; o < d; ++o) {
        double acc = 0.0;
        for (int f = 0; f < F; ++f)
            acc += h[f] * load_elem(W2, dtype, w2base + (int64_t)o * F + f);
        store_elem(yrow, dtype, o, acc);
    }
    free(h);
}

/* Expert computation over all groups: rows [offsets[e], offsets[e+1]) go
 * through expert e, i.e. row r goes through the e with
 * offsets[e] <= r < offsets[e+1] (the last e with offsets[e] <= r, so empty
 * groups are skipped).  H may be NULL. */
void oracle_expert_ffn(const void* Xp, const void* W1, const void* W2, int dtype,
                       int E, int d, int F, const int32_t* offsets, void* H, void* Yp) {
    size_t es = elem_size(dtype);
#pragma omp parallel for schedule(dynamic, 8)
    for (int row = offsets[0]; row < offsets[E]; ++row) {
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
        }
        oracle_expert_ffn_row((const char*)Xp + (size_t)row * d * es, W1, W2, dtype, lo, d, F,
                              H ? (char*)H + (size_t)row * F * es : NULL,
                              (char*)Yp + (size_t)row * d * es);
    }
}

/* Selected rows, each through its own expert: rows[i] through experts[i]
 * (the full-size parity checks sample rows this way).  H may be NULL. */
void oracle_expert_ffn_rows(const void* rows, const int32_t* experts, int n, const void* W1,
                            const void* W2, int dtype, int d, int F, void* H, void* Y) {
    size_t es = elem_size(dtype);
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; ++i)
        oracle_expert_ffn_row((const char*)rows + (size_t)i * d * es, W1, W2, dtype, experts[i],
                              d, F, H ? (char*)H + (size_t)i * F * es : NULL,
                              (char*)Y + (size_t)i * d * es);
}

/* --------------------------------------------------------- combine (a4) ---- */

/* Output decode.  [Survey-5] restores token order by the gating indices; each
 * token's output is the gate-weighted sum of its experts' outputs:
 * y[t] = sum_{j < k, slot kept} w[t][j] * Yp[slot_row[t][j]], j ascending, in
 * double, rounded once to the storage dtype.  Dropped slots add nothing, and a
 * token with no kept slot gets zeros. */
void oracle_combine(const void* Yp, int dtype, int T, int d, int k,
                    const int32_t* slot_row, const float* w, void* y) {
#pragma omp parallel
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            if (!acc) continue;
            for (int o = 0; o < d; ++o) acc[o] = 0.0;
            for (int j = 0; j < k; ++j) {
                int32_t row = slot_row[(int64_t)t * k + j];
                if (row < 0) continue;
                double wj = (double)w[(int64_t)t * k + j];
                for (int o = 0; o < d; ++o)
                    acc[o] += wj * load_elem(Yp, dtype, (int64_t)row * d + o);
            }
            for (int o = 0; o < d; ++o) store_elem(y, dtype, (int64_t)t * d + o, acc[o]);
        }
        free(acc);
    }
}

/* ------------------------------------------------------ popularity (a5) ---- */

/* Sliding-window expert popularity.  [Pop-3.1] per-expert token counts are the
 * popularity; [Pop-4.2] they are averaged over a window of recent iterations
 * (Eq. 1 is lost; reading: arithmetic mean of the last n = min(step+1, W)
 * count vectors).
 *  - hist is a ring of W count vectors; this step's counts go to slot step % W;
 *  - sum[e] = sum over the n most recent slots (int64);
 *  - mean[e] = (float)sum[e] / (float)n, one correctly rounded fp32 division;
 *  - hot = the P experts with the largest sum, ties to the lower index
 *    (the same order as the mean).
 * Returns 0, or -1 on invalid sizes. */
int oracle_popularity_update(const int32_t* counts, int E, int32_t* hist, int W,
                             int64_t step, float* mean, int P, int32_t* hot) {
    if (E <= 0 || W <= 0 || step < 0 || P < 0 || P > E) return -1;
    int slot = (int)(step % W);
    for (int e = 0; e < E; ++e) hist[(int64_t)slot * E + e] = counts[e];
    int64_t n = step + 1 < W ? step + 1 : W;
    int64_t* sum = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
    if (!sum || !taken) { free(sum); free(taken); return -1; }
    for (int64_t i = 0; i < n; ++i) {
        int s = (int)((step - i) % W);
        for (int e = 0; e < E; ++e) sum[e] += hist[(int64_t)s * E + e];
    }
    for (int e = 0; e < E; ++e) mean[e] = (float)sum[e] / (float)n;
    for (int p = 0; p < P; ++p) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || sum[e] > sum[best]) best = e;
        }
        taken[best] = 1;
        hot[p] = best;
    }
    free(sum);
    free(taken);
    return 0;
}

/* ------------------------------------------- cross-layer correlation (f2) -- */

/* Co-selection counts between consecutive MoE layers.  PopFetcher, section 4.1
 * (Fig. 6): a token that picks expert x at layer j and x' at layer j+1 forms a
 * correlated pair (x, x').  Every token t adds one to C[i][h] for each i among
 * its layer-j experts and each h among its layer-(j+1) experts.  C is [E][E]
 * int32 and is accumulated into (not cleared). */
void oracle_correlation_update(const int32_t* ids_prev, int k_prev, const int32_t* ids_next,
                               int k_next, int T, int E, int32_t* C) {
    for (int t = 0; t < T; ++t)
        for (int a = 0; a < k_prev; ++a)
            for (int b = 0; b < k_next; ++b) {
                int i = ids_prev[(int64_t)t * k_prev + a];
                int h = ids_next[(int64_t)t * k_next + b];
                C[(int64_t)i * E + h] += 1;
            }
}

/* Correlation-based popularity forecast.  PopFetcher, section 4.2, Eq. 2-3
 * (lost in extraction): the conditional probability that a token which chose
 * expert i at layer j chooses h at layer j+1, and the next layer's popularity
 * predicted from the previous layer's.  Reading taken:
 *   n_i     = tokens that chose i at layer j = (sum_h C[i][h]) / k_next
 *   P(h|i)  = C[i][h] / n_i                     (sum_h P(h|i) = k_next)
 *   pred[h] = sum_i pop_prev[i] * P(h|i) / k_prev
 * (pop_prev counts token-slots, each token k_prev times; rows with n_i = 0 add
 * nothing).  Evaluated in double in this fixed order, then rounded once to
 * fp32:  S_i = sum_h C[i][h];  q_i = (pop_prev[i] * k_next) / (S_i * k_prev);
 * pred[h] = sum over i ascending of q_i * C[i][h].  hot = the P experts with
 * the largest forecast, ties to the lower index. */
void oracle_popularity_forecast(const float* pop_prev, const int32_t* C, int E, int k_prev,
                                int k_next, float* pred, int P, int32_t* hot) {
    double* q = (double*)malloc(sizeof(double) * (size_t)E);
    unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
    if (!q || !taken) { free(q); free(taken); return; }
    for (int i = 0; i < E; ++i) {
        int64_t s = 0;
        for (int h = 0; h < E; ++h) s += C[(int64_t)i * E + h];
        q[i] = s == 0 ? 0.0
                      : ((double)pop_prev[i] * (double)k_next) / ((double)s * (double)k_prev);
    }
    for (int h = 0; h < E; ++h) {
        double a = 0.0;
        for (int i = 0; i < E; ++i) a += q[i] * (double)C[(int64_t)i * E + h];
        pred[h] = (float)a;
    }
    for (int p = 0; p < P; ++p) {
        int best = -1;
        for (int h = 0; h < E; ++h) {
            if (taken[h]) continue;
            if (best < 0 || pred[h] > pred[best]) best = h;
        }
        taken[best] = 1;
        hot[p] = best;
    }
    free(q);
    free(taken);
}

/* ----------------------------------------------- load-balancing loss (f4) -- */

/* GShard's auxiliary load-balancing loss.  PopFetcher, section 2.3.1, names it
 * (GShard spreads the workload evenly across workers with a balancing loss)
 * without the formula; reading taken (GShard / Switch form):
 *   f_e  = counts[e] / (T * k)          fraction of routed slots on expert e
 *   P_e  = (1/T) sum_t softmax(z_t)_e   mean router probability of expert e,
 *          z = logits + bias (one fp32 add, the routing keys)
 *   loss = E * sum_e f_e * P_e          (= 1 when routing and probabilities
 *                                         are both uniform)
 * In double, e ascending; loss and the P_e rounded once to fp32. */
float oracle_aux_loss(const float* logits, const float* bias, int T, int E, int k,
                      const int32_t* counts, float* prob_mean) {
    double* P = (double*)calloc((size_t)E, sizeof(double));
    double* ex = (double*)malloc(sizeof(double) * (size_t)E);
    if (!P || !ex) { free(P); free(ex); return NAN; }
    for (int t = 0; t < T; ++t) {
        double zmax = -INFINITY;
        for (int e = 0; e < E; ++e) {
            float z = logits[(int64_t)t * E + e] + (bias ? bias[e] : 0.0f);
            ex[e] = (double)z;
            if (ex[e] > zmax) zmax = ex[e];
        }
        double D = 0.0;
        for (int e = 0; e < E; ++e) {
            ex[e] = exp(ex[e] - zmax);
            D += ex[e];
        }
        for (int e = 0; e < E; ++e) P[e] += ex[e] / D;
    }
    double loss = 0.0;
    for (int e = 0; e < E; ++e) {
        double Pe = T > 0 ? P[e] / (double)T : 0.0;
        double fe = T > 0 ? (double)counts[e] / ((double)T * (double)k) : 0.0;
        loss += fe * Pe;
        if (prob_mean) prob_mean[e] = (float)Pe;
    }
    free(P);
    free(ex);
    return (float)((double)E * loss);
}

/* ------------------------------------------------------------ backward (f1) -- */

/* Backward of the MoE layer (PopFetcher, section 5.2.1: every expert GEMM of
 * the forward pass has two in the backward pass, for the input and for the
 * weights).  Gradients of the layer as written above, taken in exact
 * arithmetic at the stored forward values (the bf16 storage roundings of H and
 * Yp pass the gradient through unchanged), accumulated in double and rounded
 * once to the storage type of the tensor written.
 *
 * Output decode / combine:   dw[t][j]  = <dy[t], Yp[row]>            (fp32)
 *                            dYp[row]  = w[t][j] * dy[t]             (dtype)
 * for kept slots (row = slot_row[t][j] >= 0); dropped slots: dw = 0. */
void oracle_combine_backward(const void* dy, const void* Yp, int dtype, int T, int d, int k,
                             const int32_t* slot_row, const float* w, float* dw, void* dYp) {
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t s = (int64_t)t * k + j;
            int32_t row = slot_row[s];
            if (row < 0) { dw[s] = 0.0f; continue; }
            double dot = 0.0;
            for (int o = 0; o < d; ++o) {
                double g = load_elem(dy, dtype, (int64_t)t * d + o);
                dot += g * load_elem(Yp, dtype, (int64_t)row * d + o);
                store_elem(dYp, dtype, (int64_t)row * d + o, (double)w[s] * g);
            }
            dw[s] = (float)dot;
        }
}

/* Expert computation, backward, for the rows of each group e:
 *   dH[r][f]   = (H[r][f] > 0) ? sum_o dYp[r][o] W2[e][o][f] : 0      (ReLU)
 *   dXp[r][c]  = sum_f dH[r][f] W1[e][f][c]
 *   dW2[e][o][f] = sum_r dYp[r][o] H[r][f]      dW1[e][f][c] = sum_r dH[r][f] Xp[r][c]
 * dH is stored in dtype and that stored value feeds dXp and dW1 (as on the
 * GPU, where it is a tensor between two GEMMs).  dW1, dW2 are fp32; dH, dXp
 * dtype.  Any of dW1 / dW2 may be NULL. */
void oracle_expert_ffn_backward(const void* Xp, const void* H, const void* dYp, const void* W1,
                                const void* W2, int dtype, int E, int d, int F,
                                const int32_t* offsets, void* dH, void* dXp, float* dW1,
                                float* dW2) {
    double* g = (double*)malloc(sizeof(double) * (size_t)F);
    if (!g) return;
    for (int e = 0; e < E; ++e) {
        const int64_t w1b = (int64_t)e * F * d, w2b = (int64_t)e * d * F;
        for (int r = offsets[e]; r < offsets[e + 1]; ++r) {
            for (int f = 0; f < F; ++f) {
                double acc = 0.0;
                if (load_elem(H, dtype, (int64_t)r * F + f) > 0.0)
                    for (int o = 0; o < d; ++o)
                        acc += load_elem(dYp, dtype, (int64_t)r * d + o) *
                               load_elem(W2, dtype, w2b + (int64_t)o * F + f);
                store_elem(dH, dtype, (int64_t)r * F + f, acc);
                g[f] = load_elem(dH, dtype, (int64_t)r * F + f);
            }
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int f = 0; f < F; ++f)
                    acc += g[f] * load_elem(W1, dtype, w1b + (int64_t)f * d + c);
                store_elem(dXp, dtype, (int64_t)r * d + c, acc);
            }
        }
        if (dW2)
            for (int o = 0; o < d; ++o)
                for (int f = 0; f < F; ++f) {
                    double acc = 0.0;
                    for (int r = offsets[e]; r < offsets[e + 1]; ++r)
                        acc += load_elem(dYp, dtype, (int64_t)r * d + o) *
                               load_elem(H, dtype, (int64_t)r * F + f);
                    dW2[w2b + (int64_t)o * F + f] = (float)acc;
                }
        if (dW1)
            for (int f = 0; f < F; ++f)
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int r = offsets[e]; r < offsets[e + 1]; ++r)
                        acc += load_elem(dH, dtype, (int64_t)r * F + f) *
                               load_elem(Xp, dtype, (int64_t)r * d + c);
                    dW1[w1b + (int64_t)f * d + c] = (float)acc;
                }
    }
    free(g);
}

/* Input encode, backward: each token's rows return to it,
 * dx[t] = sum over kept slots of dXp[slot_row[t][j]], j ascending (dtype). */
void oracle_dispatch_backward(const void* dXp, int dtype, int T, int d, int k,
                              const int32_t* slot_row, void* dx) {
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int32_t row = slot_row[(int64_t)t * k + j];
                if (row >= 0) acc += load_elem(dXp, dtype, (int64_t)row * d + c);
            }
            store_elem(dx, dtype, (int64_t)t * d + c, acc);
        }
}

/* Gate routing, backward.  w_j = exp(z_j) / sum_{i in S_t} exp(z_i) over the
 * token's selected experts S_t (the renormalised softmax), so
 *   dz[t][e] = w_e (dw_e - sum_{i in S_t} w_i dw_i)  for e in S_t, else 0;
 * dlogits = dz (fp32, dense [T][E]); dbias[e] = sum_t dz[t][e] (fp32, may be
 * NULL).  The selection itself is piecewise constant and passes no gradient. */
void oracle_route_backward(const int32_t* ids, const float* w, const float* dw, int T, int E,
                           int k, float* dlogits, float* dbias) {
    double* db = (double*)calloc((size_t)E, sizeof(double));
    if (!db) return;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) dlogits[(int64_t)t * E + e] = 0.0f;
        double s = 0.0;
        for (int i = 0; i < k; ++i) s += (double)w[(int64_t)t * k + i] * (double)dw[(int64_t)t * k + i];
        for (int j = 0; j < k; ++j) {
            int e = ids[(int64_t)t * k + j];
            double dz = (double)w[(int64_t)t * k + j] * ((double)dw[(int64_t)t * k + j] - s);
            dlogits[(int64_t)t * E + e] = (float)dz;
            db[e] += dz;
        }
    }
    if (dbias)
        for (int e = 0; e < E; ++e) dbias[e] = (float)db[e];
    free(db);
}

/* Gate projection, backward: dx[t][c] += sum_e dlogits[t][e] Wg[e][c] (added
 * to the dtype values already in dx, rounded once) and
 * dWg[e][c] = sum_t dlogits[t][e] x[t][c] (fp32). */
void oracle_gate_backward(const void* x, const void* Wg, int dtype, int T, int d, int E,
                          const float* dlogits, void* dx, float* dWg) {
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = load_elem(dx, dtype, (int64_t)t * d + c);
            for (int e = 0; e < E; ++e)
                acc += (double)dlogits[(int64_t)t * E + e] * load_elem(Wg, dtype, (int64_t)e * d + c);
            store_elem(dx, dtype, (int64_t)t * d + c, acc);
        }
    for (int e = 0; e < E; ++e)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < T; ++t)
                acc += (double)dlogits[(int64_t)t * E + e] * load_elem(x, dtype, (int64_t)t * d + c);
            dWg[(int64_t)e * d + c] = (float)acc;
        }
}
