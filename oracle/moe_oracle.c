/*
 * moe_oracle.c -- float64 CPU reference for the forward pass of a sparse
 * Mixture-of-Experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE. Only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark load this library. The product path (the CUDA library)
 * never links, loads or calls it, and the two share no code.
 *
 * Style rules this file keeps so that a reader can check it against the pages:
 *   - one plain loop nest per formula, no blocking, no fusion;
 *   - every sum runs in ascending order of its reduction index;
 *   - all arithmetic is float64; BF16 / FP32 inputs are upcast exactly.
 *
 * Threads: the default build (no -fopenmp) runs on one thread.  The same
 * source compiled with -fopenmp (libmoe_oracle_omp.so, a CPU-baseline build)
 * splits the outer loops of the gate logits and of the layer rows over
 * threads: each output is still one thread's sum in the same order, so both
 * builds give the same bits.
 *
 * Sources (page title, section / equation):
 *   [ZM]  "Zen MoDE: Mixture of Distilled Experts Architecture"
 *         §3.1 Router Architecture (eq. router_standard), §5.2 Auxiliary Load
 *         Balancing Loss (eq. L_balance), §5.3 Adaptive Capacity Factors
 *         (capacity_e), §6.2 Expert Utilization (table tab:utilization),
 *         §7.1 Compute Budget (FLOPs ratio).
 *   [ZX]  "Zen-Max: Maximum Capability via Mixture-of-Experts Architecture"
 *         §2.2 Fine-Grained Expert Architecture (Expert_i, shared experts),
 *         §2.3 Auxiliary-Loss-Free Load Balancing (s_ij = softmax(x W_g)_j + b_j),
 *         §3.2 MoE-Specific Training Stability (router z-loss).
 *   [SE]  "Scaling with experts" (jeff-ong.com), sections "The gating network",
 *         "A balance penalty", "A budget", "A shared expert".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the OpenMP build uses from now on (n >= 1); returns the number it
 * will use.  The default build always returns 1. */
int oracle_set_threads(int32_t n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* Element type codes for inputs handed to the oracle. */
enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

/* Bias placement for selection (see oracle_select). */
enum { ORC_BIAS_PROB = 0, ORC_BIAS_LOGIT = 1 };

/* Bytes per element of an input type code. */
static size_t esz(int dt) { return dt == ORC_F64 ? 8 : dt == ORC_F32 ? 4 : 2; }

/* Exact upcast of element i of an input array to float64.  BF16 is the upper
 * half of an IEEE float32, so shifting it up 16 bits gives the float exactly. */
static double ld(const void* p, int dt, int64_t i) {
    if (dt == ORC_F64) return ((const double*)p)[i];
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------------------
 * Gate logits.  [ZM] §3.1: the standard router applies a linear projection
 * W_r to the token; [SE] "The gating network": one score per expert.
 *   logits[t,e] = sum_j x[t,j] * Wg[e,j]   (+ offset[e] when given)
 * Wg is stored as [E, d] (one row per expert).  The optional additive offset
 * is an input of the layer (used to impose a popularity prior on experts).
 * ------------------------------------------------------------------------- */
void oracle_gate_logits(int64_t T, int32_t d, int32_t E,
                        const void* x, int32_t x_dt,
                        const void* wg, int32_t wg_dt,
                        const float* offset, double* logits) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int32_t j = 0; j < d; ++j)
                acc += ld(x, x_dt, t * (int64_t)d + j) * ld(wg, wg_dt, (int64_t)e * d + j);
            if (offset) acc += (double)offset[e];
            logits[t * E + e] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Softmax over all E experts of one token.  [ZM] §3.1 eq. router_standard:
 * softmax(W_r x).  Shifted by the row maximum (the value is unchanged).
 *   p[t,e] = exp(l[t,e] - m_t) / sum_e' exp(l[t,e'] - m_t)
 * ------------------------------------------------------------------------- */
void oracle_softmax(int64_t T, int32_t E, const double* logits, double* p) {
    for (int64_t t = 0; t < T; ++t) {
        const double* l = logits + t * E;
        double m = l[0];
        for (int32_t e = 1; e < E; ++e)
            if (l[e] > m) m = l[e];
        double z = 0.0;
        for (int32_t e = 0; e < E; ++e) z += exp(l[e] - m);
        for (int32_t e = 0; e < E; ++e) p[t * E + e] = exp(l[e] - m) / z;
    }
}

/* ---------------------------------------------------------------------------
 * Top-K selection and renormalised gate weights.
 *
 * Selection score s[e]:
 *   no bias            : s = logit            (softmax is monotone, so this
 *                                              is TopK(softmax(W_r x)) of [ZM] §3.1)
 *   bias, BIAS_PROB    : s = p + b            ([ZX] §2.3: softmax(x W_g)_j + b_j)
 *   bias, BIAS_LOGIT   : s = logit + b        (variant: bias in logit space)
 * The bias steers selection only; gate weights never see it.
 * The K chosen experts are those with the largest s; equal scores go to the
 * lower expert index; they are listed in that order (largest s first).
 *
 * Gate weights ([SE] "The gating network": only the k best scores stay
 * non-zero and they are rescaled so that they add up to 1):
 *   w[t,k] = p[t, idx[t,k]] / sum_k' p[t, idx[t,k']]
 * which equals a softmax taken over the selected logits only.
 *
 * Returns 0, or -1 when K is outside [1, E].
 * ------------------------------------------------------------------------- */
int oracle_select(int64_t T, int32_t E, int32_t K,
                  const double* logits, const double* p,
                  const float* bias, int32_t bias_mode,
                  int32_t* idx, double* w) {
    if (K < 1 || K > E) return -1;
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) {
            double v = logits[t * E + e];
            if (bias) {
                if (bias_mode == ORC_BIAS_LOGIT) v = logits[t * E + e] + (double)bias[e];
                else                             v = p[t * E + e] + (double)bias[e];
            }
            s[e] = v;
            taken[e] = 0;
        }
        /* K passes; each takes the best remaining expert (strictly greater score
         * wins, so on a tie the earlier, i.e. lower, index is kept). */
        for (int32_t k = 0; k < K; ++k) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || s[e] > s[best]) best = e;
            }
            taken[best] = 1;
            idx[t * K + k] = best;
        }
        double denom = 0.0;
        for (int32_t k = 0; k < K; ++k) denom += p[t * E + idx[t * K + k]];
        for (int32_t k = 0; k < K; ++k) w[t * K + k] = p[t * E + idx[t * K + k]] / denom;
    }
    free(s);
    free(taken);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Per-expert capacity.  [ZM] §5.3: capacity_e = C * (batch*seq) / N_E, the
 * Switch top-1 form.  With top-K routing each token makes K assignments, so
 * the budget that keeps a uniform load whole is C * T * K / E; it is rounded
 * up to a whole number of rows.  C <= 0 means no limit (returns -1).
 * Computed in float64 as (C * (T*K)) / E, then ceil.
 * ------------------------------------------------------------------------- */
int64_t oracle_capacity(int64_t T, int32_t K, int32_t E, float C) {
    if (!(C > 0.0f)) return -1;
    double v = ((double)C * (double)(T * (int64_t)K)) / (double)E;
    return (int64_t)ceil(v);
}

/* ---------------------------------------------------------------------------
 * Capacity-limited dispatch.  [SE] "A budget": an expert accepts a bounded
 * number of tokens per batch; an assignment beyond that bound is dropped, so
 * the expert does not process that token, which keeps only its residual path.
 * [ZM] §5.3 lets that bound differ per expert (capacity_e), so it is given
 * here per expert:
 *
 *   counts[e]  = number of (t,k) with idx[t,k] == e               (pre-capacity)
 *   kept[e]    = min(counts[e], caps[e])    (counts[e] if caps[e] < 0)
 *   seg_off    = exclusive prefix sum of kept; seg_off[E] = total kept rows
 *   rank(t,k)  = number of tokens t' < t that also chose e = idx[t,k]
 *   kept iff rank < kept[e]; then slot_of[t,k] = seg_off[e] + rank and
 *   perm[slot] = t*K + k; otherwise slot_of[t,k] = -1.
 * Tokens are served in ascending token order (first come, first served).
 * Returns 0, or -1 on an expert index outside [0, E).
 * ------------------------------------------------------------------------- */
int oracle_dispatch_caps(int64_t T, int32_t K, int32_t E, const int64_t* caps,
                         const int32_t* idx,
                         int32_t* counts, int32_t* kept, int32_t* seg_off,
                         int32_t* slot_of, int32_t* perm) {
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < T * (int64_t)K; ++i) {
        if (idx[i] < 0 || idx[i] >= E) return -1;
        counts[idx[i]] += 1;
    }
    for (int32_t e = 0; e < E; ++e)
        kept[e] = (caps[e] < 0 || counts[e] < caps[e]) ? counts[e] : (int32_t)caps[e];
    seg_off[0] = 0;
    for (int32_t e = 0; e < E; ++e) seg_off[e + 1] = seg_off[e] + kept[e];

    int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int32_t e = idx[t * K + k];
            int32_t rank = seen[e];
            seen[e] += 1;
            if (rank < kept[e]) {
                int32_t slot = seg_off[e] + rank;
                slot_of[t * K + k] = slot;
                perm[slot] = (int32_t)(t * K + k);
            } else {
                slot_of[t * K + k] = -1;
            }
        }
    }
    free(seen);
    return 0;
}

/* The same dispatch with one capacity for every expert (cap < 0: no limit). */
int oracle_dispatch(int64_t T, int32_t K, int32_t E, int64_t cap,
                    const int32_t* idx,
                    int32_t* counts, int32_t* kept, int32_t* seg_off,
                    int32_t* slot_of, int32_t* perm) {
    int64_t* caps = (int64_t*)malloc((size_t)E * sizeof(int64_t));
    for (int32_t e = 0; e < E; ++e) caps[e] = cap;
    int rc = oracle_dispatch_caps(T, K, E, caps, idx, counts, kept, seg_off, slot_of, perm);
    free(caps);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Selection-bias update.  [ZX] §2.3 Auxiliary-Loss-Free Load Balancing: after
 * a training step each expert's bias b_e moves against the deviation of its
 * load from the target: an overloaded expert's bias goes down, an underloaded
 * one's up.  The page gives neither the load measure nor the step size; the
 * reading taken here: load = counts[e] (assignments before the capacity cut),
 * target = T*K / E (the mean load), step size `rate`, and either
 *   mode 0 (sign):          b_e += rate * sign(T*K - E*counts[e])
 *   mode 1 (proportional):  b_e += rate * (T*K - E*counts[e]) / (T*K)
 * (mode 1 is the relative deviation (target - load) / target).  Each update is
 * evaluated in float64 and rounded once to the float32 bias.  TK = T*K.
 * ------------------------------------------------------------------------- */
void oracle_bias_update(int32_t E, int64_t TK, const int32_t* counts, float* bias,
                        float rate, int32_t mode) {
    for (int32_t e = 0; e < E; ++e) {
        int64_t dev = TK - (int64_t)E * (int64_t)counts[e];   /* E * (target - load) */
        double step;
        if (mode == 0)
            step = (double)rate * (double)((dev > 0) - (dev < 0));
        else
            step = (double)rate * ((double)dev / (double)TK);
        bias[e] = (float)((double)bias[e] + step);
    }
}

/* ---------------------------------------------------------------------------
 * Adaptive per-expert capacity.  [ZM] §5.3 Adaptive Capacity Factors:
 *   C_e = C_base + gamma * (fbar_e - 1/N_E)
 * with fbar_e the expert's load fraction over a rolling window of recent
 * batches, so an expert that has been receiving less than its share gets a
 * smaller budget and one receiving more gets a larger one.  Reading: fbar_e is
 * the mean over the last n batches of f_e = counts[e] / (T*K) (the balance
 * statistic's f, pre-capacity); hist holds those n batches' counts, [n, E]
 * row-major (T and K fixed, so the mean of the fractions is the window's
 * summed counts over n*T*K).  The capacity is then capacity_e with C_e in
 * place of C, K-scaled like the uniform one:
 *   cap_e = ceil(C_e * (T*K) / E), clamped to [0, T].
 * ------------------------------------------------------------------------- */
void oracle_adaptive_capacity(int64_t T, int32_t K, int32_t E, const int32_t* hist, int32_t n,
                              float c_base, float gamma, int64_t* caps) {
    int64_t TK = T * (int64_t)K;
    for (int32_t e = 0; e < E; ++e) {
        int64_t s = 0;
        for (int32_t i = 0; i < n; ++i) s += hist[(int64_t)i * E + e];
        double fbar = (double)s / ((double)n * (double)TK);
        double ce = (double)c_base + (double)gamma * (fbar - 1.0 / (double)E);
        double v = ceil((ce * (double)TK) / (double)E);
        caps[e] = v <= 0.0 ? 0 : (v >= (double)T ? T : (int64_t)v);
    }
}

/* SiLU, [ZX] §2.2 (activation): silu(z) = z * sigmoid(z) = z / (1 + e^-z). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------------------
 * One SwiGLU expert applied to one token.  [ZX] §2.2 eq. Expert_i:
 *   Expert(x) = (SiLU(x W_gate) (.) x W_up) W_down
 * Storage ("linear [out, in]"): w13 is [2F, d] with rows 0..F-1 the gate
 * projection and rows F..2F-1 the up projection; w2 is [d, F].
 *   g[f] = sum_j w13[f, j]   x[j]
 *   u[f] = sum_j w13[F+f, j] x[j]
 *   h[f] = silu(g[f]) * u[f]
 *   out[i] += scale * sum_f w2[i, f] h[f]
 * h is caller scratch of F doubles.
 * ------------------------------------------------------------------------- */
void oracle_swiglu_accumulate(int32_t d, int32_t F, const double* x,
                              const void* w13, const void* w2, int32_t w_dt,
                              double scale, double* h, double* out) {
    for (int32_t f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (int32_t j = 0; j < d; ++j) {
            g += ld(w13, w_dt, (int64_t)f * d + j) * x[j];
            u += ld(w13, w_dt, (int64_t)(F + f) * d + j) * x[j];
        }
        h[f] = silu(g) * u;
    }
    for (int32_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t f = 0; f < F; ++f) acc += ld(w2, w_dt, (int64_t)i * F + f) * h[f];
        out[i] += scale * acc;
    }
}

/* One row of oracle_layer_rows (below): token t into yr (d doubles); xr, h scratch.
 * Returns -1 on an out-of-range token or expert, else 0. */
static int layer_row(int64_t T, int32_t d, int32_t E, int32_t K, int32_t F, int32_t n_shared,
                     const void* x, int32_t x_dt, const void* w13, const void* w2,
                     const void* w13_sh, const void* w2_sh, int32_t w_dt,
                     const int32_t* idx, const double* w, const int32_t* slot_of,
                     int64_t t, double* xr, double* h, double* yr) {
    const int64_t w13_stride = 2 * (int64_t)F * d;
    const int64_t w2_stride = (int64_t)d * F;
    if (t < 0 || t >= T) return -1;
    for (int32_t j = 0; j < d; ++j) xr[j] = ld(x, x_dt, t * d + j);
    for (int32_t i = 0; i < d; ++i) yr[i] = 0.0;
    for (int32_t s = 0; s < n_shared; ++s) {
        const char* a = (const char*)w13_sh + (size_t)(s * w13_stride) * esz(w_dt);
        const char* b = (const char*)w2_sh + (size_t)(s * w2_stride) * esz(w_dt);
        oracle_swiglu_accumulate(d, F, xr, a, b, w_dt, 1.0, h, yr);
    }
    for (int32_t k = 0; k < K; ++k) {
        if (slot_of[t * K + k] < 0) continue;
        int32_t e = idx[t * K + k];
        if (e < 0 || e >= E) return -1;
        const char* a = (const char*)w13 + (size_t)(e * w13_stride) * esz(w_dt);
        const char* b = (const char*)w2 + (size_t)(e * w2_stride) * esz(w_dt);
        oracle_swiglu_accumulate(d, F, xr, a, b, w_dt, w[t * K + k], h, yr);
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * The layer output for a list of tokens, given the routing.
 *   y[t] = sum_{s < N_s} Expert^shared_s(x_t)
 *        + sum_{k : slot_of[t,k] >= 0} w[t,k] * Expert_{idx[t,k]}(x_t)
 * Shared experts: always active, added unweighted ([ZX] §2.2; [SE] "A shared
 * expert").  Routed part: gate-weighted sum ([SE] "The gating network":
 * y = g1 Expert1(x) + g2 Expert2(x)).  A dropped pair contributes nothing and
 * the kept pairs are not rescaled again ([SE] "A budget").  The residual
 * add is outside the layer.
 * Layouts: x [T, d]; w13 [E, 2F, d]; w2 [E, d, F]; shared weights
 * [N_s, 2F, d] / [N_s, d, F]; y rows written for the listed tokens only:
 * y[r * d + i] for r = 0..n_rows-1 (row r is token rows[r]).
 * Returns 0, or -1 on an out-of-range token or expert.
 * ------------------------------------------------------------------------- */
int oracle_layer_rows(int64_t T, int32_t d, int32_t E, int32_t K, int32_t F, int32_t n_shared,
                      const void* x, int32_t x_dt,
                      const void* w13, const void* w2,
                      const void* w13_sh, const void* w2_sh, int32_t w_dt,
                      const int32_t* idx, const double* w, const int32_t* slot_of,
                      int64_t n_rows, const int64_t* rows, double* y) {
    int rc = 0;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)d);
        double* h = (double*)malloc(sizeof(double) * (size_t)F);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (layer_row(T, d, E, K, F, n_shared, x, x_dt, w13, w2, w13_sh, w2_sh, w_dt, idx, w, slot_of,
                          rows[r], xr, h, y + r * d) != 0) {
#pragma omp atomic write
                rc = -1;
            }
        }
        free(xr);
        free(h);
    }
    return rc;
}

/* ---------------------------------------------------------------------------
 * Combine expert-grouped outputs back to token order ([SE] "The gating
 * network": y = g1 Expert1(x) + g2 Expert2(x); "A budget": dropped pairs add
 * nothing; shared-expert output added unweighted):
 *   y[t, i] = y_shared[t, i] + sum_{k : slot_of[t,k] >= 0} w[t,k] * y_perm[slot_of[t,k], i]
 * y_perm rows and y_shared are inputs of any element type; y_shared may be NULL.
 * ------------------------------------------------------------------------- */
void oracle_combine(int64_t T, int32_t d, int32_t K,
                    const void* y_perm, int32_t yp_dt, const int32_t* slot_of, const double* w,
                    const void* y_shared, int32_t ys_dt, double* y) {
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t i = 0; i < d; ++i) {
            double acc = y_shared ? ld(y_shared, ys_dt, t * d + i) : 0.0;
            for (int32_t k = 0; k < K; ++k) {
                int32_t slot = slot_of[t * K + k];
                if (slot < 0) continue;
                acc += w[t * K + k] * ld(y_perm, yp_dt, (int64_t)slot * d + i);
            }
            y[t * d + i] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Switch balance statistics.  [ZM] §5.2 eq. L_balance and [SE] "A balance
 * penalty":  L = alpha * N * sum_e f_e P_e, with
 *   f_e = counts[e] / (T*K)   fraction of the batch's assignments sent to e
 *                             (counted before the capacity cut)
 *   P_e = (1/T) sum_t p[t,e]  mean softmax probability of e over the batch
 * With uniform routing (f_e = P_e = 1/E) the loss is exactly alpha.
 * ------------------------------------------------------------------------- */
void oracle_balance(int64_t T, int32_t E, int32_t K, const int32_t* counts,
                    const double* p, double alpha, double* f, double* P, double* loss) {
    double acc = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        f[e] = (double)counts[e] / (double)(T * (int64_t)K);
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) s += p[t * E + e];
        P[e] = s / (double)T;
    }
    for (int32_t e = 0; e < E; ++e) acc += f[e] * P[e];
    *loss = alpha * (double)E * acc;
}

/* ---------------------------------------------------------------------------
 * Router z-loss.  [ZX] §3.2: L_z = (1/B) sum_x (log sum_j e^{x_j})^2 over the
 * router logits of the B tokens.  (Coefficient applied by the caller.)
 * ------------------------------------------------------------------------- */
double oracle_router_zloss(int64_t T, int32_t E, const double* logits) {
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        const double* l = logits + t * E;
        double m = l[0];
        for (int32_t e = 1; e < E; ++e)
            if (l[e] > m) m = l[e];
        double z = 0.0;
        for (int32_t e = 0; e < E; ++e) z += exp(l[e] - m);
        double lse = m + log(z);
        acc += lse * lse;
    }
    return acc / (double)T;
}

/* ---------------------------------------------------------------------------
 * Expert utilisation statistics, [ZM] §6.2 table tab:utilization, from the
 * per-expert assignment counts (n = sum counts):
 *   out[0] entropy in bits of the load distribution q_e = counts[e]/n
 *          (0 log 0 = 0; at most log2 E, i.e. 7 bits for 128 experts)
 *   out[1] coefficient of variation of counts (population std / mean)
 *   out[2] token drop rate: dropped assignments / n
 *   out[3] experts whose load is below 50% of the mean
 *   out[4] experts whose load is above 200% of the mean
 * ------------------------------------------------------------------------- */
void oracle_utilization(int32_t E, const int32_t* counts, const int32_t* kept, double* out) {
    double n = 0.0, dropped = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        n += counts[e];
        dropped += (double)(counts[e] - kept[e]);
    }
    double mean = n / (double)E;
    double ent = 0.0, var = 0.0, below = 0.0, above = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        if (counts[e] > 0) {
            double q = (double)counts[e] / n;
            ent -= q * log2(q);
        }
        double dv = (double)counts[e] - mean;
        var += dv * dv;
        if ((double)counts[e] < 0.5 * mean) below += 1.0;
        if ((double)counts[e] > 2.0 * mean) above += 1.0;
    }
    var /= (double)E;
    out[0] = ent;
    out[1] = mean > 0.0 ? sqrt(var) / mean : 0.0;
    out[2] = n > 0.0 ? dropped / n : 0.0;
    out[3] = below;
    out[4] = above;
}

/* ---------------------------------------------------------------------------
 * Algorithmic FLOPs of one layer forward (multiply-add = 2 FLOPs):
 *   router   2 T d E
 *   experts  6 d F per kept (t,k) pair (three d x F projections)
 *   shared   6 d F N_s per token
 * and the ratio of expert FLOPs to the dense-equivalent cost of running every
 * expert on every token, T E 6 d F.  With no drops the ratio is
 * (K + N_s) / E, the [ZM] §7.1 compute-budget ratio (12/128 there).
 * out[0] = total FLOPs, out[1] = expert FLOPs, out[2] = the ratio.
 * ------------------------------------------------------------------------- */
void oracle_flops(int64_t T, int32_t d, int32_t E, int32_t F, int32_t n_shared,
                  int64_t kept_pairs, double* out) {
    double router = 2.0 * (double)T * d * E;
    double expert = 6.0 * (double)d * F * (double)kept_pairs + 6.0 * (double)d * F * n_shared * (double)T;
    out[0] = router + expert;
    out[1] = expert;
    out[2] = expert / (6.0 * (double)d * F * (double)E * (double)T);
}

/* ---------------------------------------------------------------------------
 * Backward of the layer, for training.  [SE] "The gating network": a token's
 * output is the gate-weighted sum of the experts it was sent to, so the loss
 * reaches an expert only through the tokens it processed and reaches the
 * router through those gates; [SE] "A balance penalty" and [ZX] §3.2 add two
 * scalar terms computed from the router's probabilities.
 *
 * Given dy = dJ/dy for the forward's output y, and c_bal, c_z = dJ/dL for the
 * balance loss L = alpha E sum_e f_e P_e and the router z-loss Lz =
 * (1/T) sum_t lse_t^2, with the routing held fixed (the choice of experts and
 * the capacity cut are piecewise constant, so they carry no gradient):
 *   kept pair (t,k), e = idx[t,k]:  g = Wgate_e x, u = Wup_e x, h = silu(g) u,
 *                                   o = Wdown_e h
 *     dw_k = <dy_t, o>,  do = w_k dy_t
 *     dWdown_e += do h^T;  dh = Wdown_e^T do
 *     dg = dh u silu'(g);  du = dh silu(g);  silu'(g) = s (1 + g (1 - s)), s = sigmoid(g)
 *     dWgate_e += dg x^T;  dWup_e += du x^T;  dx_t += Wgate_e^T dg + Wup_e^T du
 *   dropped pair: dw_k = 0
 *   shared expert s: the same with weight 1, for every token
 *   router (w = softmax over the K chosen logits, p = softmax over all E):
 *     dl_{i_k} += w_k (dw_k - sum_k' w_k' dw_k')
 *     dl_e += p_e (q_e - sum_j p_j q_j),  q_e = c_bal alpha E f_e / T
 *     dl_e += c_z (2 / T) lse_t p_e
 *     dWg += dl x^T;  doffset += dl;  dx_t += Wg^T dl
 * f_e = counts[e] / (T K) as in the forward statistics.  Outputs are
 * overwritten, all in float64: dx [T,d], dw13 [E,2F,d], dw2 [E,d,F],
 * dw13_sh [Ns,2F,d], dw2_sh [Ns,d,F], dwg [E,d], doff [E], and dlogits
 * [T,E] (the dl above) when not NULL.  logits [T,E] are the forward's (offset
 * included).  Returns 0, or -1 on a bad expert index.
 * ------------------------------------------------------------------------- */
int oracle_layer_backward(int64_t T, int32_t d, int32_t E, int32_t K, int32_t F, int32_t n_shared,
                          const void* x, int32_t x_dt, const void* wg, const void* w13, const void* w2,
                          const void* w13_sh, const void* w2_sh, int32_t w_dt,
                          const double* logits, const int32_t* idx, const double* w, const int32_t* slot_of,
                          const int32_t* counts, double alpha, const double* dy, double c_bal, double c_z,
                          double* dx, double* dw13, double* dw2, double* dw13_sh, double* dw2_sh,
                          double* dwg, double* doff, double* dlogits) {
    const int64_t w13_stride = 2 * (int64_t)F * d;
    const int64_t w2_stride = (int64_t)d * F;
    for (int64_t i = 0; i < T * d; ++i) dx[i] = 0.0;
    for (int64_t i = 0; i < E * w13_stride; ++i) dw13[i] = 0.0;
    for (int64_t i = 0; i < E * w2_stride; ++i) dw2[i] = 0.0;
    for (int64_t i = 0; i < n_shared * w13_stride; ++i) dw13_sh[i] = 0.0;
    for (int64_t i = 0; i < n_shared * w2_stride; ++i) dw2_sh[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)E * d; ++i) dwg[i] = 0.0;
    for (int32_t e = 0; e < E; ++e) doff[e] = 0.0;

    double* xr = (double*)malloc(sizeof(double) * (size_t)d);
    double* g = (double*)malloc(sizeof(double) * (size_t)F);
    double* u = (double*)malloc(sizeof(double) * (size_t)F);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* dh = (double*)malloc(sizeof(double) * (size_t)F);
    double* dz = (double*)malloc(sizeof(double) * (size_t)F);   /* dg */
    double* dv = (double*)malloc(sizeof(double) * (size_t)F);   /* du */
    double* dwk = (double*)malloc(sizeof(double) * (size_t)K);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    double* dl = (double*)malloc(sizeof(double) * (size_t)E);
    double* q = (double*)malloc(sizeof(double) * (size_t)E);
    int rc = 0;
    for (int32_t e = 0; e < E; ++e)
        q[e] = c_bal * alpha * (double)E * ((double)counts[e] / ((double)T * (double)K)) / (double)T;

    for (int64_t t = 0; t < T && rc == 0; ++t) {
        for (int32_t j = 0; j < d; ++j) xr[j] = ld(x, x_dt, t * d + j);
        const double* dyt = dy + t * d;
        double* dxt = dx + t * d;
        /* experts: n_shared shared ones (weight 1), then the token's K pairs */
        for (int32_t r = 0; r < n_shared + K; ++r) {
            const void *a, *b;
            double* da;
            double* db;
            double scale;
            if (r < n_shared) {
                a = (const char*)w13_sh + (size_t)(r * w13_stride) * esz(w_dt);
                b = (const char*)w2_sh + (size_t)(r * w2_stride) * esz(w_dt);
                da = dw13_sh + r * w13_stride;
                db = dw2_sh + r * w2_stride;
                scale = 1.0;
            } else {
                int32_t k = r - n_shared;
                dwk[k] = 0.0;
                if (slot_of[t * K + k] < 0) continue;
                int32_t e = idx[t * K + k];
                if (e < 0 || e >= E) { rc = -1; break; }
                a = (const char*)w13 + (size_t)(e * w13_stride) * esz(w_dt);
                b = (const char*)w2 + (size_t)(e * w2_stride) * esz(w_dt);
                da = dw13 + e * w13_stride;
                db = dw2 + e * w2_stride;
                scale = w[t * K + k];
            }
            for (int32_t f = 0; f < F; ++f) {
                double gg = 0.0, uu = 0.0;
                for (int32_t j = 0; j < d; ++j) {
                    gg += ld(a, w_dt, (int64_t)f * d + j) * xr[j];
                    uu += ld(a, w_dt, (int64_t)(F + f) * d + j) * xr[j];
                }
                g[f] = gg;
                u[f] = uu;
                h[f] = silu(gg) * uu;
            }
            if (r >= n_shared) {   /* dw_k = <dy_t, o>, o = Wdown h */
                double acc = 0.0;
                for (int32_t i = 0; i < d; ++i) {
                    double o = 0.0;
                    for (int32_t f = 0; f < F; ++f) o += ld(b, w_dt, (int64_t)i * F + f) * h[f];
                    acc += dyt[i] * o;
                }
                dwk[r - n_shared] = acc;
            }
            /* do = scale dy_t */
            for (int32_t f = 0; f < F; ++f) dh[f] = 0.0;
            for (int32_t i = 0; i < d; ++i) {
                double doi = scale * dyt[i];
                for (int32_t f = 0; f < F; ++f) {
                    db[(int64_t)i * F + f] += doi * h[f];
                    dh[f] += ld(b, w_dt, (int64_t)i * F + f) * doi;
                }
            }
            for (int32_t f = 0; f < F; ++f) {
                double sg = 1.0 / (1.0 + exp(-g[f]));
                dz[f] = dh[f] * u[f] * (sg * (1.0 + g[f] * (1.0 - sg)));
                dv[f] = dh[f] * silu(g[f]);
            }
            for (int32_t f = 0; f < F; ++f) {
                for (int32_t j = 0; j < d; ++j) {
                    da[(int64_t)f * d + j] += dz[f] * xr[j];
                    da[(int64_t)(F + f) * d + j] += dv[f] * xr[j];
                    dxt[j] += ld(a, w_dt, (int64_t)f * d + j) * dz[f] + ld(a, w_dt, (int64_t)(F + f) * d + j) * dv[f];
                }
            }
        }
        if (rc) break;
        /* router */
        const double* lt = logits + t * E;
        double m = lt[0];
        for (int32_t e = 1; e < E; ++e) if (lt[e] > m) m = lt[e];
        double zs = 0.0;
        for (int32_t e = 0; e < E; ++e) { p[e] = exp(lt[e] - m); zs += p[e]; }
        for (int32_t e = 0; e < E; ++e) p[e] /= zs;
        double lse = m + log(zs);
        for (int32_t e = 0; e < E; ++e) dl[e] = 0.0;
        double wdw = 0.0;
        for (int32_t k = 0; k < K; ++k) wdw += w[t * K + k] * dwk[k];
        for (int32_t k = 0; k < K; ++k) {
            int32_t e = idx[t * K + k];
            if (e < 0 || e >= E) { rc = -1; break; }
            dl[e] += w[t * K + k] * (dwk[k] - wdw);
        }
        if (rc) break;
        double pq = 0.0;
        for (int32_t e = 0; e < E; ++e) pq += p[e] * q[e];
        for (int32_t e = 0; e < E; ++e) {
            dl[e] += p[e] * (q[e] - pq);
            dl[e] += c_z * (2.0 / (double)T) * lse * p[e];
        }
        if (dlogits)
            for (int32_t e = 0; e < E; ++e) dlogits[t * E + e] = dl[e];
        for (int32_t e = 0; e < E; ++e) {
            doff[e] += dl[e];
            for (int32_t j = 0; j < d; ++j) {
                dwg[(int64_t)e * d + j] += dl[e] * xr[j];
                dxt[j] += ld(wg, w_dt, (int64_t)e * d + j) * dl[e];
            }
        }
    }
    free(xr); free(g); free(u); free(h); free(dh); free(dz); free(dv); free(dwk); free(p); free(dl); free(q);
    return rc;
}
