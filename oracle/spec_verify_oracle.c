/*
 * Plain fp64 CPU oracle for batched speculative-sampling verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * execute this file; only tests/, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library: it restates the method from the pages in the plainest way, one
 * sequence at a time, single threaded, every value held in double.
 *
 * Source of the method (speculative decoding encyclopedia entry "推测解码",
 * glopedia.cn/401080):
 *   - section "提议与核验的基本步骤", paragraph 2: the draft token x at
 *     position i is accepted with probability min(1, p(x)/q(x)); p and q are
 *     the conditional probabilities under the sampling settings actually in
 *     use; acceptance stops at the first rejection; the rejected position is
 *     redrawn from the normalised positive residual max(0, p - q); when every
 *     candidate passes, one extra token is drawn from the target.
 *   - same section, paragraph 3: the worked example (A/B/C, 0.6/0.3/0.1 vs
 *     0.5/0.4/0.1) used as a pin in the tests.
 *   - same section, paragraph 4: greedy verification compares the draft with
 *     the target's most probable token and replaces it at the first
 *     mismatch; temperature / top-k must be applied identically to p and q
 *     and kept consistent in the correction step.
 *   - same section, paragraph 1: the target scores the k+1 positions in one
 *     forward pass; its last step, the output projection of the hidden
 *     states, is written out in oracle_head_logits (end of this file) for
 *     greedy verification on the logits it forms.
 *
 * Readings of what the pages leave open (each stated where it is used):
 *   R1 accept iff u*q < p  (i.e. u < min(1, p/q) for u in [0,1));
 *   R2 the final draw (correction or bonus) uses its own uniform u_k;
 *   R3 inverse CDF: smallest v with C_v > u*W, C the running sum in index
 *      order, W = C_{V-1}; if none (rounding) the largest v with w_v > 0;
 *   R4 top-k keeps every logit >= tau, tau = K-th largest raw logit counted
 *      with multiplicity (ties at tau are all kept);
 *   R5 temperature divides the logits before the softmax; top-k is chosen on
 *      the raw logits;
 *   R6 greedy: lowest index among equal maxima, values compared as numbers
 *      (-0.0 == +0.0); after a full match the target's argmax at position k
 *      is emitted; temperature, top-k and uniforms are ignored;
 *   R7 row errors: a NaN or +inf logit, no finite kept logit, a draft token
 *      outside [0, V), a temperature that is not finite and > 0 (stochastic
 *      only), a uniform outside [0, 1) (stochastic only).  The whole
 *      sequence is then reported as n = -1 with every token -1;
 *   R8 if the residual mass W is zero at a rejected position the
 *      replacement is drawn from p at that position with the same rule.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_DTYPE_BF16 0
#define OR_DTYPE_F32 1
#define OR_DTYPE_F64 2 /* logits formed here (the output projection below) */

/* ---- reading logits (bf16 widening is exact) ---------------------------- */

static double or_logit(const void* row, int dtype, long v) {
    if (dtype == OR_DTYPE_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t*)row)[v]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    if (dtype == OR_DTYPE_F64) return ((const double*)row)[v];
    return (double)((const float*)row)[v];
}

static const void* or_row(const void* base, int dtype, long row, long V) {
    size_t elt = dtype == OR_DTYPE_BF16 ? 2 : (dtype == OR_DTYPE_F64 ? 8 : 4);
    return (const char*)base + (size_t)row * (size_t)V * elt;
}

static int cmp_desc(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

/*
 * Logits processing of one row, the same for target and draft (section
 * "提议与核验的基本步骤", paragraph 4: processing rules applied identically).
 *   kept = all v, or {v : z_v >= tau} when 0 < top_k < V        (R4)
 *   s_v = z_v / T, m = max_kept s, e_v = exp(s_v - m), S = sum_kept e_v
 *   prob_v = e_v / S on kept entries, 0 elsewhere.
 * Returns 0, or 1 for a row error (R7).  `work` holds V doubles.
 */
int oracle_process_row(const void* row, int dtype, int V, double T, int top_k,
                       double* prob, double* work) {
    long v;
    double tau = -INFINITY, m = -INFINITY, S = 0.0;
    if (!(T > 0.0) || isinf(T)) return 1;
    for (v = 0; v < V; ++v) {
        double z = or_logit(row, dtype, v);
        if (isnan(z) || z == INFINITY) return 1;
        work[v] = z;
    }
    if (top_k > 0 && top_k < V) {
        qsort(work, (size_t)V, sizeof(double), cmp_desc);
        tau = work[top_k - 1];
    }
    for (v = 0; v < V; ++v) {
        double z = or_logit(row, dtype, v);
        if (z >= tau && z / T > m) m = z / T;
    }
    if (m == -INFINITY) return 1;
    for (v = 0; v < V; ++v) {
        double z = or_logit(row, dtype, v);
        prob[v] = (z >= tau) ? exp(z / T - m) : 0.0;
        S += prob[v];
    }
    for (v = 0; v < V; ++v) prob[v] /= S;
    return 0;
}

/* Lowest-index argmax of the raw row (R6).  Returns -1 on a row error. */
int oracle_argmax_row(const void* row, int dtype, int V) {
    long v;
    int best = -1;
    double bv = -INFINITY;
    for (v = 0; v < V; ++v) {
        double z = or_logit(row, dtype, v);
        if (isnan(z) || z == INFINITY) return -1;
        if (z > bv) {
            bv = z;
            best = (int)v;
        }
    }
    return best; /* -1 when every entry is -inf */
}

/*
 * Inverse-CDF draw from non-negative weights w (R3).  Writes the token and
 * the two CDF points C_{y-1}/W and C_y/W around it.  Returns 1 if W == 0.
 */
int oracle_inverse_cdf(const double* w, int V, double u, int* token, double* cdf_lo,
                       double* cdf_hi) {
    long v;
    double W = 0.0, C = 0.0, x;
    int last_pos = -1;
    for (v = 0; v < V; ++v) {
        W += w[v];
        if (w[v] > 0.0) last_pos = (int)v;
    }
    if (!(W > 0.0)) return 1;
    x = u * W;
    for (v = 0; v < V; ++v) {
        double prev = C;
        C += w[v];
        if (C > x) {
            *token = (int)v;
            *cdf_lo = prev / W;
            *cdf_hi = C / W;
            return 0;
        }
    }
    /* rounding left u*W at or above the running total: largest positive v */
    C = 0.0;
    for (v = 0; v < last_pos; ++v) C += w[v];
    *token = last_pos;
    *cdf_lo = C / W;
    *cdf_hi = (C + w[last_pos]) / W;
    return 0;
}

/*
 * Batched verification, one sequence after another.
 *   target        [B][k+1][V]   dtype
 *   draft         [B][k][V]     dtype (ignored when greedy != 0)
 *   draft_tokens  [B][k]
 *   uniforms      [B][k+1]      u_0..u_{k-1} acceptance, u_k final draw (R2)
 *   temperature   [B] or NULL (all 1.0)
 * Outputs: out_tokens [B][k+1], out_n [B]; optional (NULL to skip)
 *   out_p, out_q  [B][k]   p_i(d_i), q_i(d_i) at every position i < k
 *   out_ratio     [B][k]   acceptance threshold min(1, p/q) (q = 0: 1 if p>0 else 0)
 *   out_lo, out_hi [B]     CDF points around the final token
 * Returns the number of sequences reported as row errors.
 */
int oracle_verify(const void* target, const void* draft, const int32_t* draft_tokens,
                  const float* uniforms, int B, int k, int V, const float* temperature,
                  int top_k, int greedy, int dtype, int32_t* out_tokens, int32_t* out_n,
                  double* out_p, double* out_q, double* out_ratio, double* out_lo,
                  double* out_hi) {
    int b, i, errors = 0;
    double* pt = (double*)malloc(sizeof(double) * (size_t)(k + 1) * (size_t)V);
    double* pd = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1) * (size_t)V);
    double* w = (double*)malloc(sizeof(double) * (size_t)V);
    double* work = (double*)malloc(sizeof(double) * (size_t)V);
    if (!pt || !pd || !w || !work) {
        free(pt); free(pd); free(w); free(work);
        return -1;
    }
    for (b = 0; b < B; ++b) {
        int32_t* tok = out_tokens + (size_t)b * (k + 1);
        const int32_t* d = draft_tokens + (size_t)b * k;
        const float* u = uniforms ? uniforms + (size_t)b * (k + 1) : NULL;
        double T = temperature ? (double)temperature[b] : 1.0;
        int err = 0, j = k, y = -1;
        double lo = NAN, hi = NAN;
        for (i = 0; i < k; ++i)
            if (d[i] < 0 || d[i] >= V) err = 1;
        for (i = 0; i <= k; ++i) tok[i] = -1;
        if (out_p) for (i = 0; i < k; ++i) out_p[(size_t)b * k + i] = NAN;
        if (out_q) for (i = 0; i < k; ++i) out_q[(size_t)b * k + i] = NAN;
        if (out_ratio) for (i = 0; i < k; ++i) out_ratio[(size_t)b * k + i] = NAN;

        if (greedy) {
            /* R6: g_i = argmax of target row i; the first mismatch emits g_j.
             * Every row is examined so that a bad row anywhere is reported. */
            for (i = 0; i <= k && !err; ++i) {
                int g = oracle_argmax_row(or_row(target, dtype, (long)b * (k + 1) + i, V), dtype, V);
                if (g < 0) {
                    err = 1;
                } else if (i < k && j == k && d[i] != g) {
                    j = i;
                    y = g;
                } else if (i == k && j == k) {
                    y = g;
                }
            }
        } else {
            if (!(T > 0.0) || isinf(T) || isnan(T)) err = 1;
            for (i = 0; i <= k && !err; ++i)
                if (!(u[i] >= 0.0f && u[i] < 1.0f)) err = 1;
            for (i = 0; i <= k && !err; ++i)
                err |= oracle_process_row(or_row(target, dtype, (long)b * (k + 1) + i, V), dtype,
                                          V, T, top_k, pt + (size_t)i * V, work);
            for (i = 0; i < k && !err; ++i)
                err |= oracle_process_row(or_row(draft, dtype, (long)b * k + i, V), dtype, V, T,
                                          top_k, pd + (size_t)i * V, work);
            if (!err) {
                long v;
                int found = 0;
                /* p_i(d_i), q_i(d_i) at every position; R1 for the decisions */
                for (i = 0; i < k; ++i) {
                    double p = pt[(size_t)i * V + d[i]], q = pd[(size_t)i * V + d[i]];
                    if (out_p) out_p[(size_t)b * k + i] = p;
                    if (out_q) out_q[(size_t)b * k + i] = q;
                    if (out_ratio)
                        out_ratio[(size_t)b * k + i] = q > 0.0 ? (p / q < 1.0 ? p / q : 1.0)
                                                               : (p > 0.0 ? 1.0 : 0.0);
                    if (!found && !((double)u[i] * q < p)) {
                        j = i;
                        found = 1;
                    }
                }
                if (j < k) {
                    /* residual max(0, p_j - q_j), R8 if it has no mass */
                    for (v = 0; v < V; ++v) {
                        double r = pt[(size_t)j * V + v] - pd[(size_t)j * V + v];
                        w[v] = r > 0.0 ? r : 0.0;
                    }
                    if (oracle_inverse_cdf(w, V, (double)u[k], &y, &lo, &hi))
                        oracle_inverse_cdf(pt + (size_t)j * V, V, (double)u[k], &y, &lo, &hi);
                } else {
                    /* bonus token from the processed target at position k */
                    oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[k], &y, &lo, &hi);
                }
            }
        }
        if (err) {
            out_n[b] = -1;
            errors++;
        } else {
            for (i = 0; i < j; ++i) tok[i] = d[i];
            tok[j] = y;
            out_n[b] = j;
        }
        if (out_lo) out_lo[b] = lo;
        if (out_hi) out_hi[b] = hi;
    }
    free(pt); free(pd); free(w); free(work);
    return errors;
}

/*
 * Proposer sampling step, one token per row (the draft side of a round):
 * stochastic rows draw from the processed row with the inverse CDF (R3, R4,
 * R5) and their own uniform; greedy rows take the lowest-index argmax (R6).
 *   logits [rows][V], temperature [rows] or NULL, u [rows] (stochastic)
 * out_tokens[r] = -1 on a row error.  out_lo/out_hi optional.
 */
int oracle_sample_rows(const void* logits, int dtype, int rows, int V, const float* temperature,
                       int top_k, int greedy, const float* u, int32_t* out_tokens,
                       double* out_lo, double* out_hi) {
    int r, errors = 0;
    double* prob = (double*)malloc(sizeof(double) * (size_t)V);
    double* work = (double*)malloc(sizeof(double) * (size_t)V);
    if (!prob || !work) {
        free(prob); free(work);
        return -1;
    }
    for (r = 0; r < rows; ++r) {
        const void* row = or_row(logits, dtype, r, V);
        int y = -1;
        double lo = NAN, hi = NAN;
        if (greedy) {
            y = oracle_argmax_row(row, dtype, V);
        } else {
            double T = temperature ? (double)temperature[r] : 1.0;
            if ((u[r] >= 0.0f && u[r] < 1.0f) &&
                oracle_process_row(row, dtype, V, T, top_k, prob, work) == 0) {
                if (oracle_inverse_cdf(prob, V, (double)u[r], &y, &lo, &hi)) y = -1;
            }
        }
        if (y < 0) errors++;
        out_tokens[r] = y;
        if (out_lo) out_lo[r] = lo;
        if (out_hi) out_hi[r] = hi;
    }
    free(prob); free(work);
    return errors;
}

/* ==== further logits processors ============================================
 *
 * Section "提议与核验的基本步骤", paragraph 4, names nucleus sampling,
 * repetition penalties and vocabulary masks (with temperature and top-k) among
 * the processing rules that must be applied to the target and the draft
 * distributions alike, and kept consistent in the correction step.  The page
 * does not define them; the readings taken here:
 *   R12 order: repetition penalty and vocabulary mask act on the raw logits,
 *       then top-k (R4) on the result, then temperature and the softmax (R5),
 *       then the nucleus on the resulting probabilities;
 *   R13 repetition penalty theta > 0 and finite (else a row error) on the
 *       sequence's listed token ids (each
 *       id once, ids outside [0, V) ignored): z -> z / theta if z > 0, else
 *       z * theta, the result rounded to fp32 (the logit's quotient or product
 *       of two fp32 values, correctly rounded: computing it in double and
 *       rounding once gives exactly that, as 53 >= 2 * 24 + 2 bits).  The
 *       penalised logit decides the top-k set, so both sides take that
 *       decision on the same fp32 value;
 *   R14 vocabulary mask: token v is allowed iff bit (v % 32) of word v / 32 is
 *       set; a disallowed token gets the logit -inf (probability 0);
 *   R15 nucleus 0 < top_p <= 1: order the tokens of positive probability by
 *       probability descending (equal ones by index), take the first at which
 *       the running sum reaches top_p, keep every token whose probability is
 *       >= that token's (equal probabilities are all kept), renormalise;
 *       top_p = 1 keeps every token.
 * The same processors apply to every target and draft row of a sequence. */

typedef struct {
    double top_p;           /* R15, 1 disables */
    double rep_penalty;     /* R13, 1 disables */
    const int32_t* rep_ids; /* n_rep ids, or NULL */
    int n_rep;
    const uint32_t* mask;   /* ceil(V/32) words, or NULL (all allowed) */
} or_procs_t;

typedef struct {
    double p;
    long v;
} or_pv_t;

static int cmp_pv_desc(const void* a, const void* b) {
    const or_pv_t* x = (const or_pv_t*)a;
    const or_pv_t* y = (const or_pv_t*)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->v > y->v) - (x->v < y->v);
}

/* Raw logit of token v after the repetition penalty and the mask (R13, R14). */
static double or_logit_procs(const void* row, int dtype, long v, const or_procs_t* pr) {
    double z = or_logit(row, dtype, v);
    int i;
    if (pr->mask && !((pr->mask[v / 32] >> (v % 32)) & 1u)) return -INFINITY;
    if (pr->rep_ids && pr->rep_penalty != 1.0) {
        for (i = 0; i < pr->n_rep; ++i) {
            if (pr->rep_ids[i] == v) {
                /* rounded to fp32, the precision the kernels rank and exponentiate in */
                z = z > 0.0 ? (double)(float)(z / pr->rep_penalty) : (double)(float)(z * pr->rep_penalty);
                break; /* each id once */
            }
        }
    }
    return z;
}

/*
 * oracle_process_row with the processors of R12..R15.  `work` holds V
 * doubles, `pv` V pairs (only used when top_p < 1).  Returns 0, or 1 for a
 * row error (R7; every token disallowed counts as "no finite kept logit").
 */
int oracle_process_row_procs(const void* row, int dtype, int V, double T, int top_k,
                             const or_procs_t* pr, double* prob, double* work, void* pv_buf) {
    long v, n = 0, i;
    double tau = -INFINITY, m = -INFINITY, S = 0.0;
    if (!(T > 0.0) || isinf(T)) return 1;
    if (!(pr->top_p > 0.0 && pr->top_p <= 1.0) || !(pr->rep_penalty > 0.0) || isinf(pr->rep_penalty))
        return 1;
    for (v = 0; v < V; ++v) {
        double z0 = or_logit(row, dtype, v);
        if (isnan(z0) || z0 == INFINITY) return 1;
        work[v] = or_logit_procs(row, dtype, v, pr);
    }
    for (v = 0; v < V; ++v) prob[v] = work[v]; /* processed logits, kept for below */
    if (top_k > 0 && top_k < V) {
        qsort(work, (size_t)V, sizeof(double), cmp_desc);
        tau = work[top_k - 1];
    }
    for (v = 0; v < V; ++v)
        if (prob[v] >= tau && prob[v] / T > m) m = prob[v] / T;
    if (m == -INFINITY) return 1;
    for (v = 0; v < V; ++v) {
        double z = prob[v];
        prob[v] = (z >= tau) ? exp(z / T - m) : 0.0;
        S += prob[v];
    }
    for (v = 0; v < V; ++v) prob[v] /= S;
    if (pr->top_p < 1.0) {
        or_pv_t* pv = (or_pv_t*)pv_buf;
        double run = 0.0, cut = 0.0, K2 = 0.0;
        for (v = 0; v < V; ++v)
            if (prob[v] > 0.0) {
                pv[n].p = prob[v];
                pv[n].v = v;
                ++n;
            }
        qsort(pv, (size_t)n, sizeof(or_pv_t), cmp_pv_desc);
        cut = n > 0 ? pv[n - 1].p : 0.0;
        for (i = 0; i < n; ++i) {
            run += pv[i].p;
            if (run >= pr->top_p) {
                cut = pv[i].p;
                break;
            }
        }
        for (v = 0; v < V; ++v) {
            if (!(prob[v] >= cut)) prob[v] = 0.0;
            K2 += prob[v];
        }
        for (v = 0; v < V; ++v) prob[v] /= K2;
    }
    return 0;
}

/*
 * oracle_verify with per-sequence processors (R12..R15): top_p [B] or NULL
 * (all 1), rep_penalty [B] or NULL (all 1), rep_ids [B][n_rep] (entries < 0
 * unused) or NULL, mask [B][ceil(V/32)] or NULL.  Same outputs and return
 * value as oracle_verify, whose steps it follows.
 */
int oracle_verify_procs(const void* target, const void* draft, const int32_t* draft_tokens,
                        const float* uniforms, int B, int k, int V, const float* temperature,
                        int top_k, int dtype, const float* top_p, const float* rep_penalty,
                        const int32_t* rep_ids, int n_rep, const uint32_t* mask,
                        int32_t* out_tokens, int32_t* out_n, double* out_p, double* out_q,
                        double* out_ratio, double* out_lo, double* out_hi) {
    int b, i, errors = 0;
    const long words = (V + 31) / 32;
    double* pt = (double*)malloc(sizeof(double) * (size_t)(k + 1) * (size_t)V);
    double* pd = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1) * (size_t)V);
    double* w = (double*)malloc(sizeof(double) * (size_t)V);
    double* work = (double*)malloc(sizeof(double) * (size_t)V);
    or_pv_t* pv = (or_pv_t*)malloc(sizeof(or_pv_t) * (size_t)V);
    if (!pt || !pd || !w || !work || !pv) {
        free(pt); free(pd); free(w); free(work); free(pv);
        return -1;
    }
    for (b = 0; b < B; ++b) {
        int32_t* tok = out_tokens + (size_t)b * (k + 1);
        const int32_t* d = draft_tokens + (size_t)b * k;
        const float* u = uniforms + (size_t)b * (k + 1);
        double T = temperature ? (double)temperature[b] : 1.0;
        or_procs_t pr;
        int err = 0, j = k, y = -1;
        double lo = NAN, hi = NAN;
        pr.top_p = top_p ? (double)top_p[b] : 1.0;
        pr.rep_penalty = rep_penalty ? (double)rep_penalty[b] : 1.0;
        pr.rep_ids = rep_ids ? rep_ids + (size_t)b * n_rep : NULL;
        pr.n_rep = rep_ids ? n_rep : 0;
        pr.mask = mask ? mask + (size_t)b * words : NULL;
        for (i = 0; i < k; ++i)
            if (d[i] < 0 || d[i] >= V) err = 1;
        for (i = 0; i <= k; ++i) tok[i] = -1;
        if (out_p) for (i = 0; i < k; ++i) out_p[(size_t)b * k + i] = NAN;
        if (out_q) for (i = 0; i < k; ++i) out_q[(size_t)b * k + i] = NAN;
        if (out_ratio) for (i = 0; i < k; ++i) out_ratio[(size_t)b * k + i] = NAN;
        if (!(T > 0.0) || isinf(T) || isnan(T)) err = 1;
        for (i = 0; i <= k && !err; ++i)
            if (!(u[i] >= 0.0f && u[i] < 1.0f)) err = 1;
        for (i = 0; i <= k && !err; ++i)
            err |= oracle_process_row_procs(or_row(target, dtype, (long)b * (k + 1) + i, V), dtype, V,
                                            T, top_k, &pr, pt + (size_t)i * V, work, pv);
        for (i = 0; i < k && !err; ++i)
            err |= oracle_process_row_procs(or_row(draft, dtype, (long)b * k + i, V), dtype, V, T,
                                            top_k, &pr, pd + (size_t)i * V, work, pv);
        if (!err) {
            long v;
            int found = 0;
            for (i = 0; i < k; ++i) {
                double p = pt[(size_t)i * V + d[i]], q = pd[(size_t)i * V + d[i]];
                if (out_p) out_p[(size_t)b * k + i] = p;
                if (out_q) out_q[(size_t)b * k + i] = q;
                if (out_ratio)
                    out_ratio[(size_t)b * k + i] = q > 0.0 ? (p / q < 1.0 ? p / q : 1.0)
                                                           : (p > 0.0 ? 1.0 : 0.0);
                if (!found && !((double)u[i] * q < p)) {
                    j = i;
                    found = 1;
                }
            }
            if (j < k) {
                for (v = 0; v < V; ++v) {
                    double r = pt[(size_t)j * V + v] - pd[(size_t)j * V + v];
                    w[v] = r > 0.0 ? r : 0.0;
                }
                if (oracle_inverse_cdf(w, V, (double)u[k], &y, &lo, &hi))
                    oracle_inverse_cdf(pt + (size_t)j * V, V, (double)u[k], &y, &lo, &hi);
            } else {
                oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[k], &y, &lo, &hi);
            }
        }
        if (err) {
            out_n[b] = -1;
            errors++;
        } else {
            for (i = 0; i < j; ++i) tok[i] = d[i];
            tok[j] = y;
            out_n[b] = j;
        }
        if (out_lo) out_lo[b] = lo;
        if (out_hi) out_hi[b] = hi;
    }
    free(pt); free(pd); free(w); free(work); free(pv);
    return errors;
}

/* The proposer's draw (as oracle_sample_rows, stochastic) with processors:
 * row r uses the processors of sequence r / rows_per_seq. */
int oracle_sample_rows_procs(const void* logits, int dtype, int rows, int rows_per_seq, int V,
                             const float* temperature, int top_k, const float* top_p,
                             const float* rep_penalty, const int32_t* rep_ids, int n_rep,
                             const uint32_t* mask, const float* u, int32_t* out_tokens) {
    int r, errors = 0;
    const long words = (V + 31) / 32;
    double* prob = (double*)malloc(sizeof(double) * (size_t)V);
    double* work = (double*)malloc(sizeof(double) * (size_t)V);
    or_pv_t* pv = (or_pv_t*)malloc(sizeof(or_pv_t) * (size_t)V);
    if (!prob || !work || !pv) {
        free(prob); free(work); free(pv);
        return -1;
    }
    for (r = 0; r < rows; ++r) {
        const int s = r / rows_per_seq;
        or_procs_t pr;
        int y = -1;
        double lo, hi, T = temperature ? (double)temperature[r] : 1.0;
        pr.top_p = top_p ? (double)top_p[s] : 1.0;
        pr.rep_penalty = rep_penalty ? (double)rep_penalty[s] : 1.0;
        pr.rep_ids = rep_ids ? rep_ids + (size_t)s * n_rep : NULL;
        pr.n_rep = rep_ids ? n_rep : 0;
        pr.mask = mask ? mask + (size_t)s * words : NULL;
        if ((u[r] >= 0.0f && u[r] < 1.0f) &&
            oracle_process_row_procs(or_row(logits, dtype, r, V), dtype, V, T, top_k, &pr, prob, work,
                                     pv) == 0) {
            if (oracle_inverse_cdf(prob, V, (double)u[r], &y, &lo, &hi)) y = -1;
        }
        if (y < 0) errors++;
        out_tokens[r] = y;
    }
    free(prob); free(work); free(pv);
    return errors;
}

/* ==== tree verification =====================================================
 *
 * The entry's section "提议方式与实现形态", paragraph 3, names candidate trees
 * besides chains; the pages give no acceptance rule for them.  The reading
 * taken here (R18) is the plainest one that reduces to paragraph 2 of
 * "提议与核验的基本步骤" on a chain:
 *   - node 0 is the verified context, node n >= 1 carries the draft token
 *     t_n and a parent par_n < n; target row n and draft row n are the target
 *     and draft distributions of the token that follows node n's prefix (the
 *     children of node n were drawn from draft row n);
 *   - the walk starts at node 0 with the current distribution R = p (the
 *     processed target row of the node) and tries the node's children in
 *     index order: child c is accepted iff u_c * q(t_c) < R(t_c) (R1 on the
 *     current distribution, q the processed draft row of the node, u_c the
 *     child's own uniform); a rejection replaces R by the normalised residual
 *     max(0, R - q) (left unchanged when that has no mass, the reading of R8);
 *   - an accepted child's token is emitted and the walk continues from that
 *     child; when no child of the current node is accepted (or it has none)
 *     the final token is drawn from R with the last uniform (R3);
 *   - greedy: the first child whose token is the lowest-index argmax of the
 *     node's target row is accepted; if none, that argmax is emitted (R6);
 *   - the rows a walk reads are those of the nodes it visits; a row error
 *     (R7) there, a token outside [0, V), a parent outside [0, n) or (in
 *     stochastic mode) a uniform outside [0, 1) or a bad temperature makes the
 *     sequence an error.
 * With children drawn independently from q, each emitted token follows p of
 * its prefix (rejection with the residual is the one-candidate step applied
 * again to the residual).
 *
 *   target, draft  [B][N+1][V] dtype (draft ignored when greedy)
 *   tokens, parents [B][N]  (node n at index n - 1)
 *   uniforms       [B][N+1] (u_c at index c - 1, the final draw at N)
 * Outputs: out_tokens [B][N+1] (the accepted tokens, the final token, then
 * -1), out_n [B] (accepted tokens, -1 on an error); optional: out_nodes
 * [B][N+1] (the accepted nodes, then -1), out_p / out_q / out_ratio [B][N]
 * (R(t_c), q(t_c) and min(1, R/q) for every child tested, NaN otherwise),
 * out_lo / out_hi [B] (the CDF points around the final token).
 * Returns the number of sequences reported as errors (-1: no memory).
 */
int oracle_verify_tree(const void* target, const void* draft, const int32_t* tokens,
                       const int32_t* parents, const float* uniforms, int B, int N, int V,
                       const float* temperature, int top_k, int greedy, int dtype,
                       int32_t* out_tokens, int32_t* out_n, int32_t* out_nodes, double* out_p,
                       double* out_q, double* out_ratio, double* out_lo, double* out_hi) {
    int b, i, errors = 0;
    double* R = (double*)malloc(sizeof(double) * (size_t)V);
    double* Q = (double*)malloc(sizeof(double) * (size_t)V);
    double* work = (double*)malloc(sizeof(double) * (size_t)V);
    if (!R || !Q || !work) {
        free(R); free(Q); free(work);
        return -1;
    }
    for (b = 0; b < B; ++b) {
        const int32_t* t = tokens + (size_t)b * N;
        const int32_t* par = parents + (size_t)b * N;
        const float* u = uniforms ? uniforms + (size_t)b * (N + 1) : NULL;
        int32_t* tok = out_tokens + (size_t)b * (N + 1);
        int32_t* nodes = out_nodes ? out_nodes + (size_t)b * (N + 1) : NULL;
        double T = temperature ? (double)temperature[b] : 1.0;
        int err = 0, depth = 0, a = 0, y = -1;
        double lo = NAN, hi = NAN;
        for (i = 0; i <= N; ++i) {
            tok[i] = -1;
            if (nodes) nodes[i] = -1;
        }
        for (i = 0; i < N; ++i) {
            if (out_p) out_p[(size_t)b * N + i] = NAN;
            if (out_q) out_q[(size_t)b * N + i] = NAN;
            if (out_ratio) out_ratio[(size_t)b * N + i] = NAN;
            if (t[i] < 0 || t[i] >= V || par[i] < 0 || par[i] > i) err = 1;
        }
        if (!greedy) {
            if (!(T > 0.0) || isinf(T) || isnan(T)) err = 1;
            for (i = 0; i <= N && !err; ++i)
                if (!(u[i] >= 0.0f && u[i] < 1.0f)) err = 1;
        }
        while (!err) {
            const long row = (long)b * (N + 1) + a;
            int c, next = 0;
            if (greedy) {
                int g = oracle_argmax_row(or_row(target, dtype, row, V), dtype, V);
                if (g < 0) {
                    err = 1;
                    break;
                }
                for (c = a + 1; c <= N && !next; ++c)
                    if (par[c - 1] == a && t[c - 1] == g) next = c;
                if (!next) {
                    y = g;
                    break;
                }
            } else {
                long v;
                err |= oracle_process_row(or_row(target, dtype, row, V), dtype, V, T, top_k, R, work);
                if (!err) err |= oracle_process_row(or_row(draft, dtype, row, V), dtype, V, T, top_k, Q, work);
                if (err) break;
                for (c = a + 1; c <= N && !next; ++c) {
                    double r, q, W = 0.0;
                    if (par[c - 1] != a) continue;
                    r = R[t[c - 1]];
                    q = Q[t[c - 1]];
                    if (out_p) out_p[(size_t)b * N + c - 1] = r;
                    if (out_q) out_q[(size_t)b * N + c - 1] = q;
                    if (out_ratio)
                        out_ratio[(size_t)b * N + c - 1] = q > 0.0 ? (r / q < 1.0 ? r / q : 1.0) : (r > 0.0 ? 1.0 : 0.0);
                    if ((double)u[c - 1] * q < r) {
                        next = c;
                        break;
                    }
                    /* rejected: the residual becomes the current distribution */
                    for (v = 0; v < V; ++v) W += (R[v] > Q[v]) ? R[v] - Q[v] : 0.0;
                    if (W > 0.0)
                        for (v = 0; v < V; ++v) R[v] = (R[v] > Q[v]) ? (R[v] - Q[v]) / W : 0.0;
                }
                if (!next) {
                    oracle_inverse_cdf(R, V, (double)u[N], &y, &lo, &hi);
                    break;
                }
            }
            tok[depth] = t[next - 1];
            if (nodes) nodes[depth] = next;
            depth++;
            a = next;
        }
        if (err) {
            for (i = 0; i <= N; ++i) {
                tok[i] = -1;
                if (nodes) nodes[i] = -1;
            }
            out_n[b] = -1;
            errors++;
        } else {
            tok[depth] = y;
            out_n[b] = depth;
        }
        if (out_lo) out_lo[b] = lo;
        if (out_hi) out_hi[b] = hi;
    }
    free(R); free(Q); free(work);
    return errors;
}

/*
 * The target's output projection (section "提议与核验的基本步骤", paragraph 1:
 * one forward pass scores every position; its last step maps the hidden
 * state h of a position to the logits z_v = sum_j h_j * W[v][j]).
 *   hidden  [rows][H] bf16 bits, weight [V][H] bf16 bits
 *   out_z   [rows][V] fp64: z_v summed in index order j = 0 .. H-1
 *   out_abs [rows][V] fp64 or NULL: sum_j |h_j * W[v][j]|, the scale of the
 *           rounding of any other summation of the same products
 * The products of two bf16 values are exact in double (8-bit significands);
 * only the running sum rounds.  Writes the given rows only (row0 .. row0+n).
 */
void oracle_head_logits(const uint16_t* hidden, const uint16_t* weight, long row0, long n, int V, int H,
                        double* out_z, double* out_abs) {
    long r, v, j;
    for (r = row0; r < row0 + n; ++r) {
        const void* h = hidden + (size_t)r * (size_t)H;
        for (v = 0; v < V; ++v) {
            const void* w = weight + (size_t)v * (size_t)H;
            double z = 0.0, a = 0.0;
            for (j = 0; j < H; ++j) {
                double t = or_logit(h, OR_DTYPE_BF16, j) * or_logit(w, OR_DTYPE_BF16, j);
                z += t;
                a += fabs(t);
            }
            out_z[(size_t)(r - row0) * (size_t)V + v] = z;
            if (out_abs) out_abs[(size_t)(r - row0) * (size_t)V + v] = a;
        }
    }
}
