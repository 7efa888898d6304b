/*
 * spec_oracle.c -- plain, slow, fp64 CPU oracle for the speculative-decoding
 * verify/accept step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load or call this code.  The
 * product (the CUDA library) never links or calls it and shares no code with
 * it: no header, helper, table or constant comes from here or goes there.
 *
 * Every function follows one passage of the three pages the method is taken
 * from, cited by page and section:
 *
 *   [atlas]   "Speculative Decoding —— 无损加速自回归 decode"
 *             (llm-infra-atlas, speculative_decoding chapter)
 *   [kevins]  "Speculative Decoding：投机解码的真实收益、校正采样与生产边界"
 *             (ricardokevins tech-analysis notes)
 *   [origins] zdszero "spec_origins" page (Blockwise / Speculative Decoding /
 *             SpecInfer / "In SGLang" sections)
 *
 * Notation of the pages: p = target distribution, q = draft distribution
 * ([origins] "Speculative Decoding", note on notation: Leviathan's p/q, not
 * Chen's swapped one).  Arithmetic is fp64 throughout.  Inputs (bf16 or f32)
 * are widened to fp64 exactly; a temperature is taken as its f32 value.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - temperature softmax p = softmax(logits / T), T > 0, applied to draft
 *     logits with the same T; draft probabilities are used as given;
 *   - accept iff u <= p(x)/q(x), ratio = +inf when q(x) = 0;
 *   - inverse CDF over index order 0..V-1: smallest j with u*S < C_j;
 *   - empty residual (S <= 0) falls back to sampling the target row itself;
 *   - argmax ties go to the lowest index, comparing values (-0 == +0);
 *   - tree children are visited in increasing node index;
 *   - any invalid input of a sequence (non-finite row maximum, NaN or +inf
 *     logit, token id out of range, a temperature that is not a finite
 *     normal positive f32, malformed parent array) marks the whole sequence
 *     invalid: num_accepted = -1 and every output slot -1.
 *
 * Parity margins: for each sequence the oracle also reports how close each
 * random decision came to flipping (|u - ratio|, |coin - prob_acc/theta|,
 * |p - theta_single|) and the relative distance of u*S to the nearest boundary
 * of the chosen inverse-CDF cell.  A comparison against another
 * implementation treats sequences whose margins are below its tolerance as
 * near-ties (flagged and counted), never as silent passes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_F32 0
#define OR_BF16 1

/* Mutation switch for the pin-sensitivity tests: 0 = the oracle as written.
 * A non-zero value plants one deliberate mistake so that the tests can show
 * that their pins catch it.  Never set outside tests/. */
static int g_mutation = 0;
void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

/* Exact widening of one stored element to fp64. */
static double widen(const void* base, int dtype, int64_t idx) {
    if (dtype == OR_F32) return (double)((const float*)base)[idx];
    uint16_t h = ((const uint16_t*)base)[idx];
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Temperature softmax of one logits row: p_j = exp(l_j/T - m) / sum_i exp(l_i/T - m),
 * m = max_j l_j/T.  The pages name temperature sampling ([kevins]
 * "draft / verify / accept", greedy vs temperature paragraph; "production
 * limits", higher temperature lowers acceptance) without printing the
 * formula; this is its textbook form.  Returns 0, or -1 if the row holds a
 * NaN or +inf, or has no finite maximum.
 */
static int softmax_T(const void* row, int dtype, int V, double T, double* p) {
    if (g_mutation == 11) T = 1.0 / T;                          /* l*T for l/T */
    double m = -INFINITY;
    for (int j = 0; j < V; ++j) {
        double x = widen(row, dtype, j) / T;
        if (isnan(x) || x == INFINITY) return -1;
        if (x > m) m = x;
    }
    if (!(m > -INFINITY)) return -1;
    double Z = 0.0;
    for (int j = 0; j < V; ++j) {
        p[j] = exp(widen(row, dtype, j) / T - m);
        Z += p[j];
    }
    for (int j = 0; j < V; ++j) p[j] /= Z;
    return 0;
}

/*
 * Inverse-CDF draw from the unnormalised weights w[0..V-1] with the uniform u:
 * C_j = w_0 + ... + w_j (index order), S = C_{V-1}; pick the smallest j with
 * u*S < C_j.  Zero-weight entries are never picked.  *margin receives
 * min(u*S - C_{j-1}, C_j - u*S) / S.  Returns -1 if S is not positive.
 */
static int inverse_cdf(const double* w, int V, double u, double* S_out, double* margin) {
    double S = 0.0;
    for (int j = 0; j < V; ++j) S += w[j];
    if (S_out) *S_out = S;
    if (!(S > 0.0)) return -1;
    double t = u * S;
    double C = 0.0;
    for (int j = 0; j < V; ++j) {
        double Cprev = C;
        C += w[j];
        if (t < C) {
            double a = t - Cprev, b = C - t;
            *margin = (a < b ? a : b) / S;
            return (g_mutation == 5 && j > 0) ? j - 1 : j;   /* off-by-one cell */
        }
    }
    /* Unreachable for u in [0,1): t < S = C_{V-1}.  Keep the last positive
     * entry for completeness. */
    for (int j = V - 1; j >= 0; --j)
        if (w[j] > 0.0) { *margin = 0.0; return j; }
    return -1;
}

static void fill_i32(int32_t* a, int n, int32_t v) { for (int i = 0; i < n; ++i) a[i] = v; }

/* A usable temperature: finite, positive and not subnormal as an f32. */
static int temperature_ok(double T) { return T >= 0x1p-126 && T <= 0x1.fffffep127; }

/*
 * Top-k / top-p filtering of one temperature-softmax row.  The pages name
 * top-k and top-p next to temperature as the sampling strategies a verify
 * step must stay unbiased under ([kevins] "draft / verify / accept",
 * greedy vs sampling paragraph; "production limits": a wider top-p lowers
 * acceptance) without defining them; the textbook definitions, in the order
 * temperature -> top-k -> top-p:
 *   top-k (0 < top_k < V): keep the tokens whose logit is >= the top_k-th
 *     largest logit (every token tied with it is kept);
 *   top-p (0 < top_p < 1): within the top-k set, with the distribution
 *     renormalised on it, keep the smallest set of whole groups of equal
 *     logits, taken from the largest down, whose mass reaches top_p;
 *   the kept tokens' probabilities are renormalised, the rest are 0.
 * p holds softmax(row / T) on entry and the filtered distribution on exit.
 * *margin receives |cumulative mass - top_p| at the two masses around the
 * top-p crossing (relative to the renormalised distribution; +inf when
 * top-p is off).  Returns 0, or -1 for an out-of-range top_k or top_p.
 */
typedef struct { double v; int j; } vj_t;
static int cmp_vj_desc(const void* a, const void* b) {
    const vj_t* x = (const vj_t*)a;
    const vj_t* y = (const vj_t*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return x->j - y->j;
}
static int filter_probs(const void* row, int dtype, int V, double* p, int top_k, double top_p, vj_t* sorted,
                        double* margin) {
    *margin = INFINITY;
    if (top_k < 0 || !(top_p > 0.0 && top_p <= 1.0)) return -1;
    if ((top_k == 0 || top_k >= V) && top_p == 1.0) return 0;
    for (int j = 0; j < V; ++j) {
        sorted[j].v = widen(row, dtype, j);
        sorted[j].j = j;
    }
    qsort(sorted, (size_t)V, sizeof(vj_t), cmp_vj_desc);
    /* top-k: every token whose logit is >= the top_k-th largest */
    int nA = V;
    if (top_k > 0 && top_k < V) {
        int kk = (g_mutation == 16) ? top_k - 1 : top_k;          /* keeps one group too few */
        if (kk < 1) kk = 1;
        const double th = sorted[kk - 1].v;
        nA = kk;
        while (nA < V && sorted[nA].v >= th) ++nA;
    }
    double ZA = 0.0;
    for (int i = 0; i < nA; ++i) ZA += p[sorted[i].j];
    /* top-p: whole groups of equal logits from the top until the mass reaches top_p */
    int nB = nA;
    if (top_p < 1.0) {
        double cum = 0.0;
        int i = 0;
        while (i < nA) {
            int e = i;
            double g = 0.0;
            while (e < nA && sorted[e].v == sorted[i].v) g += p[sorted[e++].j];
            const double before = cum;
            cum += g / ZA;
            if (cum >= top_p) {
                const double m1 = fabs(before - top_p), m2 = fabs(cum - top_p);
                *margin = m1 < m2 ? m1 : m2;
                nB = (g_mutation == 17 && i > 0) ? i : e;           /* drops the crossing group */
                break;
            }
            i = e;
        }
    }
    double ZB = 0.0;
    for (int i = 0; i < nB; ++i) ZB += p[sorted[i].j];
    for (int i = 0; i < nB; ++i) sorted[i].v = p[sorted[i].j];   /* the kept probabilities */
    for (int j = 0; j < V; ++j) p[j] = 0.0;
    for (int i = 0; i < nB; ++i) p[sorted[i].j] = sorted[i].v / ZB;  /* ZB > 0: the maximum is kept */
    return 0;
}

/*
 * Chain verify, one call = one round for B independent sequences.
 *
 * [origins] "Speculative Decoding: sampling can be lossless", acceptance
 * rule 1-3, with [kevins] "sampling correction" a(x) and r(x):
 *   1. accept draft x_i with probability min(1, p_i(x_i)/q_i(x_i)), i.e. iff
 *      coin_i <= p_i(x_i)/q_i(x_i);
 *   2. at the first rejection k, draw the correction from
 *      norm(max(0, p_k - q_k)) and stop;
 *   3. if all gamma drafts are accepted, draw the bonus token from p_gamma.
 *
 * Layout: target row (b,i), i in [0,gamma], starts at element
 * (b*(gamma+1)+i)*t_row_stride; draft row (b,i), i in [0,gamma), at
 * (b*gamma+i)*d_row_stride; draft_is_probs selects logits (softmax at the
 * sequence's T) or probabilities (f32, used as given).
 * Outputs: out_tokens[b*(gamma+1) + j] (accepted drafts, then the
 * correction/bonus, then -1), out_num_accepted[b] in [0,gamma] or -1.
 * Diagnostics (nullable): out_px/out_qx [b*gamma+i] = p_i(x_i), q_i(x_i)
 * for every i < gamma; out_S[b] = mass of the final distribution before
 * normalisation (sum max(0,p_k-q_k) on a rejection, 1 for the bonus);
 * out_dmargin[b] = min over the evaluated decisions of |coin - ratio|;
 * out_cmargin[b] = inverse-CDF margin.
 */
static void chain_impl(int B, int gamma, int V,
                       const void* target, int tdt, int64_t t_row_stride,
                       const void* draft, int ddt, int draft_is_probs, int64_t d_row_stride,
                       const int32_t* draft_tokens, const float* temperature,
                       const float* coins, const float* final_u,
                       const int32_t* top_k, const float* top_p,
                       int32_t* out_tokens, int32_t* out_num_accepted,
                       double* out_px, double* out_qx, double* out_S,
                       double* out_dmargin, double* out_cmargin, double* out_fmargin, int nthreads) {
    const int filtered = top_k != NULL || top_p != NULL;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* P = (double*)malloc(sizeof(double) * (size_t)V * (size_t)(gamma + 1));
        double* Q = (double*)malloc(sizeof(double) * (size_t)V * (size_t)gamma);
        double* w = (double*)malloc(sizeof(double) * (size_t)V);
        vj_t* sorted = filtered ? (vj_t*)malloc(sizeof(vj_t) * (size_t)V) : NULL;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int b = 0; b < B; ++b) {
            int32_t* toks = out_tokens + (int64_t)b * (gamma + 1);
            const int32_t* x = draft_tokens + (int64_t)b * gamma;
            double T = (double)temperature[b];
            int bad = !temperature_ok(T);
            const int K = top_k ? top_k[b] : 0;
            const double Pp = top_p ? (double)top_p[b] : 1.0;
            double fmargin = INFINITY, fm;
            for (int i = 0; i <= gamma && !bad; ++i) {
                const char* row = (const char*)target +
                    ((int64_t)b * (gamma + 1) + i) * t_row_stride * (tdt == OR_F32 ? 4 : 2);
                if (softmax_T(row, tdt, V, T, P + (int64_t)i * V)) bad = 1;
                else if (filtered) {
                    if (filter_probs(row, tdt, V, P + (int64_t)i * V, K, Pp, sorted, &fm)) bad = 1;
                    if (fm < fmargin) fmargin = fm;
                }
            }
            for (int i = 0; i < gamma && !bad; ++i) {
                const char* row = (const char*)draft +
                    ((int64_t)b * gamma + i) * d_row_stride * (ddt == OR_F32 ? 4 : 2);
                double* q = Q + (int64_t)i * V;
                if (draft_is_probs) {
                    for (int j = 0; j < V; ++j) q[j] = widen(row, OR_F32, j);
                } else if (softmax_T(row, ddt, V, g_mutation == 12 ? 1.0 : T, q)) {
                    bad = 1;
                } else if (filtered && g_mutation != 18) {              /* 18: draft left unfiltered */
                    if (filter_probs(row, ddt, V, q, K, Pp, sorted, &fm)) bad = 1;
                    if (fm < fmargin) fmargin = fm;
                }
                if (x[i] < 0 || x[i] >= V) bad = 1;
                else if (isnan(q[x[i]]) || q[x[i]] < 0.0) bad = 1;
            }
            if (out_fmargin) out_fmargin[b] = bad ? INFINITY : fmargin;
            if (bad) {
                fill_i32(toks, gamma + 1, -1);
                out_num_accepted[b] = -1;
                if (out_px) for (int i = 0; i < gamma; ++i) out_px[(int64_t)b * gamma + i] = NAN;
                if (out_qx) for (int i = 0; i < gamma; ++i) out_qx[(int64_t)b * gamma + i] = NAN;
                if (out_S) out_S[b] = NAN;
                if (out_dmargin) out_dmargin[b] = INFINITY;
                if (out_cmargin) out_cmargin[b] = INFINITY;
                continue;
            }
            /* Rule 1: accept while coin_i <= p_i(x_i)/q_i(x_i). */
            double dmargin = INFINITY;
            int k = gamma;
            for (int i = 0; i < gamma; ++i) {
                double px = P[(int64_t)i * V + x[i]];
                double qx = Q[(int64_t)i * V + x[i]];
                if (out_px) out_px[(int64_t)b * gamma + i] = px;
                if (out_qx) out_qx[(int64_t)b * gamma + i] = qx;
            }
            for (int i = 0; i < gamma; ++i) {
                double px = P[(int64_t)i * V + x[i]];
                double qx = Q[(int64_t)i * V + x[i]];
                if (g_mutation == 1) { double s = px; px = qx; qx = s; }   /* p/q swapped */
                double ratio = (qx > 0.0) ? px / qx : INFINITY;
                double u = (double)coins[(int64_t)b * gamma + (g_mutation == 4 ? 0 : i)];
                double mg = fabs(u - ratio);
                if (mg < dmargin) dmargin = mg;
                if (!(u <= ratio)) { k = i; break; }
            }
            double S = 1.0, cm = INFINITY;
            int y;
            if (k < gamma) {
                /* Rule 2: correction from norm(max(0, p_k - q_k)). */
                const double* p = P + (int64_t)k * V;
                const double* q = Q + (int64_t)k * V;
                for (int j = 0; j < V; ++j) {
                    double d = p[j] - q[j];
                    if (g_mutation == 2) w[j] = fabs(d);            /* max dropped */
                    else if (g_mutation == 3) w[j] = q[j] - p[j] > 0.0 ? q[j] - p[j] : 0.0;
                    else w[j] = d > 0.0 ? d : 0.0;
                }
                y = inverse_cdf(w, V, (double)final_u[b], &S, &cm);
                if (y < 0) {
                    /* Empty residual (reachable only through rounding, since a
                     * rejection needs p != q): draw from p_k itself. */
                    double S1;
                    y = inverse_cdf(p, V, (double)final_u[b], &S1, &cm);
                }
            } else {
                /* Rule 3: bonus token from p_gamma. */
                const double* p = P + (int64_t)(g_mutation == 6 ? gamma - 1 : gamma) * V;
                y = inverse_cdf(p, V, (double)final_u[b], &S, &cm);
                S = 1.0;
            }
            for (int i = 0; i < k; ++i) toks[i] = x[i];
            toks[k] = y;
            for (int i = k + 1; i <= gamma; ++i) toks[i] = -1;
            out_num_accepted[b] = k;
            if (out_S) out_S[b] = S;
            if (out_dmargin) out_dmargin[b] = dmargin;
            if (out_cmargin) out_cmargin[b] = cm;
        }
        free(P);
        free(Q);
        free(w);
        free(sorted);
    }
}

void oracle_chain(int B, int gamma, int V,
                  const void* target, int tdt, int64_t t_row_stride,
                  const void* draft, int ddt, int draft_is_probs, int64_t d_row_stride,
                  const int32_t* draft_tokens, const float* temperature,
                  const float* coins, const float* final_u,
                  int32_t* out_tokens, int32_t* out_num_accepted,
                  double* out_px, double* out_qx, double* out_S,
                  double* out_dmargin, double* out_cmargin, int nthreads) {
    chain_impl(B, gamma, V, target, tdt, t_row_stride, draft, ddt, draft_is_probs, d_row_stride,
               draft_tokens, temperature, coins, final_u, NULL, NULL, out_tokens, out_num_accepted,
               out_px, out_qx, out_S, out_dmargin, out_cmargin, NULL, nthreads);
}

/*
 * Chain verify with top-k / top-p filtering (filter_probs) of every target
 * row and, when the draft is given as logits, every draft row, with the
 * sequence's top_k[b] (0 = off) and top_p[b] (1 = off); draft probabilities
 * are used as given.  Rules 1-3 then run on the filtered distributions, so
 * the emitted tokens follow the filtered target distribution.  top_k < 0 or
 * top_p outside (0, 1] makes the sequence invalid.  out_fmargin[b] = the
 * smallest top-p crossing margin over the sequence's rows.
 */
void oracle_chain_filtered(int B, int gamma, int V,
                           const void* target, int tdt, int64_t t_row_stride,
                           const void* draft, int ddt, int draft_is_probs, int64_t d_row_stride,
                           const int32_t* draft_tokens, const float* temperature,
                           const float* coins, const float* final_u,
                           const int32_t* top_k, const float* top_p,
                           int32_t* out_tokens, int32_t* out_num_accepted,
                           double* out_px, double* out_qx, double* out_S,
                           double* out_dmargin, double* out_cmargin, double* out_fmargin, int nthreads) {
    chain_impl(B, gamma, V, target, tdt, t_row_stride, draft, ddt, draft_is_probs, d_row_stride,
               draft_tokens, temperature, coins, final_u, top_k, top_p, out_tokens, out_num_accepted,
               out_px, out_qx, out_S, out_dmargin, out_cmargin, out_fmargin, nthreads);
}

/* The filtered distribution of one row, as the verify above uses it (for the pins). */
int oracle_filter_row(const void* row, int dtype, int V, double T, int top_k, double top_p, double* p,
                      double* margin) {
    if (softmax_T(row, dtype, V, T, p)) return -1;
    vj_t* sorted = (vj_t*)malloc(sizeof(vj_t) * (size_t)V);
    double m = INFINITY;
    const int r = filter_probs(row, dtype, V, p, top_k, top_p, sorted, &m);
    free(sorted);
    if (margin) *margin = m;
    return r;
}

/*
 * Tree shape check shared by both tree walks: parents[0] = -1, 0 <= parents[n] < n
 * for n >= 1, node depth <= max_depth, tokens[n] in [0,V) for n >= 1 (the
 * root's token is the last verified token and is not read).  Trees are
 * flattened with ancestors first ([origins] "SpecInfer", tree attention
 * mask: every node sees only its ancestors).
 */
static int tree_ok(int N, int V, int max_depth, const int32_t* tokens, const int32_t* parents,
                   int* depth) {
    if (parents[0] != -1) return 0;
    depth[0] = 0;
    for (int n = 1; n < N; ++n) {
        int pa = parents[n];
        if (pa < 0 || pa >= n) return 0;
        depth[n] = depth[pa] + 1;
        if (depth[n] > max_depth) return 0;
        if (tokens[n] < 0 || tokens[n] >= V) return 0;
    }
    return 1;
}

/*
 * Greedy tree verify ([origins] "In SGLang": greedy goes through
 * verify_tree_greedy; "Blockwise Parallel Decoding", verify: keep the
 * longest prefix that agrees with the scoring model's own argmax, which
 * equals token-by-token greedy decoding).
 *   g_n = argmax_j logits[n][j] (lowest index among equal maxima);
 *   cur = root; repeat: the first child c of cur (increasing node index) with
 *   tokens[c] == g_cur is accepted and becomes cur; stop when none matches.
 *   Emitted tokens: the accepted draft tokens, then g_cur (the bonus).
 * Outputs (width max_depth+1 per sequence, -1 padded): accept_index (root
 * first), out_tokens, num_accepted = number of accepted draft tokens;
 * out_argmax[b*N+n] = g_n (nullable).
 */
void oracle_tree_greedy(int B, int N, int V, int max_depth,
                        const void* target, int tdt, int64_t t_row_stride,
                        const int32_t* tokens, const int32_t* parents,
                        int32_t* out_accept_index, int32_t* out_tokens,
                        int32_t* out_num_accepted, int32_t* out_argmax, int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int* g = (int*)malloc(sizeof(int) * (size_t)N);
        int* depth = (int*)malloc(sizeof(int) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int b = 0; b < B; ++b) {
            const int32_t* tk = tokens + (int64_t)b * N;
            const int32_t* pa = parents + (int64_t)b * N;
            int32_t* ai = out_accept_index + (int64_t)b * (max_depth + 1);
            int32_t* ot = out_tokens + (int64_t)b * (max_depth + 1);
            int bad = !tree_ok(N, V, max_depth, tk, pa, depth);
            for (int n = 0; n < N && !bad; ++n) {
                const char* row = (const char*)target +
                    ((int64_t)b * N + n) * t_row_stride * (tdt == OR_F32 ? 4 : 2);
                double best = -INFINITY;
                int arg = 0;
                for (int j = 0; j < V; ++j) {
                    double v = widen(row, tdt, j);
                    if (isnan(v)) { bad = 1; break; }
                    int better = (g_mutation == 7) ? (v >= best) : (v > best);
                    if (better) { best = v; arg = j; }
                }
                g[n] = arg;
            }
            if (bad) {
                fill_i32(ai, max_depth + 1, -1);
                fill_i32(ot, max_depth + 1, -1);
                out_num_accepted[b] = -1;
                if (out_argmax) fill_i32(out_argmax + (int64_t)b * N, N, -1);
                continue;
            }
            if (out_argmax) for (int n = 0; n < N; ++n) out_argmax[(int64_t)b * N + n] = g[n];
            fill_i32(ai, max_depth + 1, -1);
            fill_i32(ot, max_depth + 1, -1);
            int cur = 0, k = 0;
            ai[0] = 0;
            for (;;) {
                int next = -1;
                for (int c = cur + 1; c < N; ++c) {
                    if (pa[c] == cur && tk[c] == g[cur]) { next = c; break; }
                }
                if (next < 0) break;
                ot[k] = tk[next];
                ++k;
                ai[k] = next;
                cur = next;
            }
            ot[k] = g[cur];
            out_num_accepted[b] = k;
        }
        free(g);
        free(depth);
    }
}

/*
 * Target-only tree sampling ([origins] "In SGLang",
 * tree_speculative_sampling_target_only; the SpecInfer-style walk down the
 * tree that tries the next sibling after a rejection):
 *   cur = root.  At cur, children c_1..c_m in increasing node index,
 *   prob_acc = 0; for each child: prob_acc += p_cur(tok_c); accept c iff
 *   coin_cur <= prob_acc / threshold_acc or p_cur(tok_c) >= threshold_single;
 *   a child that is not accepted is rejected, its target probability is
 *   written into the draft-probability row of cur at tok_c.  On acceptance
 *   cur = c and the walk continues one level down with coin_c; it stops when
 *   no child of cur is accepted or cur has no children.
 *   Final token: drawn from relu(p_cur - d_cur), d_cur = draft_probs row of
 *   cur (zeros when draft_probs is NULL) with the rejected children's
 *   entries overwritten by their target probabilities.
 * coins[b*N + n] is the coin used while visiting node n.  draft_probs rows
 * (nullable) start at element (b*N+n)*dp_row_stride; they are not modified.
 * Outputs as oracle_tree_greedy; out_pchild[b*N+n] = p_parent(n)(tokens[n])
 * for n >= 1 and 0 for the root; margins as oracle_chain.
 */
static void tree_sample_impl(int B, int N, int V, int max_depth,
                             const void* target, int tdt, int64_t t_row_stride,
                             const int32_t* tokens, const int32_t* parents,
                             const float* temperature, const float* coins, const float* final_u,
                             const float* draft_probs, int64_t dp_row_stride,
                             float threshold_single, float threshold_acc,
                             const int32_t* top_k, const float* top_p,
                             int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted,
                             double* out_pchild, double* out_S, double* out_dmargin,
                             double* out_cmargin, double* out_fmargin, int nthreads) {
    const int filtered = top_k != NULL || top_p != NULL;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* P = (double*)malloc(sizeof(double) * (size_t)V * (size_t)N);
        double* d = (double*)malloc(sizeof(double) * (size_t)V);
        double* w = (double*)malloc(sizeof(double) * (size_t)V);
        int* depth = (int*)malloc(sizeof(int) * (size_t)N);
        int* rej = (int*)malloc(sizeof(int) * (size_t)N);
        vj_t* sorted = filtered ? (vj_t*)malloc(sizeof(vj_t) * (size_t)V) : NULL;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int b = 0; b < B; ++b) {
            const int32_t* tk = tokens + (int64_t)b * N;
            const int32_t* pa = parents + (int64_t)b * N;
            int32_t* ai = out_accept_index + (int64_t)b * (max_depth + 1);
            int32_t* ot = out_tokens + (int64_t)b * (max_depth + 1);
            double T = (double)temperature[b];
            int bad = !temperature_ok(T) || !tree_ok(N, V, max_depth, tk, pa, depth);
            const int K = top_k ? top_k[b] : 0;
            const double Pp = top_p ? (double)top_p[b] : 1.0;
            double fmargin = INFINITY, fm;
            for (int n = 0; n < N && !bad; ++n) {
                const char* row = (const char*)target +
                    ((int64_t)b * N + n) * t_row_stride * (tdt == OR_F32 ? 4 : 2);
                if (softmax_T(row, tdt, V, T, P + (int64_t)n * V)) bad = 1;
                else if (filtered && g_mutation != 19) {              /* 19: tree rows left unfiltered */
                    if (filter_probs(row, tdt, V, P + (int64_t)n * V, K, Pp, sorted, &fm)) bad = 1;
                    if (fm < fmargin) fmargin = fm;
                }
            }
            if (out_fmargin) out_fmargin[b] = bad ? INFINITY : fmargin;
            fill_i32(ai, max_depth + 1, -1);
            fill_i32(ot, max_depth + 1, -1);
            if (bad) {
                out_num_accepted[b] = -1;
                if (out_pchild) for (int n = 0; n < N; ++n) out_pchild[(int64_t)b * N + n] = NAN;
                if (out_S) out_S[b] = NAN;
                if (out_dmargin) out_dmargin[b] = INFINITY;
                if (out_cmargin) out_cmargin[b] = INFINITY;
                continue;
            }
            if (out_pchild) {
                out_pchild[(int64_t)b * N] = 0.0;
                for (int n = 1; n < N; ++n)
                    out_pchild[(int64_t)b * N + n] = P[(int64_t)pa[n] * V + tk[n]];
            }
            double th_s = (double)threshold_single, th_a = (double)threshold_acc;
            double dmargin = INFINITY;
            int cur = 0, k = 0, nrej = 0;
            ai[0] = 0;
            for (;;) {
                const double* p = P + (int64_t)cur * V;
                double u = (double)coins[(int64_t)b * N + (g_mutation == 8 ? 0 : cur)];
                double acc = 0.0;
                int next = -1;
                nrej = 0;
                for (int c = cur + 1; c < N; ++c) {
                    if (pa[c] != cur) continue;
                    double pc = p[tk[c]];
                    acc = (g_mutation == 9) ? pc : acc + pc;
                    double r = acc / th_a;
                    double m1 = fabs(u - r), m2 = fabs(pc - th_s);
                    /* accept iff (u <= r) or (pc >= th_s): an acceptance flips only if every
                     * condition that holds can flip, a rejection if either can */
                    const int a1 = u <= r, a2 = pc >= th_s;
                    const double mm = (a1 || a2) ? fmax(a1 ? m1 : 0.0, a2 ? m2 : 0.0) : fmin(m1, m2);
                    if (mm < dmargin) dmargin = mm;
                    if (a1 || a2) { next = c; break; }
                    rej[nrej++] = tk[c];
                }
                if (next < 0) break;
                ot[k] = tk[next];
                ++k;
                ai[k] = next;
                cur = next;
            }
            /* Final draw from relu(p_cur - d_cur). */
            const double* p = P + (int64_t)cur * V;
            if (draft_probs) {
                const float* drow = draft_probs + ((int64_t)b * N + cur) * dp_row_stride;
                for (int j = 0; j < V; ++j) d[j] = (double)drow[j];
            } else {
                for (int j = 0; j < V; ++j) d[j] = 0.0;
            }
            if (g_mutation != 10)
                for (int r = 0; r < nrej; ++r) d[rej[r]] = p[rej[r]];
            for (int j = 0; j < V; ++j) {
                double x = p[j] - d[j];
                w[j] = x > 0.0 ? x : 0.0;
            }
            double S, cm = INFINITY;
            int y = inverse_cdf(w, V, (double)final_u[b], &S, &cm);
            if (y < 0) {
                double S1;
                y = inverse_cdf(p, V, (double)final_u[b], &S1, &cm);
            }
            ot[k] = y;
            out_num_accepted[b] = k;
            if (out_S) out_S[b] = S;
            if (out_dmargin) out_dmargin[b] = dmargin;
            if (out_cmargin) out_cmargin[b] = cm;
        }
        free(P);
        free(d);
        free(w);
        free(depth);
        free(rej);
        free(sorted);
    }
}

void oracle_tree_sample(int B, int N, int V, int max_depth,
                        const void* target, int tdt, int64_t t_row_stride,
                        const int32_t* tokens, const int32_t* parents,
                        const float* temperature, const float* coins, const float* final_u,
                        const float* draft_probs, int64_t dp_row_stride,
                        float threshold_single, float threshold_acc,
                        int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted,
                        double* out_pchild, double* out_S, double* out_dmargin,
                        double* out_cmargin, int nthreads) {
    tree_sample_impl(B, N, V, max_depth, target, tdt, t_row_stride, tokens, parents, temperature, coins,
                     final_u, draft_probs, dp_row_stride, threshold_single, threshold_acc, NULL, NULL,
                     out_accept_index, out_tokens, out_num_accepted, out_pchild, out_S, out_dmargin,
                     out_cmargin, NULL, nthreads);
}

/*
 * Target-only tree sampling under top-k / top-p filtering: every node's
 * target row is filtered (filter_probs, the sequence's top_k[b] / top_p[b])
 * before the walk above uses it, so prob_acc, the thresholds and the final
 * relu(p_cur - d_cur) all see the filtered distribution; draft_probs rows are
 * used as given.  out_fmargin[b] = the smallest top-p margin over the rows.
 */
void oracle_tree_sample_filtered(int B, int N, int V, int max_depth,
                                 const void* target, int tdt, int64_t t_row_stride,
                                 const int32_t* tokens, const int32_t* parents,
                                 const float* temperature, const float* coins, const float* final_u,
                                 const float* draft_probs, int64_t dp_row_stride,
                                 float threshold_single, float threshold_acc,
                                 const int32_t* top_k, const float* top_p,
                                 int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted,
                                 double* out_pchild, double* out_S, double* out_dmargin,
                                 double* out_cmargin, double* out_fmargin, int nthreads) {
    tree_sample_impl(B, N, V, max_depth, target, tdt, t_row_stride, tokens, parents, temperature, coins,
                     final_u, draft_probs, dp_row_stride, threshold_single, threshold_acc, top_k, top_p,
                     out_accept_index, out_tokens, out_num_accepted, out_pchild, out_S, out_dmargin,
                     out_cmargin, out_fmargin, nthreads);
}

/*
 * Tree verification with a draft distribution: SpecInfer's multi-step
 * speculative sampling ([origins] "SpecInfer", the MSS bullet: after a child
 * is rejected the target distribution becomes the residual
 * norm(max(0, p - q)) and the next sibling is tried; the output keeps the
 * target distribution).
 *   cur = root.  p = softmax(target row cur / T); q = draft_probs row cur,
 *   the distribution the children of cur were drawn from.  Children c_1..c_m
 *   in increasing node index: child c is accepted iff
 *   coins[c] <= p(tok_c) / q(tok_c) (ratio +inf when q(tok_c) = 0); on
 *   acceptance cur = c and the walk continues one level down with that
 *   node's p and q; on rejection p <- max(0, p - q) / S, S = sum of
 *   max(0, p - q) (p is kept when S is not positive: rounding only), and the
 *   next sibling is tried.  When no child of cur is accepted, or cur is a
 *   leaf, the last token is drawn with final_u from the current p.
 * coins[b*N + c] is the uniform of the test of child c (coins[b*N] unused).
 * draft_probs rows start at element (b*N+n)*dp_row_stride.  A drafted
 * token's q(tok_c) must be finite and >= 0, else the sequence is invalid.
 * Outputs as oracle_tree_greedy; out_ptest[b*N+c] = p(tok_c) at the test of
 * child c (NaN for children never tested); out_S[b] = the last residual mass
 * S at the final node (1 when it had no rejection); margins as oracle_chain.
 */
void oracle_tree_mss(int B, int N, int V, int max_depth,
                     const void* target, int tdt, int64_t t_row_stride,
                     const int32_t* tokens, const int32_t* parents,
                     const float* temperature, const float* coins, const float* final_u,
                     const float* draft_probs, int64_t dp_row_stride,
                     int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted,
                     double* out_ptest, double* out_S, double* out_dmargin, double* out_cmargin,
                     int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* P = (double*)malloc(sizeof(double) * (size_t)V * (size_t)N);
        double* p = (double*)malloc(sizeof(double) * (size_t)V);
        double* p0 = (double*)malloc(sizeof(double) * (size_t)V);
        int* depth = (int*)malloc(sizeof(int) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int b = 0; b < B; ++b) {
            const int32_t* tk = tokens + (int64_t)b * N;
            const int32_t* pa = parents + (int64_t)b * N;
            int32_t* ai = out_accept_index + (int64_t)b * (max_depth + 1);
            int32_t* ot = out_tokens + (int64_t)b * (max_depth + 1);
            double* pt = out_ptest ? out_ptest + (int64_t)b * N : NULL;
            double T = (double)temperature[b];
            int bad = !temperature_ok(T) || !tree_ok(N, V, max_depth, tk, pa, depth);
            for (int n = 0; n < N && !bad; ++n) {
                const char* row = (const char*)target +
                    ((int64_t)b * N + n) * t_row_stride * (tdt == OR_F32 ? 4 : 2);
                if (softmax_T(row, tdt, V, T, P + (int64_t)n * V)) bad = 1;
            }
            fill_i32(ai, max_depth + 1, -1);
            fill_i32(ot, max_depth + 1, -1);
            if (pt) for (int n = 0; n < N; ++n) pt[n] = NAN;
            double dmargin = INFINITY, S_last = 1.0;
            int cur = 0, k = 0;
            if (!bad) {
                ai[0] = 0;
                for (;;) {
                    const float* q = draft_probs + ((int64_t)b * N + cur) * dp_row_stride;
                    for (int j = 0; j < V; ++j) p[j] = p0[j] = P[(int64_t)cur * V + j];
                    S_last = 1.0;
                    int next = -1;
                    for (int c = cur + 1; c < N && !bad; ++c) {
                        if (pa[c] != cur) continue;
                        const double qx = (double)q[tk[c]];
                        if (!(qx >= 0.0 && qx <= 0x1.fffffep127)) { bad = 1; break; }
                        const double px = p[tk[c]];
                        if (pt) pt[c] = px;
                        const double ratio = qx > 0.0 ? px / qx : INFINITY;
                        const double u = (double)coins[(int64_t)b * N + (g_mutation == 15 ? cur : c)];
                        const double m = fabs(u - ratio);
                        if (m < dmargin) dmargin = m;
                        if (u <= ratio) { next = c; break; }
                        if (g_mutation == 13) continue;                 /* residual never taken */
                        const double* base = (g_mutation == 14) ? p0 : p; /* residual of the first p */
                        double S = 0.0;
                        for (int j = 0; j < V; ++j) {
                            const double d = base[j] - (double)q[j];
                            S += d > 0.0 ? d : 0.0;
                        }
                        if (!(S <= 0x1.fffffffffffffp1023)) { bad = 1; break; }   /* NaN or inf */
                        if (S > 0.0) {
                            for (int j = 0; j < V; ++j) {
                                const double d = base[j] - (double)q[j];
                                p[j] = (d > 0.0 ? d : 0.0) / S;
                            }
                            S_last = S;
                        }
                    }
                    if (bad || next < 0) break;
                    ot[k] = tk[next];
                    ++k;
                    ai[k] = next;
                    cur = next;
                }
            }
            if (bad) {
                fill_i32(ai, max_depth + 1, -1);
                fill_i32(ot, max_depth + 1, -1);
                out_num_accepted[b] = -1;
                if (pt) for (int n = 0; n < N; ++n) pt[n] = NAN;
                if (out_S) out_S[b] = NAN;
                if (out_dmargin) out_dmargin[b] = INFINITY;
                if (out_cmargin) out_cmargin[b] = INFINITY;
                continue;
            }
            double S1, cm = INFINITY;
            const int y = inverse_cdf(p, V, (double)final_u[b], &S1, &cm);
            ot[k] = y;
            out_num_accepted[b] = k;
            if (out_S) out_S[b] = S_last;
            if (out_dmargin) out_dmargin[b] = dmargin;
            if (out_cmargin) out_cmargin[b] = cm;
        }
        free(P);
        free(p);
        free(p0);
        free(depth);
    }
}

/* Exposed for the pins: the temperature softmax of one row, and the
 * inverse-CDF draw, exactly as the verify functions above use them. */
int oracle_softmax_row(const void* row, int dtype, int V, double T, double* p) {
    return softmax_T(row, dtype, V, T, p);
}

int oracle_inverse_cdf(const double* w, int V, double u, double* S, double* margin) {
    double m = INFINITY;
    int j = inverse_cdf(w, V, u, S, &m);
    if (margin) *margin = m;
    return j;
}
