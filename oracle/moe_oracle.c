/*
 * moe_oracle.c -- plain fp64 CPU oracle of the dropless Mixture-of-Experts
 * layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library: it is a second, independent statement of what
 * the layer computes, written to be read against the pages by eye.
 *
 * Single thread, fp64, no BLAS, no fast-math.  Build with
 *   gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared moe_oracle.c -lm
 * (-ffp-contract=off keeps a*b+c as two roundings everywhere, so the
 * per-token loop and the sorted-dispatch path below round identically.)
 *
 * Sources (page title, section):
 *  - "Mixture of Experts: routing, sorted dispatch, Switch aux loss, aux-free
 *    bias" (openlearn course module): sec. 2 symbol table (z_n = W_g x_n,
 *    p_n = softmax(z_n), f_e, P_e, b_e); sec. 2.1 router table (softmax_topk,
 *    topk_softmax, sigmoid; ties to the lowest id; routed_scaling);
 *    sec. 2.2 sorted dispatch (a = n k + j, stable sort, perm, inv_perm,
 *    offsets); sec. 2.3 L_aux = E sum_e f_e P_e; sec. 2.5 sign rule for b_e;
 *    sec. 3 worked example; sec. 4 "your graded tests" (per-token loop in
 *    float64 with an explicit (score, id) key).
 *  - "nano-moe" (cameronrwolfe substack): MLP experts with nn.GELU() (exact
 *    erf form) and biases.
 *  - "Extending Raschka's GPT-2: an MoE trained from scratch on an RTX 3090":
 *    masked top-k softmax example next to Diagram 4.
 *
 * Layout conventions (all row-major):
 *   x    [N, d]            token activations
 *   Wg   [E, d]            router, z_n[e] = sum_i Wg[e, i] x[n, i]
 *   W1   [E, F, d]         expert e: row f holds the weights of hidden unit f
 *   W3   [E, F, d]         SwiGLU "up" projection (unused for GELU)
 *   W2   [E, d, F]         expert e: row c holds the weights of output c
 *   b1   [E, F], b2 [E, d] optional biases
 *
 * Readings where the pages leave a step open:
 *   - selection for the softmax routers compares logits z (softmax is
 *     strictly increasing, so the chosen set and order equal those of p);
 *   - slot j of token n holds the j-th expert in (score desc, id asc) order;
 *   - SwiGLU hidden unit: silu(W1 x) * (W3 x);
 *   - GELU is the exact erf form;
 *   - f_e counts assignments; P_e averages the full softmax p (for the
 *     sigmoid router too);
 *   - sign(0) = 0 in the bias rule, evaluated on integers as
 *     sign(N k - E count_e).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_ID 2

#define ORC_SOFTMAX_TOPK 0
#define ORC_TOPK_SOFTMAX 1
#define ORC_SIGMOID 2

#define ORC_GELU 0
#define ORC_SWIGLU 1

/* ---------------------------------------------------------------- helpers */

/* Expert a ranks ahead of expert b: higher score, or equal score and lower
 * id ("ties go to the lowest id", router table of the course module). */
static int ranks_ahead(double score_a, int a, double score_b, int b)
{
    if (score_a > score_b) return 1;
    if (score_a < score_b) return 0;
    return a < b;
}

/* Order the ids 0..E-1 by (score desc, id asc); insertion sort, E is small. */
static void order_by_score(int E, const double *score, int *order)
{
    for (int e = 0; e < E; ++e) {
        int pos = e;
        while (pos > 0 && ranks_ahead(score[e], e, score[order[pos - 1]], order[pos - 1])) {
            order[pos] = order[pos - 1];
            --pos;
        }
        order[pos] = e;
    }
}

static double gelu_exact(double v) { return 0.5 * v * (1.0 + erf(v / sqrt(2.0))); }
static double silu(double v) { return v / (1.0 + exp(-v)); }
static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* ---------------------------------------------------------------- routing */

/*
 * Router for all N tokens.
 *
 *   z_n[e]  = sum_i Wg[e,i] x[n,i]                        (symbol table)
 *   p_n     = softmax(z_n)                                 (symbol table)
 *   chosen T_n: softmax routers -> top k of z_n (= of p_n);
 *               sigmoid router  -> top k of sigma(z_n) + b (router table,
 *               sec. 2.5: the bias only chooses)
 *   weights:  softmax_topk -> p_{n,e}, renormalised over T_n if norm_topk;
 *             topk_softmax -> softmax over the chosen logits;
 *             sigmoid      -> sigma(z_{n,e}), renormalised if norm_topk;
 *   then every weight times routed_scaling.
 *
 * margin[n] (optional): smallest gap between neighbours among the first
 * min(k+1, E) scores in ranked order, measured on p (softmax routers) or on
 * sigma(z)+b (sigmoid router); +inf when there is only one score.
 *
 * forced[n] != 0 (optional) makes token n use forced_ids[n, :] as its chosen
 * experts, in that slot order, with weights computed from this oracle's own
 * fp64 scores; it lets a caller evaluate the oracle on another party's
 * selection for near-tie tokens.
 */
int oracle_route(int64_t N, int d, int E, int k, int router, int norm_topk,
                 double routed_scaling, const double *x, const double *Wg,
                 const double *b_sel, const int32_t *forced_ids,
                 const uint8_t *forced, int32_t *ids, double *w, double *probs,
                 double *logits, double *margin)
{
    if (N < 0 || d < 1 || E < 1 || k < 1 || k > E) return ORC_ERR_ARG;
    if (router < ORC_SOFTMAX_TOPK || router > ORC_SIGMOID) return ORC_ERR_ARG;
    if (!x || !Wg || !ids || !w) return ORC_ERR_ARG;

    double *z = malloc(sizeof(double) * E);
    double *p = malloc(sizeof(double) * E);
    double *sel = malloc(sizeof(double) * E);
    double *gap_score = malloc(sizeof(double) * E);
    int *order = malloc(sizeof(int) * E);
    if (!z || !p || !sel || !gap_score || !order) {
        free(z); free(p); free(sel); free(gap_score); free(order);
        return ORC_ERR_ARG;
    }

    for (int64_t n = 0; n < N; ++n) {
        const double *xn = x + n * d;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += Wg[(int64_t)e * d + i] * xn[i];
            z[e] = acc;
        }
        double zmax = z[0];
        for (int e = 1; e < E; ++e) if (z[e] > zmax) zmax = z[e];
        double denom = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp(z[e] - zmax); denom += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= denom;

        for (int e = 0; e < E; ++e) {
            if (router == ORC_SIGMOID) {
                sel[e] = sigmoid(z[e]) + (b_sel ? b_sel[e] : 0.0);
                gap_score[e] = sel[e];
            } else {
                sel[e] = z[e];
                gap_score[e] = p[e];
            }
        }
        order_by_score(E, sel, order);

        if (margin) {
            int m = (k + 1 < E) ? k + 1 : E;
            double mg = INFINITY;
            for (int r = 0; r + 1 < m; ++r) {
                double g = gap_score[order[r]] - gap_score[order[r + 1]];
                if (g < mg) mg = g;
            }
            margin[n] = mg;
        }

        int32_t *idn = ids + n * k;
        double *wn = w + n * k;
        for (int j = 0; j < k; ++j)
            idn[j] = (forced && forced[n]) ? forced_ids[n * k + j] : order[j];
        for (int j = 0; j < k; ++j)
            if (idn[j] < 0 || idn[j] >= E) {
                free(z); free(p); free(sel); free(gap_score); free(order);
                return ORC_ERR_ID;
            }

        if (router == ORC_SOFTMAX_TOPK) {
            double s = 0.0;
            for (int j = 0; j < k; ++j) { wn[j] = p[idn[j]]; s += wn[j]; }
            if (norm_topk) for (int j = 0; j < k; ++j) wn[j] /= s;
        } else if (router == ORC_TOPK_SOFTMAX) {
            double cmax = z[idn[0]];
            for (int j = 1; j < k; ++j) if (z[idn[j]] > cmax) cmax = z[idn[j]];
            double s = 0.0;
            for (int j = 0; j < k; ++j) { wn[j] = exp(z[idn[j]] - cmax); s += wn[j]; }
            for (int j = 0; j < k; ++j) wn[j] /= s;
        } else {
            double s = 0.0;
            for (int j = 0; j < k; ++j) { wn[j] = sigmoid(z[idn[j]]); s += wn[j]; }
            if (norm_topk) for (int j = 0; j < k; ++j) wn[j] /= s;
        }
        for (int j = 0; j < k; ++j) wn[j] *= routed_scaling;

        if (probs) for (int e = 0; e < E; ++e) probs[n * E + e] = p[e];
        if (logits) for (int e = 0; e < E; ++e) logits[n * E + e] = z[e];
    }
    free(z); free(p); free(sel); free(gap_score); free(order);
    return ORC_OK;
}

/* ----------------------------------------------------------------- expert */

/*
 * One expert on one token.
 *   GELU  : h = gelu(W1 x + b1),           o = W2 h + b2   ("nano-moe" MLP)
 *   SwiGLU: h = silu(W1 x) * (W3 x),       o = W2 h (+ b2) (course module,
 *           act="silu" gated MLP)
 * W1/W3 point at one expert's [F, d] block, W2 at its [d, F] block;
 * b1 ([F], GELU only: the SwiGLU experts on the pages carry no hidden bias)
 * and b2 ([d]) may be NULL.  h is caller scratch of F doubles.
 */
void oracle_expert_ffn(int d, int F, int act, const double *x,
                       const double *W1, const double *b1, const double *W3,
                       const double *W2, const double *b2, double *h,
                       double *out)
{
    for (int f = 0; f < F; ++f) {
        double g = 0.0;
        for (int i = 0; i < d; ++i) g += W1[(int64_t)f * d + i] * x[i];
        if (act == ORC_SWIGLU) {
            double u = 0.0;
            for (int i = 0; i < d; ++i) u += W3[(int64_t)f * d + i] * x[i];
            h[f] = silu(g) * u;
        } else {
            if (b1) g += b1[f];
            h[f] = gelu_exact(g);
        }
    }
    for (int c = 0; c < d; ++c) {
        double o = 0.0;
        for (int f = 0; f < F; ++f) o += W2[(int64_t)c * F + f] * h[f];
        if (b2) o += b2[c];
        out[c] = o;
    }
}

static void expert_on_token(int d, int F, int act, int e, const double *xrow,
                            const double *W1, const double *b1,
                            const double *W3, const double *W2,
                            const double *b2, double *h, double *out)
{
    oracle_expert_ffn(d, F, act, xrow, W1 + (int64_t)e * F * d,
                      b1 ? b1 + (int64_t)e * F : NULL,
                      W3 ? W3 + (int64_t)e * F * d : NULL,
                      W2 + (int64_t)e * d * F,
                      b2 ? b2 + (int64_t)e * d : NULL, h, out);
}

/*
 * Per-token loop: y_n = sum_j w_{n,j} Expert_{T_n[j]}(x_n), the sum taken in
 * slot order starting from zero (sec. 2.1 equation, no shared expert).
 */
int oracle_dense_forward(int64_t N, int d, int F, int E, int k, int act,
                         const double *x, const double *W1, const double *b1,
                         const double *W3, const double *W2, const double *b2,
                         const int32_t *ids, const double *w, double *y)
{
    if (N < 0 || d < 1 || F < 1 || E < 1 || k < 1) return ORC_ERR_ARG;
    if (act == ORC_SWIGLU && !W3) return ORC_ERR_ARG;
    double *h = malloc(sizeof(double) * F);
    double *o = malloc(sizeof(double) * d);
    if (!h || !o) { free(h); free(o); return ORC_ERR_ARG; }
    for (int64_t n = 0; n < N; ++n) {
        double *yn = y + n * d;
        for (int c = 0; c < d; ++c) yn[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[n * k + j];
            if (e < 0 || e >= E) { free(h); free(o); return ORC_ERR_ID; }
            expert_on_token(d, F, act, e, x + n * d, W1, b1, W3, W2, b2, h, o);
            for (int c = 0; c < d; ++c) yn[c] += w[n * k + j] * o[c];
        }
    }
    free(h); free(o);
    return ORC_OK;
}

/* --------------------------------------------------------------- dispatch */

typedef struct { int32_t expert; int64_t a; } assignment;

static int cmp_assignment(const void *pa, const void *pb)
{
    const assignment *u = pa, *v = pb;
    if (u->expert != v->expert) return u->expert < v->expert ? -1 : 1;
    return (u->a > v->a) - (u->a < v->a);
}

/*
 * Sorted dispatch (sec. 2.2): assignments a = n k + j, stably sorted by
 * expert id.  Sorting on the key (expert, a) is that stable sort, because a
 * is unique.  perm[i] = the assignment at sorted position i;
 * inv_perm[perm[i]] = i; counts[e] = assignments to e; offsets[e] = start of
 * e's slice (offsets[0] = 0, offsets[E] = N k).  Any of perm, inv_perm,
 * offsets, counts may be NULL.
 */
int oracle_dispatch(int64_t N, int E, int k, const int32_t *ids,
                    int32_t *perm, int32_t *inv_perm, int32_t *offsets,
                    int32_t *counts)
{
    if (N < 0 || E < 1 || k < 1) return ORC_ERR_ARG;
    int64_t A = N * k;
    for (int64_t a = 0; a < A; ++a)
        if (ids[a] < 0 || ids[a] >= E) return ORC_ERR_ID;
    assignment *as = malloc(sizeof(assignment) * (A > 0 ? A : 1));
    if (!as) return ORC_ERR_ARG;
    for (int64_t a = 0; a < A; ++a) { as[a].expert = ids[a]; as[a].a = a; }
    qsort(as, (size_t)A, sizeof(assignment), cmp_assignment);
    if (perm) for (int64_t i = 0; i < A; ++i) perm[i] = (int32_t)as[i].a;
    if (inv_perm) for (int64_t i = 0; i < A; ++i) inv_perm[as[i].a] = (int32_t)i;
    if (counts || offsets) {
        int32_t *cnt = calloc((size_t)E, sizeof(int32_t));
        if (!cnt) { free(as); return ORC_ERR_ARG; }
        for (int64_t a = 0; a < A; ++a) cnt[ids[a]] += 1;
        if (counts) memcpy(counts, cnt, sizeof(int32_t) * E);
        if (offsets) {
            offsets[0] = 0;
            for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + cnt[e];
        }
        free(cnt);
    }
    free(as);
    return ORC_OK;
}

/*
 * Combine (sec. 2.2): y_n = sum_j w_{n,j} y_sorted[inv_perm[n k + j]], slot
 * order, starting from zero.  y_sorted is [N k, d].
 */
void oracle_combine(int64_t N, int d, int k, const double *y_sorted,
                    const double *w, const int32_t *inv_perm, double *y)
{
    for (int64_t n = 0; n < N; ++n) {
        double *yn = y + n * d;
        for (int c = 0; c < d; ++c) yn[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            const double *src = y_sorted + (int64_t)inv_perm[n * k + j] * d;
            for (int c = 0; c < d; ++c) yn[c] += w[n * k + j] * src[c];
        }
    }
}

/*
 * The sorted path end to end: dispatch, x_sorted = x[perm // k], each expert
 * on its own slice offsets[e] .. offsets[e+1]-1, then combine through
 * inv_perm.  Optional outputs x_sorted [N k, d] and y_sorted [N k, d].
 */
int oracle_sorted_forward(int64_t N, int d, int F, int E, int k, int act,
                          const double *x, const double *W1, const double *b1,
                          const double *W3, const double *W2, const double *b2,
                          const int32_t *ids, const double *w, double *y,
                          double *x_sorted_out, double *y_sorted_out)
{
    if (N < 0 || d < 1 || F < 1 || E < 1 || k < 1) return ORC_ERR_ARG;
    if (act == ORC_SWIGLU && !W3) return ORC_ERR_ARG;
    int64_t A = N * k;
    size_t nA = (size_t)(A > 0 ? A : 1);
    int32_t *perm = malloc(sizeof(int32_t) * nA);
    int32_t *inv = malloc(sizeof(int32_t) * nA);
    int32_t *offsets = malloc(sizeof(int32_t) * (E + 1));
    double *xs = malloc(sizeof(double) * nA * d);
    double *ys = malloc(sizeof(double) * nA * d);
    double *h = malloc(sizeof(double) * F);
    int rc = ORC_ERR_ARG;
    if (!perm || !inv || !offsets || !xs || !ys || !h) goto done;
    rc = oracle_dispatch(N, E, k, ids, perm, inv, offsets, NULL);
    if (rc != ORC_OK) goto done;
    for (int64_t i = 0; i < A; ++i)
        memcpy(xs + i * d, x + (int64_t)(perm[i] / k) * d, sizeof(double) * d);
    for (int e = 0; e < E; ++e)
        for (int64_t i = offsets[e]; i < offsets[e + 1]; ++i)
            expert_on_token(d, F, act, e, xs + i * d, W1, b1, W3, W2, b2, h,
                            ys + i * d);
    oracle_combine(N, d, k, ys, w, inv, y);
    if (x_sorted_out) memcpy(x_sorted_out, xs, sizeof(double) * A * d);
    if (y_sorted_out) memcpy(y_sorted_out, ys, sizeof(double) * A * d);
    rc = ORC_OK;
done:
    free(perm); free(inv); free(offsets); free(xs); free(ys); free(h);
    return rc;
}

/* ----------------------------------------------------------- aux and bias */

/*
 * Switch load-balance loss (sec. 2.3): f_e = (assignments to e) / N,
 * P_e = (1/N) sum_n p_{n,e}, L = E sum_e f_e P_e.  probs is [N, E].
 * counts_out (optional) receives the assignment counts.
 */
double oracle_aux_loss(int64_t N, int E, int k, const double *probs,
                       const int32_t *ids, int32_t *counts_out)
{
    if (N <= 0 || E < 1 || k < 1) return NAN;
    int32_t *cnt = calloc((size_t)E, sizeof(int32_t));
    double *P = calloc((size_t)E, sizeof(double));
    if (!cnt || !P) { free(cnt); free(P); return NAN; }
    for (int64_t a = 0; a < N * k; ++a) {
        if (ids[a] < 0 || ids[a] >= E) { free(cnt); free(P); return NAN; }
        cnt[ids[a]] += 1;
    }
    for (int64_t n = 0; n < N; ++n)
        for (int e = 0; e < E; ++e) P[e] += probs[n * E + e];
    double L = 0.0;
    for (int e = 0; e < E; ++e) {
        double f = (double)cnt[e] / (double)N;
        double Pe = P[e] / (double)N;
        L += f * Pe;
    }
    L *= (double)E;
    if (counts_out) memcpy(counts_out, cnt, sizeof(int32_t) * E);
    free(cnt); free(P);
    return L;
}

/*
 * The Switch loss of a batch split into parts (course module sec. 2.3: f_e
 * and P_e are averages over the whole batch of N tokens), from each part's
 * assignment counts and probability sums added up over the parts:
 * counts[e] = assignments to e in the whole batch, psum[e] = sum over the
 * whole batch of p_{n,e}.  Every token makes k assignments, so
 * N = (sum_e counts[e]) / k; then f_e = counts[e] / N, P_e = psum[e] / N and
 * L = E sum_e f_e P_e as in oracle_aux_loss.  0 for an empty batch.
 */
double oracle_aux_from_partials(int E, int k, const int32_t *counts, const double *psum)
{
    if (E < 1 || k < 1) return NAN;
    int64_t total = 0;
    for (int e = 0; e < E; ++e) total += counts[e];
    if (total == 0) return 0.0;
    const double N = (double)total / (double)k;
    double L = 0.0;
    for (int e = 0; e < E; ++e) {
        double f = (double)counts[e] / N;
        double Pe = psum[e] / N;
        L += f * Pe;
    }
    return L * (double)E;
}

/*
 * Aux-free bias rule (sec. 2.5): b_e <- b_e + gamma sign(mean load - load_e)
 * with mean load = N k / E, i.e. the sign of the integer N k - E count_e.
 */
void oracle_bias_update(int64_t N, int E, int k, const int32_t *counts,
                        double gamma, double *b)
{
    for (int e = 0; e < E; ++e) {
        int64_t diff = N * (int64_t)k - (int64_t)E * counts[e];
        int s = (diff > 0) - (diff < 0);
        b[e] += gamma * (double)s;
    }
}

/* ------------------------------------------------------ router z-loss, shared */

/*
 * Router z-loss ("nano-moe", "Router z-loss"; RustingBrain tutorial chapter
 * "Mixture of Experts", sec. 15.3 "The z-loss"): the mean over tokens of the squared log-sum-exp of the
 * router logits, (1/N) sum_n (log sum_e exp z_{n,e})^2.  logits is [N, E].
 */
double oracle_z_loss(int64_t N, int E, const double *logits)
{
    if (N <= 0 || E < 1) return N == 0 ? 0.0 : NAN;
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        const double *z = logits + n * E;
        double zmax = z[0];
        for (int e = 1; e < E; ++e) if (z[e] > zmax) zmax = z[e];
        double s = 0.0;
        for (int e = 0; e < E; ++e) s += exp(z[e] - zmax);
        const double lse = zmax + log(s);
        total += lse * lse;
    }
    return total / (double)N;
}

/*
 * Shared expert (course module sec. 2.1: y_n = sum_{e in T_n} w_{n,e}
 * Expert_e(x_n) + Shared(x_n); S shared experts of width f act as one FFN of
 * width S f; RustingBrain chapter sec. 15.4 "The shared expert"): adds Shared(x_n) to y_n for every token, after the routed sum.
 * Ws1/Ws3 are [Fs, d], Ws2 [d, Fs]; bs1 [Fs] (GELU only) and bs2 [d] may be
 * NULL.
 */
int oracle_shared_add(int64_t N, int d, int Fs, int act, const double *x,
                      const double *Ws1, const double *bs1, const double *Ws3,
                      const double *Ws2, const double *bs2, double *y)
{
    if (N < 0 || d < 1 || Fs < 1) return ORC_ERR_ARG;
    if (act == ORC_SWIGLU && !Ws3) return ORC_ERR_ARG;
    double *h = malloc(sizeof(double) * Fs);
    double *o = malloc(sizeof(double) * d);
    if (!h || !o) { free(h); free(o); return ORC_ERR_ARG; }
    for (int64_t n = 0; n < N; ++n) {
        oracle_expert_ffn(d, Fs, act, x + n * d, Ws1, bs1, Ws3, Ws2, bs2, h, o);
        for (int c = 0; c < d; ++c) y[n * d + c] += o[c];
    }
    free(h); free(o);
    return ORC_OK;
}

/* --------------------------------------------------------------- backward */

/*
 * One FFN (an expert or the shared expert) on one token, backward: given the
 * gradient `go` of its output o, adds the parameter gradients and the input
 * gradient.  Recomputes the pre-activations from x.
 *   GELU  : a = W1 x + b1, h = gelu(a), o = W2 h + b2;
 *           gelu'(a) = Phi(a) + a phi(a)
 *   SwiGLU: g = W1 x, u = W3 x, h = silu(g) u, o = W2 h (+ b2);
 *           silu'(g) = s (1 + g (1 - s)), s = sigmoid(g)
 * dh = W2^T go; dW2 += go h^T; db2 += go; then da (dg, du) through the
 * activation; dW1 += da x^T (dW3 += du x^T); db1 += da; dx += W1^T da
 * (+ W3^T du).  Gradient pointers other than dx may be NULL (not wanted).
 */
static void ffn_backward(int d, int F, int act, const double *x, const double *W1, const double *b1,
                         const double *W3, const double *W2, const double *go, double *dW1, double *db1,
                         double *dW3, double *dW2, double *db2, double *dx, double *scratch)
{
    double *a = scratch, *u = scratch + F, *h = scratch + 2 * F, *dh = scratch + 3 * F;
    for (int f = 0; f < F; ++f) {
        double g = 0.0;
        for (int i = 0; i < d; ++i) g += W1[(int64_t)f * d + i] * x[i];
        if (act == ORC_SWIGLU) {
            double v = 0.0;
            for (int i = 0; i < d; ++i) v += W3[(int64_t)f * d + i] * x[i];
            a[f] = g;
            u[f] = v;
            h[f] = silu(g) * v;
        } else {
            if (b1 != NULL) g += b1[f];
            a[f] = g;
            h[f] = gelu_exact(g);
        }
    }
    for (int f = 0; f < F; ++f) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += W2[(int64_t)c * F + f] * go[c];
        dh[f] = s;
    }
    if (dW2)
        for (int c = 0; c < d; ++c)
            for (int f = 0; f < F; ++f) dW2[(int64_t)c * F + f] += go[c] * h[f];
    if (db2) for (int c = 0; c < d; ++c) db2[c] += go[c];
    for (int f = 0; f < F; ++f) {
        double da, du = 0.0;
        if (act == ORC_SWIGLU) {
            const double sg = sigmoid(a[f]);
            da = dh[f] * u[f] * sg * (1.0 + a[f] * (1.0 - sg));
            du = dh[f] * silu(a[f]);
        } else {
            const double Phi = 0.5 * (1.0 + erf(a[f] / sqrt(2.0)));
            const double phi = exp(-0.5 * a[f] * a[f]) / sqrt(2.0 * acos(-1.0));
            da = dh[f] * (Phi + a[f] * phi);
            if (db1) db1[f] += da;
        }
        for (int i = 0; i < d; ++i) {
            if (dW1) dW1[(int64_t)f * d + i] += da * x[i];
            dx[i] += W1[(int64_t)f * d + i] * da;
            if (act == ORC_SWIGLU) {
                if (dW3) dW3[(int64_t)f * d + i] += du * x[i];
                dx[i] += W3[(int64_t)f * d + i] * du;
            }
        }
    }
}

/*
 * Backward of the layer (course module sec. 2.1 forward with the sec. 2.3
 * Switch loss; "nano-moe" router z-loss) for the scalar
 *   loss = <dy, y> + aux_coef * L_aux + z_coef * L_z,
 * y = sum_j w_j Expert_{T_n[j]}(x_n) + Shared(x_n).  The expert choice and
 * f_e = count_e / N are piecewise constant (no gradient, sec. 2.4); the
 * selection bias b_sel selects only.  Per token:
 *   dw_j = <dy_n, o_j> for the j-th expert output o_j; the expert gets the
 *   output gradient w_j dy_n; the shared expert gets dy_n;
 *   gates w_j = routed_scaling * g_{T[j]}:
 *     softmax_topk: g_e = p_e (/ S, S = sum_T p, if norm_topk)
 *     topk_softmax: g = softmax over z_T
 *     sigmoid:      g_e = s_e = sigmoid(z_e) (/ sum_T s, if norm_topk)
 *   L_aux = E sum_e f_e P_e gives dL_aux/dp_{n,e} = E f_e / N (sec. 2.3,
 *   through P_e = mean_n p_{n,e}, p = softmax(z) for every router);
 *   L_z = mean_n lse(z_n)^2 gives dL_z/dz_{n,e} = 2 lse(z_n) p_{n,e} / N;
 *   through p = softmax(z): dz = p (dp - <p, dp>);
 *   dW_g += dz x_n^T; dx_n += W_g^T dz.
 * forced_ids / forced replay the routing as in oracle_route.  Every gradient
 * is zeroed first; shared-expert pointers are NULL when Fs = 0; dWs*, db*
 * may be NULL where the activation has no such parameter.
 */
int oracle_backward(int64_t N, int d, int F, int E, int k, int router, int norm_topk,
                    double routed_scaling, int act, const double *x, const double *Wg,
                    const double *b_sel, const double *W1, const double *b1,
                    const double *W3, const double *W2, const double *b2, int Fs,
                    const double *Ws1, const double *bs1, const double *Ws3,
                    const double *Ws2, const double *bs2, const double *dy,
                    double aux_coef, double z_coef, const int32_t *forced_ids,
                    const uint8_t *forced, double *dx, double *dWg, double *dW1,
                    double *db1, double *dW3, double *dW2, double *db2, double *dWs1,
                    double *dbs1, double *dWs3, double *dWs2, double *dbs2)
{
    if (N < 0 || d < 1 || F < 1 || E < 1 || k < 1 || k > E || Fs < 0) return ORC_ERR_ARG;
    if (act == ORC_SWIGLU && (!W3 || !dW3)) return ORC_ERR_ARG;
    if (Fs > 0 && (!Ws1 || !Ws2 || !dWs1 || !dWs2 || (act == ORC_SWIGLU && (!Ws3 || !dWs3)))) return ORC_ERR_ARG;
    memset(dx, 0, sizeof(double) * N * d);
    memset(dWg, 0, sizeof(double) * E * d);
    memset(dW1, 0, sizeof(double) * E * F * d);
    memset(dW2, 0, sizeof(double) * E * d * F);
    if (dW3) memset(dW3, 0, sizeof(double) * E * F * d);
    if (db1) memset(db1, 0, sizeof(double) * E * F);
    if (db2) memset(db2, 0, sizeof(double) * E * d);
    if (Fs > 0) {
        memset(dWs1, 0, sizeof(double) * Fs * d);
        memset(dWs2, 0, sizeof(double) * d * Fs);
        if (dWs3) memset(dWs3, 0, sizeof(double) * Fs * d);
        if (dbs1) memset(dbs1, 0, sizeof(double) * Fs);
        if (dbs2) memset(dbs2, 0, sizeof(double) * d);
    }
    if (N == 0) return ORC_OK;

    int32_t *ids = malloc(sizeof(int32_t) * N * k);
    double *w = malloc(sizeof(double) * N * k);
    double *probs = malloc(sizeof(double) * N * E);
    double *logits = malloc(sizeof(double) * N * E);
    double *cnt = calloc(E, sizeof(double));
    int Fmax = F > Fs ? F : Fs;
    double *scratch = malloc(sizeof(double) * 4 * Fmax);
    double *hbuf = malloc(sizeof(double) * F);
    double *o = malloc(sizeof(double) * d);
    double *go = malloc(sizeof(double) * d);
    double *dp = malloc(sizeof(double) * E);
    double *dz = malloc(sizeof(double) * E);
    double *dg = malloc(sizeof(double) * E);
    if (!ids || !w || !probs || !logits || !cnt || !scratch || !hbuf || !o || !go || !dp || !dz || !dg) {
        free(ids); free(w); free(probs); free(logits); free(cnt); free(scratch); free(hbuf);
        free(o); free(go); free(dp); free(dz); free(dg);
        return ORC_ERR_ARG;
    }
    int rc = oracle_route(N, d, E, k, router, norm_topk, routed_scaling, x, Wg, b_sel, forced_ids, forced,
                          ids, w, probs, logits, NULL);
    if (rc == ORC_OK) {
        for (int64_t a = 0; a < N * k; ++a) cnt[ids[a]] += 1.0;
        for (int64_t n = 0; n < N; ++n) {
            const double *xn = x + n * d, *dyn = dy + n * d, *p = probs + n * E, *z = logits + n * E;
            const int32_t *idn = ids + n * k;
            double *dxn = dx + n * d;
            for (int e = 0; e < E; ++e) dg[e] = 0.0;
            for (int j = 0; j < k; ++j) {
                const int e = idn[j];
                expert_on_token(d, F, act, e, xn, W1, b1, W3, W2, b2, hbuf, o);
                double dwj = 0.0;
                for (int c = 0; c < d; ++c) dwj += dyn[c] * o[c];
                dg[e] += routed_scaling * dwj;  /* gradient of the unscaled gate */
                for (int c = 0; c < d; ++c) go[c] = w[n * k + j] * dyn[c];
                ffn_backward(d, F, act, xn, W1 + (int64_t)e * F * d, b1 ? b1 + (int64_t)e * F : NULL,
                             W3 ? W3 + (int64_t)e * F * d : NULL, W2 + (int64_t)e * d * F, go,
                             dW1 + (int64_t)e * F * d, db1 ? db1 + (int64_t)e * F : NULL,
                             dW3 ? dW3 + (int64_t)e * F * d : NULL, dW2 + (int64_t)e * d * F,
                             db2 ? db2 + (int64_t)e * d : NULL, dxn, scratch);
            }
            if (Fs > 0)
                ffn_backward(d, Fs, act, xn, Ws1, bs1, Ws3, Ws2, dyn, dWs1, dbs1, dWs3, dWs2, dbs2, dxn,
                             scratch);

            /* gates -> dp (softmax probabilities) and dz (direct) */
            for (int e = 0; e < E; ++e) { dp[e] = 0.0; dz[e] = 0.0; }
            if (router == ORC_SOFTMAX_TOPK) {
                if (norm_topk) {
                    double S = 0.0, gp = 0.0;
                    for (int j = 0; j < k; ++j) { S += p[idn[j]]; gp += dg[idn[j]] * p[idn[j]]; }
                    for (int j = 0; j < k; ++j) dp[idn[j]] += dg[idn[j]] / S - gp / (S * S);
                } else {
                    for (int j = 0; j < k; ++j) dp[idn[j]] += dg[idn[j]];
                }
            } else if (router == ORC_TOPK_SOFTMAX) {
                double cmax = z[idn[0]], s = 0.0, gdot = 0.0;
                for (int j = 1; j < k; ++j) if (z[idn[j]] > cmax) cmax = z[idn[j]];
                for (int j = 0; j < k; ++j) s += exp(z[idn[j]] - cmax);
                for (int j = 0; j < k; ++j) gdot += exp(z[idn[j]] - cmax) / s * dg[idn[j]];
                for (int j = 0; j < k; ++j) {
                    const double gj = exp(z[idn[j]] - cmax) / s;
                    dz[idn[j]] += gj * (dg[idn[j]] - gdot);
                }
            } else {
                double S = 0.0, gs = 0.0;
                for (int j = 0; j < k; ++j) { S += sigmoid(z[idn[j]]); gs += dg[idn[j]] * sigmoid(z[idn[j]]); }
                for (int j = 0; j < k; ++j) {
                    const int e = idn[j];
                    const double s = sigmoid(z[e]);
                    const double ds = norm_topk ? dg[e] / S - gs / (S * S) : dg[e];
                    dz[e] += ds * s * (1.0 - s);
                }
            }
            /* Switch loss through P_e = mean_n p_{n,e} */
            for (int e = 0; e < E; ++e) dp[e] += aux_coef * (double)E * (cnt[e] / (double)N) / (double)N;
            double pdp = 0.0;
            for (int e = 0; e < E; ++e) pdp += p[e] * dp[e];
            for (int e = 0; e < E; ++e) dz[e] += p[e] * (dp[e] - pdp);
            /* router z-loss */
            if (z_coef != 0.0) {
                double zmax = z[0], s = 0.0;
                for (int e = 1; e < E; ++e) if (z[e] > zmax) zmax = z[e];
                for (int e = 0; e < E; ++e) s += exp(z[e] - zmax);
                const double lse_n = zmax + log(s);
                for (int e = 0; e < E; ++e) dz[e] += z_coef * 2.0 * lse_n * p[e] / (double)N;
            }
            for (int e = 0; e < E; ++e)
                for (int i = 0; i < d; ++i) {
                    dWg[(int64_t)e * d + i] += dz[e] * xn[i];
                    dxn[i] += Wg[(int64_t)e * d + i] * dz[e];
                }
        }
    }
    free(ids); free(w); free(probs); free(logits); free(cnt); free(scratch); free(hbuf);
    free(o); free(go); free(dp); free(dz); free(dg);
    return rc;
}
