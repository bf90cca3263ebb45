/*
 * fp64 CPU oracle of the Mixtral-style sparse MoE feed-forward layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
 * baseline leg may load or call this.  It shares no code with the CUDA path:
 * no headers, helpers, tables or constants.  It is plain and slow on purpose:
 * every sum runs in double, index ascending, with no blocking or reordering.
 *
 * What it computes, per token x (a row of the input), following the
 * "Mistral/Mixtral architecture" page (disassemble-channel.com,
 * "Mistral/Mixtralのアーキテクチャ — Sliding Window AttentionとMoEの融合"),
 * section "MoEの数学 — ルーターとゲーティング機構":
 *
 *   1. router scores   s = Wg x, Wg in R^{E x d}, no bias
 *                      (subsection "Top-2ゲーティングの定式化", score equation;
 *                       the "Mixtral of Experts" summary page writes the same
 *                       thing as H(x)_i = (x . Wg)_i)
 *   2. top-k selection of the k largest scores, ordered by descending score
 *                      (same subsection, Top-2 equation with s_i1 >= s_i2);
 *                      equal scores go to the lower expert index
 *   3. gate weights    g_j = exp(s_ij) / sum_m exp(s_im) over the k selected
 *                      only (same subsection, gate equation; the summary page's
 *                      Softmax(KeepTopK(H, 2)) with the others at -inf is the
 *                      same thing).  Evaluated as exp(s_ij - s_i1) / sum, which
 *                      is the same number, to keep exp() in range.
 *   4. experts         E_i(x) = W2_i (SiLU(W1_i x) * W3_i x), SiLU(a) = a sigmoid(a)
 *                      (subsection "各エキスパートの構造"; the page's code
 *                       "MoEレイヤー全体の実装" applies w2 on the left, so
 *                       W2_i in R^{d x F} multiplies the F-vector)
 *   5. output          MoE(x) = sum_j g_j E_ij(x), j = 0 .. k-1 in selection
 *                      order (subsection "Top-2ゲーティングの定式化", output
 *                      equation; the page's code adds slot 0 of every expert
 *                      first, then slot 1, which is the same per-token order)
 *
 * Only selected experts are evaluated: an unselected expert has gate weight
 * exactly zero, so it adds nothing.
 *
 * Two steps around the layer, from the same page:
 *
 *   6. the block       out = h + MoE(RMSNorm(h)): section "Mixtral 8x7B — Sparse
 *                      MoEの導入", subsection "Mixtralのアーキテクチャ" (the second
 *                      sub-layer of every Transformer block: RMSNorm, then the MoE
 *                      layer, then the residual connection).  The page names
 *                      RMSNorm without printing it; this file uses the usual
 *                      definition RMSNorm(h)_j = gamma_j h_j / sqrt(mean_i(h_i^2) + eps)
 *                      with a per-channel gain gamma and the caller's eps.
 *   7. load balance    f_i = (1/T) #{t : i among the top-k of s_t},
 *                      p_i = (1/T) sum_t softmax(s_t)_i over all E experts,
 *                      L = alpha * E * sum_i f_i p_i: subsection "ロードバランス損失"
 *                      (f, p and loss equations), with f counting all k
 *                      selections as the page's load_balance_loss code does.
 *   8. backward        gradients of a scalar loss L through the layer, given
 *                      dout = dL/dout (the training step the page's subsection
 *                      "ロードバランス損失" closes with: the layer is trained
 *                      by gradient descent on L_LM + L_balance).  The top-k
 *                      choice is piecewise constant, so no gradient flows
 *                      through it; for each selected slot j with expert e:
 *                        dy_j  = g_j dout                      dg_j = <dout, y_j>
 *                        ds_e  = g_j (dg_j - sum_m g_m dg_m)   (softmax over the k)
 *                        dh    = W2_e^T dy_j
 *                        da    = dh * b * SiLU'(a),  db = dh * SiLU(a)
 *                        dx   += W1_e^T da + W3_e^T db,  plus Wg^T ds from the router
 *                        dW2_e += dy_j h^T, dW1_e += da x^T, dW3_e += db x^T,
 *                        dWg   += ds x^T
 *                      with SiLU'(a) = sigmoid(a) (1 + a (1 - sigmoid(a))).
 *                      With alpha != 0 the loss also holds step 7's L_balance
 *                      (the page's total loss L_LM + L_balance): f is piecewise
 *                      constant, p = mean softmax(s), so each token's scores get
 *                        ds_e += (alpha E / T) p_te (f_e - sum_m p_tm f_m)
 *                      on every expert e, and that reaches dx and dWg through
 *                      the router like the rest of ds.
 *
 * Operands are row-major: x[T][d], Wg[E][d], W1[E][F][d], W3[E][F][d],
 * W2[E][d][F].  dtype 0 = float32 storage, 1 = bfloat16 bit patterns, 2 =
 * double (for operands that are themselves exact results, such as the
 * normalised rows of the block form); every element is widened exactly to
 * double before use.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of one stored element to double */
static double elem(const void* base, int dtype, size_t i) {
    if (dtype == 0) return (double)((const float*)base)[i];
    if (dtype == 2) return ((const double*)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* step 1 for one token: s[e] = sum_j x[j] * Wg[e][j], j ascending */
static void token_scores(int d, int E, const void* x, const void* Wg, int dtype, size_t t, double* s) {
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += elem(x, dtype, t * (size_t)d + j) * elem(Wg, dtype, (size_t)e * d + j);
        s[e] = acc;
    }
}

/* e beats f in the selection order: higher score, or equal score and lower index */
static int beats(const double* s, int e, int f) {
    return s[e] > s[f] || (s[e] == s[f] && e < f);
}

/*
 * steps 2-3 for one token.  idx[0..k) and g[0..k) in selection order.
 * margin = s_(k) - s_(k+1) (k-th minus (k+1)-th largest score, +inf when k == E)
 * mingap = smallest gap between consecutive selected scores (+inf when k == 1)
 */
static void token_select(int E, int k, const double* s, int32_t* idx, double* g,
                         double* margin, double* mingap) {
    int chosen[64] = {0};
    int order[65];
    int n_order = (k < E) ? k + 1 : k;       /* also find the best unselected one */
    for (int r = 0; r < n_order; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (chosen[e]) continue;
            if (best < 0 || beats(s, e, best)) best = e;
        }
        chosen[best] = 1;
        order[r] = best;
    }
    for (int j = 0; j < k; ++j) idx[j] = order[j];
    double top = s[order[0]];
    double denom = 0.0;
    for (int j = 0; j < k; ++j) denom += exp(s[order[j]] - top);
    for (int j = 0; j < k; ++j) g[j] = exp(s[order[j]] - top) / denom;
    if (margin) *margin = (k < E) ? s[order[k - 1]] - s[order[k]] : INFINITY;
    if (mingap) {
        double m = INFINITY;
        for (int j = 0; j + 1 < k; ++j) {
            double gap = s[order[j]] - s[order[j + 1]];
            if (gap < m) m = gap;
        }
        *mingap = m;
    }
}

/* step 4 for one token vector xv (already widened): y = W2_e (SiLU(W1_e xv) * W3_e xv) */
static void expert_apply(int d, int F, const double* xv, const void* W1, const void* W3, const void* W2,
                         int dtype, int e, double* h, double* y) {
    size_t w13 = (size_t)e * F * d;
    for (int f = 0; f < F; ++f) {
        double a = 0.0, b = 0.0;
        for (int j = 0; j < d; ++j) {
            a += elem(W1, dtype, w13 + (size_t)f * d + j) * xv[j];
            b += elem(W3, dtype, w13 + (size_t)f * d + j) * xv[j];
        }
        double silu = a / (1.0 + exp(-a));
        h[f] = silu * b;
    }
    size_t w2 = (size_t)e * d * F;
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += elem(W2, dtype, w2 + (size_t)i * F + f) * h[f];
        y[i] = acc;
    }
}

/* router scores for all tokens: logits[T][E] */
int oracle_scores(int T, int d, int E, const void* x, const void* Wg, int dtype, double* logits,
                  int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || E > 64) return 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) token_scores(d, E, x, Wg, dtype, (size_t)t, logits + (size_t)t * E);
    return 0;
}

/* selection + gates from given scores (used by tests to pin the selection) */
int oracle_select(int T, int E, int k, const double* logits, int32_t* idx, double* g, double* margin,
                  double* mingap) {
    if (T < 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
    for (int t = 0; t < T; ++t)
        token_select(E, k, logits + (size_t)t * E, idx + (size_t)t * k, g + (size_t)t * k,
                     margin ? margin + t : NULL, mingap ? mingap + t : NULL);
    return 0;
}

/* routing of all tokens (steps 1-3) */
int oracle_route(int T, int d, int E, int k, const void* x, const void* Wg, int dtype, int32_t* idx,
                 double* g, double* margin, double* mingap, int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        double s[64];
        token_scores(d, E, x, Wg, dtype, (size_t)t, s);
        token_select(E, k, s, idx + (size_t)t * k, g + (size_t)t * k, margin + t, mingap + t);
    }
    return 0;
}

/* one expert on one token row of x (step 4 alone) */
int oracle_expert(int d, int F, const void* x, const void* W1, const void* W3, const void* W2, int dtype,
                  int e, int t, double* y) {
    if (d <= 0 || F <= 0) return 1;
    double* xv = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * F);
    if (!xv || !h) { free(xv); free(h); return 2; }
    for (int j = 0; j < d; ++j) xv[j] = elem(x, dtype, (size_t)t * d + j);
    expert_apply(d, F, xv, W1, W3, W2, dtype, e, h, y);
    free(xv);
    free(h);
    return 0;
}

/*
 * The whole layer for the tokens listed in tokens[0..n) (all tokens when
 * tokens == NULL, n == T).  out[n][d] in double; idx/g [n][k]; margin/mingap [n].
 */
int oracle_moe(int T, int d, int F, int E, int k, const void* x, const void* Wg, const void* W1,
               const void* W3, const void* W2, int dtype, const int32_t* tokens, int n, double* out,
               int32_t* idx, double* g, double* margin, double* mingap, int nthreads) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E || n < 0) return 1;
    if (!tokens && n != T) return 1;
    for (int r = 0; r < n; ++r)
        if (tokens && (tokens[r] < 0 || tokens[r] >= T)) return 1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* xv = (double*)malloc(sizeof(double) * d);
        double* h = (double*)malloc(sizeof(double) * F);
        double* y = (double*)malloc(sizeof(double) * d);
        if (!xv || !h || !y) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                size_t t = tokens ? (size_t)tokens[r] : (size_t)r;
                double s[64];
                token_scores(d, E, x, Wg, dtype, t, s);
                int32_t* ir = idx + (size_t)r * k;
                double* gr = g + (size_t)r * k;
                token_select(E, k, s, ir, gr, margin + r, mingap + r);
                for (int j = 0; j < d; ++j) xv[j] = elem(x, dtype, t * d + j);
                double* o = out + (size_t)r * d;
                for (int i = 0; i < d; ++i) o[i] = 0.0;
                for (int j = 0; j < k; ++j) {
                    expert_apply(d, F, xv, W1, W3, W2, dtype, ir[j], h, y);
                    for (int i = 0; i < d; ++i) o[i] += gr[j] * y[i];
                }
            }
        }
        free(xv);
        free(h);
        free(y);
    }
    return fail ? 2 : 0;
}

/* ------------------------------------------------------------------ block */

/* step 6, the norm, for one row: u_j = gamma_j * h_j / sqrt((1/d) sum_i h_i^2 + eps) */
static void row_rmsnorm(int d, const void* h, const void* gamma, double eps, int dtype, size_t t, double* u) {
    double ss = 0.0;
    for (int j = 0; j < d; ++j) {
        double v = elem(h, dtype, t * (size_t)d + j);
        ss += v * v;
    }
    double r = 1.0 / sqrt(ss / (double)d + eps);
    for (int j = 0; j < d; ++j) u[j] = elem(gamma, dtype, (size_t)j) * (elem(h, dtype, t * (size_t)d + j) * r);
}

/* step 1 on a vector already in double: s[e] = sum_j v[j] * Wg[e][j], j ascending */
static void vector_scores(int d, int E, const double* v, const void* Wg, int dtype, double* s) {
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += v[j] * elem(Wg, dtype, (size_t)e * d + j);
        s[e] = acc;
    }
}

/* the norm alone for every row: u[T][d] */
int oracle_rmsnorm(int T, int d, const void* h, const void* gamma, double eps, int dtype, double* u) {
    if (T < 0 || d <= 0 || !(eps >= 0.0)) return 1;
    for (int t = 0; t < T; ++t) row_rmsnorm(d, h, gamma, eps, dtype, (size_t)t, u + (size_t)t * d);
    return 0;
}

/* router scores of the normalised rows: logits[T][E] = Wg RMSNorm(h_t) */
int oracle_block_scores(int T, int d, int E, const void* h, const void* gamma, double eps, const void* Wg,
                        int dtype, double* logits, int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || E > 64 || !(eps >= 0.0)) return 1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * d);
        if (!u) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int t = 0; t < T; ++t) {
                row_rmsnorm(d, h, gamma, eps, dtype, (size_t)t, u);
                vector_scores(d, E, u, Wg, dtype, logits + (size_t)t * E);
            }
        }
        free(u);
    }
    return fail ? 2 : 0;
}

/*
 * The block out = h + MoE(RMSNorm(h)) for the tokens listed in tokens[0..n)
 * (all tokens when tokens == NULL, n == T).  Steps 1-5 run on u = RMSNorm(h_t)
 * exactly as in oracle_moe, then the row h_t is added.  out[n][d] in double.
 */
int oracle_block(int T, int d, int F, int E, int k, const void* h, const void* gamma, double eps, const void* Wg,
                 const void* W1, const void* W3, const void* W2, int dtype, const int32_t* tokens, int n,
                 double* out, int32_t* idx, double* g, double* margin, double* mingap, int nthreads) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E || n < 0 || !(eps >= 0.0)) return 1;
    if (!tokens && n != T) return 1;
    for (int r = 0; r < n; ++r)
        if (tokens && (tokens[r] < 0 || tokens[r] >= T)) return 1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * d);
        double* hh = (double*)malloc(sizeof(double) * F);
        double* y = (double*)malloc(sizeof(double) * d);
        double* m = (double*)malloc(sizeof(double) * d);
        if (!u || !hh || !y || !m) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                size_t t = tokens ? (size_t)tokens[r] : (size_t)r;
                row_rmsnorm(d, h, gamma, eps, dtype, t, u);
                double s[64];
                vector_scores(d, E, u, Wg, dtype, s);
                int32_t* ir = idx + (size_t)r * k;
                double* gr = g + (size_t)r * k;
                token_select(E, k, s, ir, gr, margin + r, mingap + r);
                for (int i = 0; i < d; ++i) m[i] = 0.0;
                for (int j = 0; j < k; ++j) {
                    expert_apply(d, F, u, W1, W3, W2, dtype, ir[j], hh, y);
                    for (int i = 0; i < d; ++i) m[i] += gr[j] * y[i];
                }
                double* o = out + (size_t)r * d;
                for (int i = 0; i < d; ++i) o[i] = elem(h, dtype, t * (size_t)d + i) + m[i];
            }
        }
        free(u);
        free(hh);
        free(y);
        free(m);
    }
    return fail ? 2 : 0;
}

/* ------------------------------------------------------------ load balance */

/*
 * step 7 from given scores logits[T][E]: f[E], p[E] and the loss.
 * softmax over all E is evaluated as exp(s_e - max) / sum, the same number.
 */
int oracle_balance(int T, int E, int k, const double* logits, double alpha, double* f, double* p, double* loss) {
    if (T <= 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
    for (int e = 0; e < E; ++e) f[e] = p[e] = 0.0;
    for (int t = 0; t < T; ++t) {
        const double* s = logits + (size_t)t * E;
        int32_t idx[64];
        double g[64];
        token_select(E, k, s, idx, g, NULL, NULL);
        for (int j = 0; j < k; ++j) f[idx[j]] += 1.0;
        double mx = s[0];
        for (int e = 1; e < E; ++e)
            if (s[e] > mx) mx = s[e];
        double denom = 0.0;
        for (int e = 0; e < E; ++e) denom += exp(s[e] - mx);
        for (int e = 0; e < E; ++e) p[e] += exp(s[e] - mx) / denom;
    }
    double acc = 0.0;
    for (int e = 0; e < E; ++e) {
        f[e] /= (double)T;
        p[e] /= (double)T;
        acc += f[e] * p[e];
    }
    *loss = alpha * (double)E * acc;
    return 0;
}

/* ------------------------------------------------------------------ backward */

static double sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

/* the forward of one expert on xv, keeping a, b and h (step 4 with its intermediates) */
static void expert_forward_keep(int d, int F, const double* xv, const void* W1, const void* W3, const void* W2,
                                int dtype, int e, double* a, double* b, double* h, double* y) {
    size_t w13 = (size_t)e * F * d;
    for (int f = 0; f < F; ++f) {
        double sa = 0.0, sb = 0.0;
        for (int j = 0; j < d; ++j) {
            sa += elem(W1, dtype, w13 + (size_t)f * d + j) * xv[j];
            sb += elem(W3, dtype, w13 + (size_t)f * d + j) * xv[j];
        }
        a[f] = sa;
        b[f] = sb;
        h[f] = sa / (1.0 + exp(-sa)) * sb;
    }
    size_t w2 = (size_t)e * d * F;
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += elem(W2, dtype, w2 + (size_t)i * F + f) * h[f];
        y[i] = acc;
    }
}

struct bwd_scratch {
    double *xv, *go, *a, *b, *h, *y, *dy, *dh, *da, *db;   /* a, b, h: [k][F]; y: [k][d] */
};

static int scratch_alloc(struct bwd_scratch* w, int d, int F, int k) {
    w->xv = (double*)malloc(sizeof(double) * d);
    w->go = (double*)malloc(sizeof(double) * d);
    w->a = (double*)malloc(sizeof(double) * (size_t)k * F);
    w->b = (double*)malloc(sizeof(double) * (size_t)k * F);
    w->h = (double*)malloc(sizeof(double) * (size_t)k * F);
    w->y = (double*)malloc(sizeof(double) * (size_t)k * d);
    w->dy = (double*)malloc(sizeof(double) * d);
    w->dh = (double*)malloc(sizeof(double) * F);
    w->da = (double*)malloc(sizeof(double) * F);
    w->db = (double*)malloc(sizeof(double) * F);
    return w->xv && w->go && w->a && w->b && w->h && w->y && w->dy && w->dh && w->da && w->db;
}

static void scratch_free(struct bwd_scratch* w) {
    free(w->xv); free(w->go); free(w->a); free(w->b); free(w->h);
    free(w->y); free(w->dy); free(w->dh); free(w->da); free(w->db);
}

/*
 * step 8 for one token t: dx_t [d] and the router-score gradient ds [E]
 * (zero for unselected experts).  When dWg/dW1/dW3/dW2 are non-null the
 * token's contributions are added to them (the caller runs tokens in order).
 */
static void token_backward(int d, int F, int E, int k, const void* x, int xdtype, const void* Wg, const void* W1,
                           const void* W3, const void* W2, int dtype, const void* dout, size_t t,
                           struct bwd_scratch* w, double* dx, double* ds, int32_t* idx, double* g, double* margin,
                           double* mingap, double* dWg, double* dW1, double* dW3, double* dW2,
                           const double* ds_extra) {
    /* x is read as xdtype (the layer's dtype, or double for the block form's exact normalised rows) */
    for (int j = 0; j < d; ++j) {
        w->xv[j] = elem(x, xdtype, t * (size_t)d + j);
        w->go[j] = elem(dout, dtype, t * (size_t)d + j);
    }
    double s[64], dg[64];
    for (int e = 0; e < E; ++e) {   /* step 1, as token_scores: j ascending */
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += w->xv[j] * elem(Wg, dtype, (size_t)e * d + j);
        s[e] = acc;
    }
    token_select(E, k, s, idx, g, margin, mingap);
    for (int j = 0; j < k; ++j) {
        expert_forward_keep(d, F, w->xv, W1, W3, W2, dtype, idx[j], w->a + (size_t)j * F, w->b + (size_t)j * F,
                            w->h + (size_t)j * F, w->y + (size_t)j * d);
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += w->go[i] * w->y[(size_t)j * d + i];
        dg[j] = acc;
    }
    double gdg = 0.0;
    for (int j = 0; j < k; ++j) gdg += g[j] * dg[j];
    for (int e = 0; e < E; ++e) ds[e] = 0.0;
    for (int j = 0; j < k; ++j) ds[idx[j]] = g[j] * (dg[j] - gdg);
    if (ds_extra)
        for (int e = 0; e < E; ++e) ds[e] += ds_extra[e];
    /* router path: dx = Wg^T ds */
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int e = 0; e < E; ++e) acc += elem(Wg, dtype, (size_t)e * d + i) * ds[e];
        dx[i] = acc;
    }
    if (dWg)
        for (int e = 0; e < E; ++e)
            for (int i = 0; i < d; ++i) dWg[(size_t)e * d + i] += ds[e] * w->xv[i];
    for (int j = 0; j < k; ++j) {
        const int e = idx[j];
        const double* a = w->a + (size_t)j * F;
        const double* b = w->b + (size_t)j * F;
        const double* h = w->h + (size_t)j * F;
        for (int i = 0; i < d; ++i) w->dy[i] = g[j] * w->go[i];
        const size_t w2 = (size_t)e * d * F, w13 = (size_t)e * F * d;
        for (int f = 0; f < F; ++f) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += elem(W2, dtype, w2 + (size_t)i * F + f) * w->dy[i];
            w->dh[f] = acc;
            const double sg = sigmoid(a[f]);
            w->da[f] = acc * b[f] * sg * (1.0 + a[f] * (1.0 - sg));
            w->db[f] = acc * a[f] * sg;
        }
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int f = 0; f < F; ++f)
                acc += elem(W1, dtype, w13 + (size_t)f * d + i) * w->da[f] +
                       elem(W3, dtype, w13 + (size_t)f * d + i) * w->db[f];
            dx[i] += acc;
        }
        if (dW2)
            for (int i = 0; i < d; ++i)
                for (int f = 0; f < F; ++f) dW2[w2 + (size_t)i * F + f] += w->dy[i] * h[f];
        if (dW1)
            for (int f = 0; f < F; ++f)
                for (int i = 0; i < d; ++i) {
                    dW1[w13 + (size_t)f * d + i] += w->da[f] * w->xv[i];
                    dW3[w13 + (size_t)f * d + i] += w->db[f] * w->xv[i];
                }
    }
}

/*
 * Step 8's load-balance part from given scores logits[T][E]: the gradient of
 * alpha E sum_e f_e p_e with respect to every score, f held fixed (it is
 * piecewise constant): dbal[t][e] = (alpha E / T) p_te (f_e - sum_m p_tm f_m),
 * p_t = softmax(s_t) over all E.
 */
int oracle_balance_grad(int T, int E, int k, const double* logits, double alpha, double* dbal) {
    if (T <= 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
    double f[64], p[64], loss;
    if (oracle_balance(T, E, k, logits, alpha, f, p, &loss)) return 1;
    const double c = alpha * (double)E / (double)T;
    for (int t = 0; t < T; ++t) {
        const double* s = logits + (size_t)t * E;
        double mx = s[0];
        for (int e = 1; e < E; ++e)
            if (s[e] > mx) mx = s[e];
        double den = 0.0;
        for (int e = 0; e < E; ++e) den += exp(s[e] - mx);
        double pf = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp(s[e] - mx) / den;
            pf += p[e] * f[e];
        }
        for (int e = 0; e < E; ++e) dbal[(size_t)t * E + e] = c * p[e] * (f[e] - pf);
    }
    return 0;
}

/* router scores of every token (step 1) and, when alpha != 0, the load-balance part of ds; NULL when alpha == 0 */
static double* balance_part(int T, int d, int E, int k, const void* x, const void* Wg, int dtype, double alpha,
                            int* fail) {
    *fail = 0;
    if (alpha == 0.0 || T <= 0) return NULL;
    double* s = (double*)malloc(sizeof(double) * (size_t)T * E);
    double* b = (double*)malloc(sizeof(double) * (size_t)T * E);
    if (!s || !b) {
        free(s);
        free(b);
        *fail = 2;
        return NULL;
    }
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) token_scores(d, E, x, Wg, dtype, (size_t)t, s + (size_t)t * E);
    if (oracle_balance_grad(T, E, k, s, alpha, b)) *fail = 1;
    free(s);
    return b;
}

/*
 * Every gradient of L = sum_t <dout_t, out_t> (+ alpha L_balance) (step 8), tokens in order.
 * dx [T][d], dlogits [T][E] (the router-score gradient ds), dWg [E][d],
 * dW1/dW3 [E][F][d], dW2 [E][d][F]; idx/g [T][k], margin/mingap [T] as in
 * oracle_route.  Slow by design: for small shapes.
 */
int oracle_backward(int T, int d, int F, int E, int k, const void* x, const void* Wg, const void* W1, const void* W3,
                    const void* W2, int dtype, const void* dout, double alpha, double* dx, double* dlogits,
                    double* dWg, double* dW1, double* dW3, double* dW2, int32_t* idx, double* g, double* margin,
                    double* mingap) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
    int bfail = 0;
    double* bal = balance_part(T, d, E, k, x, Wg, dtype, alpha, &bfail);
    if (bfail) return bfail;
    struct bwd_scratch w;
    if (!scratch_alloc(&w, d, F, k)) {
        scratch_free(&w);
        free(bal);
        return 2;
    }
    memset(dWg, 0, sizeof(double) * (size_t)E * d);
    memset(dW1, 0, sizeof(double) * (size_t)E * F * d);
    memset(dW3, 0, sizeof(double) * (size_t)E * F * d);
    memset(dW2, 0, sizeof(double) * (size_t)E * d * F);
    for (int t = 0; t < T; ++t)
        token_backward(d, F, E, k, x, dtype, Wg, W1, W3, W2, dtype, dout, (size_t)t, &w, dx + (size_t)t * d,
                       dlogits + (size_t)t * E, idx + (size_t)t * k, g + (size_t)t * k, margin + t, mingap + t, dWg,
                       dW1, dW3, dW2, bal ? bal + (size_t)t * E : NULL);
    scratch_free(&w);
    free(bal);
    return 0;
}

/* dx and ds of the listed tokens only (no weight gradients); rows in list order */
int oracle_backward_tokens(int T, int d, int F, int E, int k, const void* x, const void* Wg, const void* W1,
                           const void* W3, const void* W2, int dtype, const void* dout, double alpha,
                           const int32_t* tokens, int n, double* dx, double* dlogits, int32_t* idx, double* g,
                           double* margin, double* mingap, int nthreads) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E || n < 0) return 1;
    for (int r = 0; r < n; ++r)
        if (tokens[r] < 0 || tokens[r] >= T) return 1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    int bfail = 0;
    double* bal = balance_part(T, d, E, k, x, Wg, dtype, alpha, &bfail);
    if (bfail) return bfail;
#pragma omp parallel
    {
        struct bwd_scratch w;
        if (!scratch_alloc(&w, d, F, k)) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r)
                token_backward(d, F, E, k, x, dtype, Wg, W1, W3, W2, dtype, dout, (size_t)tokens[r], &w,
                               dx + (size_t)r * d, dlogits + (size_t)r * E, idx + (size_t)r * k, g + (size_t)r * k,
                               margin + r, mingap + r, NULL, NULL, NULL, NULL,
                               bal ? bal + (size_t)tokens[r] * E : NULL);
        }
        scratch_free(&w);
    }
    free(bal);
    return fail ? 2 : 0;
}

/*
 * dx and ds (step 8, output path only: alpha = 0) of n given input rows held in
 * double, x_rows [n][d], with the operands Wg, W1, W3, W2 and the upstream
 * gradient rows dout_rows [n][d] stored as dtype.  The block form's backward
 * needs this: the MoE layer's input there is the exact normalised row u, which
 * no stored dtype holds, while its weights stay in theirs.  Rows are
 * independent (without the load-balance part nothing couples them).
 */
int oracle_backward_rows(int n, int d, int F, int E, int k, const double* x_rows, const void* Wg, const void* W1,
                         const void* W3, const void* W2, int dtype, const void* dout_rows, double* dx,
                         double* dlogits, int32_t* idx, double* g, double* margin, double* mingap, int nthreads) {
    if (n < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E) return 1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        struct bwd_scratch w;
        if (!scratch_alloc(&w, d, F, k)) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r)
                token_backward(d, F, E, k, x_rows, 2, Wg, W1, W3, W2, dtype, dout_rows, (size_t)r, &w,
                               dx + (size_t)r * d, dlogits + (size_t)r * E, idx + (size_t)r * k, g + (size_t)r * k,
                               margin + r, mingap + r, NULL, NULL, NULL, NULL, NULL);
        }
        scratch_free(&w);
    }
    return fail ? 2 : 0;
}

/*
 * Selected slices of expert e's weight gradients over all tokens (step 8):
 * rows f of dW1_e and dW3_e ([nf][d] each) and columns f of dW2_e ([d][nf]),
 * for f in fs[0..nf).  Each needs only row f of W1_e/W3_e and column f of
 * W2_e per routed token, so full-size batches stay cheap.
 */
int oracle_weight_grad_slices(int T, int d, int F, int E, int k, const void* x, const void* Wg, const void* W1,
                              const void* W3, const void* W2, int dtype, const void* dout, int e, const int32_t* fs,
                              int nf, double* dW1_rows, double* dW3_rows, double* dW2_cols, int nthreads) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || E > 64 || k <= 0 || k > E || e < 0 || e >= E || nf < 0) return 1;
    for (int r = 0; r < nf; ++r)
        if (fs[r] < 0 || fs[r] >= F) return 1;
    /* routing of every token: slot of e and its gate (0 when e is not selected) */
    double* ge = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!ge) return 2;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        double s[64], g[64];
        int32_t idx[64];
        token_scores(d, E, x, Wg, dtype, (size_t)t, s);
        token_select(E, k, s, idx, g, NULL, NULL);
        ge[t] = 0.0;
        for (int j = 0; j < k; ++j)
            if (idx[j] == e) ge[t] = g[j];
    }
    const size_t w13 = (size_t)e * F * d, w2 = (size_t)e * d * F;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nf; ++r) {
        const int f = fs[r];
        double* r1 = dW1_rows + (size_t)r * d;
        double* r3 = dW3_rows + (size_t)r * d;
        for (int i = 0; i < d; ++i) {
            r1[i] = r3[i] = 0.0;
            dW2_cols[(size_t)i * nf + r] = 0.0;
        }
        for (int t = 0; t < T; ++t) {
            if (ge[t] == 0.0) continue;
            double a = 0.0, b = 0.0, dh = 0.0;
            for (int j = 0; j < d; ++j) {
                const double xj = elem(x, dtype, (size_t)t * d + j);
                a += elem(W1, dtype, w13 + (size_t)f * d + j) * xj;
                b += elem(W3, dtype, w13 + (size_t)f * d + j) * xj;
            }
            const double sg = sigmoid(a);
            const double h = a * sg * b;
            for (int i = 0; i < d; ++i) dh += elem(W2, dtype, w2 + (size_t)i * F + f) * ge[t] * elem(dout, dtype, (size_t)t * d + i);
            const double da = dh * b * sg * (1.0 + a * (1.0 - sg));
            const double db = dh * a * sg;
            for (int i = 0; i < d; ++i) {
                const double xi = elem(x, dtype, (size_t)t * d + i);
                r1[i] += da * xi;
                r3[i] += db * xi;
                dW2_cols[(size_t)i * nf + r] += ge[t] * elem(dout, dtype, (size_t)t * d + i) * h;
            }
        }
    }
    free(ge);
    return 0;
}

/* per-expert assignment counts: counts[e] = #{(t, j) : idx[t][j] == e} */
int oracle_counts(int T, int k, int E, const int32_t* idx, int64_t* counts) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (size_t a = 0; a < (size_t)T * k; ++a) {
        if (idx[a] < 0 || idx[a] >= E) return 1;
        counts[idx[a]] += 1;
    }
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
