/*
 * Plain fp64 CPU oracle for the GLM-4.5 / GLM-5 sparse MoE feed-forward forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA path and never calls it.
 *
 * Every stored input (fp32 or bf16) is widened exactly to double on read; all
 * arithmetic is fp64; there is no blocking, fusion or reordering beyond the
 * definitions cited below.  Sources (page title, section, equation):
 *
 *   [GR]  "GLM-4.5 Group Router", section "How it works": the gate is a bias-free
 *         float32 linear map followed by a sigmoid; the correction bias b is added
 *         only for selection (s' = s + b); experts fall into G contiguous groups of
 *         E/G; a group's score is the sum of its two largest s'; the topk_group
 *         best groups are kept; T = top-k of s' inside the kept groups; weights use
 *         the raw s, renormalised over T with eps = 1e-20 when norm_topk_prob, then
 *         scaled by alpha (routed_scaling_factor).  G = 1 reduces to plain top-k.
 *   [MF]  "GLM-4.5 MoE Forward", section "How it works": each routed expert is a
 *         bias-free SwiGLU E_i(x) = W_down,i (SiLU(W_gate,i x) (.) W_up,i x) with
 *         gate and up packed as gate_up_proj[i] of shape (2 d_moe, D), gate rows
 *         first; y_n = sum_{i in T(n)} w_{n,i} E_i(x_n) + E_sh(x_n), the shared
 *         expert at scale 1.
 *   [G5]  "GLM-5 Mixture of experts", code excerpt of the experts' forward: an
 *         index equal to E (the number of routed experts) is a sentinel that is
 *         skipped; down_proj[i] has shape (D, d_moe).
 *   [SH]  "GLM-5 Shared output", MLP excerpt: the shared expert is
 *         down(silu(gate x) * up x) with gate/up of shape (d_sh, D) and down (D, d_sh),
 *         applied to the same input as the routed experts.
 *   [CL]  "GLM-5.3-Flash Module 02", section 3: the clamped SwiGLU variant of
 *         another model, a = min(W_g x, 10) (gate clamped above only),
 *         u = clip(W_u x, -10, 10), f = W_d (SiLU(a) (.) u), for every expert,
 *         routed or shared.  Here the limits are parameters (gate_max, up_max);
 *         +infinity gives the plain SwiGLU of [MF].
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes): discarded groups are masked to -infinity (the zero-fill
 * alternative is evaluated too and reported); ties go to the lower index for
 * both groups and experts; topk_idx is ordered by descending s', then ascending
 * index.
 *
 * Parity pins for every function here live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1 };

/* Exact widening of one stored element to double. */
static double widen(const void *base, int dt, size_t i)
{
    if (dt == OR_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static void widen_row(const void *base, int dt, size_t offset, int len, double *out)
{
    for (int i = 0; i < len; ++i)
        out[i] = widen(base, dt, offset + (size_t)i);
}

static double dot(const double *a, const double *b, int len)
{
    double acc = 0.0;
    for (int i = 0; i < len; ++i)
        acc += a[i] * b[i];
    return acc;
}

/* Logistic sigmoid, [GR] s = sigma(r). */
static double sigmoid(double r) { return 1.0 / (1.0 + exp(-r)); }

/* SiLU(a) = a * sigma(a), [MF] expert definition. */
static double silu(double a) { return a * sigmoid(a); }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Router logits r[n,e] = sum_d x[n,d] W_g[e,d]   ([GR] "s = sigma(x W_g^T)").
 * x: [N,D] (x_dt), W_g: [E,D] (wg_dt), r: [N,E] double.
 */
void oracle_router_logits(const void *x, int x_dt, const void *wg, int wg_dt,
                          int N, int D, int E, double *r)
{
#pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * (size_t)D);
        double *wr = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
        for (int n = 0; n < N; ++n) {
            widen_row(x, x_dt, (size_t)n * D, D, xr);
            for (int e = 0; e < E; ++e) {
                widen_row(wg, wg_dt, (size_t)e * D, D, wr);
                r[(size_t)n * E + e] = dot(xr, wr, D);
            }
        }
        free(xr);
        free(wr);
    }
}

/* Index of the largest value among v[i] with allowed[i] != 0; lower index wins ties.
 * Returns -1 when nothing is allowed. */
static int argmax_allowed(const double *v, const unsigned char *allowed, int len)
{
    int best = -1;
    for (int i = 0; i < len; ++i) {
        if (!allowed[i])
            continue;
        if (best < 0 || v[i] > v[best])
            best = i;
    }
    return best;
}

/*
 * Selection and weighting from logits, one token at a time ([GR] steps after the
 * linear map).  Inputs: r [N,E] double logits, b [E] float correction bias.
 * Outputs:
 *   idx   [N,k] int32  selected experts, descending s' then ascending index
 *   w     [N,k] double mixture weights (alpha included)
 *   s_out [N,E] double raw sigmoid scores (may be NULL)
 *   margin_exp [N] double  s'_(k) - s'_(k+1) among candidates (+inf if none left)
 *   margin_grp [N] double  g_(tg) - g_(tg+1) (+inf when G == 1 or tg == G)
 *   zero_fill_differs [N] int  1 if masking discarded groups with 0 instead of
 *                              -inf would select a different set
 * Returns 0, or -1 on an invalid configuration.
 */
int oracle_select(const double *r, const float *b, int N, int E, int G, int tg, int k,
                  int norm, double alpha, int32_t *idx, double *w, double *s_out,
                  double *margin_exp, double *margin_grp, int32_t *zero_fill_differs)
{
    if (N < 0 || E <= 0 || G <= 0 || E % G != 0 || tg <= 0 || tg > G || k <= 0 || k > E)
        return -1;
    const int m = E / G;
    if (G > 1 && m < 2)
        return -1;
    if (tg * m < k)
        return -1;

    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)E);
        double *sp = (double *)malloc(sizeof(double) * (size_t)E);
        double *zf = (double *)malloc(sizeof(double) * (size_t)E);
        double *gs = (double *)malloc(sizeof(double) * (size_t)G);
        unsigned char *kept = (unsigned char *)malloc((size_t)G);
        unsigned char *cand = (unsigned char *)malloc((size_t)E);
        unsigned char *left = (unsigned char *)malloc((size_t)E);
        unsigned char *all = (unsigned char *)malloc((size_t)E);
        int32_t *chosen = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            const double *rn = r + (size_t)n * E;
            /* s = sigma(r); s' = s + b (bias used for selection only). */
            for (int e = 0; e < E; ++e) {
                s[e] = sigmoid(rn[e]);
                sp[e] = s[e] + (double)b[e];
            }
            /* Group scores: sum of the two largest s' of each contiguous group. */
            memset(kept, 0, (size_t)G);
            double mgrp = INFINITY;
            if (G > 1) {
                for (int g = 0; g < G; ++g) {
                    int i1 = -1, i2 = -1;
                    for (int j = g * m; j < (g + 1) * m; ++j) {
                        if (i1 < 0 || sp[j] > sp[i1]) {
                            i2 = i1;
                            i1 = j;
                        } else if (i2 < 0 || sp[j] > sp[i2]) {
                            i2 = j;
                        }
                    }
                    gs[g] = sp[i1] + sp[i2];
                }
                /* Keep the tg groups with the largest score. */
                unsigned char *gleft = (unsigned char *)malloc((size_t)G);
                memset(gleft, 1, (size_t)G);
                double last = 0.0;
                for (int t = 0; t < tg; ++t) {
                    int g = argmax_allowed(gs, gleft, G);
                    kept[g] = 1;
                    gleft[g] = 0;
                    last = gs[g];
                }
                int nxt = argmax_allowed(gs, gleft, G);
                if (nxt >= 0)
                    mgrp = last - gs[nxt];
                free(gleft);
            } else {
                kept[0] = 1;
            }
            /* Candidates: experts of kept groups (discarded groups are -inf). */
            for (int e = 0; e < E; ++e) {
                cand[e] = kept[e / m];
                left[e] = cand[e];
            }
            double last = 0.0;
            for (int t = 0; t < k; ++t) {
                int e = argmax_allowed(sp, left, E);
                chosen[t] = e;
                left[e] = 0;
                last = sp[e];
            }
            int nxt = argmax_allowed(sp, left, E);
            double mexp = (nxt >= 0) ? last - sp[nxt] : INFINITY;

            /* Weights from the raw scores of the chosen set. */
            double sum = 0.0;
            for (int t = 0; t < k; ++t)
                sum += s[chosen[t]];
            for (int t = 0; t < k; ++t) {
                double sv = s[chosen[t]];
                w[(size_t)n * k + t] = norm ? alpha * sv / (sum + 1e-20) : alpha * sv;
                idx[(size_t)n * k + t] = chosen[t];
            }
            if (s_out)
                memcpy(s_out + (size_t)n * E, s, sizeof(double) * (size_t)E);
            if (margin_exp)
                margin_exp[n] = mexp;
            if (margin_grp)
                margin_grp[n] = mgrp;

            /* Alternative reading: discarded groups filled with 0 instead of -inf. */
            if (zero_fill_differs) {
                for (int e = 0; e < E; ++e) {
                    zf[e] = cand[e] ? sp[e] : 0.0;
                    all[e] = 1;
                }
                int differs = 0;
                for (int t = 0; t < k; ++t) {
                    int e = argmax_allowed(zf, all, E);
                    all[e] = 0;
                    if (!cand[e])
                        differs = 1;
                }
                zero_fill_differs[n] = differs;
            }
        }
        free(s);
        free(sp);
        free(zf);
        free(gs);
        free(kept);
        free(cand);
        free(left);
        free(all);
        free(chosen);
    }
    return bad;
}

/*
 * Full router: logits then selection.  r_out [N,E] may be NULL (scratch is
 * allocated here then).
 */
int oracle_router(const void *x, int x_dt, const void *wg, int wg_dt, const float *b,
                  int N, int D, int E, int G, int tg, int k, int norm, double alpha,
                  int32_t *idx, double *w, double *r_out, double *s_out,
                  double *margin_exp, double *margin_grp, int32_t *zero_fill_differs)
{
    double *r = r_out ? r_out : (double *)malloc(sizeof(double) * (size_t)N * (size_t)E);
    if (!r)
        return -2;
    oracle_router_logits(x, x_dt, wg, wg_dt, N, D, E, r);
    int rc = oracle_select(r, b, N, E, G, tg, k, norm, alpha, idx, w, s_out, margin_exp,
                           margin_grp, zero_fill_differs);
    if (!r_out)
        free(r);
    return rc;
}

/*
 * One SwiGLU expert applied to one token ([MF] E_i(x), [SH] for the shared one):
 *   a_r = W_gate[r,:] . x,  u_r = W_up[r,:] . x,  h_r = SiLU(a_r) u_r,
 *   o_c = W_down[c,:] . h.
 * gate_base/up_base: element offsets of the first gate / up row in w_gu (row-major,
 * row length D); down_base: offset of row 0 of W_down (row length dd).
 * Result is ADDED, scaled by `scale`, into y[D].
 */
static void swiglu_accumulate(const void *w_gu, size_t gate_base, const void *w_up,
                              size_t up_base, const void *w_down, size_t down_base, int dt,
                              int D, int dd, const double *xn, double scale, double *y,
                              double *row, double *h, double gate_max, double up_max)
{
    for (int r = 0; r < dd; ++r) {
        widen_row(w_gu, dt, gate_base + (size_t)r * D, D, row);
        double a = dot(row, xn, D);
        widen_row(w_up, dt, up_base + (size_t)r * D, D, row);
        double u = dot(row, xn, D);
        /* [CL]: the gate is clamped from above only, the up projection both sides */
        if (a > gate_max)
            a = gate_max;
        if (u > up_max)
            u = up_max;
        if (u < -up_max)
            u = -up_max;
        h[r] = silu(a) * u;
    }
    for (int c = 0; c < D; ++c) {
        widen_row(w_down, dt, down_base + (size_t)c * dd, dd, row);
        y[c] += scale * dot(row, h, dd);
    }
}

/*
 * MoE forward for a list of tokens ([MF] y_n formula, token-major):
 *   y_n = sum_{j<k, idx[n,j] != E} w[n,j] * E_idx(x_n)  +  E_sh(x_n)
 * x [N,D]; gate_up [E,2d,D] (gate rows 0..d-1, up rows d..2d-1); down [E,D,d];
 * sh_gate/sh_up [d_sh,D]; sh_down [D,d_sh]; all in dtype dt.  idx [N,k] int32,
 * w [N,k] double.  tokens[0..n_tokens) lists which rows to evaluate;
 * y [n_tokens, D] double receives them in list order.
 * Indices outside [0, E] are rejected (-1); the sentinel E contributes nothing.
 * gate_max / up_max: the [CL] limits (+infinity for the plain SwiGLU).
 */
int oracle_forward(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                   const void *sh_up, const void *sh_down, int dt, const int32_t *idx,
                   const double *w, int N, int D, int E, int d, int d_sh, int k,
                   const int32_t *tokens, int n_tokens, double gate_max, double up_max,
                   double *y)
{
    for (int t = 0; t < n_tokens; ++t)
        if (tokens[t] < 0 || tokens[t] >= N)
            return -1;
    for (int t = 0; t < n_tokens; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t i = idx[(size_t)tokens[t] * k + j];
            if (i < 0 || i > E)
                return -1;
        }
    const int dmax = d > d_sh ? d : d_sh;
    const int rowlen = D > dmax ? D : dmax;
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * (size_t)D);
        double *row = (double *)malloc(sizeof(double) * (size_t)rowlen);
        double *h = (double *)malloc(sizeof(double) * (size_t)dmax);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < n_tokens; ++t) {
            const int n = tokens[t];
            double *yn = y + (size_t)t * D;
            for (int c = 0; c < D; ++c)
                yn[c] = 0.0;
            widen_row(x, dt, (size_t)n * D, D, xn);
            for (int j = 0; j < k; ++j) {
                const int i = idx[(size_t)n * k + j];
                if (i == E)
                    continue; /* sentinel: no expert */
                const size_t gu = (size_t)i * 2 * (size_t)d * D;
                swiglu_accumulate(gate_up, gu, gate_up, gu + (size_t)d * D, down,
                                  (size_t)i * D * (size_t)d, dt, D, d, xn,
                                  w[(size_t)n * k + j], yn, row, h, gate_max, up_max);
            }
            /* Always-on shared expert, scale 1. */
            swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 1.0, yn, row,
                              h, gate_max, up_max);
        }
        free(xn);
        free(row);
        free(h);
    }
    return 0;
}
