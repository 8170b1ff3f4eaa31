/*
 * moe_oracle.c -- plain fp64 CPU oracle of the sigmoid-bias top-k MoE block.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use this file; the CUDA library never links,
 * loads or calls it, and the two share no code.
 *
 * What it computes follows "LFM2.5-24B-A2B: Biased Routing, Short Convolutions
 * and Ten KV Caches" (flozi.net, English page):
 *   - section "The exact checkpoint": a block applies RMS normalization before
 *     its feed-forward network and adds a residual;
 *   - section "The router has two different scores": X in R^{N x 2048}, a router
 *     matrix W_r in R^{64 x 2048} gives 64 logits per token, sigmoid is applied
 *     to each logit independently, a stored 64-element bias takes part in the
 *     top-4 selection but not in the mixture weights; the weights are
 *     normalised with an epsilon (they sum to slightly less than one) and the
 *     routed scaling factor is 1; each selected expert is a gated SiLU MLP of
 *     three matrices, whose two input matrices may be packed together; the
 *     worked example: the bias is added after the activation, and a displaced
 *     expert contributes with its unbiased score;
 *   - section "What to verify in a deployment": tokens are grouped by expert and
 *     the weighted outputs accumulated.
 * Every value is read from its stored type (f32 or bf16) and widened to double
 * exactly; all arithmetic is double with no intermediate rounding.
 *
 * Readings taken where the page is silent (its display equations were lost):
 * RMSNorm is x / sqrt(mean(x^2) + eps) * g with the gain multiplied as stored,
 * and the same eps serves the RMSNorm and the weight normalisation; the
 * weights are scale * s_i / (sum of the k selected s + eps); top-k ties go to
 * the lower expert index and slots are ordered by biased score, descending;
 * the gated MLP is down( silu(gate x) * (up x) ) with gate rows first in the
 * packed matrix; the combine sums slots in slot order and adds the residual.
 *
 * Planted mistakes (the `mutation` argument) exist only so that the tests can
 * show that each plausible error would be caught by a pin; 0 = the method.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

enum {
    MUT_NONE = 0,
    MUT_BIASED_WEIGHTS = 1,   /* mixture weights from s + b instead of s       */
    MUT_SOFTMAX = 2,          /* softmax over logits instead of sigmoid        */
    MUT_BIAS_BEFORE_ACT = 3,  /* sigmoid(l + b) used for selection             */
    MUT_NO_EPS = 4,           /* weights normalised by the plain sum           */
    MUT_NO_GAIN = 5,          /* RMSNorm without its gain                      */
    MUT_SILU_ON_UP = 6,       /* SiLU applied to the up half, not the gate     */
    MUT_TIE_HIGH = 7,         /* ties go to the higher index                   */
    MUT_NO_RESIDUAL = 8,      /* output without the residual                   */
    MUT_MEAN_NOT_SUM = 9,     /* RMS uses sum of squares without the 1/d       */
    MUT_SLOT_SWAP = 10,       /* slots ordered ascending instead of descending */
    MUT_DOWN_TRANSPOSED = 11, /* down matrix read as [I][d]                    */
    MUT_COUNT = 12
};

static double ld(const void *p, int dtype, size_t i)
{
    if (dtype == OR_F32) return (double)((const float *)p)[i];
    if (dtype == OR_BF16) {
        uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return ((const double *)p)[i];
}

/* Pre-FFN RMSNorm of one row. */
static void rmsnorm_row(int d, double eps, const void *x, int xdt, size_t row,
                        const float *gain, double *xn, int mutation)
{
    double ss = 0.0;
    for (int j = 0; j < d; ++j) {
        double v = ld(x, xdt, row * (size_t)d + j);
        ss += v * v;
    }
    double ms = (mutation == MUT_MEAN_NOT_SUM) ? ss : ss / (double)d;
    double r = sqrt(ms + eps);
    for (int j = 0; j < d; ++j) {
        double g = (mutation == MUT_NO_GAIN) ? 1.0 : (double)gain[j];
        xn[j] = ld(x, xdt, row * (size_t)d + j) / r * g;
    }
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Router, activation, biased selection and weights for one token.
 * xn[d] in; s[E], c[E] scratch/out; sel[k], w[k] out; returns the margin
 * c_(k) - c_(k+1) between the last selected and the best unselected biased
 * score (INFINITY when k == E). When forced != NULL, the selection (and slot
 * order) is taken from it instead of being chosen. */
static double route_one(int d, int E, int k, double eps, double scale,
                        const double *xn, const float *router_w, const float *bias,
                        double *s, double *c, int32_t *sel, double *w,
                        const int32_t *forced, int mutation)
{
    double lmax = -INFINITY;
    for (int e = 0; e < E; ++e) {
        double l = 0.0;
        for (int j = 0; j < d; ++j) l += (double)router_w[(size_t)e * d + j] * xn[j];
        c[e] = l;                       /* c holds the logits until the bias step */
        if (l > lmax) lmax = l;
    }
    if (mutation == MUT_SOFTMAX) {
        double z = 0.0;
        for (int e = 0; e < E; ++e) z += exp(c[e] - lmax);
        for (int e = 0; e < E; ++e) s[e] = exp(c[e] - lmax) / z;
    } else {
        for (int e = 0; e < E; ++e) s[e] = sigmoid(c[e]);
    }
    for (int e = 0; e < E; ++e) {
        if (mutation == MUT_BIAS_BEFORE_ACT)
            c[e] = sigmoid(c[e] + (double)bias[e]);
        else
            c[e] = s[e] + (double)bias[e];
    }

    double margin = INFINITY;
    if (forced) {
        for (int j = 0; j < k; ++j) sel[j] = forced[j];
    } else {
        unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || c[e] > c[best] ||
                    (mutation == MUT_TIE_HIGH && c[e] == c[best]))
                    best = e;
            }
            taken[best] = 1;
            sel[j] = best;
        }
        if (k < E) {
            int nxt = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (nxt < 0 || c[e] > c[nxt])) nxt = e;
            margin = c[sel[k - 1]] - c[nxt];
        }
        free(taken);
        if (mutation == MUT_SLOT_SWAP)
            for (int j = 0; j < k / 2; ++j) {
                int32_t t = sel[j]; sel[j] = sel[k - 1 - j]; sel[k - 1 - j] = t;
            }
    }

    double sum = 0.0;
    for (int j = 0; j < k; ++j)
        sum += (mutation == MUT_BIASED_WEIGHTS) ? c[sel[j]] : s[sel[j]];
    double den = (mutation == MUT_NO_EPS) ? sum : sum + eps;
    for (int j = 0; j < k; ++j) {
        double num = (mutation == MUT_BIASED_WEIGHTS) ? c[sel[j]] : s[sel[j]];
        w[j] = scale * (num / den);
    }
    return margin;
}

int oracle_num_mutations(void) { return MUT_COUNT; }

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* RMSNorm of N rows: xn[N][d]. */
int oracle_rmsnorm(int N, int d, double eps, const void *x, int xdt,
                   const float *gain, double *xn, int mutation)
{
    if (N < 0 || d <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < N; ++t)
        rmsnorm_row(d, eps, x, xdt, (size_t)t, gain, xn + (size_t)t * d, mutation);
    return 0;
}

/* Routing of N tokens. Outputs: idx[N][k] expert indices in slot order,
 * w[N][k] mixture weights, s[N][E] unbiased scores (may be NULL),
 * margin[N] (may be NULL). */
int oracle_route(int N, int d, int E, int k, double eps, double scale,
                 const void *x, int xdt, const float *gain, const float *router_w,
                 const float *bias, int32_t *idx, double *w, double *s_out,
                 double *margin, int mutation)
{
    if (N < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return -1;
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)E);
        double *c = (double *)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(dynamic, 4)
        for (int t = 0; t < N; ++t) {
            rmsnorm_row(d, eps, x, xdt, (size_t)t, gain, xn, mutation);
            double m = route_one(d, E, k, eps, scale, xn, router_w, bias, s, c,
                                 idx + (size_t)t * k, w + (size_t)t * k, NULL, mutation);
            if (margin) margin[t] = m;
            if (s_out) memcpy(s_out + (size_t)t * E, s, sizeof(double) * (size_t)E);
        }
        free(xn); free(s); free(c);
    }
    return 0;
}

/* Full block output for a subset of tokens: out[n][d] (double) for the rows
 * tokens[0..n-1] of x. forced (may be NULL) gives each listed token's
 * selection [n][k] in slot order, used in place of the oracle's own choice;
 * idx_out/w_out (may be NULL) receive the selection and weights used. */
int oracle_forward(int n, const int64_t *tokens, int N, int d, int E, int k, int I,
                   double eps, double scale, const void *x, int xdt,
                   const float *gain, const float *router_w, const float *bias,
                   const void *w_gate_up, const void *w_down, int wdt,
                   const int32_t *forced, double *out, int32_t *idx_out,
                   double *w_out, int mutation)
{
    if (n < 0 || N < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || I <= 0) return -1;
    for (int i = 0; i < n; ++i)
        if (tokens[i] < 0 || tokens[i] >= N) return -2;
    int bad = 0;
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)E);
        double *c = (double *)malloc(sizeof(double) * (size_t)E);
        double *gt = (double *)malloc(sizeof(double) * (size_t)I);
        double *up = (double *)malloc(sizeof(double) * (size_t)I);
        double *a = (double *)malloc(sizeof(double) * (size_t)I);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n; ++i) {
            size_t t = (size_t)tokens[i];
            double *o = out + (size_t)i * d;
            rmsnorm_row(d, eps, x, xdt, t, gain, xn, mutation);
            route_one(d, E, k, eps, scale, xn, router_w, bias, s, c, sel, w,
                      forced ? forced + (size_t)i * k : NULL, mutation);
            int ok = 1;
            for (int j = 0; j < k; ++j) if (sel[j] < 0 || sel[j] >= E) ok = 0;
            if (!ok) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            if (idx_out) memcpy(idx_out + (size_t)i * k, sel, sizeof(int32_t) * (size_t)k);
            if (w_out) memcpy(w_out + (size_t)i * k, w, sizeof(double) * (size_t)k);
            for (int j = 0; j < d; ++j)
                o[j] = (mutation == MUT_NO_RESIDUAL) ? 0.0 : ld(x, xdt, t * (size_t)d + j);
            for (int slot = 0; slot < k; ++slot) {
                size_t e = (size_t)sel[slot];
                size_t gbase = e * (size_t)(2 * I) * (size_t)d;
                for (int f = 0; f < I; ++f) {
                    double g = 0.0, u = 0.0;
                    size_t rg = gbase + (size_t)f * d, ru = gbase + (size_t)(I + f) * d;
                    for (int j = 0; j < d; ++j) {
                        g += ld(w_gate_up, wdt, rg + j) * xn[j];
                        u += ld(w_gate_up, wdt, ru + j) * xn[j];
                    }
                    gt[f] = g;
                    up[f] = u;
                }
                for (int f = 0; f < I; ++f)
                    a[f] = (mutation == MUT_SILU_ON_UP) ? up[f] * sigmoid(up[f]) * gt[f]
                                                         : gt[f] * sigmoid(gt[f]) * up[f];
                size_t dbase = e * (size_t)d * (size_t)I;
                for (int j = 0; j < d; ++j) {
                    double y = 0.0;
                    for (int f = 0; f < I; ++f) {
                        size_t off = (mutation == MUT_DOWN_TRANSPOSED)
                                         ? dbase + (size_t)f * d + j
                                         : dbase + (size_t)j * I + f;
                        y += ld(w_down, wdt, off) * a[f];
                    }
                    o[j] += w[slot] * y;
                }
            }
        }
        free(xn); free(s); free(c); free(gt); free(up); free(a); free(sel); free(w);
    }
    return bad ? -3 : 0;
}

/* Grouping of the N*k assignments by expert: counts[E], offsets[E+1]
 * (exclusive prefix sum), perm[N*k] listing assignment ids t*k+j expert by
 * expert, ascending token index within an expert. */
int oracle_dispatch(int N, int E, int k, const int32_t *idx, int32_t *counts,
                    int32_t *offsets, int32_t *perm)
{
    if (N < 0 || E <= 0 || k <= 0) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (size_t a = 0; a < (size_t)N * k; ++a) {
        if (idx[a] < 0 || idx[a] >= E) return -2;
        counts[idx[a]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    size_t pos = 0;
    for (int e = 0; e < E; ++e)
        for (int t = 0; t < N; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e) perm[pos++] = t * k + j;
    return 0;
}
