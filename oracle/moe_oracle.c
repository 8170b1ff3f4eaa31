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
 * FP8_BLOCK experts, from "LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell"
 * (inferencekey.com, section "Für Engineers", paragraph "Quantisierung"):
 * expert weights are stored as FP8 statically in 128x128
 * blocks, activations are quantised to FP8 dynamically per group of 128; the
 * router stays unquantised. Readings taken: the FP8 format is e4m3 with no
 * infinities (largest finite 448), decoded from its definition; a weight is
 * its code's value times the fp32 scale of its 128x128 block ([row/128]
 * [col/128] of each matrix); both expert inputs (the normalised row before
 * gate/up, SiLU(gate)*up before down) are quantised per token in groups of
 * 128 consecutive columns with s = amax/448 and code = e4m3(v/s) rounded to
 * nearest even (saturating at 448), an all-zero group giving s = 0 and zero
 * codes. That code decision is taken in fp32 like the kernel's: v is rounded
 * to float first and amax, s and v/s are float operations. Everything else
 * stays exact double arithmetic on the decoded values.
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

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2, OR_E4M3 = 3 };

/* FP8_BLOCK: weight blocks of FP8_B x FP8_B, activation groups of FP8_B. */
enum { FP8_B = 128 };

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
    MUT_FP8_SCALE_T = 12,     /* weight block scales read as [col/128][row/128] */
    MUT_FP8_NO_ACT_QUANT = 13,/* SiLU(gate)*up not quantised before down       */
    MUT_FP8_NO_MAX = 14,      /* activation scale amax instead of amax/448     */
    MUT_MARGIN_ZERO = 15,     /* margin reported as 0 for every token          */
    MUT_MARGIN_WORST = 16,    /* margin against the WORST unselected expert    */
    MUT_MARGIN_ON_S = 17,     /* margin on the unbiased s instead of c = s + b */
    MUT_FORCED_IGNORED = 18,  /* a forced selection is ignored                 */
    MUT_FORCED_WEIGHTS_OWN = 19, /* forced experts, but weights of the oracle's own choice */
    MUT_CONV_LAG_REVERSED = 20, /* conv tap l applied at lag 2 - l               */
    MUT_CONV_CENTERED = 21,   /* conv window t-1 .. t+1 instead of t-2 .. t      */
    MUT_CONV_GATE_AFTER = 22, /* g multiplied after the convolution, not before  */
    MUT_CONV_SEQ_LEAK = 23,   /* history carried across sequences of the batch   */
    MUT_CONV_UV_SWAPPED = 24, /* streams u and v taken in the other order        */
    MUT_COUNT = 25
};

/* Value of an e4m3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent 0 is subnormal; S.1111.111 is NaN; no infinities). */
static double e4m3_value(uint8_t c)
{
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (c & 0x80) ? -v : v;
}

/* e4m3 code of a float, rounded to nearest with ties to even, saturating to
 * +-448. The spacing of e4m3 values is 2^-9 below 2^-6 and 2^(E-3) in the
 * binade [2^E, 2^(E+1)); a / spacing is exact (a power-of-two division) and
 * rint() rounds it to the nearest integer, ties to even. */
static uint8_t e4m3_encode(float f)
{
    uint8_t sign = signbit(f) ? 0x80 : 0;
    double a = fabs((double)f);
    if (a != a) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    double q;
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);              /* a in [2^(ex-1), 2^ex) */
        q = ldexp(1.0, ex - 1 - 3);
    }
    double v = rint(a / q) * q;     /* the nearest e4m3 magnitude */
    if (v >= 448.0) return sign | 0x7E;
    if (v < ldexp(1.0, -6)) return sign | (uint8_t)(v / ldexp(1.0, -9));
    int ex;
    double fr = frexp(v, &ex);      /* v = fr * 2^ex, fr in [0.5, 1) */
    int mant = (int)(fr * 16.0) - 8;  /* (8 + mant) / 16 = fr */
    return sign | (uint8_t)(((ex - 1 + 7) << 3) | mant);
}

/* Dynamic FP8 quantisation of n values in groups of FP8_B (the last group
 * may be shorter): codes, per-group scales and the dequantised values
 * (code value * scale, exact in double) replacing v. codes/scales may be
 * NULL. */
static void quant_groups(int n, double *v, uint8_t *codes, float *scales, int mutation)
{
    for (int g0 = 0; g0 < n; g0 += FP8_B) {
        int g1 = g0 + FP8_B < n ? g0 + FP8_B : n;
        float amax = 0.0f;
        for (int j = g0; j < g1; ++j) {
            float a = fabsf((float)v[j]);
            if (a > amax) amax = a;
        }
        float sc = (mutation == MUT_FP8_NO_MAX) ? amax : amax / 448.0f;
        if (scales) scales[g0 / FP8_B] = sc;
        for (int j = g0; j < g1; ++j) {
            uint8_t c = (sc > 0.0f) ? e4m3_encode((float)v[j] / sc) : 0;
            if (codes) codes[j] = c;
            v[j] = e4m3_value(c) * (double)sc;
        }
    }
}

static inline __attribute__((always_inline)) double ld(const void *p, int dtype, size_t i)
{
    if (dtype == OR_F32) return (double)((const float *)p)[i];
    if (dtype == OR_BF16) {
        uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    if (dtype == OR_E4M3) return e4m3_value(((const uint8_t *)p)[i]);
    return ((const double *)p)[i];
}

/* Element (r, c) of a [rows][cols] expert matrix starting at element `base`
 * of w: the stored value, times its 128x128 block's scale when sc != NULL
 * (sc points at this matrix's [rows/128][cols/128] scales). */
static inline __attribute__((always_inline)) double wval(const void *w, int wdt, size_t base,
                                                          int cols, int rows, int r, int c,
                   const float *sc, int mutation)
{
    double v = ld(w, wdt, base + (size_t)r * cols + c);
    if (!sc) return v;
    int rb = r / FP8_B, cb = c / FP8_B;
    int nrb = (rows + FP8_B - 1) / FP8_B, ncb = (cols + FP8_B - 1) / FP8_B;
    size_t bi = (mutation == MUT_FP8_SCALE_T) ? (size_t)cb * nrb + rb : (size_t)rb * ncb + cb;
    return v * (double)sc[bi];
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

    /* The oracle's own choice: k rounds of arg-max over the biased scores,
     * then the margin between the last selected and the best unselected. */
    double margin = INFINITY;
    unsigned char *taken = (unsigned char *)calloc((size_t)(unsigned)E, 1);
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
        const double *key = (mutation == MUT_MARGIN_ON_S) ? s : c;
        int nxt = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (nxt < 0 || (mutation == MUT_MARGIN_WORST ? key[e] < key[nxt] : key[e] > key[nxt]))
                nxt = e;
        }
        margin = key[sel[k - 1]] - key[nxt];
        if (mutation == MUT_MARGIN_ZERO) margin = 0.0;
    }
    free(taken);
    if (mutation == MUT_SLOT_SWAP)
        for (int j = 0; j < k / 2; ++j) {
            int32_t t = sel[j]; sel[j] = sel[k - 1 - j]; sel[k - 1 - j] = t;
        }
    /* A forced selection (slot order as given) replaces the own choice; the
     * margin then does not apply. */
    const int use_forced = forced && mutation != MUT_FORCED_IGNORED;
    if (use_forced) {
        margin = INFINITY;
        if (mutation != MUT_FORCED_WEIGHTS_OWN)
            for (int j = 0; j < k; ++j) sel[j] = forced[j];
    }

    double sum = 0.0;
    for (int j = 0; j < k; ++j)
        sum += (mutation == MUT_BIASED_WEIGHTS) ? c[sel[j]] : s[sel[j]];
    double den = (mutation == MUT_NO_EPS) ? sum : sum + eps;
    for (int j = 0; j < k; ++j) {
        double num = (mutation == MUT_BIASED_WEIGHTS) ? c[sel[j]] : s[sel[j]];
        w[j] = scale * (num / den);
    }
    if (use_forced && mutation == MUT_FORCED_WEIGHTS_OWN)
        for (int j = 0; j < k; ++j) sel[j] = forced[j];
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

/* One gated SiLU expert e on the row xin[d] (read only): y[d] =
 * down( silu(gate xin) * (up xin) ). For e4m3 weights (FP8_BLOCK) the
 * weights carry their block scales (sgu, sdn: all experts' scales,
 * [E][2I/128][d/128] and [E][d/128][I/128]) and both inputs are quantised
 * per group of 128 first. Scratch: xq[d], gt/up/a[I]. */
static void expert_mlp(int d, int I, const double *xin, const void *w_gate_up,
                       const void *w_down, int wdt, const float *sgu, const float *sdn,
                       size_t e, double *xq, double *gt, double *up, double *a, double *y,
                       int mutation)
{
    const int fp8 = (wdt == OR_E4M3);
    const size_t ngu = (size_t)((2 * I + FP8_B - 1) / FP8_B) * ((d + FP8_B - 1) / FP8_B);
    const size_t ndn = (size_t)((d + FP8_B - 1) / FP8_B) * ((I + FP8_B - 1) / FP8_B);
    const float *sg = fp8 ? sgu + e * ngu : NULL;
    const float *sd = fp8 ? sdn + e * ndn : NULL;
    memcpy(xq, xin, sizeof(double) * (size_t)d);
    if (fp8) quant_groups(d, xq, NULL, NULL, mutation);
    size_t gbase = e * (size_t)(2 * I) * (size_t)d;
    for (int f = 0; f < I; ++f) {
        double g = 0.0, u = 0.0;
        for (int j = 0; j < d; ++j) {
            g += wval(w_gate_up, wdt, gbase, d, 2 * I, f, j, sg, mutation) * xq[j];
            u += wval(w_gate_up, wdt, gbase, d, 2 * I, I + f, j, sg, mutation) * xq[j];
        }
        gt[f] = g;
        up[f] = u;
    }
    for (int f = 0; f < I; ++f)
        a[f] = (mutation == MUT_SILU_ON_UP) ? up[f] * sigmoid(up[f]) * gt[f]
                                             : gt[f] * sigmoid(gt[f]) * up[f];
    if (fp8 && mutation != MUT_FP8_NO_ACT_QUANT) quant_groups(I, a, NULL, NULL, mutation);
    size_t dbase = e * (size_t)d * (size_t)I;
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int f = 0; f < I; ++f) {
            double wv = (mutation == MUT_DOWN_TRANSPOSED)
                            ? ld(w_down, wdt, dbase + (size_t)f * d + j)
                            : wval(w_down, wdt, dbase, I, d, j, f, sd, mutation);
            acc += wv * a[f];
        }
        y[j] = acc;
    }
}

/* Full block output for a subset of tokens: out[n][d] (double) for the rows
 * tokens[0..n-1] of x. forced (may be NULL) gives each listed token's
 * selection [n][k] in slot order, used in place of the oracle's own choice;
 * idx_out/w_out (may be NULL) receive the selection and weights used.
 * wdt == e4m3 selects the FP8_BLOCK experts with block scales sgu/sdn. */
int oracle_forward(int n, const int64_t *tokens, int N, int d, int E, int k, int I,
                   double eps, double scale, const void *x, int xdt,
                   const float *gain, const float *router_w, const float *bias,
                   const void *w_gate_up, const void *w_down, int wdt,
                   const float *sgu, const float *sdn,
                   const int32_t *forced, double *out, int32_t *idx_out,
                   double *w_out, int mutation)
{
    if (n < 0 || N < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || I <= 0) return -1;
    if (wdt == OR_E4M3 && (!sgu || !sdn)) return -1;
    for (int i = 0; i < n; ++i)
        if (tokens[i] < 0 || tokens[i] >= N) return -2;
    int bad = 0;
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * (size_t)d);
        double *xq = (double *)malloc(sizeof(double) * (size_t)d);
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
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
                expert_mlp(d, I, xn, w_gate_up, w_down, wdt, sgu, sdn, (size_t)sel[slot],
                           xq, gt, up, a, y, mutation);
                for (int j = 0; j < d; ++j) o[j] += w[slot] * y[j];
            }
        }
        free(xn); free(xq); free(y); free(s); free(c); free(gt); free(up); free(a);
        free(sel); free(w);
    }
    return bad ? -3 : 0;
}

/* Expert e alone on n input rows xin[n][d]: y[n][d] (the step each selected
 * slot takes inside oracle_forward). */
int oracle_expert(int n, int d, int I, const double *xin, const void *w_gate_up,
                  const void *w_down, int wdt, const float *sgu, const float *sdn, int e,
                  double *y, int mutation)
{
    if (n < 0 || d <= 0 || I <= 0 || e < 0) return -1;
    if (wdt == OR_E4M3 && (!sgu || !sdn)) return -1;
    double *xq = (double *)malloc(sizeof(double) * (size_t)d);
    double *gt = (double *)malloc(sizeof(double) * (size_t)I);
    double *up = (double *)malloc(sizeof(double) * (size_t)I);
    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < n; ++i)
        expert_mlp(d, I, xin + (size_t)i * d, w_gate_up, w_down, wdt, sgu, sdn, (size_t)e,
                   xq, gt, up, a, y + (size_t)i * d, mutation);
    free(xq); free(gt); free(up); free(a);
    return 0;
}

/* FP8_BLOCK quantisation of rows v[n_rows][n] in groups of 128: codes
 * [n_rows][n], scales [n_rows][ceil(n/128)], dequantised values deq[n_rows][n]. */
int oracle_quant(int n_rows, int n, const double *v, uint8_t *codes, float *scales,
                 double *deq, int mutation)
{
    if (n_rows < 0 || n <= 0) return -1;
    const int ng = (n + FP8_B - 1) / FP8_B;
    for (int r = 0; r < n_rows; ++r) {
        memcpy(deq + (size_t)r * n, v + (size_t)r * n, sizeof(double) * (size_t)n);
        quant_groups(n, deq + (size_t)r * n, codes + (size_t)r * n, scales + (size_t)r * ng,
                     mutation);
    }
    return 0;
}

/* e4m3 code of each float (round to nearest even, saturating), and the value
 * of each code: the format conversions alone, for the pins. */
int oracle_e4m3(int n, const float *f, uint8_t *codes, const uint8_t *in_codes, double *values)
{
    if (n < 0) return -1;
    for (int i = 0; i < n; ++i) {
        if (f && codes) codes[i] = e4m3_encode(f[i]);
        if (in_codes && values) values[i] = e4m3_value(in_codes[i]);
    }
    return 0;
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


/* ------------------------------------------------------------------------
 * The neighbouring steps of the block ("LFM2.5-24B-A2B: Biased Routing,
 * Short Convolutions and Ten KV Caches", section "The exact checkpoint": the
 * first two layers are dense and convolutional; a block normalises before
 * its mixer and before its feed-forward network, each with a residual).
 *
 * Dense feed-forward: out = x + down( silu(gate xn) * (up xn) ), xn the
 * RMSNorm of x, gate/up packed [2I][d] (gate rows first), down [d][I]: the
 * gated SiLU MLP of one expert, applied to every token with weight 1. */
int oracle_dense_ffn(int N, int d, int I, double eps, const void *x, int xdt, const float *gain,
                     const void *w_gate_up, const void *w_down, int wdt, double *out,
                     int mutation)
{
    if (N < 0 || d <= 0 || I <= 0 || wdt == OR_E4M3) return -1;
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * (size_t)d);
        double *xq = (double *)malloc(sizeof(double) * (size_t)d);
        double *gt = (double *)malloc(sizeof(double) * (size_t)I);
        double *up = (double *)malloc(sizeof(double) * (size_t)I);
        double *a = (double *)malloc(sizeof(double) * (size_t)I);
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < N; ++t) {
            rmsnorm_row(d, eps, x, xdt, (size_t)t, gain, xn, mutation);
            expert_mlp(d, I, xn, w_gate_up, w_down, wdt, NULL, NULL, 0, xq, gt, up, a, y,
                       mutation);
            double *o = out + (size_t)t * d;
            for (int j = 0; j < d; ++j)
                o[j] = ((mutation == MUT_NO_RESIDUAL) ? 0.0 : ld(x, xdt, (size_t)t * d + j)) + y[j];
        }
        free(xn); free(xq); free(gt); free(up); free(a); free(y);
    }
    return 0;
}

/* Short-convolution block ("LFM2.5-24B-A2B: Biased Routing, Short
 * Convolutions and Ten KV Caches", section "A short convolution is a local
 * mixer, not an embedding lookup"): the normalised row is projected into
 * three width-d streams g, u, v (B, C and x of the implementation; packed
 * w_in [3d][d] in that order); a = g * v; a depthwise causal convolution of
 * width three, c_t = sum_{l=0..2} k[l] * a_{t-l} per channel (k indexed by
 * lag: kconv[channel][l] multiplies a_{t-l}); y = u * c; out = x + w_out y,
 * w_out [d][d]. No bias in the projections or the convolution, no
 * activation on the gates (the page: direct linear projections).
 * x is [B][T][d]; each of the B sequences has its own history: the a vectors
 * of its two positions before t = 0, state_in[b][0] (position -2) and
 * state_in[b][1] (position -1), or zeros when state_in is NULL. state_out
 * (may be NULL) receives each sequence's a vectors of its last two
 * positions in the same layout (for T = 1: the old position -1, then a_0),
 * so that running T1 then T2 tokens with the state carried equals running
 * T1 + T2 at once. */
int oracle_shortconv(int B, int T, int d, double eps, const void *x, int xdt, const float *gain,
                     const void *w_in, const void *w_out, int wdt, const float *kconv,
                     const double *state_in, double *out, double *state_out, int mutation)
{
    if (B < 0 || T < 0 || d <= 0 || wdt == OR_E4M3) return -1;
    const size_t D = (size_t)d;
    /* a of every position, with two history positions in front per sequence */
    double *a = (double *)malloc(sizeof(double) * (size_t)B * (size_t)(T + 2) * D);
    double *u = (double *)malloc(sizeof(double) * (size_t)B * (size_t)T * D);
    double *g = (double *)malloc(sizeof(double) * (size_t)B * (size_t)T * D);
    if (!a || !u || !g) { free(a); free(u); free(g); return -4; }
    const int uo = (mutation == MUT_CONV_UV_SWAPPED) ? 2 : 1;   /* row block of u */
    const int vo = (mutation == MUT_CONV_UV_SWAPPED) ? 1 : 2;   /* row block of v */
    for (int b = 0; b < B; ++b) {
        double *ab = a + (size_t)b * (T + 2) * D;
        for (int j = 0; j < 2; ++j)
            for (size_t c = 0; c < D; ++c) {
                int src = b;
                if (mutation == MUT_CONV_SEQ_LEAK) src = b - 1;  /* previous sequence's state */
                ab[j * D + c] = (state_in && src >= 0) ? state_in[((size_t)src * 2 + j) * D + c] : 0.0;
            }
    }
#pragma omp parallel
    {
        double *xn = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < B * T; ++r) {
            const int b = r / T, t = r % T;
            rmsnorm_row(d, eps, x, xdt, (size_t)r, gain, xn, mutation);
            double *ab = a + ((size_t)b * (T + 2) + 2 + t) * D;
            for (size_t c = 0; c < D; ++c) {
                double sg = 0.0, su = 0.0, sv = 0.0;
                for (size_t j = 0; j < D; ++j) {
                    sg += ld(w_in, wdt, c * D + j) * xn[j];
                    su += ld(w_in, wdt, ((size_t)uo * D + c) * D + j) * xn[j];
                    sv += ld(w_in, wdt, ((size_t)vo * D + c) * D + j) * xn[j];
                }
                g[(size_t)r * D + c] = sg;
                u[(size_t)r * D + c] = su;
                ab[c] = (mutation == MUT_CONV_GATE_AFTER) ? sv : sg * sv;
            }
        }
        free(xn);
    }
    if (mutation == MUT_CONV_SEQ_LEAK) {
        /* the history of sequence b > 0 is the previous sequence's last two a */
        for (int b = B - 1; b >= 1; --b)
            for (int j = 0; j < 2; ++j)
                for (size_t c = 0; c < D; ++c)
                    a[((size_t)b * (T + 2) + j) * D + c] =
                        (T >= 2 - j) ? a[((size_t)(b - 1) * (T + 2) + T + j) * D + c] : 0.0;
    }
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < B * T; ++r) {
            const int b = r / T, t = r % T;
            const double *ab = a + (size_t)b * (T + 2) * D;   /* position p at ab[(p + 2) D] */
            for (size_t c = 0; c < D; ++c) {
                double cv = 0.0;
                for (int l = 0; l < 3; ++l) {
                    int p = t - l;                               /* lag l */
                    double k = (double)kconv[c * 3 + l];
                    if (mutation == MUT_CONV_LAG_REVERSED) k = (double)kconv[c * 3 + (2 - l)];
                    if (mutation == MUT_CONV_CENTERED) p = t + 1 - l;
                    double av = (p + 2 < T + 2) ? ab[(size_t)(p + 2) * D + c] : 0.0;
                    cv += k * av;
                }
                if (mutation == MUT_CONV_GATE_AFTER) cv *= g[(size_t)r * D + c];
                y[c] = u[(size_t)r * D + c] * cv;
            }
            double *o = out + (size_t)r * D;
            for (size_t j = 0; j < D; ++j) {
                double acc = 0.0;
                for (size_t c = 0; c < D; ++c) acc += ld(w_out, wdt, j * D + c) * y[c];
                o[j] = ((mutation == MUT_NO_RESIDUAL) ? 0.0 : ld(x, xdt, (size_t)r * D + j)) + acc;
            }
        }
        free(y);
    }
    if (state_out)
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < 2; ++j)
                memcpy(state_out + ((size_t)b * 2 + j) * D, a + ((size_t)b * (T + 2) + T + j) * D,
                       sizeof(double) * D);
    free(a); free(u); free(g);
    return 0;
}
