/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the routed-MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and
 * the bench's CPU-baseline / reference arm may load this library. The CUDA path
 * shares no code, header, table or helper with it.
 *
 * What it computes, per token t (sources: "Tencent Hy3-295B 架构深度拆解",
 * pillumina.github.io, §4.1 "Sigmoid 路由 vs Softmax" -- the router source lines
 * and the five-step routing flow; "DeepSeek V4-Flash 架构 QA",
 * cctoctofx.netlify.app, Q4.5 (SwiGLU expert) and Q8.4 (expert loop and
 * weighted accumulation); Hy3 commentary, wmrh.cn/news/24252, §2.3
 * (enable_moe_fp32_combine)):
 *
 *   1. logit_e = sum_c x[t,c] * Wg[e,c]  (+ gate_bias[e] when given)
 *   2. s_e     = 1 / (1 + exp(-logit_e))
 *   3. the k experts of largest s_e; equal scores go to the lower expert index
 *      (a full sort of (-s_e, e), then the first k). Both score functions
 *      below are strictly increasing, so the order of the exact scores is the
 *      order of the logits: the sort ranks the logits, which fp64 holds apart
 *      where the rounded scores are not (every logit above ~37 has the fp64
 *      sigmoid 1.0), and equal scores are exactly equal logits.
 *   4. w_j     = scale * s_j / sum_{i in top-k} s_i
 *   5. for each selected expert e:
 *        g_f = sum_c x_c Wgu[e, f, c],  u_f = sum_c x_c Wgu[e, F+f, c]
 *        h_f = SiLU(g_f) * u_f,  SiLU(z) = z / (1 + exp(-z))
 *        y_i = sum_f h_f Wd[e, i, f]
 *   6. out_i   = bf16_rne( sum_j w_j * y_{j,i} )
 *
 * The complete Hy3 MoE block adds two optional pieces (same pages: §4.1 step 2
 * and the Flash QA's Q4.3 / Q4.7):
 *   - e_score_correction_bias b_e, added to the sigmoid scores for the choice
 *     only: step 3 ranks c_e = s_e + b_e, while step 4 still renormalises the
 *     unbiased s_j of the chosen experts;
 *   - one shared expert (a SwiGLU with its own weights, applied to every
 *     token with weight 1): step 6 becomes
 *       out_i = bf16_rne( sum_j w_j * y_{j,i} + y_shared_i ),
 *     the shared term added last, inside the same fp64 sum.
 * and route_norm (Flash QA Q4.9): the router scores an RMS-normalised copy of
 * the token, xn_c = x_c / sqrt(mean_c' x_c'^2 + eps) * g_c (g: the norm's
 * weight); step 1 uses xn in place of x, the experts still take x.
 *
 * The second routing and precision variant of the pages ("Tencent Hy3-295B
 * 架构深度拆解" §2.2 and §2.7, the V4-Flash column): the score of step 2 may
 * be sqrt(softplus(logit)) instead of the sigmoid (same steps 3-4, with its own
 * scale, 1.5 on the page), and the routed experts may be FP4: E2M1 codes (1
 * sign, 2 exponent bits with bias 1, 1 mantissa bit; two per byte, the even
 * element in the low nibble) with one E8M0 scale 2^(b-127) per 32 consecutive
 * elements of a row; the weight value is code * scale.
 *
 * Every sum is a plain left-to-right fp64 loop; inputs are bf16 bit patterns
 * (or e4m3 codes with fp32 scales) widened exactly to double. The only
 * rounding to a narrow type is the single final bf16 cast of step 6.
 *
 * Weight layouts: Wg [E, d]; Wgu [E, 2F, d] with rows [0,F) = gate and
 * [F,2F) = up; Wd [E, d, F]. FP8 weights use the same layouts as uint8 e4m3
 * codes, with per-row fp32 scales s_gu [E, 2F] and s_d [E, d]; the weight
 * value is code * scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- formats */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* e4m3 (OCP FP8 "E4M3FN"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN. exp 0 is subnormal: mant/8 * 2^-6. */
static double e4m3_to_double(uint8_t q)
{
    int sign = (q >> 7) & 1;
    int ex = (q >> 3) & 0xF;
    int mant = q & 0x7;
    double v;
    if (ex == 0xF && mant == 0x7)
        return NAN;
    if (ex == 0)
        v = ldexp((double)mant / 8.0, -6);
    else
        v = ldexp(1.0 + (double)mant / 8.0, ex - 7);
    return sign ? -v : v;
}

/* e2m1 (OCP MX FP4): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no
 * infinities or NaN. exp 0 is subnormal: mant/2 * 2^0. */
static double e2m1_to_double(uint8_t nib)
{
    int sign = (nib >> 3) & 1;
    int ex = (nib >> 1) & 0x3;
    int mant = nib & 0x1;
    double v = (ex == 0) ? 0.5 * mant : ldexp(1.0 + 0.5 * mant, ex - 1);
    return sign ? -v : v;
}

/* e8m0 (OCP MX scale): 2^(b - 127); 0xFF is NaN. */
static double e8m0_to_double(uint8_t b)
{
    return (b == 0xFF) ? NAN : ldexp(1.0, (int)b - 127);
}

/* Round half to even of a non-negative double to an integer-valued double. */
static double round_half_even(double n)
{
    double fl = floor(n);
    double frac = n - fl;
    if (frac > 0.5)
        return fl + 1.0;
    if (frac < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Direct double -> bf16 with round-to-nearest-even (no intermediate float).
 * bf16: 8 exponent bits (bias 127), 7 stored mantissa bits. A normal value
 * with unbiased exponent E has quantum 2^(E-7); below 2^-126 the quantum is
 * fixed at 2^-133 (subnormals). */
static uint16_t double_to_bf16(double v)
{
    uint16_t sign;
    double a;
    int ex;
    if (isnan(v))
        return 0x7FC0;
    sign = signbit(v) ? 0x8000 : 0;
    a = fabs(v);
    if (isinf(a))
        return sign | 0x7F80;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &ex);          /* a = m * 2^ex, m in [0.5, 1) */
    ex -= 1;                      /* a = (2m) * 2^ex, 2m in [1, 2) */
    if (ex < -126) {
        double r = round_half_even(a / ldexp(1.0, -133));
        return sign | (uint16_t)r;              /* r = 128 is 2^-126 exactly */
    } else {
        double r = round_half_even(a / ldexp(1.0, ex - 7));  /* r in [128, 256] */
        long bits = ((long)(ex + 127) << 7) + ((long)r - 128);
        if (bits >= 0x7F80)
            return sign | 0x7F80;               /* overflow rounds to infinity */
        return sign | (uint16_t)bits;
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* SwiGLU's SiLU(g) * u, SiLU(z) = z * sigmoid(z). */
static double silu_times(double g, double u) { return g * sigmoid(g) * u; }

/* softplus(z) = ln(1 + e^z), evaluated without overflow. */
static double softplus(double z) { return (z > 0.0) ? z + log1p(exp(-z)) : log1p(exp(z)); }

/* Step 2's score: 0 = sigmoid (Hy3), 1 = sqrt(softplus) (the V4-Flash router). */
static double score_of(double z, int score_fn)
{
    return score_fn == 1 ? sqrt(softplus(z)) : sigmoid(z);
}

/* Weight element (expert e, row r, column c) of a [E, rows, cols] block that is
 * either bf16 (scales == NULL) or e4m3 codes with per-row fp32 scales. */
static double weight_at(const void* w, const float* scales, long e, long rows, long cols,
                        long r, long c)
{
    long off = (e * rows + r) * cols + c;
    if (scales == NULL)
        return bf16_to_double(((const uint16_t*)w)[off]);
    return e4m3_to_double(((const uint8_t*)w)[off]) * (double)scales[e * rows + r];
}

/* Weight element (expert e, row r, column c) of a [E, rows, cols] block of FP4
 * codes (two per byte, the even element in the low nibble) with E8M0 scales
 * [E, rows, cols/32], one per 32 consecutive elements of a row. */
static double weight_at_fp4(const uint8_t* w, const uint8_t* scales, long e, long rows, long cols,
                            long r, long c)
{
    long off = (e * rows + r) * cols + c;
    uint8_t byte = w[off >> 1];
    uint8_t nib = (off & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
    return e2m1_to_double(nib) * e8m0_to_double(scales[(e * rows + r) * (cols / 32) + c / 32]);
}

/* ---------------------------------------------------------------- routing */

typedef struct {
    double key; /* what the choice ranks: the logit (the order of the exact
                   scores), or s plus the score bias when that is given */
    double v;   /* the ranked value in score units: s, or s + score bias */
    double s;   /* sigmoid score */
    int e;
} scored_expert;

/* Descending key; equal keys: lower expert index first. */
static int by_score_then_index(const void* pa, const void* pb)
{
    const scored_expert* a = (const scored_expert*)pa;
    const scored_expert* b = (const scored_expert*)pb;
    if (a->key > b->key)
        return -1;
    if (a->key < b->key)
        return 1;
    return (a->e < b->e) ? -1 : (a->e > b->e);
}

/* Route one token: steps 1-4 above. Writes k indices (descending key), their
 * k weights, optionally all E logits and scores, and the gap between the
 * ranked values (in score units) of the k-th and (k+1)-th expert of the order
 * (+inf when k == E). score_bias may be NULL. */
static void route_token(int d, int E, int k, double scale, const uint16_t* xrow,
                        const uint16_t* wg, const float* gate_bias, const float* score_bias,
                        const float* norm_w, double norm_eps, int score_fn, int32_t* idx,
                        double* w, double* logits_out, double* scores_out, double* gap)
{
    scored_expert* order = (scored_expert*)malloc(sizeof(scored_expert) * (size_t)E);
    double* xr = (double*)malloc(sizeof(double) * (size_t)d);
    double sel_sum = 0.0;
    int e, c, j;
    for (c = 0; c < d; ++c)
        xr[c] = bf16_to_double(xrow[c]);
    if (norm_w) {
        /* route_norm: RMSNorm of the token for the router only */
        double ms = 0.0, inv;
        for (c = 0; c < d; ++c)
            ms += xr[c] * xr[c];
        inv = 1.0 / sqrt(ms / d + norm_eps);
        for (c = 0; c < d; ++c)
            xr[c] = xr[c] * inv * (double)norm_w[c];
    }
    for (e = 0; e < E; ++e) {
        double logit = 0.0;
        for (c = 0; c < d; ++c)
            logit += xr[c] * bf16_to_double(wg[(long)e * d + c]);
        if (gate_bias)
            logit += (double)gate_bias[e];
        order[e].s = score_of(logit, score_fn);
        order[e].v = score_bias ? order[e].s + (double)score_bias[e] : order[e].s;
        order[e].key = score_bias ? order[e].v : logit;
        order[e].e = e;
        if (logits_out)
            logits_out[e] = logit;
        if (scores_out)
            scores_out[e] = order[e].s;
    }
    qsort(order, (size_t)E, sizeof(scored_expert), by_score_then_index);
    for (j = 0; j < k; ++j)
        sel_sum += order[j].s;
    for (j = 0; j < k; ++j) {
        idx[j] = order[j].e;
        w[j] = scale * order[j].s / sel_sum;
    }
    *gap = (k < E) ? order[k - 1].v - order[k].v : INFINITY;
    free(xr);
    free(order);
}

/* ---------------------------------------------------------------- experts */

/* One SwiGLU expert on one token: step 5. h may be NULL. */
static void expert_token(int d, int F, long e, const uint16_t* xrow, const void* wgu,
                         const float* s_gu, const void* wd, const float* s_d, double* h,
                         double* y)
{
    double* hh = h ? h : (double*)malloc(sizeof(double) * (size_t)F);
    int f, c, i;
    for (f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (c = 0; c < d; ++c) {
            double xc = bf16_to_double(xrow[c]);
            g += xc * weight_at(wgu, s_gu, e, 2L * F, d, f, c);
            u += xc * weight_at(wgu, s_gu, e, 2L * F, d, (long)F + f, c);
        }
        hh[f] = silu_times(g, u);
    }
    for (i = 0; i < d; ++i) {
        double acc = 0.0;
        for (f = 0; f < F; ++f)
            acc += hh[f] * weight_at(wd, s_d, e, d, F, i, f);
        y[i] = acc;
    }
    if (!h)
        free(hh);
}

/* Step 5 with FP4 expert weights (same mathematics). */
static void expert_token_fp4(int d, int F, long e, const uint16_t* xrow, const uint8_t* wgu,
                             const uint8_t* s_gu, const uint8_t* wd, const uint8_t* s_d,
                             double* h, double* y)
{
    double* hh = h ? h : (double*)malloc(sizeof(double) * (size_t)F);
    int f, c, i;
    for (f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (c = 0; c < d; ++c) {
            double xc = bf16_to_double(xrow[c]);
            g += xc * weight_at_fp4(wgu, s_gu, e, 2L * F, d, f, c);
            u += xc * weight_at_fp4(wgu, s_gu, e, 2L * F, d, (long)F + f, c);
        }
        hh[f] = silu_times(g, u);
    }
    for (i = 0; i < d; ++i) {
        double acc = 0.0;
        for (f = 0; f < F; ++f)
            acc += hh[f] * weight_at_fp4(wd, s_d, e, d, F, i, f);
        y[i] = acc;
    }
    if (!h)
        free(hh);
}

/* ---------------------------------------------------------------- combine */

/* Step 6 for one token: out_i = bf16_rne( sum_j w_j * y_{j,i} ), the sum in
 * fp64 over j = 0..k-1 in order. y is [k, d]. acc (may be NULL) receives the
 * sum before the cast. */
static void combine_token(int k, int d, const double* y, const double* w, const double* y_shared,
                          double* acc, uint16_t* out)
{
    int i, j;
    for (i = 0; i < d; ++i) {
        double a = 0.0;
        for (j = 0; j < k; ++j)
            a += w[j] * y[(long)j * d + i];
        if (y_shared)
            a += y_shared[i];
        if (acc)
            acc[i] = a;
        out[i] = double_to_bf16(a);
    }
}

/* ---------------------------------------------------------------- exported */

/* Step 6 for n tokens: y [n, k, d] (fp64), w [n, k] -> out_bf16 [n, d]. */
void oracle_combine(int n, int k, int d, const double* y, const double* w, uint16_t* out)
{
    long r;
    for (r = 0; r < n; ++r)
        combine_token(k, d, y + r * (long)k * d, w + r * (long)k, NULL, NULL, out + r * (long)d);
}


int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

void oracle_bf16_from_double(const double* v, uint16_t* out, long n)
{
    long i;
    for (i = 0; i < n; ++i)
        out[i] = double_to_bf16(v[i]);
}

void oracle_double_from_bf16(const uint16_t* b, double* out, long n)
{
    long i;
    for (i = 0; i < n; ++i)
        out[i] = bf16_to_double(b[i]);
}

void oracle_double_from_e4m3(const uint8_t* q, double* out, long n)
{
    long i;
    for (i = 0; i < n; ++i)
        out[i] = e4m3_to_double(q[i]);
}

/* Steps 1-4 for tokens [0, T), with the optional score bias [E] (NULL: none)
 * and route_norm weight [d] (NULL: no route_norm; norm_eps its epsilon).
 * logits/scores may be NULL ([T, E] otherwise). */
int oracle_route2(int T, int d, int E, int k, double scale, const uint16_t* x,
                  const uint16_t* wg, const float* gate_bias, const float* score_bias,
                  const float* norm_w, double norm_eps, int score_fn, int32_t* idx, double* w,
                  double* logits, double* scores, double* gap)
{
    long t;
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || (norm_w && !(norm_eps > 0.0)) ||
        score_fn < 0 || score_fn > 1)
        return -1;
#pragma omp parallel for schedule(dynamic, 4)
    for (t = 0; t < T; ++t)
        route_token(d, E, k, scale, x + t * (long)d, wg, gate_bias, score_bias, norm_w, norm_eps,
                    score_fn, idx + t * (long)k, w + t * (long)k,
                    logits ? logits + t * (long)E : NULL, scores ? scores + t * (long)E : NULL,
                    gap + t);
    return 0;
}

/* Steps 1-4 without a score bias. */
int oracle_route(int T, int d, int E, int k, double scale, const uint16_t* x,
                 const uint16_t* wg, const float* gate_bias, int32_t* idx, double* w,
                 double* logits, double* scores, double* gap)
{
    return oracle_route2(T, d, E, k, scale, x, wg, gate_bias, NULL, NULL, 0.0, 0, idx, w, logits,
                         scores, gap);
}

/* Step 5 for n (row, expert) pairs: rows of xrows [n, d], experts[n]. h [n, F]
 * may be NULL; y is [n, d]. */
int oracle_expert_rows(int n, int d, int F, const uint16_t* xrows, const int32_t* experts,
                       const void* wgu, const float* s_gu, const void* wd, const float* s_d,
                       double* h, double* y)
{
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n; ++r)
        expert_token(d, F, experts[r], xrows + r * (long)d, wgu, s_gu, wd, s_d,
                     h ? h + r * (long)F : NULL, y + r * (long)d);
    return 0;
}

/* Steps 1-6 for the n tokens listed in tokens[] (indices into x [T, d]), with
 * the optional score bias [E], the optional RMSNorm of the router input
 * (norm_w [d], norm_eps), the score function (0 sigmoid, 1 sqrt-softplus) and
 * the optional shared expert (sh_wgu [2F, d], sh_wd [d, F]
 * in the routed experts' format, with row scales sh_s_gu [2F] / sh_s_d [d] for
 * e4m3 codes; sh_wgu NULL: no shared expert).
 * Outputs per listed token: out_f64 [n, d] (the fp64 sum before the cast),
 * out_bf16 [n, d], idx [n, k], w [n, k], gap [n]. */
int oracle_forward_tokens2(int T, int d, int E, int k, int F, double scale, const uint16_t* x,
                           const uint16_t* wg, const float* gate_bias, const float* score_bias,
                           const float* norm_w, double norm_eps, int score_fn,
                           const void* wgu, const float* s_gu, const void* wd, const float* s_d,
                           const void* sh_wgu, const float* sh_s_gu, const void* sh_wd,
                           const float* sh_s_d, const int32_t* tokens, int n, double* out_f64,
                           uint16_t* out_bf16, int32_t* idx, double* w, double* gap)
{
    long r;
    if (d <= 0 || E <= 0 || k <= 0 || k > E || F <= 0)
        return -1;
    if ((sh_wgu == NULL) != (sh_wd == NULL) || (norm_w && !(norm_eps > 0.0)) || score_fn < 0 ||
        score_fn > 1)
        return -1;
    for (r = 0; r < n; ++r)
        if (tokens[r] < 0 || tokens[r] >= T)
            return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n; ++r) {
        const uint16_t* xrow = x + (long)tokens[r] * d;
        double* y = (double*)malloc(sizeof(double) * (size_t)k * d);
        double* ysh = sh_wgu ? (double*)malloc(sizeof(double) * (size_t)d) : NULL;
        int j;
        route_token(d, E, k, scale, xrow, wg, gate_bias, score_bias, norm_w, norm_eps, score_fn,
                    idx + r * (long)k, w + r * (long)k, NULL, NULL, gap + r);
        for (j = 0; j < k; ++j)
            expert_token(d, F, idx[r * (long)k + j], xrow, wgu, s_gu, wd, s_d, NULL,
                         y + (long)j * d);
        if (ysh)
            expert_token(d, F, 0, xrow, sh_wgu, sh_s_gu, sh_wd, sh_s_d, NULL, ysh);
        combine_token(k, d, y, w + r * (long)k, ysh, out_f64 + r * (long)d,
                      out_bf16 + r * (long)d);
        free(ysh);
        free(y);
    }
    return 0;
}

/* Steps 1-6 without a score bias or shared expert. */
int oracle_forward_tokens(int T, int d, int E, int k, int F, double scale, const uint16_t* x,
                          const uint16_t* wg, const float* gate_bias, const void* wgu,
                          const float* s_gu, const void* wd, const float* s_d,
                          const int32_t* tokens, int n, double* out_f64, uint16_t* out_bf16,
                          int32_t* idx, double* w, double* gap)
{
    return oracle_forward_tokens2(T, d, E, k, F, scale, x, wg, gate_bias, NULL, NULL, 0.0, 0, wgu,
                                  s_gu, wd, s_d, NULL, NULL, NULL, NULL, tokens, n, out_f64,
                                  out_bf16, idx, w, gap);
}

void oracle_double_from_e2m1(const uint8_t* nibbles, double* out, long n)
{
    long i;
    for (i = 0; i < n; ++i)
        out[i] = e2m1_to_double(nibbles[i] & 0xF);
}

void oracle_double_from_e8m0(const uint8_t* b, double* out, long n)
{
    long i;
    for (i = 0; i < n; ++i)
        out[i] = e8m0_to_double(b[i]);
}

/* Step 5 with FP4 experts for n (row, expert) pairs (see oracle_expert_rows). */
int oracle_expert_rows_fp4(int n, int d, int F, const uint16_t* xrows, const int32_t* experts,
                           const uint8_t* wgu, const uint8_t* s_gu, const uint8_t* wd,
                           const uint8_t* s_d, double* h, double* y)
{
    long r;
    if (d % 32 || F % 32)
        return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n; ++r)
        expert_token_fp4(d, F, experts[r], xrows + r * (long)d, wgu, s_gu, wd, s_d,
                         h ? h + r * (long)F : NULL, y + r * (long)d);
    return 0;
}

/* Steps 1-6 of the second variant for the listed tokens: score_fn as in
 * oracle_route2, FP4 routed experts, optional score bias; no shared expert. */
int oracle_forward_tokens_fp4(int T, int d, int E, int k, int F, double scale, const uint16_t* x,
                              const uint16_t* wg, const float* gate_bias, const float* score_bias,
                              int score_fn, const uint8_t* wgu, const uint8_t* s_gu,
                              const uint8_t* wd, const uint8_t* s_d, const int32_t* tokens, int n,
                              double* out_f64, uint16_t* out_bf16, int32_t* idx, double* w,
                              double* gap)
{
    long r;
    if (d <= 0 || E <= 0 || k <= 0 || k > E || F <= 0 || d % 32 || F % 32 || score_fn < 0 ||
        score_fn > 1)
        return -1;
    for (r = 0; r < n; ++r)
        if (tokens[r] < 0 || tokens[r] >= T)
            return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n; ++r) {
        const uint16_t* xrow = x + (long)tokens[r] * d;
        double* y = (double*)malloc(sizeof(double) * (size_t)k * d);
        int j;
        route_token(d, E, k, scale, xrow, wg, gate_bias, score_bias, NULL, 0.0, score_fn,
                    idx + r * (long)k, w + r * (long)k, NULL, NULL, gap + r);
        for (j = 0; j < k; ++j)
            expert_token_fp4(d, F, idx[r * (long)k + j], xrow, wgu, s_gu, wd, s_d, NULL,
                             y + (long)j * d);
        combine_token(k, d, y, w + r * (long)k, NULL, out_f64 + r * (long)d,
                      out_bf16 + r * (long)d);
        free(y);
    }
    return 0;
}

/* The grouping that the library's permute step defines (integer work):
 * counts[e] = number of slots s = t*k + j with idx[s] == e;
 * offsets[e] = sum_{e' < e} counts[e'], offsets[E] = T*k;
 * row_of[s] = offsets[idx[s]] + #{ s' < s : idx[s'] == idx[s] }  (stable). */
int oracle_permute(int T, int k, int E, const int32_t* idx, int32_t* counts, int32_t* offsets,
                   int32_t* row_of)
{
    long s, n = (long)T * k;
    int e;
    int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (e = 0; e < E; ++e)
        counts[e] = 0;
    for (s = 0; s < n; ++s) {
        if (idx[s] < 0 || idx[s] >= E) {
            free(seen);
            return -1;
        }
        counts[idx[s]] += 1;
    }
    offsets[0] = 0;
    for (e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    for (s = 0; s < n; ++s) {
        row_of[s] = offsets[idx[s]] + seen[idx[s]];
        seen[idx[s]] += 1;
    }
    free(seen);
    return 0;
}
