/*
 * moe_oracle.c -- CPU oracle for the forward of one fused routed-expert FP8 MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, obviously-correct restatement of
 * what the layer computes.  Only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg may load it.  The CUDA library never includes, links or calls it, and the
 * two share no code, header, table or constant generator.
 *
 * Sources (web pages, cited by title and section):
 *   [MindIE]   "MindIE-SD Fused MoE" (fused_moe.md): function signature, parameter table,
 *              execution flow (prepare / select_experts / dispatch / mlp / combine), routing
 *              selection, quantization configs, the custom routing function example.
 *   [MATE]     "MATE Mega MoE" (mega_moe.rst): Typical Flow, Current Limits, API.
 *   [metrale]  "metrale_model_layers fp8_grouped_tc_w8a8.rs": module doc and
 *              run_fp8_grouped_w8a8 (act-quant E4M3 per (row,128) -> gate+up -> SiLU
 *              product requantized -> down).
 *   [DeepGEMM] "DeepGEMM PR #371: Add W8A8 (FP8xFP8) Mega MoE support": Changes (UE8M0
 *              4-packed scale factors, per-32 activation scale factors), Testing.
 *   [mlx]      "mlx_native ops/moe_gate.rs": moe_gate doc (top-K sort, softmax,
 *              per_expert_scale) and its argument validation.
 *   [W4A8]     "DeepGEMM PR #371", Changes: the W4A8 (FP8 x FP4) path it derives from uses
 *              e2m1 weights with the same 4-packed UE8M0 scale factors; "MATE Mega MoE",
 *              Use Mega MoE when: the W4A8 mixed-dtype GEMM path.
 *
 * Precision: decisions that turn floating point into integers (expert selection, group
 * selection, E4M3 codes, scales) are taken in fp32, the precision of the kernels; every
 * accumulation (the two grouped GEMMs, SwiGLU, combine) is carried in fp64, and the output is
 * rounded once to bf16 (round to nearest even).
 *
 * Readings of points the pages leave open are marked "Reading:" below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_EUNSUPPORTED (-2)

/* ------------------------------------------------------------------------------------------
 * Problem description (the oracle's own; not shared with the library's header).
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    int32_t num_tokens, hidden, inter, num_experts, top_k;
    int32_t routing;            /* 0 softmax, 1 sigmoid                                      */
    int32_t renormalize;        /* softmax only; sigmoid weights are always normalized       */
    int32_t group_count, k_group, group_select_mode;
    float routed_scaling_factor;
    int32_t recipe;             /* 0: fp32 scale per (row,128); 1: UE8M0 scale per 32 (MXFP8);
                                   2: W4A8, E2M1 weights with UE8M0 per 32, MXFP8 activations */
    int32_t shared_experts;     /* 0 or 1: one more expert, index num_experts, that every token
                                   uses with weight 1 ([metrale] run_fp8_grouped_w8a8: the shared
                                   expert's gate/up/down run in the same grouped steps)          */
} orc_cfg;

/* ------------------------------------------------------------------------------------------
 * E4M3 ("float8_e4m3fn", named in [MindIE] MXFP8 example): 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448;
 * subnormals m * 2^-9.
 * ---------------------------------------------------------------------------------------- */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);             /* subnormal: m/8 * 2^-6 */
    else v = ldexp((double)(8 + m), e - 10);          /* (1 + m/8) * 2^(e-7)   */
    return s ? -v : v;
}

/* Round half to even of a non-negative double. */
static double rne(double m)
{
    double fl = floor(m), d = m - fl;
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;
}

/* fp32 -> E4M3, round to nearest even, saturating to +-448 (the "satfinite" rule: values at or
 * beyond the largest finite magnitude become that magnitude; NaN stays NaN). */
uint8_t orc_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v), quantum, n;
    int ex;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {                         /* subnormal range: step 2^-9 */
        n = rne(a / ldexp(1.0, -9));                  /* 0..8; 8 is the smallest normal */
        return (uint8_t)(sign | (int)n);
    }
    frexp(a, &ex);                                    /* a = f * 2^ex, f in [0.5,1) */
    ex -= 1;                                          /* floor(log2 a) */
    quantum = ldexp(1.0, ex - 3);                     /* 3 mantissa bits */
    n = rne(a / quantum);                             /* 8..16 */
    if (n == 16.0) { n = 8.0; ex += 1; }
    return (uint8_t)(sign | ((ex + 7) << 3) | ((int)n - 8));
}

/* Decoded values of all 256 codes, filled from orc_e4m3_decode when the library loads. */
static double e4m3_table[256];

__attribute__((constructor)) static void fill_e4m3_table(void)
{
    for (int c = 0; c < 256; c++) e4m3_table[c] = orc_e4m3_decode((uint8_t)c);
}

/* ------------------------------------------------------------------------------------------
 * E2M1 (FP4, the "e2m1" weights of [W4A8]; the element format of the OCP microscaling
 * formats): 1 sign, 2 exponent (bias 1), 1 mantissa bit; no infinities or NaN.  Exponent 0 is
 * subnormal, m * 0.5; otherwise (1 + m/2) * 2^(e-1).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * Reading: two codes per byte, the lower-indexed element in the low nibble.
 * ---------------------------------------------------------------------------------------- */
double orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* Weight element n of row k of a [Kdim, N] weight matrix: an E4M3 byte (recipes 0, 1) or an
 * E2M1 nibble of a byte packed along N (recipe 2). */
static double weight_value(int recipe, const uint8_t *wq, int N, int k, int n)
{
    if (recipe == 2) {
        const uint8_t b = wq[(size_t)k * (N / 2) + n / 2];
        return orc_e2m1_decode((uint8_t)((n & 1) ? (b >> 4) : (b & 15)));
    }
    return e4m3_table[wq[(size_t)k * N + n]];
}

/* Bytes of a [Kdim, N] weight matrix's codes. */
static size_t weight_bytes(int recipe, int Kdim, int N)
{
    return recipe == 2 ? (size_t)Kdim * N / 2 : (size_t)Kdim * N;
}

/* UE8M0: an unsigned biased power-of-two exponent, value 2^(b - 127). */
static double ue8m0_value(uint8_t b) { return ldexp(1.0, (int)b - 127); }

/* ------------------------------------------------------------------------------------------
 * Dynamic activation quantization ([metrale] module doc: "quantized to E4M3 per (row, 128
 * group)"; [DeepGEMM] Changes: UE8M0 scale factors, per 32 K-elements).
 *
 * Reading (recipe 0): s = amax / 448 in fp32, q = e4m3_rn_satfinite(x / s) with an IEEE fp32
 * division; amax == 0 gives s = 1.
 * Reading (recipe 1): the scale is the smallest power of two 2^e with amax <= 448 * 2^e, found
 * exactly from amax's binary exponent; its UE8M0 byte is e + 127 clamped to [0, 254]; amax == 0
 * gives byte 127; q = e4m3_rn_satfinite(x / 2^e).  No value saturates.
 * ---------------------------------------------------------------------------------------- */
void orc_quant_group_fp32(const float *x, int n, uint8_t *q, float *s_out)
{
    float amax = 0.0f, s;
    for (int i = 0; i < n; i++) amax = fmaxf(amax, fabsf(x[i]));
    s = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int i = 0; i < n; i++) q[i] = orc_e4m3_encode(x[i] / s);
    *s_out = s;
}

int orc_mx_exponent(float amax)
{
    int ex, e;
    double f;
    if (!(amax > 0.0f)) return 0;
    f = frexp((double)amax, &ex);                     /* amax = (2f) * 2^(ex-1), 2f in [1,2) */
    /* amax <= 448 * 2^e  <=>  (2f) * 2^(ex-1) <= 1.75 * 2^(8+e) */
    e = (ex - 1) - 8 + ((2.0 * f) > 1.75 ? 1 : 0);
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

void orc_quant_group_mx(const float *x, int n, uint8_t *q, uint8_t *e8_out)
{
    float amax = 0.0f, scale;
    int e;
    for (int i = 0; i < n; i++) amax = fmaxf(amax, fabsf(x[i]));
    e = orc_mx_exponent(amax);
    scale = ldexpf(1.0f, e);
    for (int i = 0; i < n; i++) q[i] = orc_e4m3_encode(x[i] / scale);
    *e8_out = (uint8_t)(e + 127);
}

/* Quantize one row of n values in groups: recipe 0 -> n/128 fp32 scales, recipes 1 and 2
 * (W4A8 activations are MXFP8) -> n/32 UE8M0 bytes.  `scales` points at float or uint8_t
 * storage accordingly. */
void orc_quant_row(const float *x, int n, int recipe, uint8_t *q, void *scales)
{
    if (recipe == 0) {
        for (int g = 0; g < n / 128; g++)
            orc_quant_group_fp32(x + 128 * g, 128, q + 128 * g, (float *)scales + g);
    } else {
        for (int g = 0; g < n / 32; g++)
            orc_quant_group_mx(x + 32 * g, 32, q + 32 * g, (uint8_t *)scales + g);
    }
}

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* double -> bf16 bits, round to nearest even, directly from the double (one rounding). */
uint16_t orc_bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v), quantum, n, r;
    int ex;
    float f;
    uint32_t u;
    if (isnan(v)) return 0x7FC0;
    if (a == 0.0) return sign;
    frexp(a, &ex);
    ex -= 1;                                          /* floor(log2 a) */
    if (ex < -126) ex = -126;                         /* bf16 subnormals: step 2^-133 */
    quantum = ldexp(1.0, ex - 7);                     /* 7 stored mantissa bits */
    n = rne(a / quantum);
    r = n * quantum;
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);   /* overflow to infinity */
    f = (float)r;                                     /* exact: r is a bf16 value */
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (u >> 16));
}

/* ------------------------------------------------------------------------------------------
 * Routing ([MindIE] routing selection and parameter table; [mlx] moe_gate doc).
 *
 *   softmax: p_e = exp(l_e - max) / sum_e' exp(l_e' - max); the weights of the selected experts
 *            are p; with renormalize they are divided by their sum.
 *   sigmoid: s_e = 1 / (1 + exp(-l_e)); weights are s divided by their sum over the selected
 *            experts (the page: sigmoid routing outputs normalized weights).
 *   groups:  the E experts form group_count contiguous groups; a group's score is the max of
 *            its experts' scores (mode 0) or the sum of its two largest (mode 1); the k_group
 *            best groups are kept and the top_k experts are chosen inside them.
 *   then     weights *= per_expert_scale[id] (when given), then *= routed_scaling_factor,
 *            which the page says takes effect at expert selection.
 *
 * Reading: experts are chosen by their raw logits, which order them exactly as softmax or
 * sigmoid scores do; ties go to the lower expert index and groups' ties to the lower group
 * index; slots are emitted in descending order (the page's custom routing example uses topk,
 * and moe_gate sorts).  Group scores are computed from fp32 scores (the kernels' precision);
 * a token whose k_group-th and (k_group+1)-th group scores lie within 1e-5 relative is
 * flagged as a near tie.
 * ---------------------------------------------------------------------------------------- */
static int better(float va, int ia, float vb, int ib)   /* is (va, ia) ahead of (vb, ib)? */
{
    return va > vb || (va == vb && ia < ib);
}

int orc_check_cfg(const orc_cfg *c)
{
    if (c->num_tokens <= 0 || c->hidden <= 0 || c->inter <= 0 || c->num_experts <= 0 ||
        c->top_k <= 0 || c->top_k > c->num_experts)
        return ORC_EINVAL;
    if (c->hidden % 128 || c->inter % 128 || c->num_experts > 256) return ORC_EUNSUPPORTED;
    if (c->group_count < 1 || c->num_experts % c->group_count) return ORC_EUNSUPPORTED;
    if (c->k_group < 1 || c->k_group > c->group_count) return ORC_EUNSUPPORTED;
    if (c->top_k > c->k_group * (c->num_experts / c->group_count)) return ORC_EUNSUPPORTED;
    if (c->group_select_mode == 1 && c->num_experts / c->group_count < 2) return ORC_EUNSUPPORTED;
    if (c->routing != 0 && c->routing != 1) return ORC_EINVAL;
    if (c->recipe < 0 || c->recipe > 2) return ORC_EINVAL;
    if (c->shared_experts != 0 && c->shared_experts != 1) return ORC_EUNSUPPORTED;
    return ORC_OK;
}

/* fp32 scores of one token's experts (used only for the group scores): sigmoid, or softmax
 * over all E. */
static void token_scores(const orc_cfg *c, const float *l, float *score)
{
    const int E = c->num_experts;
    if (c->routing == 1) {
        for (int e = 0; e < E; e++) score[e] = 1.0f / (1.0f + expf(-l[e]));
    } else {
        float m = l[0], z = 0.0f;
        for (int e = 1; e < E; e++) m = fmaxf(m, l[e]);
        for (int e = 0; e < E; e++) z += expf(l[e] - m);
        for (int e = 0; e < E; e++) score[e] = expf(l[e] - m) / z;
    }
}

/* fp32 group scores of one token from its expert scores: the max of the group's scores
 * (mode 0) or the sum of its two largest (mode 1). */
static void group_scores(const orc_cfg *c, const float *score, float *gscore)
{
    const int G = c->group_count, gs = c->num_experts / G;
    for (int g = 0; g < G; g++) {
        const float *s = score + g * gs;
        if (c->group_select_mode == 0) {
            float mx = s[0];
            for (int i = 1; i < gs; i++) mx = fmaxf(mx, s[i]);
            gscore[g] = mx;
        } else {
            int i1 = 0, i2 = -1;
            for (int i = 1; i < gs; i++) if (s[i] > s[i1]) i1 = i;
            for (int i = 0; i < gs; i++)
                if (i != i1 && (i2 < 0 || s[i] > s[i2])) i2 = i;
            gscore[g] = s[i1] + s[i2];
        }
    }
}

/* Weights of the selected experts ids[k] of one token, in fp64, rounded once to fp32. */
static void route_weights(const orc_cfg *c, const float *l, const float *per_expert_scale,
                          const int32_t *ids, float *w)
{
    const int E = c->num_experts, K = c->top_k;
    double wsum = 0.0, wd[256];
    if (c->routing == 1) {
        for (int j = 0; j < K; j++) wd[j] = 1.0 / (1.0 + exp(-(double)l[ids[j]]));
        for (int j = 0; j < K; j++) wsum += wd[j];
        for (int j = 0; j < K; j++) wd[j] /= wsum;
    } else {
        double m = l[0], z = 0.0;
        for (int e = 1; e < E; e++) m = fmax(m, (double)l[e]);
        for (int e = 0; e < E; e++) z += exp((double)l[e] - m);
        for (int j = 0; j < K; j++) wd[j] = exp((double)l[ids[j]] - m) / z;
        if (c->renormalize) {
            for (int j = 0; j < K; j++) wsum += wd[j];
            for (int j = 0; j < K; j++) wd[j] /= wsum;
        }
    }
    for (int j = 0; j < K; j++) {
        if (per_expert_scale) wd[j] *= (double)per_expert_scale[ids[j]];
        wd[j] *= (double)c->routed_scaling_factor;
        w[j] = (float)wd[j];
    }
}

/* Route one token: logits l[E] -> ids[k], weights[k]; returns 1 if the group choice was a
 * near tie, else 0. */
static int route_token(const orc_cfg *c, const float *l, const float *per_expert_scale,
                       int32_t *ids, float *w)
{
    const int E = c->num_experts, K = c->top_k, G = c->group_count, gs = E / G;
    float score[256];
    unsigned char eligible[256], taken[256];
    int near_tie = 0;

    token_scores(c, l, score);
    for (int e = 0; e < E; e++) eligible[e] = 1;
    if (G > 1) {
        float gscore[256];
        unsigned char gtaken[256];
        int order[256];
        group_scores(c, score, gscore);
        for (int g = 0; g < G; g++) gtaken[g] = 0;
        for (int r = 0; r < G; r++) {                 /* full order of groups */
            int best = -1;
            for (int g = 0; g < G; g++)
                if (!gtaken[g] && (best < 0 || better(gscore[g], g, gscore[best], best))) best = g;
            order[r] = best;
            gtaken[best] = 1;
        }
        if (c->k_group < G) {
            double a = gscore[order[c->k_group - 1]], b = gscore[order[c->k_group]];
            if (fabs(a - b) <= 1e-5 * fmax(fabs(a), fabs(b))) near_tie = 1;
        }
        for (int e = 0; e < E; e++) eligible[e] = 0;
        for (int r = 0; r < c->k_group; r++)
            for (int i = 0; i < gs; i++) eligible[order[r] * gs + i] = 1;
    }

    for (int e = 0; e < E; e++) taken[e] = 0;
    for (int j = 0; j < K; j++) {
        int best = -1;
        for (int e = 0; e < E; e++)
            if (eligible[e] && !taken[e] && (best < 0 || better(l[e], e, l[best], best))) best = e;
        ids[j] = best;
        taken[best] = 1;
    }
    route_weights(c, l, per_expert_scale, ids, w);
    return near_tie;
}

/* The fp32 group scores of every token, [T, group_count] (the values the near-tie flag and
 * the group choice above are taken on); for checking another implementation's group choice. */
int orc_group_scores(const orc_cfg *c, const float *logits, float *gscores)
{
    int rc = orc_check_cfg(c);
    if (rc) return rc;
    const int E = c->num_experts, G = c->group_count;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < c->num_tokens; t++) {
        float score[256];
        token_scores(c, logits + (size_t)t * E, score);
        group_scores(c, score, gscores + (size_t)t * G);
    }
    return ORC_OK;
}

/* Routing weights of caller-chosen experts topk_idx [T, k] (each id in [0, E)): the same
 * weight rule as orc_route, for checking the weights that go with another implementation's
 * valid selection. */
int orc_route_weights(const orc_cfg *c, const float *logits, const float *per_expert_scale,
                      const int32_t *topk_idx, float *topk_w)
{
    int rc = orc_check_cfg(c);
    if (rc) return rc;
    for (size_t i = 0; i < (size_t)c->num_tokens * c->top_k; i++)
        if (topk_idx[i] < 0 || topk_idx[i] >= c->num_experts) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < c->num_tokens; t++)
        route_weights(c, logits + (size_t)t * c->num_experts, per_expert_scale,
                      topk_idx + (size_t)t * c->top_k, topk_w + (size_t)t * c->top_k);
    return ORC_OK;
}

int orc_route(const orc_cfg *c, const float *logits, const float *per_expert_scale,
              int32_t *topk_idx, float *topk_w, uint8_t *near_tie)
{
    int rc = orc_check_cfg(c);
    if (rc) return rc;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < c->num_tokens; t++) {
        int f = route_token(c, logits + (size_t)t * c->num_experts, per_expert_scale,
                            topk_idx + (size_t)t * c->top_k, topk_w + (size_t)t * c->top_k);
        if (near_tie) near_tie[t] = (uint8_t)f;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * The gate in front of the router ([mlx_native] moe_gate: RMS-Norm of the token's hidden state,
 * then the router matmul, then top-K with softmax and per-expert scale), up to the logits:
 *   xn[h]      = x[h] / sqrt( mean_h x[h]^2 + eps ) * norm_w[h]
 *   logits[e]  = sum_h xn[h] * router_w[e, h]          (router_w fp32 [E, H], row-major)
 * in fp64, rounded once to fp32 (the router takes fp32 logits).  Reading: the learned norm
 * weight multiplies the normalized value (the page names it "RMS norm learned weight").
 * ---------------------------------------------------------------------------------------- */
void orc_gate_logits(int T, int H, int E, const uint16_t *x, const float *norm_w,
                     const float *router_w, float eps, float *logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        double ss = 0.0;
        double *xn = (double *)malloc(sizeof(double) * (size_t)H);
        for (int h = 0; h < H; h++) {
            const double v = (double)bf16_to_f32(x[(size_t)t * H + h]);
            ss += v * v;
        }
        const double r = 1.0 / sqrt(ss / (double)H + (double)eps);
        for (int h = 0; h < H; h++)
            xn[h] = (double)bf16_to_f32(x[(size_t)t * H + h]) * r * (double)norm_w[h];
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int h = 0; h < H; h++) acc += xn[h] * (double)router_w[(size_t)e * H + h];
            logits[(size_t)t * E + e] = (float)acc;
        }
        free(xn);
    }
}

/* ------------------------------------------------------------------------------------------
 * Permutation into expert-contiguous order ([MindIE] execution flow, dispatch: tokens are
 * reordered by expert and the tokens per expert counted; combine restores token order).
 * Routed row a = t*k + j.  Reading: inside one expert, rows ascend by token index.
 * ---------------------------------------------------------------------------------------- */
void orc_permute(int T, int K, int E, const int32_t *topk_idx, int32_t *counts,
                 int32_t *offsets, int32_t *row_src, int32_t *row_of)
{
    int pos = 0;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int a = 0; a < T * K; a++) counts[topk_idx[a]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    for (int e = 0; e < E; e++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < K; j++)
                if (topk_idx[t * K + j] == e) {
                    row_src[pos] = t * K + j;
                    row_of[t * K + j] = pos;
                    pos++;
                }
}

/* ------------------------------------------------------------------------------------------
 * One grouped, block-scaled FP8 GEMM row:
 *   out[n] = sum_g  sa[g] * sw[g][n] * sum_{k in group g} dec(aq[k]) * dec(wq[k][n])
 * (dec = E4M3, or E2M1 for the W4A8 weights of recipe 2, which are packed two per byte along N)
 * with wq stored K rows x N columns (the pages' w13 [E, hidden, 2*inter] and
 * w2 [E, inter, hidden] orientation, [MindIE] parameter table) and the weight scales stored
 * [K/g][N] ([MindIE] MXFP8 example: the scale tensor is transposed to put the K blocks
 * before N).  Accumulated in fp64; each group's inner sum is exact there.
 * ---------------------------------------------------------------------------------------- */
static double act_scale(int recipe, const void *s, size_t i)
{
    return recipe == 0 ? (double)((const float *)s)[i] : ue8m0_value(((const uint8_t *)s)[i]);
}

void orc_scaled_gemv(int recipe, int Kdim, int N, const uint8_t *aq, const void *as,
                     const uint8_t *wq, const void *ws, double *out)
{
    const int g = recipe == 0 ? 128 : 32;
    double *part = (double *)malloc(sizeof(double) * (size_t)N);
    for (int n = 0; n < N; n++) out[n] = 0.0;
    for (int grp = 0; grp < Kdim / g; grp++) {
        double sa = act_scale(recipe, as, (size_t)grp);
        for (int n = 0; n < N; n++) part[n] = 0.0;
        for (int k = grp * g; k < (grp + 1) * g; k++) {
            double a = e4m3_table[aq[k]];
            for (int n = 0; n < N; n++) part[n] += a * weight_value(recipe, wq, N, k, n);
        }
        for (int n = 0; n < N; n++)
            out[n] += sa * act_scale(recipe, ws, (size_t)grp * N + n) * part[n];
    }
    free(part);
}

/* ------------------------------------------------------------------------------------------
 * One expert's MLP on one routed row ([metrale] run_fp8_grouped_w8a8; [MATE] API:
 * activation "swiglu"; [MindIE] parameter table for w13/w2 and their biases):
 *   h    = gemm(x_q, W13_e) + b13_e                           (2I values, fp64)
 *   a_i  = silu(h_i) * h_{I+i},  silu(z) = z / (1 + exp(-z))   (gate = columns 0:I, up = I:2I)
 *   a_q  = quantize(a) per the recipe, decisions in fp32
 *   o    = gemm(a_q, W2_e) + b2_e                             (H values, fp64)
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    const uint8_t *w13;   const void *w13s;   /* [E,H,2I] codes (recipe 2: [E,H,I] bytes of
                                                 two E2M1 codes), scales [E,H/g,2I]      */
    const uint8_t *w2;    const void *w2s;    /* [E,I,H] codes (recipe 2: [E,I,H/2]), scales
                                                 [E,I/g,H]                               */
    const uint16_t *b13;  const uint16_t *b2; /* bf16 [E,2I], [E,H], or NULL         */
} orc_weights;

static size_t scale_bytes(int recipe) { return recipe == 0 ? 4 : 1; }

static void expert_mlp_row(const orc_cfg *c, const orc_weights *W, int e, const uint8_t *xq,
                           const void *xs, double *o, uint8_t *act_q_out, void *act_s_out)
{
    const int H = c->hidden, I = c->inter, g = c->recipe == 0 ? 128 : 32;
    const size_t sb = scale_bytes(c->recipe);
    double *h = (double *)malloc(sizeof(double) * 2 * (size_t)I);
    float *a = (float *)malloc(sizeof(float) * (size_t)I);
    uint8_t *aq = (uint8_t *)malloc((size_t)I);
    void *as = malloc(sb * (size_t)(I / g));

    orc_scaled_gemv(c->recipe, H, 2 * I, xq, xs, W->w13 + (size_t)e * weight_bytes(c->recipe, H, 2 * I),
                    (const uint8_t *)W->w13s + (size_t)e * (H / g) * 2 * I * sb, h);
    if (W->b13)
        for (int n = 0; n < 2 * I; n++) h[n] += (double)bf16_to_f32(W->b13[(size_t)e * 2 * I + n]);
    for (int i = 0; i < I; i++) {
        double z = h[i];
        a[i] = (float)(z / (1.0 + exp(-z)) * h[I + i]);
    }
    orc_quant_row(a, I, c->recipe, aq, as);
    orc_scaled_gemv(c->recipe, I, H, aq, as, W->w2 + (size_t)e * weight_bytes(c->recipe, I, H),
                    (const uint8_t *)W->w2s + (size_t)e * (I / g) * H * sb, o);
    if (W->b2)
        for (int n = 0; n < H; n++) o[n] += (double)bf16_to_f32(W->b2[(size_t)e * H + n]);
    if (act_q_out) memcpy(act_q_out, aq, (size_t)I);
    if (act_s_out) memcpy(act_s_out, as, sb * (size_t)(I / g));
    free(h); free(a); free(aq); free(as);
}

/* ------------------------------------------------------------------------------------------
 * The layer forward, written per token ([MindIE] execution flow; [MATE] Current Limits: the
 * output is a contiguous bf16 tensor):
 *   for each token t: route, quantize x_t, run each selected expert, and
 *   y_t = bf16_rn( sum_j w_j * o_j )   (fp64 sum in slot order j = 0..k-1)
 * With a shared expert (cfg->shared_experts = 1; [metrale] run_fp8_grouped_w8a8 runs it in the
 * same grouped steps as the routed experts), slot k is expert num_experts with weight 1, added
 * after the routed slots.
 *
 * `tokens` (n_sel entries) lists which tokens to compute, or is NULL for all of them; y and
 * the per-token outputs are indexed by position in that list.  When topk_idx_in is non-NULL
 * the routing is taken from it and topk_w_in (the custom routing function path of [MindIE]);
 * otherwise it is computed from the logits.  act_q/act_s (optional) receive each slot's
 * requantized SwiGLU product, [n_sel, k + S, I] and [n_sel, k + S, I/g] (S = shared_experts).
 * ---------------------------------------------------------------------------------------- */
int orc_forward(const orc_cfg *c, const uint16_t *x, const float *logits,
                const float *per_expert_scale, const int32_t *topk_idx_in,
                const float *topk_w_in, const uint8_t *w13, const void *w13s,
                const uint8_t *w2, const void *w2s, const uint16_t *b13, const uint16_t *b2,
                const int32_t *tokens, int n_sel, uint16_t *y, uint8_t *act_q, void *act_s)
{
    const int H = c->hidden, I = c->inter, K = c->top_k, g = c->recipe == 0 ? 128 : 32;
    const int KT = K + c->shared_experts;             /* slots per token */
    const size_t sb = scale_bytes(c->recipe);
    orc_weights W = {w13, w13s, w2, w2s, b13, b2};
    int rc = orc_check_cfg(c);
    if (rc) return rc;
    if (!tokens) n_sel = c->num_tokens;
    if (!topk_idx_in && !logits) return ORC_EINVAL;

#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < n_sel; p++) {
        const int t = tokens ? tokens[p] : p;
        int32_t ids[257];
        float wts[257];
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *xq = (uint8_t *)malloc((size_t)H);
        void *xs = malloc(sb * (size_t)(H / g));
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
        double *acc = (double *)calloc((size_t)H, sizeof(double));

        if (topk_idx_in) {
            for (int j = 0; j < K; j++) {
                ids[j] = topk_idx_in[(size_t)t * K + j];
                wts[j] = topk_w_in[(size_t)t * K + j];
            }
        } else {
            route_token(c, logits + (size_t)t * c->num_experts, per_expert_scale, ids, wts);
        }
        if (c->shared_experts) {                       /* the shared expert: slot k, weight 1 */
            ids[K] = c->num_experts;
            wts[K] = 1.0f;
        }
        for (int h = 0; h < H; h++) xf[h] = bf16_to_f32(x[(size_t)t * H + h]);
        orc_quant_row(xf, H, c->recipe, xq, xs);
        for (int j = 0; j < KT; j++) {
            uint8_t *aq = act_q ? act_q + ((size_t)p * KT + j) * I : NULL;
            void *as = act_s ? (uint8_t *)act_s + ((size_t)p * KT + j) * (I / g) * sb : NULL;
            expert_mlp_row(c, &W, ids[j], xq, xs, o, aq, as);
            for (int h = 0; h < H; h++) acc[h] += (double)wts[j] * o[h];
        }
        for (int h = 0; h < H; h++) y[(size_t)p * H + h] = orc_bf16_from_double(acc[h]);
        free(xf); free(xq); free(xs); free(o); free(acc);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Expert parallelism, the two sides of the exchange ([MindIE] execution flow: dispatch, mlp,
 * combine; the dynamic dispatcher's all-to-all).  A rank that owns some experts receives token
 * rows, each tagged with one of its experts, and returns each row's expert output; the token's
 * home rank then forms the weighted sum.
 *
 * orc_expert_rows: for each row n, quantize x_n as the layer does and run expert e_n's MLP:
 *   o[n] = expert_mlp(quantize(x_n), e_n)                    (fp64, H values)
 * c describes the owning rank: num_experts = its experts, weights indexed by local id.
 * Returns ORC_EINVAL for an expert id outside [0, num_experts).
 * ---------------------------------------------------------------------------------------- */
int orc_expert_rows(const orc_cfg *c, int N, const uint16_t *x, const int32_t *expert_of_row,
                    const uint8_t *w13, const void *w13s, const uint8_t *w2, const void *w2s,
                    const uint16_t *b13, const uint16_t *b2, double *o)
{
    const int H = c->hidden, g = c->recipe == 0 ? 128 : 32;
    const size_t sb = scale_bytes(c->recipe);
    orc_weights W = {w13, w13s, w2, w2s, b13, b2};
    int bad = 0;
    for (int n = 0; n < N; n++)
        if (expert_of_row[n] < 0 || expert_of_row[n] >= c->num_experts) bad = 1;
    if (bad) return ORC_EINVAL;

#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < N; n++) {
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *xq = (uint8_t *)malloc((size_t)H);
        void *xs = malloc(sb * (size_t)(H / g));
        for (int h = 0; h < H; h++) xf[h] = bf16_to_f32(x[(size_t)n * H + h]);
        orc_quant_row(xf, H, c->recipe, xq, xs);
        expert_mlp_row(c, &W, expert_of_row[n], xq, xs, o + (size_t)n * H, NULL, NULL);
        free(xf); free(xq); free(xs);
    }
    return ORC_OK;
}

/* orc_combine_rows: on the home rank, y_t = bf16_rn( sum_j w_tj * o[pos_tj] ), the sum in fp64
 * in slot order j = 0..K-1, as in orc_forward.  pos indexes the A = T*K returned rows. */
int orc_combine_rows(int T, int K, int H, const double *o, const int32_t *pos, const float *w,
                     uint16_t *y)
{
    const int A = T * K;
    for (int i = 0; i < A; i++)
        if (pos[i] < 0 || pos[i] >= A) return ORC_EINVAL;
    for (int t = 0; t < T; t++)
        for (int h = 0; h < H; h++) {
            double acc = 0.0;
            for (int j = 0; j < K; j++)
                acc += (double)w[(size_t)t * K + j] * o[(size_t)pos[(size_t)t * K + j] * H + h];
            y[(size_t)t * H + h] = orc_bf16_from_double(acc);
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * The same forward through the permuted formulation: route all tokens, permute rows into
 * expert-contiguous order, run each expert over its rows, then combine back in token order.
 * Used to check that the per-token loop and the dispatch/combine plumbing agree bit for bit.
 * ---------------------------------------------------------------------------------------- */
int orc_forward_permuted(const orc_cfg *c, const uint16_t *x, const float *logits,
                         const float *per_expert_scale, const uint8_t *w13, const void *w13s,
                         const uint8_t *w2, const void *w2s, const uint16_t *b13,
                         const uint16_t *b2, uint16_t *y)
{
    const int T = c->num_tokens, H = c->hidden, E = c->num_experts + c->shared_experts;
    const int K = c->top_k + c->shared_experts;   /* slots per token, the shared one last */
    const int g = c->recipe == 0 ? 128 : 32, A = T * K;
    const size_t sb = scale_bytes(c->recipe);
    orc_weights W = {w13, w13s, w2, w2s, b13, b2};
    int32_t *idx, *counts, *offsets, *row_src, *row_of;
    float *wts;
    double *o;
    int rc = orc_check_cfg(c);
    if (rc) return rc;
    idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    wts = (float *)malloc(sizeof(float) * (size_t)A);
    counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    row_src = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    row_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    o = (double *)malloc(sizeof(double) * (size_t)A * H);
    {
        const int k = c->top_k;
        int32_t *ridx = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k);
        float *rw = (float *)malloc(sizeof(float) * (size_t)T * k);
        orc_route(c, logits, per_expert_scale, ridx, rw, NULL);
        for (int t = 0; t < T; t++) {
            for (int j = 0; j < k; j++) {
                idx[t * K + j] = ridx[t * k + j];
                wts[t * K + j] = rw[t * k + j];
            }
            if (c->shared_experts) {
                idx[t * K + k] = c->num_experts;
                wts[t * K + k] = 1.0f;
            }
        }
        free(ridx); free(rw);
    }
    orc_permute(T, K, E, idx, counts, offsets, row_src, row_of);

    /* mlp: expert by expert over its contiguous rows */
    for (int e = 0; e < E; e++) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int r = offsets[e]; r < offsets[e + 1]; r++) {
            int t = row_src[r] / K;
            float *xf = (float *)malloc(sizeof(float) * (size_t)H);
            uint8_t *xq = (uint8_t *)malloc((size_t)H);
            void *xs = malloc(sb * (size_t)(H / g));
            for (int h = 0; h < H; h++) xf[h] = bf16_to_f32(x[(size_t)t * H + h]);
            orc_quant_row(xf, H, c->recipe, xq, xs);
            expert_mlp_row(c, &W, e, xq, xs, o + (size_t)r * H, NULL, NULL);
            free(xf); free(xq); free(xs);
        }
    }
    /* combine: token order, slot order */
    for (int t = 0; t < T; t++)
        for (int h = 0; h < H; h++) {
            double acc = 0.0;
            for (int j = 0; j < K; j++)
                acc += (double)wts[t * K + j] * o[(size_t)row_of[t * K + j] * H + h];
            y[(size_t)t * H + h] = orc_bf16_from_double(acc);
        }
    free(idx); free(wts); free(counts); free(offsets); free(row_src); free(row_of); free(o);
    return ORC_OK;
}

/* Quantize every token's row of x (bf16 [T,H]) as the dispatch does before the first GEMM. */
void orc_quantize_tokens(int T, int H, int recipe, const uint16_t *x, uint8_t *q, void *scales)
{
    const int g = recipe == 0 ? 128 : 32;
    const size_t sb = scale_bytes(recipe);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        for (int h = 0; h < H; h++) xf[h] = bf16_to_f32(x[(size_t)t * H + h]);
        orc_quant_row(xf, H, recipe, q + (size_t)t * H, (uint8_t *)scales + (size_t)t * (H / g) * sb);
        free(xf);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
