/*
 * Plain CPU oracle for the expert-parallel MoE layer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm may load this.  It shares no code,
 * header, table or constant with the CUDA library: every constant below is
 * derived here from its mathematical definition.
 *
 * Single-threaded, slow, and written to be read against its sources:
 *
 *  - axolotl docs, "integrations.expert_parallel.args", ExpertParallelArgs:
 *      expert_parallel_backend (torch: all_to_all_single over the EP group),
 *      expert_parallel_dispatch_chunks, expert_parallel_size,
 *      expert_parallel_token_capacity ("lowest-weight excess (token,expert)
 *      assignments are dropped").
 *  - LightLLM PR 1687 review page: _select_experts (top-k over the logical
 *      experts, norm_topk_prob renormalisation), the expert prefix-sum
 *      ("psum") contiguous layout for the grouped GEMM, SwiGLU
 *      (silu_and_mul) between the two grouped GEMMs, decode reducing expert
 *      outputs straight into a dense output, the FP8 grouped GEMM with UE8M0
 *      (power-of-two) scales and the quantisation of h after silu_and_mul.
 *  - the same axolotl page, expert_parallel_save_dispatch: the layer's
 *      backward with the dispatch outputs saved or recomputed.
 *
 * Readings of points the pages leave open are marked "Reading:".
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC -lm.
 * -ffp-contract=off matters: the routing weights must come out of exactly the
 * IEEE operations written here, one rounding each.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NONFINITE 2

/* ------------------------------------------------------------------------- */
/* Deterministic exponential for r <= 0 (Cody & Waite argument reduction,    */
/* "Software Manual for the Elementary Functions", 1980, then a Taylor        */
/* polynomial).  Reading: the pages only say "softmax"; a bit-reproducible    */
/* exp is needed because the capacity clip compares weights across tokens.    */
/* ------------------------------------------------------------------------- */

/* 1/ln 2 rounded to fp32. */
static float orc_log2e(void) { return (float)(1.0 / 0.69314718055994530941723212145818); }
/* ln 2 truncated to 16 significant bits: 45426 / 2^16.  n * LN2_HI is exact for
 * |n| <= 127 and r - n*LN2_HI is exact for |r| < 88, so the reduction loses
 * nothing in its first step. */
static float orc_ln2_hi(void) { return 45426.0f / 65536.0f; }
/* the rest of ln 2, rounded to fp32 */
static float orc_ln2_lo(void) { return (float)(0.69314718055994530941723212145818 - 45426.0 / 65536.0); }

float orc_exp_det(float r)
{
    if (r < -87.0f) return 0.0f;
    float t = r * orc_log2e();              /* one fp32 multiply */
    float n = rintf(t);                     /* round half to even */
    float f = fmaf(-n, orc_ln2_hi(), r);    /* exact */
    f = fmaf(-n, orc_ln2_lo(), f);          /* one rounding */
    /* Taylor coefficients 1/j!, j = 7..0, each rounded to fp32 once. */
    double fact = 1.0;
    float c[8];
    for (int j = 0; j < 8; ++j) { if (j > 0) fact *= (double)j; c[j] = (float)(1.0 / fact); }
    float p = c[7];
    for (int j = 6; j >= 0; --j) p = fmaf(p, f, c[j]);
    /* 2^n by assembling the exponent field; n is in [-126, 0] here. */
    int ni = (int)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;
    float two_n;
    memcpy(&two_n, &bits, sizeof two_n);
    return p * two_n;                       /* one fp32 multiply (may round to subnormal) */
}

/* ------------------------------------------------------------------------- */
/* Step 1: router top-k with renormalised softmax weights.                    */
/* LightLLM PR 1687, "_select_experts" (top-k over logical experts, weights    */
/* renormalised with norm_topk_prob); axolotl: "routing topk ... always saved".*/
/* ------------------------------------------------------------------------- */

/* Returns 1 if (va, a) ranks before (vb, b): larger value first, lower expert
 * index first among equal values (IEEE ==, so -0 == +0). */
static int orc_before(float va, int a, float vb, int b)
{
    if (va > vb) return 1;
    if (va < vb) return 0;
    return a < b;
}

/*
 * logits fp32 [T, E]; bias fp32 [E] or NULL.
 * topk_idx int32 [T, k], topk_w fp32 [T, k] in rank order; counts int32 [E]
 * (assignments per expert before any clip).
 *
 * Weights: with v_j the logits of the selected experts in slot order and
 * m = max_j v_j,
 *   w_j = exp(v_j - m) / sum_{i<k} exp(v_i - m),
 * which equals the full softmax restricted to the top k and renormalised (the
 * softmax denominator cancels).  Reading: the bias (skewed-router workload)
 * enters both the selection and the weights (v_j = l'_j, so m = l'_0); the sum
 * runs in slot order.
 *
 * Routing variants (LightLLM PR 1687: "grouped top-k" kept inside experts()
 * for DeepSeek-V2, GLM-4-MoE-Lite and Qwen3-MoE).  The page names them only;
 * the plainest readings, stated:
 *  - grouped top-k (n_group > 1): experts form n_group contiguous groups of
 *    E / n_group.  A group's score is its best biased logit (group_score 0) or
 *    the fp32 sum of its two best (group_score 1).  The topk_group groups with
 *    the best scores are kept (larger score first, lower group index among
 *    equal scores); the top-k is then taken among their experts only.
 *  - bias_select_only: the bias steers the choice of experts (and of groups)
 *    but the weights use the unbiased logits, v_j = logit_j (+0 for -0).
 */
int orc_route_topk_ex(int T, int E, int k, const float *logits, const float *bias,
                      int n_group, int topk_group, int group_score, int bias_select_only,
                      int32_t *topk_idx, float *topk_w, int32_t *counts)
{
    if (T < 0 || E <= 0 || k <= 0 || k > E) return ORC_ERR_ARG;
    const int grouped = n_group > 1;
    if (grouped) {
        if (E % n_group != 0 || topk_group < 1 || topk_group > n_group ||
            k > topk_group * (E / n_group) || (group_score != 0 && group_score != 1) ||
            (group_score == 1 && E / n_group < 2))
            return ORC_ERR_ARG;
    }
    const int gs = grouped ? E / n_group : E;
    float *l = (float *)malloc(sizeof(float) * (size_t)E);
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    float *ev = (float *)malloc(sizeof(float) * (size_t)k);
    float *gscore = (float *)malloc(sizeof(float) * (size_t)(grouped ? n_group : 1));
    unsigned char *gkeep = (unsigned char *)malloc((size_t)(grouped ? n_group : 1));
    int status = ORC_OK;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            float b = bias ? bias[e] : 0.0f;
            l[e] = logits[(size_t)t * E + e] + b;   /* -0 + +0 = +0: canonicalises -0 */
            if (!isfinite(l[e])) status = ORC_ERR_NONFINITE;
            taken[e] = 0;
        }
        if (grouped) {
            /* group scores, then keep the best topk_group groups by repeated selection */
            for (int g = 0; g < n_group; ++g) {
                int b1 = -1, b2 = -1;       /* the group's best and second-best experts */
                for (int e = g * gs; e < (g + 1) * gs; ++e) {
                    if (b1 < 0 || l[e] > l[b1]) { b2 = b1; b1 = e; }
                    else if (b2 < 0 || l[e] > l[b2]) b2 = e;
                }
                gscore[g] = group_score == 0 ? l[b1] : l[b1] + l[b2];
                gkeep[g] = 0;
            }
            for (int j = 0; j < topk_group; ++j) {
                int best = -1;
                for (int g = 0; g < n_group; ++g) {
                    if (gkeep[g]) continue;
                    if (best < 0 || orc_before(gscore[g], g, gscore[best], best)) best = g;
                }
                gkeep[best] = 1;
            }
            /* experts of the dropped groups cannot be chosen */
            for (int e = 0; e < E; ++e)
                if (!gkeep[e / gs]) taken[e] = 1;
        }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || orc_before(l[e], e, l[best], best)) best = e;
            }
            taken[best] = 1;
            topk_idx[(size_t)t * k + j] = best;
            counts[best] += 1;
        }
        /* the weights' logits: biased, or unbiased when the bias only selects */
        float m = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(size_t)t * k + j];
            const float v = bias_select_only ? logits[(size_t)t * E + e] + 0.0f : l[e];
            ev[j] = v;
            if (j == 0 || v > m) m = v;
        }
        float S = 0.0f;
        for (int j = 0; j < k; ++j) {
            ev[j] = orc_exp_det(ev[j] - m);
            S = S + ev[j];
        }
        for (int j = 0; j < k; ++j) topk_w[(size_t)t * k + j] = ev[j] / S;
    }
    free(l); free(taken); free(ev); free(gscore); free(gkeep);
    return status;
}

int orc_route_topk(int T, int E, int k, const float *logits, const float *bias,
                   int32_t *topk_idx, float *topk_w, int32_t *counts)
{
    return orc_route_topk_ex(T, E, k, logits, bias, 0, 0, 0, 0, topk_idx, topk_w, counts);
}

/* ------------------------------------------------------------------------- */
/* Step 2: per-expert token capacity (axolotl ExpertParallelArgs,              */
/* expert_parallel_token_capacity): at most C assignments per expert per       */
/* forward; the lowest-weight excess (token, expert) pairs are dropped.        */
/* Tie rule: among equal weights the higher token index is dropped first.      */
/* Reading: the weight compared is the renormalised top-k weight (the combine  */
/* weight); survivors are not re-renormalised.  C < 0 means no cap; C = 0    */
/* drops every assignment.                                                     */
/* ------------------------------------------------------------------------- */

typedef struct { float w; int t; int j; } orc_assign;

static int orc_cmp_keep_first(const void *pa, const void *pb)
{
    const orc_assign *a = (const orc_assign *)pa, *b = (const orc_assign *)pb;
    if (a->w > b->w) return -1;
    if (a->w < b->w) return 1;
    return (a->t < b->t) ? -1 : (a->t > b->t);
}

int orc_capacity_clip(int T, int E, int k, int C, const int32_t *topk_idx,
                      const float *topk_w, uint8_t *keep, int32_t *kept_counts)
{
    if (T < 0 || E <= 0 || k <= 0) return ORC_ERR_ARG;
    for (size_t i = 0; i < (size_t)T * k; ++i) keep[i] = 1;
    orc_assign *seg = (orc_assign *)malloc(sizeof(orc_assign) * ((size_t)T + 1));
    for (int e = 0; e < E; ++e) {
        int n = 0;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (topk_idx[(size_t)t * k + j] == e) {
                    seg[n].w = topk_w[(size_t)t * k + j]; seg[n].t = t; seg[n].j = j; ++n;
                }
        if (C >= 0 && n > C) {
            qsort(seg, (size_t)n, sizeof(orc_assign), orc_cmp_keep_first);
            for (int i = C; i < n; ++i) keep[(size_t)seg[i].t * k + seg[i].j] = 0;
            kept_counts[e] = C;
        } else {
            kept_counts[e] = n;
        }
    }
    free(seg);
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Step 3: dispatch layout.  The torch backend sends rows with                 */
/* all_to_all_single over the EP group (axolotl, expert_parallel_backend) and  */
/* the receiver runs its experts on the expert-contiguous prefix-sum layout    */
/* (LightLLM PR 1687, "use_psum_layout").  Readings:                           */
/*  - source rank of token t in a chunk [b, b+n): s = (t - b) / (n / EP)       */
/*    (contiguous equal token blocks, as in a data-parallel split);            */
/*  - destination rank of expert e: d = e / (E / EP);                          */
/*  - receive order: by destination rank, then expert, then token; with the    */
/*    two readings above this is simply the stable order by (e, t).            */
/* Outputs: expert_offsets [E+1], rank_offsets [EP+1], recv_token [N]          */
/* (absolute token index), recv_slot [N], pos [n, k] (chunk-relative rows; -1  */
/* where dropped), send_splits [EP, EP] (row s = source, column d = dest).     */
/* Returns N (>= 0) or -ORC_ERR_ARG.                                           */
/* ------------------------------------------------------------------------- */

int orc_dispatch_layout(int T, int E, int k, int EP, int tok_begin, int tok_count,
                        const int32_t *topk_idx, const uint8_t *keep,
                        int32_t *expert_offsets, int32_t *rank_offsets,
                        int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                        int32_t *send_splits)
{
    if (EP <= 0 || E % EP != 0 || tok_count < 0 || tok_begin < 0 ||
        tok_begin + tok_count > T || tok_count % EP != 0)
        return -ORC_ERR_ARG;
    int tpr = tok_count / EP;          /* tokens per source rank */
    int epr = E / EP;                  /* experts per destination rank */
    for (size_t i = 0; i < (size_t)tok_count * k; ++i) pos[i] = -1;
    for (int i = 0; i < EP * EP; ++i) send_splits[i] = 0;
    int n = 0;
    for (int e = 0; e < E; ++e) {
        expert_offsets[e] = n;
        for (int t = tok_begin; t < tok_begin + tok_count; ++t)
            for (int j = 0; j < k; ++j) {
                size_t a = (size_t)t * k + j;
                if (topk_idx[a] == e && keep[a]) {
                    recv_token[n] = t;
                    recv_slot[n] = j;
                    pos[(size_t)(t - tok_begin) * k + j] = n;
                    int s = (t - tok_begin) / tpr;
                    int d = e / epr;
                    send_splits[s * EP + d] += 1;
                    ++n;
                }
            }
    }
    expert_offsets[E] = n;
    for (int d = 0; d <= EP; ++d) rank_offsets[d] = expert_offsets[d * epr];
    return n;
}

/* ------------------------------------------------------------------------- */
/* Step 4: permute.  xr[p, :] = x[recv_token[p], :] (bytewise copy).            */
/* ------------------------------------------------------------------------- */
void orc_permute(int H, int elem_bytes, int N, const void *x, const int32_t *recv_token,
                 void *xr)
{
    size_t row = (size_t)H * elem_bytes;
    for (int p = 0; p < N; ++p)
        memcpy((char *)xr + (size_t)p * row, (const char *)x + (size_t)recv_token[p] * row, row);
}

/* ------------------------------------------------------------------------- */
/* Storage types.  dtype 0 = fp32, 1 = bf16 (stored as uint16 bit patterns),   */
/* 2 = fp64 (for the backward's finite-difference checks: no rounding at all). */
/* ------------------------------------------------------------------------- */
static double orc_load(const void *base, size_t i, int dtype)
{
    if (dtype == 2) return ((const double *)base)[i];
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even) in one step and return its
 * bit pattern.  Normal range only matters here; tiny values flush through the
 * fp32 path, overflow gives +-inf. */
uint16_t orc_bf16_from_double(double v)
{
    if (v != v) return 0x7FC0;
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    float out;
    if (a < 1.1754943508222875e-38) {
        out = (float)v;                                     /* subnormal region */
        uint32_t u; memcpy(&u, &out, 4);
        uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);
        return (uint16_t)(r >> 16);
    }
    int ex;
    double m = frexp(a, &ex);                 /* a = m * 2^ex, m in [0.5, 1) */
    double q = nearbyint(ldexp(m, 8));        /* 8 significant bits, ties to even */
    double r = ldexp(q, ex - 8);
    if (r > 3.3895313892515355e38) {          /* above the largest finite bf16 */
        return signbit(v) ? 0xFF80 : 0x7F80;
    }
    out = (float)(signbit(v) ? -r : r);       /* exact: r has 8 significant bits */
    uint32_t u; memcpy(&u, &out, 4);
    return (uint16_t)(u >> 16);
}

static void orc_store(void *base, size_t i, int dtype, double v)
{
    if (dtype == 2) ((double *)base)[i] = v;
    else if (dtype == 0) ((float *)base)[i] = (float)v;
    else ((uint16_t *)base)[i] = orc_bf16_from_double(v);
}

/* ------------------------------------------------------------------------- */
/* Step 5: one expert's SwiGLU FFN on one row (LightLLM PR 1687: grouped GEMM  */
/* on the psum layout, then silu_and_mul, then the second grouped GEMM).       */
/*   g_i = sum_c W13[i, c] x[c],  u_i = sum_c W13[I + i, c] x[c]   (i < I)     */
/*   h_i = silu(g_i) * u_i,  silu(a) = a / (1 + exp(-a))                       */
/*   y_o = sum_i W2[o, i] h_i                                                  */
/* Dot products in double.  h is rounded to the storage type before the        */
/* second GEMM when round_h (the CUDA path stores h); y_store (optional) gets  */
/* y rounded to the storage type, y_exact (optional) the unrounded y.          */
/* w13 is one expert's [2I, H], w2 one expert's [H, I].                        */
/* ------------------------------------------------------------------------- */
void orc_ffn_row(int H, int I, int dtype, const void *x_row, const void *w13_e,
                 const void *w2_e, int round_h, void *h_store, void *y_store,
                 double *y_exact)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            double xv = orc_load(x_row, (size_t)c, dtype);
            g += orc_load(w13_e, (size_t)i * H + c, dtype) * xv;
            u += orc_load(w13_e, (size_t)(I + i) * H + c, dtype) * xv;
        }
        double hv = g / (1.0 + exp(-g)) * u;
        if (h_store) orc_store(h_store, (size_t)i, dtype, hv);
        if (round_h && dtype != 2) {
            if (dtype == 0) hv = (double)(float)hv;
            else {
                uint32_t bits = (uint32_t)orc_bf16_from_double(hv) << 16;
                float f; memcpy(&f, &bits, 4); hv = (double)f;
            }
        }
        h[i] = hv;
    }
    for (int o = 0; o < H; ++o) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += orc_load(w2_e, (size_t)o * I + i, dtype) * h[i];
        if (y_exact) y_exact[o] = acc;
        if (y_store) orc_store(y_store, (size_t)o, dtype, acc);
    }
    free(h);
}

/* ------------------------------------------------------------------------- */
/* Step 6: weighted combine back to token order.                               */
/*   out[t, :] = sum over kept slots j (in slot order) of w[t, j] * y[pos[t,j]] */
/* accumulated in double, rounded once to the storage type; a token with every */
/* slot dropped gets zeros.  pos is chunk-relative [n, k], -1 where dropped.   */
/* Shared expert (LightLLM PR 1687: the shared expert's output is added in the */
/* combine, which overlaps it): y_shared [n, H], the chunk's rows of the       */
/* shared expert's stored output, or NULL; reading: it enters the same sum     */
/* before the one rounding.                                                    */
/* ------------------------------------------------------------------------- */
void orc_combine(int H, int k, int dtype, int tok_begin, int tok_count, const void *y,
                 const int32_t *pos, const float *topk_w, const void *y_shared, void *out)
{
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    for (int i = 0; i < tok_count; ++i) {
        int t = tok_begin + i;
        for (int c = 0; c < H; ++c)
            acc[c] = y_shared ? orc_load(y_shared, (size_t)i * H + c, dtype) : 0.0;
        for (int j = 0; j < k; ++j) {
            int p = pos[(size_t)i * k + j];
            if (p < 0) continue;
            double w = (double)topk_w[(size_t)t * k + j];
            for (int c = 0; c < H; ++c) acc[c] += w * orc_load(y, (size_t)p * H + c, dtype);
        }
        for (int c = 0; c < H; ++c) orc_store(out, (size_t)t * H + c, dtype, acc[c]);
    }
    free(acc);
}

/* Decode form of step 6 (LightLLM PR 1687: decode reduces expert outputs into
 * a dense output): the same sum, but over unrounded expert outputs, because
 * the reduce consumes y before it is ever stored.  y_exact is [N, H] double. */
void orc_combine_exact(int H, int k, int dtype, int tok_begin, int tok_count,
                       const double *y_exact, const int32_t *pos, const float *topk_w,
                       const void *y_shared, void *out)
{
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    for (int i = 0; i < tok_count; ++i) {
        int t = tok_begin + i;
        for (int c = 0; c < H; ++c)
            acc[c] = y_shared ? orc_load(y_shared, (size_t)i * H + c, dtype) : 0.0;
        for (int j = 0; j < k; ++j) {
            int p = pos[(size_t)i * k + j];
            if (p < 0) continue;
            double w = (double)topk_w[(size_t)t * k + j];
            for (int c = 0; c < H; ++c) acc[c] += w * y_exact[(size_t)p * H + c];
        }
        for (int c = 0; c < H; ++c) orc_store(out, (size_t)t * H + c, dtype, acc[c]);
    }
    free(acc);
}

/* ------------------------------------------------------------------------- */
/* FP8 expert FFN (LightLLM PR 1687: the DeepGEMM FP8 grouped GEMM over the    */
/* psum layout, UE8M0 quantisation, silu_and_mul followed by quantisation of  */
/* h before the second grouped GEMM).                                          */
/*                                                                             */
/* E4M3 (the variant without infinities): 1 sign bit, 4 exponent bits with     */
/* bias 7, 3 fraction bits; exponent field 15 with fraction 7 is NaN, so the   */
/* largest finite magnitude is 1.75 * 2^8 = 448; normals reach down to 2^-6,   */
/* subnormals are j * 2^-9 for j = 1..7.                                       */
/* UE8M0: an unsigned 8-bit biased exponent (bias 127) with no mantissa, i.e.  */
/* a power-of-two scale.                                                       */
/* Reading: the pages fix power-of-two (UE8M0) scales but not their            */
/* granularity; here one scale per row: per token for activations, per output  */
/* channel (weight row) for weights.                                           */
/* ------------------------------------------------------------------------- */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, f = c & 7;
    if (e == 15 && f == 7) return NAN;
    double v = e == 0 ? ldexp((double)f, -9) : ldexp(8.0 + f, e - 10);
    return s ? -v : v;
}

/* Nearest E4M3 value, ties to the even fraction; magnitudes beyond 448 give
 * +-448 ("satfinite"); NaN gives 0x7F. */
uint8_t orc_e4m3_encode(double v)
{
    if (v != v) return 0x7F;
    uint8_t s = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return s | 0x7E;
    if (a == 0.0) return s;
    int ex;
    frexp(a, &ex);                         /* a in [2^(ex-1), 2^ex) */
    int e = ex - 1;
    if (e < -6) e = -6;                    /* the subnormal quantum is 2^-9 */
    double n = nearbyint(ldexp(a, 3 - e)); /* a in quanta of 2^(e-3), ties to even */
    double r = ldexp(n, e - 3);            /* <= 448: the largest a below 448 rounds to it */
    if (r == 0.0) return s;
    frexp(r, &ex);
    e = ex - 1;
    if (e < -6) return s | (uint8_t)ldexp(r, 9);            /* subnormal: j * 2^-9 */
    int f = (int)ldexp(r, 3 - e) - 8;                        /* r = (8 + f) 2^(e-3) */
    return s | (uint8_t)((e + 7) << 3) | (uint8_t)f;
}

/* UE8M0 scale of a row with largest magnitude amax: the smallest power of two
 * 2^e with amax <= 448 * 2^e, so that every scaled value fits E4M3 and the
 * largest uses its top binade; e clamped to [-126, 127]; a zero row takes
 * e = 0.  Returns the biased byte e + 127. */
uint8_t orc_ue8m0_scale(double amax)
{
    if (!(amax > 0.0)) return 127;
    int e = (int)ceil(log2(amax / 448.0));
    while (ldexp(448.0, e) < amax) ++e;          /* exact comparisons fix any */
    while (ldexp(448.0, e - 1) >= amax) --e;     /* rounding of the logarithm */
    if (e < -126) e = -126;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* Row-wise quantisation: scales[r] = UE8M0 scale of row r, codes[r, c] =
 * E4M3(in[r, c] / 2^e) (the division by a power of two is exact). */
void orc_quantize_rows(int64_t rows, int cols, int dtype, const void *in, uint8_t *codes,
                       uint8_t *scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        double amax = 0.0;
        for (int c = 0; c < cols; ++c) {
            double a = fabs(orc_load(in, (size_t)r * cols + c, dtype));
            if (a > amax) amax = a;
        }
        uint8_t b = orc_ue8m0_scale(amax);
        scales[r] = b;
        for (int c = 0; c < cols; ++c)
            codes[(size_t)r * cols + c] =
                orc_e4m3_encode(ldexp(orc_load(in, (size_t)r * cols + c, dtype), 127 - (int)b));
    }
}

static double orc_dq(uint8_t code, uint8_t scale) { return ldexp(orc_e4m3_decode(code), (int)scale - 127); }

/* One expert's SwiGLU FFN on one receive row in FP8: the steps of
 * orc_ffn_row on dequantised operands (value = E4M3(code) * 2^(scale - 127)).
 *   x [H] codes with scale sx; w13 [2I, H] codes with row scales w13_s [2I];
 *   w2 [H, I] codes with row scales w2_s [H].
 *   g_i, u_i: dot products in double; h_i = silu(g_i) u_i rounded to bf16
 *   (h_store, bf16 bits: the CUDA path stores h); h then quantised as one row
 *   (hq_store [I] codes, *sh_store its scale); y_o = sum_i dq(W2[o,i]) dq(hq_i)
 *   in double (y_exact, optional) and rounded to bf16 (y_store, optional). */
void orc_ffn_row_fp8(int H, int I, const uint8_t *x, uint8_t sx, const uint8_t *w13,
                     const uint8_t *w13_s, const uint8_t *w2, const uint8_t *w2_s,
                     uint16_t *h_store, uint8_t *hq_store, uint8_t *sh_store, uint16_t *y_store,
                     double *y_exact)
{
    /* dequantised value = dec[code] * 2^(scale - 127), both factors exact */
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = orc_e4m3_decode((uint8_t)c);
    double *xv = (double *)malloc(sizeof(double) * (size_t)H);
    for (int c = 0; c < H; ++c) xv[c] = orc_dq(x[c], sx);
    uint16_t *h = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)I);
    uint8_t *hq = (uint8_t *)malloc((size_t)I);
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    uint8_t sh;
    for (int i = 0; i < I; ++i) {
        const double sg = ldexp(1.0, (int)w13_s[i] - 127), su = ldexp(1.0, (int)w13_s[I + i] - 127);
        const uint8_t *wg = w13 + (size_t)i * H, *wu = w13 + (size_t)(I + i) * H;
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += dec[wg[c]] * sg * xv[c];
            u += dec[wu[c]] * su * xv[c];
        }
        h[i] = orc_bf16_from_double(g / (1.0 + exp(-g)) * u);
    }
    orc_quantize_rows(1, I, 1, h, hq, &sh);
    for (int i = 0; i < I; ++i) hv[i] = orc_dq(hq[i], sh);
    for (int o = 0; o < H; ++o) {
        const double so = ldexp(1.0, (int)w2_s[o] - 127);
        const uint8_t *wo = w2 + (size_t)o * I;
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += dec[wo[i]] * so * hv[i];
        if (y_exact) y_exact[o] = acc;
        if (y_store) y_store[o] = orc_bf16_from_double(acc);
    }
    if (h_store) memcpy(h_store, h, sizeof(uint16_t) * (size_t)I);
    if (hq_store) memcpy(hq_store, hq, (size_t)I);
    if (sh_store) *sh_store = sh;
    free(xv);
    free(h);
    free(hq);
    free(hv);
}

/* ------------------------------------------------------------------------- */
/* Backward of the layer (axolotl ExpertParallelArgs, expert_parallel_save_   */
/* dispatch: under activation checkpointing the backward either holds the     */
/* dispatch / combine all-to-all outputs from the forward or re-issues them;  */
/* the routing top-k and the split counts are always saved).                  */
/* Reading: the backward is the gradient of the layer's exact function at the */
/* stored inputs: fp64 throughout, h and y not rounded; the top-k selection   */
/* and the capacity clip are piecewise constant (no gradient through them).   */
/*   out[t] = sum over kept slots j of w[t,j] * FFN_{e_j}(x[t])               */
/*   w[t,:] = softmax over the k selected (biased, or with bias_select_only   */
/*            unbiased) logits z[t,:]                                          */
/* For L = <dout, out>:                                                        */
/*   dy[t,j] = w[t,j] dout[t];  dw[t,j] = <dout[t], FFN_{e_j}(x[t])> (kept j,   */
/*   else 0);  dz[t,j] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]).              */
/* ------------------------------------------------------------------------- */

/* One expert's SwiGLU FFN backward on one row, for an incoming dy [H]:
 *   g_i, u_i as in orc_ffn_row (double);  s_i = 1 / (1 + exp(-g_i));
 *   h_i = g_i s_i u_i;  dh_i = sum_o W2[o,i] dy_o;
 *   dg_i = dh_i u_i s_i (1 + g_i (1 - s_i))     (d silu(g) / dg)
 *   du_i = dh_i g_i s_i
 *   dx_c += sum_i W13[i,c] dg_i + W13[I+i,c] du_i
 *   dW2[o,i] += dy_o h_i;  dW13[i,c] += dg_i x_c;  dW13[I+i,c] += du_i x_c.
 * dx, dW13 [2I, H] and dW2 [H, I] accumulate (double); y_exact (optional)
 * gets the row's forward output. */
void orc_ffn_row_bwd(int H, int I, int dtype, const void *x_row, const void *w13_e,
                     const void *w2_e, const double *dy, double *dx, double *dW13,
                     double *dW2, double *y_exact)
{
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        double gi = 0.0, ui = 0.0;
        for (int c = 0; c < H; ++c) {
            double xv = orc_load(x_row, (size_t)c, dtype);
            gi += orc_load(w13_e, (size_t)i * H + c, dtype) * xv;
            ui += orc_load(w13_e, (size_t)(I + i) * H + c, dtype) * xv;
        }
        g[i] = gi;
        u[i] = ui;
        h[i] = gi / (1.0 + exp(-gi)) * ui;
    }
    if (y_exact)
        for (int o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int i = 0; i < I; ++i) acc += orc_load(w2_e, (size_t)o * I + i, dtype) * h[i];
            y_exact[o] = acc;
        }
    for (int i = 0; i < I; ++i) {
        double dh = 0.0;
        for (int o = 0; o < H; ++o) dh += orc_load(w2_e, (size_t)o * I + i, dtype) * dy[o];
        const double s = 1.0 / (1.0 + exp(-g[i]));
        const double dg = dh * u[i] * s * (1.0 + g[i] * (1.0 - s));
        const double du = dh * g[i] * s;
        for (int c = 0; c < H; ++c) {
            const double xv = orc_load(x_row, (size_t)c, dtype);
            dx[c] += orc_load(w13_e, (size_t)i * H + c, dtype) * dg +
                     orc_load(w13_e, (size_t)(I + i) * H + c, dtype) * du;
            dW13[(size_t)i * H + c] += dg * xv;
            dW13[(size_t)(I + i) * H + c] += du * xv;
        }
    }
    for (int o = 0; o < H; ++o)
        for (int i = 0; i < I; ++i) dW2[(size_t)o * I + i] += dy[o] * h[i];
    free(g);
    free(u);
    free(h);
}

/* The routed part of the backward for tokens [0, T): every kept slot (t, j)
 * of expert e = topk_idx[t, j] takes its row backward with dy = w dout[t]
 * (x[t] read as x_rows[row_of[t*k + j]]: the saved receive rows, or x itself
 * with row_of = the token, when they are recomputed) and gives dw[t, j];
 * then dz[t, :] by the softmax backward over the token's k slots.
 * dx [T, H], dW13 [E, 2I, H], dW2 [E, H, I] accumulate; dz [T, k] is written. */
void orc_layer_bwd(int T, int H, int E, int k, int I, int dtype, const int32_t *topk_idx,
                   const float *topk_w, const uint8_t *keep, const void *x_rows,
                   const int32_t *row_of, const void *w13, const void *w2, const double *dout,
                   double *dx, double *dz, double *dW13, double *dW2)
{
    const size_t eb = dtype == 2 ? 8 : dtype == 0 ? 4 : 2;
    double *dy = (double *)malloc(sizeof(double) * (size_t)H);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *dw = (double *)malloc(sizeof(double) * (size_t)k);
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            dw[j] = 0.0;
            if (!keep[(size_t)t * k + j]) continue;
            const int e = topk_idx[(size_t)t * k + j];
            const double w = (double)topk_w[(size_t)t * k + j];
            for (int c = 0; c < H; ++c) dy[c] = w * dout[(size_t)t * H + c];
            const void *xr = (const char *)x_rows + (size_t)row_of[(size_t)t * k + j] * H * eb;
            orc_ffn_row_bwd(H, I, dtype, xr, (const char *)w13 + (size_t)e * 2 * I * H * eb,
                            (const char *)w2 + (size_t)e * H * I * eb, dy, dx + (size_t)t * H,
                            dW13 + (size_t)e * 2 * I * H, dW2 + (size_t)e * H * I, y);
            double acc = 0.0;
            for (int c = 0; c < H; ++c) acc += dout[(size_t)t * H + c] * y[c];
            dw[j] = acc;
        }
        double sw = 0.0;
        for (int j = 0; j < k; ++j) sw += (double)topk_w[(size_t)t * k + j] * dw[j];
        for (int j = 0; j < k; ++j)
            dz[(size_t)t * k + j] = (double)topk_w[(size_t)t * k + j] * (dw[j] - sw);
    }
    free(dy);
    free(y);
    free(dw);
}

/* Backward of step 6 for tokens [tok_begin, tok_begin + tok_count): for each
 * kept slot (pos >= 0) dy[p] = w[t,j] dout[t] (rounded once to the storage
 * type) and dw[t,j] = sum_c dout[t,c] y[p,c] (double, y as stored); dw of a
 * dropped slot is 0.  dout [T, H], y / dy [N, H], dw [T, k]. */
void orc_combine_bwd(int H, int k, int dtype, int tok_begin, int tok_count, const void *dout,
                     const void *y, const int32_t *pos, const float *topk_w, void *dy, double *dw)
{
    for (int i = 0; i < tok_count; ++i) {
        int t = tok_begin + i;
        for (int j = 0; j < k; ++j) {
            int p = pos[(size_t)i * k + j];
            double acc = 0.0;
            if (p >= 0) {
                double w = (double)topk_w[(size_t)t * k + j];
                for (int c = 0; c < H; ++c) {
                    double d = orc_load(dout, (size_t)t * H + c, dtype);
                    orc_store(dy, (size_t)p * H + c, dtype, w * d);
                    acc += d * orc_load(y, (size_t)p * H + c, dtype);
                }
            }
            dw[(size_t)t * k + j] = acc;
        }
    }
}

/* Backward of step 1 (reading: the softmax over the k selected logits):
 * dz[t,j] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]); dlogits [T, E] is dz at
 * the selected experts and 0 elsewhere. */
void orc_route_bwd(int T, int E, int k, const int32_t *topk_idx, const float *topk_w,
                   const double *dw, double *dlogits)
{
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) dlogits[(size_t)t * E + e] = 0.0;
        double sw = 0.0;
        for (int j = 0; j < k; ++j) sw += (double)topk_w[(size_t)t * k + j] * dw[(size_t)t * k + j];
        for (int j = 0; j < k; ++j)
            dlogits[(size_t)t * E + topk_idx[(size_t)t * k + j]] =
                (double)topk_w[(size_t)t * k + j] * (dw[(size_t)t * k + j] - sw);
    }
}

/* FP8 with K-blocked scales (the finer granularity of the FP8 grouped GEMM on
 * the LightLLM PR 1687 page, DeepGEMM's UE8M0 layout): one UE8M0 scale per row
 * and per block of `block` columns, chosen and applied as orc_quantize_rows does
 * for a whole row.  scales is [rows, ceil(cols / block)]. */
void orc_quantize_blocks(int64_t rows, int cols, int block, int dtype, const void *in,
                         uint8_t *codes, uint8_t *scales)
{
    const int nb = (cols + block - 1) / block;
    for (int64_t r = 0; r < rows; ++r)
        for (int b = 0; b < nb; ++b) {
            const int c0 = b * block, c1 = c0 + block < cols ? c0 + block : cols;
            double amax = 0.0;
            for (int c = c0; c < c1; ++c) {
                double a = fabs(orc_load(in, (size_t)r * cols + c, dtype));
                if (a > amax) amax = a;
            }
            uint8_t s = orc_ue8m0_scale(amax);
            scales[(size_t)r * nb + b] = s;
            for (int c = c0; c < c1; ++c)
                codes[(size_t)r * cols + c] =
                    orc_e4m3_encode(ldexp(orc_load(in, (size_t)r * cols + c, dtype), 127 - (int)s));
        }
}

/* Dot product of two K-blocked FP8 rows of length K (same block size): the sum
 * over blocks of 2^(sa + sb - 254) times the sum of the blocks' decoded code
 * products, in double (each block's partial sum is exact in double for
 * E4M3 operands and block <= 2^20).  dec: the decoded value of every code. */
static double orc_dot_blocked_dec(int K, int block, const uint8_t *a, const uint8_t *sa,
                                  const uint8_t *b, const uint8_t *sb, const double *dec)
{
    const int nb = (K + block - 1) / block;
    double acc = 0.0;
    for (int q = 0; q < nb; ++q) {
        double part = 0.0;
        for (int c = q * block; c < K && c < (q + 1) * block; ++c)
            part += dec[a[c]] * dec[b[c]];
        acc += ldexp(part, (int)sa[q] + (int)sb[q] - 254);
    }
    return acc;
}

double orc_dot_blocked(int K, int block, const uint8_t *a, const uint8_t *sa, const uint8_t *b,
                       const uint8_t *sb)
{
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = orc_e4m3_decode((uint8_t)c);
    return orc_dot_blocked_dec(K, block, a, sa, b, sb, dec);
}

/* One expert's SwiGLU FFN on one receive row in FP8 with K-blocked scales (the
 * finer granularity of the LightLLM PR 1687 page's FP8 grouped GEMM: UE8M0
 * scales along K, four of them packed in an int32).  Reading: one UE8M0 scale
 * per row and per `block` consecutive K values, chosen as orc_quantize_rows does
 * for a whole row, for x, W13 and W2 alike, and h quantised by blocks of its I
 * values.  The steps of orc_ffn_row_fp8 with the blocked dot products:
 *   x [H] codes, xs [H/block]; w13 [2I, H] codes, w13_s [2I, H/block];
 *   w2 [H, I] codes, w2_s [H, I/block];
 *   g_i = orc_dot_blocked(w13 row i, x), u_i = the same with row I + i;
 *   h_i = silu(g_i) u_i rounded to bf16 (h_store, bf16 bits, optional);
 *   (hq_store [I], hs_store [I/block]) = orc_quantize_blocks of that bf16 row;
 *   y_o = orc_dot_blocked(w2 row o, hq) (y_exact optional; y_store bf16). */
void orc_ffn_row_fp8_blocked(int H, int I, int block, const uint8_t *x, const uint8_t *xs,
                             const uint8_t *w13, const uint8_t *w13_s, const uint8_t *w2,
                             const uint8_t *w2_s, uint16_t *h_store, uint8_t *hq_store,
                             uint8_t *hs_store, uint16_t *y_store, double *y_exact)
{
    const int nbh = (H + block - 1) / block, nbi = (I + block - 1) / block;
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = orc_e4m3_decode((uint8_t)c);
    uint16_t *h = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)I);
    uint8_t *hq = (uint8_t *)malloc((size_t)I);
    uint8_t *hs = (uint8_t *)malloc((size_t)nbi);
    for (int i = 0; i < I; ++i) {
        const double g = orc_dot_blocked_dec(H, block, w13 + (size_t)i * H, w13_s + (size_t)i * nbh, x, xs, dec);
        const double u = orc_dot_blocked_dec(H, block, w13 + (size_t)(I + i) * H,
                                             w13_s + (size_t)(I + i) * nbh, x, xs, dec);
        h[i] = orc_bf16_from_double(g / (1.0 + exp(-g)) * u);
    }
    orc_quantize_blocks(1, I, block, 1, h, hq, hs);
    for (int o = 0; o < H; ++o) {
        const double acc = orc_dot_blocked_dec(I, block, w2 + (size_t)o * I, w2_s + (size_t)o * nbi, hq, hs, dec);
        if (y_exact) y_exact[o] = acc;
        if (y_store) y_store[o] = orc_bf16_from_double(acc);
    }
    if (h_store) memcpy(h_store, h, sizeof(uint16_t) * (size_t)I);
    if (hq_store) memcpy(hq_store, hq, (size_t)I);
    if (hs_store) memcpy(hs_store, hs, (size_t)nbi);
    free(h);
    free(hq);
    free(hs);
}
