/*
 * moe_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of one sparse-MoE FFN layer
 * (router -> top-k gates -> permutation -> expert-cache lookup -> SwiGLU experts
 * on 2/3-bit block-quantised weights -> gate-weighted combine + shared expert).
 * Only the tests, the package smoke check and the bench's CPU-baseline leg may
 * load it. It shares no source with the CUDA library and is never on the
 * product path.
 *
 * Sources (page titles; each function names the section it follows):
 *   [SAITO]  "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的
 *             Qwen 3.8 Flash Next" (attain.fans repost of an X article)
 *   [EN]     "Running Qwen3.8-Flash-Next on a 12GB GPU: Custom Engine Hits 65 tok/s"
 *   [JDSSL]  "5070ti16g单卡跑qwen 3.8 flash next 新方案最高90t/s Hermes调用60t/s"
 * The pages fix the structure (top-10 of 512 routed experts plus one shared
 * expert, a hot-expert cache in VRAM whose misses go to the CPU, 2-bit and
 * 3-bit weight tiers) but not the arithmetic. The arithmetic below is this
 * library's own definition, stated at each function.
 *
 * Precision: everything is fp64 except the router logit, which is defined as an
 * fp32 value with a fixed operation order (orc_router_logit) so that expert
 * selection is reproducible bit-for-bit. Build with -ffp-contract=off and
 * without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16: the upper 16 bits of an IEEE binary32. */
double orc_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* IEEE binary16, decoded from its definition: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 is subnormal (fraction * 2^-24). */
double orc_fp16_value(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Dequantisation (library-defined formats; the pages name Q2_0 and    */
/* IQ3_XXS tiers in [EN] "Detailed Performance Numbers" but print no   */
/* bit layout).                                                        */
/* ------------------------------------------------------------------ */

/* Q2: 64-weight blocks along K; code q in {0..3} of weight k at byte k/4,
 * bits 2(k%4); block scale s and min m (fp16); w = s*q + m. */
void orc_dequant_q2(const uint8_t *codes, const uint16_t *scale, const uint16_t *mn,
                    int R, int K, double *W)
{
    for (int r = 0; r < R; ++r)
        for (int k = 0; k < K; ++k) {
            int q = (codes[(size_t)r * (K / 4) + k / 4] >> (2 * (k % 4))) & 3;
            double s = orc_fp16_value(scale[(size_t)r * (K / 64) + k / 64]);
            double m = orc_fp16_value(mn[(size_t)r * (K / 64) + k / 64]);
            W[(size_t)r * K + k] = s * (double)q + m;
        }
}

/* Q3: 64-weight blocks along K; code q in {0..7}: low two bits as in Q2, third
 * bit of weight k at byte k/8, bit k%8 of the hi plane; fp16 scale s;
 * w = s*(q-4). */
void orc_dequant_q3(const uint8_t *lo, const uint8_t *hi, const uint16_t *scale,
                    int R, int K, double *W)
{
    for (int r = 0; r < R; ++r)
        for (int k = 0; k < K; ++k) {
            int q_lo = (lo[(size_t)r * (K / 4) + k / 4] >> (2 * (k % 4))) & 3;
            int q_hi = (hi[(size_t)r * (K / 8) + k / 8] >> (k % 8)) & 1;
            int q = q_lo + 4 * q_hi;
            double s = orc_fp16_value(scale[(size_t)r * (K / 64) + k / 64]);
            W[(size_t)r * K + k] = s * (double)(q - 4);
        }
}

/* ------------------------------------------------------------------ */
/* Router ([SAITO] "1250 亿参数，每个词只用得上 2%": each token picks 10 of the */
/* layer's 512 experts; the router stays pinned in VRAM per            */
/* "命中率七成，代价是答案会变").                                          */
/* ------------------------------------------------------------------ */

/* The router logit as an fp32 value with a fixed order of operations:
 * d is cut into d/128 chunks; inside chunk i, accumulator l (0..31) takes the
 * four products of elements 128i+4l+j, j=0..3, each with one fused multiply-add
 * (single rounding), chunks in increasing order. The 32 accumulators are then
 * combined by pairwise fp32 additions acc[l] += acc[l^o] for o=16,8,4,2,1 and
 * the result is accumulator 0. The bias, if any, is added last in fp32. */
float orc_router_logit(const uint16_t *x, const float *w, int d, const float *bias_or_null)
{
    float acc[32];
    for (int l = 0; l < 32; ++l)
        acc[l] = 0.0f;
    for (int i = 0; i < d / 128; ++i)
        for (int l = 0; l < 32; ++l)
            for (int j = 0; j < 4; ++j) {
                int kk = 128 * i + 4 * l + j;
                acc[l] = fmaf((float)orc_bf16_value(x[kk]), w[kk], acc[l]);
            }
    for (int o = 16; o >= 1; o >>= 1) {
        float nxt[32];
        for (int l = 0; l < 32; ++l)
            nxt[l] = acc[l] + acc[l ^ o];
        memcpy(acc, nxt, sizeof acc);
    }
    float r = acc[0];
    if (bias_or_null)
        r = r + *bias_or_null;
    return r;
}

/* All T*E logits in fp32 (above) and in fp64 (plain dot product), plus
 * sum_k |x_k w_k| for the rounding-error bound the tests check. */
void orc_router(const uint16_t *x, const float *Wr, const float *bias, int T, int d, int E,
                float *logit32, double *logit64, double *absdot)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            const uint16_t *xt = x + (size_t)t * d;
            const float *we = Wr + (size_t)e * d;
            double s = 0.0, a = 0.0;
            for (int kk = 0; kk < d; ++kk) {
                double p = orc_bf16_value(xt[kk]) * (double)we[kk];
                s += p;
                a += fabs(p);
            }
            if (bias)
                s += (double)bias[e];
            logit32[(size_t)t * E + e] = orc_router_logit(xt, we, d, bias ? bias + e : NULL);
            if (logit64)
                logit64[(size_t)t * E + e] = s;
            if (absdot)
                absdot[(size_t)t * E + e] = a;
        }
}

typedef struct {
    float v;
    int id;
} orc_cand;

/* Order: larger logit first; equal logits (+0 and -0 are equal) by lower id. */
static int orc_cmp_cand(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    if (a->v > b->v)
        return -1;
    if (a->v < b->v)
        return 1;
    return (a->id > b->id) - (a->id < b->id);
}

static int orc_cmp_int(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* Top-k selection and gates. The k experts are the first k in the order
 * (logit desc, id asc); they are reported in ascending id. Gate j is the
 * softmax of the selected logits, exp(l_j - l_max) / sum_i exp(l_i - l_max),
 * in fp64 from the fp32 logits -- the same as a softmax over all E experts
 * renormalised over the selected k. Returns -1 if a logit is not finite. */
int orc_topk(const float *logits, int T, int E, int k, int32_t *idx, double *gate)
{
    orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)E);
    int *sel = (int *)malloc(sizeof(int) * (size_t)k);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            float v = logits[(size_t)t * E + e];
            if (!isfinite(v)) {
                free(c);
                free(sel);
                return -1;
            }
            c[e].v = v;
            c[e].id = e;
        }
        qsort(c, (size_t)E, sizeof(orc_cand), orc_cmp_cand);
        for (int j = 0; j < k; ++j)
            sel[j] = c[j].id;
        qsort(sel, (size_t)k, sizeof(int), orc_cmp_int);
        double lmax = (double)c[0].v;
        double z = 0.0;
        for (int j = 0; j < k; ++j)
            z += exp((double)logits[(size_t)t * E + sel[j]] - lmax);
        for (int j = 0; j < k; ++j) {
            idx[(size_t)t * k + j] = sel[j];
            gate[(size_t)t * k + j] = exp((double)logits[(size_t)t * E + sel[j]] - lmax) / z;
        }
    }
    free(c);
    free(sel);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Token -> expert permutation: the T*k (token, slot) pairs, numbered  */
/* p = t*k + j, sorted by expert id and, within an expert, by p.       */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t e;
    int32_t p;
} orc_pair;

static int orc_cmp_pair(const void *pa, const void *pb)
{
    const orc_pair *a = (const orc_pair *)pa, *b = (const orc_pair *)pb;
    if (a->e != b->e)
        return (a->e > b->e) - (a->e < b->e);
    return (a->p > b->p) - (a->p < b->p);
}

/* counts[E], offsets[E+1], sorted_tok/sorted_j/inv[T*k], active[E+1]
 * (active[0] = number of experts with a token, then those ids ascending).
 * Returns -1 on an id outside [0,E). */
int orc_permute(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *active)
{
    int n = T * k;
    orc_pair *pr = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int p = 0; p < n; ++p) {
        if (idx[p] < 0 || idx[p] >= E) {
            free(pr);
            return -1;
        }
        pr[p].e = idx[p];
        pr[p].p = p;
    }
    qsort(pr, (size_t)n, sizeof(orc_pair), orc_cmp_pair);
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (int s = 0; s < n; ++s) {
        sorted_tok[s] = pr[s].p / k;
        sorted_j[s] = pr[s].p % k;
        inv[pr[s].p] = s;
        counts[pr[s].e] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int na = 0;
    for (int e = 0; e < E; ++e)
        if (counts[e] > 0)
            active[1 + na++] = e;
    active[0] = na;
    free(pr);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Expert cache ([JDSSL] "为什么从 18t/s 变成 60-90t/s": hot experts live in */
/* a VRAM cache; [SAITO] "命中率七成，代价是答案会变": experts not in the */
/* cache are computed by the CPU instead).                             */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t layer, expert, token, j;
    float gate;
} orc_miss;

/* slot_of_pair[p] = slot_of[idx[p]] (-1 = not resident). Every pair whose
 * expert is not resident becomes a miss record, ordered by (expert, token);
 * records beyond miss_cap are counted but not stored. Returns the miss count. */
int orc_cache_lookup(const int32_t *slot_of, int layer, const int32_t *idx, const double *gate,
                     int T, int k, int E, int32_t *slot_of_pair, orc_miss *miss, int miss_cap)
{
    for (int p = 0; p < T * k; ++p)
        slot_of_pair[p] = slot_of[idx[p]];
    int nm = 0;
    for (int e = 0; e < E; ++e) {
        if (slot_of[e] >= 0)
            continue;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e) {
                    if (nm < miss_cap) {
                        miss[nm].layer = layer;
                        miss[nm].expert = e;
                        miss[nm].token = t;
                        miss[nm].j = j;
                        miss[nm].gate = (float)gate[(size_t)t * k + j];
                    }
                    nm++;
                }
    }
    return nm;
}

/* ------------------------------------------------------------------ */
/* SwiGLU expert FFN, fp64: a = Wg x, u = Wu x, h = silu(a) * u with   */
/* silu(a) = a / (1 + exp(-a)), y = Wd h. Wg, Wu are [f][d], Wd is     */
/* [d][f], all dequantised. The shared expert has the same form.       */
/* ------------------------------------------------------------------ */

void orc_expert_ffn(const double *Wg, const double *Wu, const double *Wd, const double *x,
                    int d, int f, double *y, double *h_out)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)f);
    for (int r = 0; r < f; ++r) {
        double a = 0.0, u = 0.0;
        for (int c = 0; c < d; ++c) {
            a += Wg[(size_t)r * d + c] * x[c];
            u += Wu[(size_t)r * d + c] * x[c];
        }
        h[r] = a / (1.0 + exp(-a)) * u;
        if (h_out)
            h_out[r] = h[r];
    }
    for (int r = 0; r < d; ++r) {
        double s = 0.0;
        for (int c = 0; c < f; ++c)
            s += Wd[(size_t)r * f + c] * h[c];
        y[r] = s;
    }
    free(h);
}

/* Same FFN for a batch of tokens: x is [n][d], y is [n][d]. */
void orc_expert_ffn_batch(const double *Wg, const double *Wu, const double *Wd, const double *x,
                          int n, int d, int f, double *y)
{
    for (int i = 0; i < n; ++i)
        orc_expert_ffn(Wg, Wu, Wd, x + (size_t)i * d, d, f, y + (size_t)i * d, NULL);
}
