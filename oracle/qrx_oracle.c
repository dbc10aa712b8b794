/*
 * qrx_oracle.c -- plain, slow CPU reference of the routed-MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only in the seeded inputs they are both given.
 *
 * What it computes (sources are the three web pages on colibri, the pure-C
 * GLM-5.2 engine):
 *   - colibri README ("JustVugg/colibri"), section "已实现的功能" (implemented
 *     features): a DeepSeek-V3-like sigmoid router (noaux_tc,
 *     routed_scaling_factor) and a shared expert; Q8_0-style int8-activation
 *     integer dot kernels; int8 / packed int4 / packed int2 weights with
 *     per-row scales, dequantised on use, packing bit-consistent with the int8
 *     container; the batch-union MoE in which each unique expert of a batch
 *     is read once and applied to every position routed to it.
 *   - blog "GLM-5.2 on slow computers", section "让它变得可以忍受的那些装置"
 *     (the devices that make it bearable): same expert read once per batch;
 *     int4 container with per-row scale, dequant-on-use.
 * The pages give no formulas.  Every formula below is the plainest reading
 * of that prose, fixed by the workload definitions (SwiGLU experts, scale =
 * absmax/7, two codes per byte low nibble first, Q8_0 blocks of 32 with an
 * f32 absmax scale, group-limited top-k with bias used for selection only).
 * Each reading is tagged [reading] where the pages leave it open.
 *
 * Arithmetic: every inner product is summed in double in index order and
 * rounded to f32 once, so this is the definition written out, not a fast
 * kernel.  Build: gcc -O2 -fopenmp -ffp-contract=off (no fast-math), so f32
 * operations are single IEEE operations exactly as written.
 *
 * Parity pins (tests/test_oracle_pins.py) tie each function to something
 * other than itself.  The pages print no example of a whole layer; the layer
 * composition is pinned by a closed form instead: one-hot tokens, chosen
 * router logits and single-entry expert rows make every stage a scalar
 * expression the test evaluates in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* configuration                                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    int hidden;         /* H */
    int n_experts;      /* E, routed experts */
    int inter;          /* I, expert intermediate size */
    int n_group;        /* G */
    int topk_group;     /* Gk */
    int top_k;          /* k */
    float routed_scaling_factor;
    int wbits;          /* 8, 4 or 2: routed and shared expert weight format */
    int afmt;           /* 0 = f32 activations, 1 = Q8_0, 2 = bf16 */
} qo_cfg;

/* One expert: SwiGLU FFN, three packed matrices in [out][in] orientation. */
typedef struct {
    const uint8_t *gate_q;  /* [I][H*bits/8] */
    const float *gate_s;    /* [I] */
    const uint8_t *up_q;    /* [I][H*bits/8] */
    const float *up_s;      /* [I] */
    const uint8_t *down_q;  /* [H][I*bits/8] */
    const float *down_s;    /* [H] */
} qo_expert;

enum { QO_A_F32 = 0, QO_A_Q8 = 1, QO_A_BF16 = 2 };

int qo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void qo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* codes and packing                                                        */
/* ------------------------------------------------------------------------ */
/* Symmetric per-row quantisation [workload definition: scale = absmax/7 for
 * int4, codes in [-8, 7]].  [reading] int8 and int2 follow the same rule
 * "scale = absmax / largest positive code": qmax 127 and 1, qmin -128 and
 * -2.  The quantiser never emits qmin but every decoder accepts it.
 * Packing [workload definition: two per byte, low nibble first]: element 2i
 * in bits [3:0], 2i+1 in bits [7:4]; [reading] the nibble holds the 4-bit
 * two's-complement code, so a packed value is bit-consistent with the same
 * code in an int8 container (README, "已实现的功能": packing verified
 * bit-consistent with the int8 container).  int2: element 4i in bits [1:0]
 * ... 4i+3 in bits [7:6], two's complement {-2..1}. */

int qo_qmax(int bits) { return bits == 8 ? 127 : (bits == 4 ? 7 : 1); }
int qo_qmin(int bits) { return bits == 8 ? -128 : (bits == 4 ? -8 : -2); }
int64_t qo_row_bytes(int bits, int64_t K) { return K * bits / 8; }

int qo_get_code(const uint8_t *row, int bits, int64_t i)
{
    if (bits == 8) return (int)(int8_t)row[i];
    if (bits == 4) {
        int v = (row[i / 2] >> ((int)(i % 2) * 4)) & 0xF;
        return v >= 8 ? v - 16 : v;
    }
    int v = (row[i / 4] >> ((int)(i % 4) * 2)) & 0x3;
    return v >= 2 ? v - 4 : v;
}

void qo_put_code(uint8_t *row, int bits, int64_t i, int code)
{
    if (bits == 8) {
        row[i] = (uint8_t)(int8_t)code;
    } else if (bits == 4) {
        int sh = (int)(i % 2) * 4;
        row[i / 2] = (uint8_t)((row[i / 2] & ~(0xF << sh)) | ((code & 0xF) << sh));
    } else {
        int sh = (int)(i % 4) * 2;
        row[i / 4] = (uint8_t)((row[i / 4] & ~(0x3 << sh)) | ((code & 0x3) << sh));
    }
}

/* w [rows][K] f32 -> q [rows][K*bits/8] packed codes, s [rows] f32.
 * s = absmax / qmax (one f32 division); code = clamp(round-half-away(w / s)).
 * A row of zeros gets s = 0 and all codes 0. */
void qo_quantize_rows(const float *w, int64_t rows, int64_t K, int bits,
                      uint8_t *q, float *s)
{
    const int qmax = qo_qmax(bits), qmin = qo_qmin(bits);
    const int64_t rb = qo_row_bytes(bits, K);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float *wr = w + r * K;
        uint8_t *qr = q + r * rb;
        float amax = 0.0f;
        for (int64_t i = 0; i < K; ++i) {
            float a = fabsf(wr[i]);
            if (a > amax) amax = a;
        }
        float sc = amax / (float)qmax;
        s[r] = sc;
        memset(qr, 0, (size_t)rb);
        if (sc == 0.0f) continue;
        for (int64_t i = 0; i < K; ++i) {
            float v = wr[i] / sc;
            int c = (int)roundf(v);           /* C99 roundf: half away from zero */
            if (c > qmax) c = qmax;
            if (c < qmin) c = qmin;
            qo_put_code(qr, bits, i, c);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 (128x128 block scales) -> per-row packed requantisation              */
/* ------------------------------------------------------------------------ */
/* FP8 e4m3 (the "fn" variant: 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent 0 is subnormal; no infinities; S.1111.111 is NaN),
 * decoded from that definition: (-1)^s * 2^(e-7) * (1 + m/8), or
 * (-1)^s * 2^-6 * (m/8) when e = 0. */
float qo_fp8_e4m3_to_f32(uint8_t b)
{
    const int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(sgn ? -v : v);
}

/* README "JustVugg/colibri", section "已实现的功能": the offline FP8->int4
 * converter dequantises FP8 weights with 128x128 block scales and requantises
 * them into the engine's container.  Per element: w[r][c] = f32(fp8[r][c]) *
 * bscale[r/128][c/128] (one f32 multiply; [reading] a NaN code counts as 0);
 * then each row as qo_quantize_rows (s = absmax / qmax, codes
 * clamp(round-half-away(w / s))).  w8 [rows][K] with row stride ld8 bytes;
 * bscale [ceil(rows/128)][ceil(K/128)] row-major. */
void qo_requant_fp8(const uint8_t *w8, int64_t rows, int64_t K, int64_t ld8, const float *bscale,
                    int bits, uint8_t *q, float *s)
{
    const int64_t nbk = (K + 127) / 128, rb = qo_row_bytes(bits, K);
    #pragma omp parallel
    {
        float *row = (float *)malloc(sizeof(float) * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t c = 0; c < K; ++c) {
                float f = qo_fp8_e4m3_to_f32(w8[r * ld8 + c]);
                if (isnan(f)) f = 0.0f;
                row[c] = f * bscale[(r / 128) * nbk + c / 128];
            }
            qo_quantize_rows(row, 1, K, bits, q + r * rb, s + r);
        }
        free(row);
    }
}

/* Decode packed rows to their integer codes (test helper). */
void qo_unpack_rows(const uint8_t *q, int64_t rows, int64_t K, int bits, int8_t *codes)
{
    const int64_t rb = qo_row_bytes(bits, K);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i)
            codes[r * K + i] = (int8_t)qo_get_code(q + r * rb, bits, i);
}

/* ------------------------------------------------------------------------ */
/* Q8_0-style activations                                                   */
/* ------------------------------------------------------------------------ */
/* README "已实现的功能": integer dot kernels with Q8_0-style int8
 * activations.  Workload definition: blocks of 32, f32 absmax scale.
 * [reading] d = amax/127 (f32 division); q = clamp(round-half-away(x * f),
 * -127, 127) with f = 127/amax (one f32 division, one f32 multiply per
 * element); the clamp applies to the f32 product (so a block whose amax is
 * below 127/FLT_MAX, where f overflows, still maps to +-127 and 0); a zero
 * block has d = 0 and q = 0. */
void qo_quantize_q8(const float *x, int64_t n, int8_t *q, float *d)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        const float *xb = x + b * 32;
        float amax = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float a = fabsf(xb[i]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            d[b] = 0.0f;
            for (int i = 0; i < 32; ++i) q[b * 32 + i] = 0;
            continue;
        }
        d[b] = amax / 127.0f;
        float f = 127.0f / amax;      /* +inf when amax < 127/FLT_MAX */
        for (int i = 0; i < 32; ++i) {
            /* the clamp is taken on the product, so an infinite factor still
             * gives +-127, and 0 * inf (a zero beside a tiny amax) gives 0 */
            float v = xb[i] * f;
            int c;
            if (v != v) c = 0;
            else if (v >= 127.0f) c = 127;
            else if (v <= -127.0f) c = -127;
            else c = (int)roundf(v);
            q[b * 32 + i] = (int8_t)c;
        }
    }
}

/* Exact int32 block accumulators acc[r][b] = sum over the 32-block of
 * code(r, i) * xq[i]: the integer part of a Q8_0 dot, compared bit for bit. */
void qo_block_dots_q8(const uint8_t *q, int64_t rows, int64_t K, int bits,
                      const int8_t *xq, int32_t *acc)
{
    const int64_t rb = qo_row_bytes(bits, K);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            int32_t s = 0;
            for (int64_t i = b * 32; i < b * 32 + 32; ++i)
                s += (int32_t)qo_get_code(q + r * rb, bits, i) * (int32_t)xq[i];
            acc[r * (K / 32) + b] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* bf16                                                                     */
/* ------------------------------------------------------------------------ */
float qo_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round-to-nearest-even of an f32 to bf16, from the definition: keep the top
 * 16 bits, rounding on the 16 dropped bits with ties to the even result. */
uint16_t qo_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040u);        /* quiet NaN */
    uint32_t lower = u & 0xFFFFu, upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* router                                                                   */
/* ------------------------------------------------------------------------ */
/* README "已实现的功能": DeepSeek-V3-like sigmoid router, noaux_tc,
 * routed_scaling_factor.  Workload definition: the score-correction bias is
 * used for selection only; group-limited top-k; weights renormalised and
 * scaled by routed_scaling_factor.  Readings (DeepSeek-V3 convention, since
 * the pages say only "DeepSeek-V3-like"):
 *   logit_e = x . Wr[e] summed in double, rounded to f32;
 *   s_e = 1/(1+exp(-logit_e)) in double, rounded to f32;  sc_e = s_e + b_e (f32);
 *   groups are contiguous blocks of E/G experts; a group's score is the sum
 *   (f32) of its two largest sc (its only one if a group has one expert);
 *   keep the Gk best groups (ties to the lower group index); among experts of
 *   kept groups take the k largest sc (ties to the lower expert id), in that
 *   order; w_j = s_j / sum_j s_j * rsf, sum and quotient in double, rounded
 *   to f32 (no epsilon: s > 0 always).
 * ties[t] bit 0: the k-th and (k+1)-th candidate sc are within 1e-5;
 *         bit 1: the Gk-th and (Gk+1)-th group scores are within 1e-5. */
static double act_value(const qo_cfg *c, const void *act, int64_t t, int64_t h)
{
    if (c->afmt == QO_A_BF16)
        return (double)qo_bf16_to_f32(((const uint16_t *)act)[t * c->hidden + h]);
    return (double)((const float *)act)[t * c->hidden + h];
}

void qo_router(const qo_cfg *c, const void *act, int T, const float *Wr,
               const float *bias, int32_t *idx, float *wout, float *logits,
               float *scores, int32_t *ties)
{
    const int H = c->hidden, E = c->n_experts, G = c->n_group;
    const int Gk = c->topk_group, k = c->top_k, gs = E / G;

    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        float *s = (float *)malloc(sizeof(float) * (size_t)E);
        float *sc = (float *)malloc(sizeof(float) * (size_t)E);
        float *gscore = (float *)malloc(sizeof(float) * (size_t)G);
        char *gkeep = (char *)calloc((size_t)G, 1);
        char *taken = (char *)calloc((size_t)E, 1);

        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += act_value(c, act, t, h) * (double)Wr[(int64_t)e * H + h];
            float lg = (float)acc;
            s[e] = (float)(1.0 / (1.0 + exp(-(double)lg)));
            sc[e] = s[e] + bias[e];
            if (logits) logits[(int64_t)t * E + e] = lg;
            if (scores) scores[(int64_t)t * E + e] = s[e];
        }
        for (int g = 0; g < G; ++g) {
            float top1 = -INFINITY, top2 = -INFINITY;
            for (int e = g * gs; e < (g + 1) * gs; ++e) {
                if (sc[e] > top1) { top2 = top1; top1 = sc[e]; }
                else if (sc[e] > top2) { top2 = sc[e]; }
            }
            gscore[g] = gs >= 2 ? top1 + top2 : top1;
        }
        int tie = 0;
        float last_kept_g = 0.0f;
        for (int r = 0; r < Gk; ++r) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
            gkeep[best] = 1;
            last_kept_g = gscore[best];
        }
        if (Gk < G) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
            if (last_kept_g - gscore[best] < 1e-5f) tie |= 2;
        }
        float last_sc = 0.0f;
        double ssum = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (gkeep[e / gs] && !taken[e] && (best < 0 || sc[e] > sc[best])) best = e;
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
            last_sc = sc[best];
            ssum += (double)s[best];
        }
        {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (gkeep[e / gs] && !taken[e] && (best < 0 || sc[e] > sc[best])) best = e;
            if (best >= 0 && last_sc - sc[best] < 1e-5f) tie |= 1;
        }
        for (int j = 0; j < k; ++j) {
            int e = idx[(int64_t)t * k + j];
            wout[(int64_t)t * k + j] =
                (float)((double)s[e] / ssum * (double)c->routed_scaling_factor);
        }
        if (ties) ties[t] = tie;
        free(s); free(sc); free(gscore); free(gkeep); free(taken);
    }
}

/* ------------------------------------------------------------------------ */
/* adaptive expert top-p                                                    */
/* ------------------------------------------------------------------------ */
/* README "JustVugg/colibri", section "快速开始" (the --topp knob, adaptive
 * expert top-p, default 0.7) and "社区基准（实测）" (its measured effect):
 * drop the low-weight experts of each token so fewer experts are read.
 * [reading] applied to the router's output, per token: the k selections are
 * ordered by weight, largest first (equal weights: the lower slot j first);
 * the shortest leading run whose weights summed in that order (in double)
 * reach p * rsf (p of the total weight, which is rsf) is kept; every other
 * slot becomes idx = -1, w = 0.  [reading] the kept weights are not
 * renormalised.  p outside (0, 1) keeps every slot (so does k > 64, beyond
 * this reference's scratch).  Returns the number of slots kept. */
int64_t qo_topp_prune(int T, int k, double p, float rsf, int32_t *idx, float *w)
{
    if (!(p > 0.0 && p < 1.0) || k > 64) return (int64_t)T * k;
    const double thr = p * (double)rsf;
    int64_t kept = 0;
    int order[64];
    for (int t = 0; t < T; ++t) {
        int32_t *it = idx + (int64_t)t * k;
        float *wt = w + (int64_t)t * k;
        for (int j = 0; j < k; ++j) order[j] = j;
        /* insertion sort: weight descending, slot ascending */
        for (int i = 1; i < k; ++i) {
            int j = i, v = order[i];
            while (j > 0 && (wt[order[j - 1]] < wt[v] || (wt[order[j - 1]] == wt[v] && order[j - 1] > v))) {
                order[j] = order[j - 1];
                --j;
            }
            order[j] = v;
        }
        double c = 0.0;
        int n = 0;
        while (n < k) {
            c += (double)wt[order[n]];
            ++n;
            if (c >= thr) break;
        }
        for (int i = n; i < k; ++i) {
            it[order[i]] = -1;
            wt[order[i]] = 0.0f;
        }
        kept += n;
    }
    return kept;
}

/* ------------------------------------------------------------------------ */
/* permutation (batch-union)                                                */
/* ------------------------------------------------------------------------ */
/* README "已实现的功能" (batch-union MoE) and the blog's "同一批次里相同的专家
 * 只读一次": group the T*k assignments a = t*k + j by expert so each expert
 * present in the batch is visited once for all its positions.
 * [reading] the order is fixed so the result is unique: a stable counting
 * sort by (expert, a).  counts[E], offsets[E+1] (exclusive prefix sum),
 * sorted[p] = a, inv[a] = p, union_ids = experts with count > 0 ascending.
 * A slot with idx = -1 (dropped by adaptive top-p, below) takes no position:
 * it is not counted and inv[a] = -1. */
void qo_permute(const int32_t *idx, int T, int k, int E, int32_t *counts,
                int32_t *offsets, int32_t *sorted, int32_t *inv,
                int32_t *union_ids, int32_t *n_union)
{
    const int64_t A = (int64_t)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < A; ++a)
        if (idx[a] >= 0) counts[idx[a]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t a = 0; a < A; ++a) {
        if (idx[a] < 0) {          /* slot dropped by adaptive top-p: no position */
            inv[a] = -1;
            continue;
        }
        int32_t p = cursor[idx[a]]++;
        sorted[p] = (int32_t)a;
        inv[a] = p;
    }
    free(cursor);
    int32_t n = 0;
    for (int e = 0; e < E; ++e)
        if (counts[e] > 0) union_ids[n++] = e;
    *n_union = n;
}

/* ------------------------------------------------------------------------ */
/* expert FFN                                                               */
/* ------------------------------------------------------------------------ */
/* SwiGLU expert: g = s_g * (Q_g x), u = s_u * (Q_u x), h = silu(g) * u,
 * y = s_d * (Q_d h), every row dot summed in double and rounded to f32.
 * Activation modes:
 *   f32  ([reading] "int4 single row stays on the f32 path", README
 *        "已实现的功能"): codes times f32 activations;
 *   Q8_0 (README: integer dot with Q8_0-style int8 activations): x and, by
 *        [reading], h are quantised to Q8_0; per block the exact int32
 *        accumulator is scaled by d_b, blocks summed in double;
 *   bf16 ([reading]): x is bf16 (widened exactly); h is rounded to bf16
 *        (nearest-even, from its f32 value) before the down projection. */
static float dot_f(const uint8_t *row, float scale, int bits, const double *x, int64_t K)
{
    double acc = 0.0;
    for (int64_t i = 0; i < K; ++i) acc += (double)qo_get_code(row, bits, i) * x[i];
    return (float)((double)scale * acc);
}

static float dot_q8(const uint8_t *row, float scale, int bits, const int8_t *xq,
                    const float *xd, int64_t K)
{
    double acc = 0.0;
    for (int64_t b = 0; b < K / 32; ++b) {
        int32_t ib = 0;
        for (int64_t i = b * 32; i < b * 32 + 32; ++i)
            ib += (int32_t)qo_get_code(row, bits, i) * (int32_t)xq[i];
        acc += (double)xd[b] * (double)ib;
    }
    return (float)((double)scale * acc);
}

static float silu_mul(float g, float u)
{
    double gd = (double)g;
    return (float)(gd / (1.0 + exp(-gd)) * (double)u);
}

/* gate/up for one token row through one expert -> h [I] */
static void ffn_gateup_one(const qo_cfg *c, const qo_expert *ex, const void *act,
                           int64_t t, float *h)
{
    const int H = c->hidden, I = c->inter, bits = c->wbits;
    const int64_t rb = qo_row_bytes(bits, H);
    if (c->afmt == QO_A_Q8) {
        int8_t *xq = (int8_t *)malloc((size_t)H);
        float *xd = (float *)malloc(sizeof(float) * (size_t)(H / 32));
        qo_quantize_q8((const float *)act + t * H, H, xq, xd);
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < I; ++i) {
            float g = dot_q8(ex->gate_q + (int64_t)i * rb, ex->gate_s[i], bits, xq, xd, H);
            float u = dot_q8(ex->up_q + (int64_t)i * rb, ex->up_s[i], bits, xq, xd, H);
            h[i] = silu_mul(g, u);
        }
        free(xq); free(xd);
    } else {
        double *x = (double *)malloc(sizeof(double) * (size_t)H);
        for (int i = 0; i < H; ++i) x[i] = act_value(c, act, t, i);
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < I; ++i) {
            float g = dot_f(ex->gate_q + (int64_t)i * rb, ex->gate_s[i], bits, x, H);
            float u = dot_f(ex->up_q + (int64_t)i * rb, ex->up_s[i], bits, x, H);
            h[i] = silu_mul(g, u);
        }
        free(x);
    }
}

/* down for one h row through one expert -> y [H] */
static void ffn_down_one(const qo_cfg *c, const qo_expert *ex, const float *h, float *y)
{
    const int H = c->hidden, I = c->inter, bits = c->wbits;
    const int64_t rb = qo_row_bytes(bits, I);
    if (c->afmt == QO_A_Q8) {
        int8_t *hq = (int8_t *)malloc((size_t)I);
        float *hd = (float *)malloc(sizeof(float) * (size_t)(I / 32));
        qo_quantize_q8(h, I, hq, hd);
        #pragma omp parallel for schedule(static)
        for (int r = 0; r < H; ++r)
            y[r] = dot_q8(ex->down_q + (int64_t)r * rb, ex->down_s[r], bits, hq, hd, I);
        free(hq); free(hd);
    } else {
        double *hx = (double *)malloc(sizeof(double) * (size_t)I);
        for (int i = 0; i < I; ++i)
            hx[i] = c->afmt == QO_A_BF16 ? (double)qo_bf16_to_f32(qo_f32_to_bf16(h[i]))
                                         : (double)h[i];
        #pragma omp parallel for schedule(static)
        for (int r = 0; r < H; ++r)
            y[r] = dot_f(ex->down_q + (int64_t)r * rb, ex->down_s[r], bits, hx, I);
        free(hx);
    }
}

/* One token through one expert (the per-token loop the union is checked
 * against). */
void qo_ffn_token(const qo_cfg *c, const qo_expert *ex, const void *act, int64_t t,
                  float *h, float *y)
{
    ffn_gateup_one(c, ex, act, t, h);
    ffn_down_one(c, ex, h, y);
}

/* Batch-union routed FFN: for each expert of the union, for each of its
 * positions p in sorted order (token t = sorted[p] / k), h_sorted[p] and
 * y_sorted[p].  experts[e] may hold NULL pointers for experts not in the
 * union.  h_sorted may be NULL. */
void qo_expert_ffn(const qo_cfg *c, const qo_expert *experts, const int32_t *offsets,
                   const int32_t *sorted, const int32_t *union_ids, int n_union,
                   const void *act, float *h_sorted, float *y_sorted)
{
    const int I = c->inter, H = c->hidden, k = c->top_k;
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    for (int u = 0; u < n_union; ++u) {
        int e = union_ids[u];
        for (int32_t p = offsets[e]; p < offsets[e + 1]; ++p) {
            int64_t t = sorted[p] / k;
            qo_ffn_token(c, &experts[e], act, t, h, y_sorted + (int64_t)p * H);
            if (h_sorted) memcpy(h_sorted + (int64_t)p * I, h, sizeof(float) * (size_t)I);
        }
    }
    free(h);
}

/* The same result reached token by token: for t, for j, expert idx[t*k+j],
 * written at its sorted position inv[t*k+j]. */
void qo_expert_ffn_per_token(const qo_cfg *c, const qo_expert *experts,
                             const int32_t *idx, const int32_t *inv, int T,
                             const void *act, float *y_sorted)
{
    const int I = c->inter, H = c->hidden, k = c->top_k;
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t a = (int64_t)t * k + j;
            qo_ffn_token(c, &experts[idx[a]], act, t, h, y_sorted + (int64_t)inv[a] * H);
        }
    free(h);
}

/* Down stage alone, given h in sorted order (stage isolation). */
void qo_expert_down(const qo_cfg *c, const qo_expert *experts, const int32_t *offsets,
                    const int32_t *union_ids, int n_union, const float *h_sorted,
                    float *y_sorted)
{
    const int I = c->inter, H = c->hidden;
    for (int u = 0; u < n_union; ++u) {
        int e = union_ids[u];
        for (int32_t p = offsets[e]; p < offsets[e + 1]; ++p)
            ffn_down_one(c, &experts[e], h_sorted + (int64_t)p * I, y_sorted + (int64_t)p * H);
    }
}

/* Shared expert (README "已实现的功能": shared expert): [reading] every
 * token, weight 1, not gated (DeepSeek-V3 convention). */
void qo_shared_ffn(const qo_cfg *c, const qo_expert *shared, const void *act, int T,
                   float *h_sh, float *y_sh)
{
    const int I = c->inter, H = c->hidden;
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    for (int t = 0; t < T; ++t) {
        qo_ffn_token(c, shared, act, t, h, y_sh + (int64_t)t * H);
        if (h_sh) memcpy(h_sh + (int64_t)t * I, h, sizeof(float) * (size_t)I);
    }
    free(h);
}

/* Weighted combine: out[t] = y_sh[t] + sum_j w[t,j] * y_sorted[inv[t*k+j]],
 * summed in double in j order, rounded to f32.  y_sh may be NULL (no shared
 * expert term).  Slots with inv = -1 (dropped) contribute nothing. */
void qo_combine(const qo_cfg *c, int T, const float *y_sorted, const float *y_sh,
                const float *w, const int32_t *inv, float *out)
{
    const int H = c->hidden, k = c->top_k;
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = y_sh ? (double)y_sh[(int64_t)t * H + h] : 0.0;
            for (int j = 0; j < k; ++j) {
                int64_t a = (int64_t)t * k + j;
                if (inv[a] < 0) continue;          /* dropped slot */
                acc += (double)w[a] * (double)y_sorted[(int64_t)inv[a] * H + h];
            }
            out[(int64_t)t * H + h] = (float)acc;
        }
}

/* The whole layer: route, (adaptive top-p when 0 < topp < 1), permute,
 * routed FFN over the union, shared expert, combine.  Scratch is allocated
 * here (this is the slow reference). */
void qo_moe_forward_opts(const qo_cfg *c, const void *act, int T, const float *Wr,
                         const float *bias, const qo_expert *experts, const qo_expert *shared,
                         double topp, int32_t *idx, float *w, float *out)
{
    const int E = c->n_experts, k = c->top_k, H = c->hidden;
    const int64_t A = (int64_t)T * k;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *sorted = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    int32_t *uid = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    float *ys = (float *)malloc(sizeof(float) * (size_t)(A * H));
    float *ysh = shared ? (float *)malloc(sizeof(float) * (size_t)T * H) : NULL;
    int32_t nu = 0;
    qo_router(c, act, T, Wr, bias, idx, w, NULL, NULL, NULL);
    qo_topp_prune(T, k, topp, c->routed_scaling_factor, idx, w);
    qo_permute(idx, T, k, E, counts, offsets, sorted, inv, uid, &nu);
    qo_expert_ffn(c, experts, offsets, sorted, uid, nu, act, NULL, ys);
    if (shared) qo_shared_ffn(c, shared, act, T, NULL, ysh);
    qo_combine(c, T, ys, ysh, w, inv, out);
    free(counts); free(offsets); free(sorted); free(inv); free(uid); free(ys); free(ysh);
}

void qo_moe_forward(const qo_cfg *c, const void *act, int T, const float *Wr,
                    const float *bias, const qo_expert *experts, const qo_expert *shared,
                    int32_t *idx, float *w, float *out)
{
    qo_moe_forward_opts(c, act, T, Wr, bias, experts, shared, 0.0, idx, w, out);
}
