/*
 * moe_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU statement of what the 4-bit mixture-of-experts layer computes, used to check
 * the CUDA library.  Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load it; the library itself never links, calls or falls back to it, and it shares no code,
 * header or table with the CUDA sources.
 *
 * What it follows:
 *  - "Perplexity Open-Sources Lily, a Qwen-Specific Mac Engine That Beats MLX-LM in Its Test",
 *    section "A runtime shaped around one model": every token goes to 8 of 256 routed experts and
 *    additionally to one shared expert; experts receive uneven numbers of tokens.
 *  - same page, section "The optimizations follow the workload": 4-bit weights are reconstructed
 *    inside the matrix products (so the result is the product with the dequantised weights), and
 *    routing happens on the device (no host step changes the result).
 *  - the layer definition this library implements (not on the pages): router softmax over the E
 *    experts, the top-k kept and their probabilities renormalised; a sigmoid gate on the shared
 *    expert; SwiGLU experts down(silu(gate x) * (up x)); int4 weights with an asymmetric
 *    per-64-column group scale and bias stored in bf16.
 *
 * Precision: each weight is dequantised in fp32 as  W = fp32(q) * fp32(s)  then  + fp32(b)  (two
 * fp32 roundings; compile with -ffp-contract=off), every product and sum after that is fp64.
 *
 * Readings taken where the definition is silent (each listed in the design notes):
 *  - top-k order is descending logit; equal logits go to the lower expert index;
 *  - gates are softmax over all E logits, restricted to the k selected and renormalised;
 *  - the shared expert has the same intermediate size and quantisation format as the routed ones,
 *    and its gate is sigmoid(x . w_sg) with an fp32 vector w_sg;
 *  - a router bias (when given) is added to the logits before selection and before the softmax;
 *  - bucketing is a stable counting sort: bucket e lists its (token, slot) entries in token order.
 *
 * Pins for every function live in tests/test_oracle_pins.py (closed forms, brute force,
 * invariants and library special cases); nothing here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t H, I, E, k, group, has_shared;
    /* routed experts: gate/up [E, I, H/8] words, down [E, H, I/8]; scale/bias [E, rows, cols/group] */
    const uint32_t *q_gate, *q_up, *q_down;
    const uint16_t *s_gate, *b_gate, *s_up, *b_up, *s_down, *b_down;
    /* shared expert: the same with E = 1 (may be NULL when has_shared == 0) */
    const uint32_t *qs_gate, *qs_up, *qs_down;
    const uint16_t *ss_gate, *bs_gate, *ss_up, *bs_up, *ss_down, *bs_down;
    const float *router;        /* [E, H] */
    const float *router_bias;   /* [E] or NULL */
    const float *shared_gate;   /* [H] or NULL */
} oracle_layer;

/* bf16 bit pattern -> fp32 value (bf16 is the top half of an IEEE binary32) */
static float bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* One dequantised weight: element (r, c) of a packed [rows, cols] matrix. */
static float weight_at(const uint32_t *q, const uint16_t *s, const uint16_t *b,
                       int cols, int group, int r, int c)
{
    uint32_t word = q[(size_t)r * (size_t)(cols / 8) + (size_t)(c / 8)];
    uint32_t nibble = (word >> (4 * (c % 8))) & 0xFu;
    size_t gi = (size_t)r * (size_t)(cols / group) + (size_t)(c / group);
    float scaled = (float)nibble * bf16_value(s[gi]);
    return scaled + bf16_value(b[gi]);
}

void oracle_dequant(const uint32_t *q, const uint16_t *s, const uint16_t *b,
                    int rows, int cols, int group, float *out)
{
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            out[(size_t)r * cols + c] = weight_at(q, s, b, cols, group, r, c);
}

/* logits[t, e] = x_t . router_e (+ bias_e), fp64 */
void oracle_router_logits(const oracle_layer *L, const uint16_t *x, int T, double *logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < L->E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < L->H; ++h)
                acc += (double)bf16_value(x[(size_t)t * L->H + h]) * (double)L->router[(size_t)e * L->H + h];
            if (L->router_bias)
                acc += (double)L->router_bias[e];
            logits[(size_t)t * L->E + e] = acc;
        }
    }
}

/* Top-k of one token's logits, then softmax over all E restricted to the selection. */
static void select_one(const double *l, int E, int k, int32_t *idx, double *gates)
{
    char *taken = (char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || l[e] > l[best]) best = e;   /* strict '>' keeps the lower index on ties */
        }
        taken[best] = 1;
        idx[j] = best;
    }
    free(taken);
    double lmax = l[0];
    for (int e = 1; e < E; ++e) if (l[e] > lmax) lmax = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += exp(l[e] - lmax);
    double sel = 0.0;
    for (int j = 0; j < k; ++j) sel += exp(l[idx[j]] - lmax) / z;
    for (int j = 0; j < k; ++j) gates[j] = (exp(l[idx[j]] - lmax) / z) / sel;
}

void oracle_select(const double *logits, int T, int E, int k, int32_t *idx, double *gates)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        select_one(logits + (size_t)t * E, E, k, idx + (size_t)t * k, gates + (size_t)t * k);
}

/* sg[t] = sigmoid(x_t . w_sg) */
void oracle_shared_gate(const oracle_layer *L, const uint16_t *x, int T, double *sg)
{
    for (int t = 0; t < T; ++t) {
        double z = 0.0;
        for (int h = 0; h < L->H; ++h)
            z += (double)bf16_value(x[(size_t)t * L->H + h]) * (double)L->shared_gate[h];
        sg[t] = 1.0 / (1.0 + exp(-z));
    }
}

/* Stable counting sort of the T*k (token, slot) entries by expert.
 * counts[e]; offsets[e] = sum of counts before e, offsets[E] = T*k;
 * perm[p] = t*k + j of the entry at bucket position p (bucket-major, token ascending). */
void oracle_bucket(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                   int32_t *perm)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int i = 0; i < T * k; ++i) counts[idx[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            perm[fill[e]++] = t * k + j;
        }
    free(fill);
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y = down(silu(gate x) * (up x)) for one token; e == L->E selects the shared expert. */
void oracle_expert_ffn(const oracle_layer *L, int e, const double *xt, double *y)
{
    const int H = L->H, I = L->I, G = L->group;
    const uint32_t *qg, *qu, *qd;
    const uint16_t *sg, *bg, *su, *bu, *sd, *bd;
    if (e == L->E) {
        qg = L->qs_gate; qu = L->qs_up; qd = L->qs_down;
        sg = L->ss_gate; bg = L->bs_gate; su = L->ss_up; bu = L->bs_up; sd = L->ss_down; bd = L->bs_down;
    } else {
        size_t wu = (size_t)e * I * (H / 8), gu = (size_t)e * I * (H / G);
        size_t wd = (size_t)e * H * (I / 8), gd = (size_t)e * H * (I / G);
        qg = L->q_gate + wu; qu = L->q_up + wu; qd = L->q_down + wd;
        sg = L->s_gate + gu; bg = L->b_gate + gu; su = L->s_up + gu; bu = L->b_up + gu;
        sd = L->s_down + gd; bd = L->b_down + gd;
    }
    double *act = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            g += (double)weight_at(qg, sg, bg, H, G, i, h) * xt[h];
            u += (double)weight_at(qu, su, bu, H, G, i, h) * xt[h];
        }
        act[i] = silu(g) * u;
    }
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i)
            acc += (double)weight_at(qd, sd, bd, I, G, h, i) * act[i];
        y[h] = acc;
    }
    free(act);
}

/* Forward of the listed tokens: route, run the k selected experts and the shared expert, combine.
 * y: [ntok, H] fp64.  idx/gates/sg outputs may be NULL.  dense != 0 runs every one of the E routed
 * experts, with a zero gate for the ones not selected (brute-force check of the sparse path). */
static void forward_impl(const oracle_layer *L, const uint16_t *x, int T, const int32_t *tokens,
                         int ntok, double *y, int32_t *idx_out, double *gates_out, double *sg_out,
                         int dense)
{
    (void)T;
    const int H = L->H, E = L->E, k = L->k;
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < ntok; ++n) {
        int t = tokens ? tokens[n] : n;
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *fe = (double *)malloc(sizeof(double) * (size_t)H);
        double *gate_of = (double *)calloc((size_t)E, sizeof(double));
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *g = (double *)malloc(sizeof(double) * (size_t)k);
        double *yt = y + (size_t)n * H;
        for (int h = 0; h < H; ++h) xt[h] = (double)bf16_value(x[(size_t)t * H + h]);
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h) acc += xt[h] * (double)L->router[(size_t)e * H + h];
            if (L->router_bias) acc += (double)L->router_bias[e];
            l[e] = acc;
        }
        select_one(l, E, k, sel, g);
        for (int j = 0; j < k; ++j) gate_of[sel[j]] = g[j];
        for (int h = 0; h < H; ++h) yt[h] = 0.0;
        if (dense) {
            for (int e = 0; e < E; ++e) {
                oracle_expert_ffn(L, e, xt, fe);
                for (int h = 0; h < H; ++h) yt[h] += gate_of[e] * fe[h];
            }
        } else {
            for (int j = 0; j < k; ++j) {
                oracle_expert_ffn(L, sel[j], xt, fe);
                for (int h = 0; h < H; ++h) yt[h] += g[j] * fe[h];
            }
        }
        double s = 0.0;
        if (L->has_shared) {
            double z = 0.0;
            for (int h = 0; h < H; ++h) z += xt[h] * (double)L->shared_gate[h];
            s = 1.0 / (1.0 + exp(-z));
            oracle_expert_ffn(L, E, xt, fe);
            for (int h = 0; h < H; ++h) yt[h] += s * fe[h];
        }
        if (idx_out) for (int j = 0; j < k; ++j) idx_out[(size_t)n * k + j] = sel[j];
        if (gates_out) for (int j = 0; j < k; ++j) gates_out[(size_t)n * k + j] = g[j];
        if (sg_out) sg_out[n] = s;
        free(xt); free(l); free(fe); free(gate_of); free(sel); free(g);
    }
}

void oracle_forward(const oracle_layer *L, const uint16_t *x, int T, const int32_t *tokens,
                    int ntok, double *y, int32_t *idx_out, double *gates_out, double *sg_out)
{
    forward_impl(L, x, T, tokens, ntok, y, idx_out, gates_out, sg_out, 0);
}

void oracle_forward_dense(const oracle_layer *L, const uint16_t *x, int T, const int32_t *tokens,
                          int ntok, double *y)
{
    forward_impl(L, x, T, tokens, ntok, y, NULL, NULL, NULL, 1);
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
