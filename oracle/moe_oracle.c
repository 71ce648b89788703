/*
 * moe_oracle.c -- fp64 CPU oracle, one literal step at a time.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
 * Shares no code with the CUDA library.  See moe_oracle.h for the sources,
 * the conventions and what each function computes.
 *
 * Build: cc -O2 -std=c11 -shared -fPIC moe_oracle.c -lm (see build_oracle.py).
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 --- */

double oracle_bf16_to_f64(uint16_t h)
{
    /* a bf16 value is the upper half of an IEEE binary32 */
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80);
    /* a = m * 2^e with m in [0.5, 1).  bf16 keeps 8 significant bits, so the
     * spacing of representable values near a is 2^(e-8); below the smallest
     * normal (2^-126) the spacing is fixed at 2^-133. */
    int e;
    (void)frexp(a, &e);
    int qe = e - 8;
    if (qe < -133)
        qe = -133;
    double n = nearbyint(ldexp(a, -qe)); /* round half to even (default mode) */
    double r = ldexp(n, qe);
    if (r >= 0x1p128)
        return (uint16_t)(sign | 0x7F80); /* rounds past the largest bf16 */
    float f = (float)r;                  /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ------------------------------------------------------------- format --- */

/* Code widths: 2, 3 or 4 bits.  A row of `cols` codes is a little-endian bit
 * stream of cols*bits/32 uint32 words: code j takes stream bits
 * [bits*j, bits*j + bits), and word w holds stream bits [32w, 32w + 32).  With
 * 2 or 4 bits no code straddles two words (code j is then at bit
 * bits*(j % (32/bits)) of word j / (32/bits)); 3-bit codes may. */
static int valid_bits(int bits)
{
    return bits == 2 || bits == 3 || bits == 4;
}

static int row_words(int bits, int64_t cols, int64_t *wpr)
{
    if (!valid_bits(bits) || cols < 0 || (cols * bits) % 32)
        return -1;
    *wpr = cols * bits / 32;
    return 0;
}

/* code j of a row's bit stream */
static unsigned stream_code(const uint32_t *row, int bits, int64_t j)
{
    int64_t o = (int64_t)bits * j;
    uint64_t pair = row[o / 32];
    if (o % 32 + bits > 32)
        pair |= (uint64_t)row[o / 32 + 1] << 32;
    return (unsigned)((pair >> (o % 32)) & ((1u << bits) - 1u));
}

int oracle_pack(int bits, const uint8_t *q, int64_t rows, int64_t cols, uint32_t *words)
{
    int64_t wpr;
    if (row_words(bits, cols, &wpr) || rows < 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r) {
        uint32_t *row = words + r * wpr;
        for (int64_t w = 0; w < wpr; ++w)
            row[w] = 0u;
        for (int64_t j = 0; j < cols; ++j) {
            uint32_t c = q[r * cols + j];
            if (c >> bits)
                return -1;
            int64_t o = (int64_t)bits * j;
            row[o / 32] |= c << (o % 32);
            if (o % 32 + bits > 32)
                row[o / 32 + 1] |= c >> (32 - o % 32);
        }
    }
    return 0;
}

int oracle_unpack(int bits, const uint32_t *words, int64_t rows, int64_t cols, uint8_t *q)
{
    int64_t wpr;
    if (row_words(bits, cols, &wpr) || rows < 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j)
            q[r * cols + j] = (uint8_t)stream_code(words + r * wpr, bits, j);
    return 0;
}

static int check_mat(int bits, int group, int64_t rows, int64_t cols)
{
    int64_t wpr;
    if (row_words(bits, cols, &wpr) || group <= 0 || rows < 0 || cols <= 0)
        return -1;
    if (cols % group)
        return -1;
    return 0;
}

/* one code of a quantised matrix */
static unsigned code_at(int bits, const uint32_t *codes, int64_t cols, int64_t r, int64_t j)
{
    return stream_code(codes + r * (cols * bits / 32), bits, j);
}

int oracle_dequant(int bits, int group, int64_t rows, int64_t cols,
                   const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                   double *W)
{
    if (check_mat(bits, group, rows, cols))
        return -1;
    int64_t gpr = cols / group;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j) {
            double s = oracle_bf16_to_f64(scale[r * gpr + j / group]);
            double b = oracle_bf16_to_f64(bias[r * gpr + j / group]);
            W[r * cols + j] = (double)code_at(bits, codes, cols, r, j) * s + b;
        }
    return 0;
}

int oracle_qmatvec(int bits, int group, int64_t rows, int64_t cols,
                   const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                   const double *v, double *y)
{
    if (check_mat(bits, group, rows, cols))
        return -1;
    double *W = malloc(sizeof(double) * (size_t)(rows * cols));
    if (!W && rows > 0)
        return -3;
    oracle_dequant(bits, group, rows, cols, codes, scale, bias, W);
    for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t j = 0; j < cols; ++j)
            acc += W[r * cols + j] * v[j];
        y[r] = acc;
    }
    free(W);
    return 0;
}

int oracle_qmatvec_grouped(int bits, int group, int64_t rows, int64_t cols,
                           const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                           const double *v, double *y)
{
    if (check_mat(bits, group, rows, cols))
        return -1;
    int64_t gpr = cols / group;
    for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t g = 0; g < gpr; ++g) {
            double sq = 0.0, sv = 0.0;
            for (int64_t j = g * group; j < (g + 1) * group; ++j) {
                sq += (double)code_at(bits, codes, cols, r, j) * v[j];
                sv += v[j];
            }
            acc += oracle_bf16_to_f64(scale[r * gpr + g]) * sq
                 + oracle_bf16_to_f64(bias[r * gpr + g]) * sv;
        }
        y[r] = acc;
    }
    return 0;
}

/* ------------------------------------------------------------- router --- */

int oracle_route(int32_t E, int32_t H, int32_t k, const double *xhat,
                 const void *w_router, int router_is_f32, const double *logit_bias,
                 double *logits, int32_t *idx, double *w)
{
    if (E <= 0 || H <= 0 || k <= 0 || k > E || !xhat || !w_router || !idx || !w)
        return -1;
    double *l = malloc(sizeof(double) * (size_t)E);
    double *p = malloc(sizeof(double) * (size_t)E);
    char *taken = calloc((size_t)E, 1);
    if (!l || !p || !taken) {
        free(l); free(p); free(taken);
        return -3;
    }
    /* logits: router matrix times the normalised input, fp64 */
    for (int32_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int32_t h = 0; h < H; ++h) {
            double wr = router_is_f32
                ? (double)((const float *)w_router)[(int64_t)e * H + h]
                : oracle_bf16_to_f64(((const uint16_t *)w_router)[(int64_t)e * H + h]);
            acc += wr * xhat[h];
        }
        if (logit_bias)
            acc += logit_bias[e];
        l[e] = acc;
    }
    /* softmax over all experts (max-subtracted) */
    double mx = l[0];
    for (int32_t e = 1; e < E; ++e)
        if (l[e] > mx)
            mx = l[e];
    double z = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        p[e] = exp(l[e] - mx);
        z += p[e];
    }
    for (int32_t e = 0; e < E; ++e)
        p[e] /= z;
    /* top-k: k passes, each takes the largest remaining logit, lower index
     * first among equal values */
    for (int32_t i = 0; i < k; ++i) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || l[e] > l[best])
                best = e;
        }
        taken[best] = 1;
        idx[i] = best;
    }
    /* renormalise the selected probabilities to sum to one */
    double s = 0.0;
    for (int32_t i = 0; i < k; ++i)
        s += p[idx[i]];
    for (int32_t i = 0; i < k; ++i)
        w[i] = p[idx[i]] / s;
    if (logits)
        memcpy(logits, l, sizeof(double) * (size_t)E);
    free(l); free(p); free(taken);
    return 0;
}

/* --------------------------------------------------------- expert FFN --- */

static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

static int qmat_ok(const oracle_qmat *m)
{
    return m->codes && m->scale && m->bias;
}

int oracle_expert_ffn(int bits, int group, int32_t H, int32_t I, const oracle_qexpert *ex,
                      const double *xhat, double *h, double *y)
{
    if (H <= 0 || I <= 0 || !ex || !xhat || !y)
        return -1;
    if (!qmat_ok(&ex->gate) || !qmat_ok(&ex->up) || !qmat_ok(&ex->down))
        return -2;
    double *g = malloc(sizeof(double) * (size_t)I);
    double *u = malloc(sizeof(double) * (size_t)I);
    double *a = malloc(sizeof(double) * (size_t)I);
    if (!g || !u || !a) {
        free(g); free(u); free(a);
        return -3;
    }
    int rc = oracle_qmatvec(bits, group, I, H, ex->gate.codes, ex->gate.scale, ex->gate.bias, xhat, g);
    if (!rc)
        rc = oracle_qmatvec(bits, group, I, H, ex->up.codes, ex->up.scale, ex->up.bias, xhat, u);
    if (!rc) {
        for (int32_t i = 0; i < I; ++i)
            a[i] = silu(g[i]) * u[i]; /* SwiGLU */
        rc = oracle_qmatvec(bits, group, H, I, ex->down.codes, ex->down.scale, ex->down.bias, a, y);
    }
    if (!rc && h)
        memcpy(h, a, sizeof(double) * (size_t)I);
    free(g); free(u); free(a);
    return rc;
}

/* -------------------------------------------------------------- layer --- */

int oracle_layer_forward(const oracle_desc *d, int32_t T,
                         const uint16_t *xhat, const uint16_t *residual,
                         const void *w_router, int router_is_f32, const double *logit_bias,
                         const oracle_qexpert *experts, const oracle_qexpert *shared,
                         const uint16_t *shared_gate,
                         double *out, int32_t *idx, double *w, double *gamma)
{
    if (!d || T < 0)
        return -1;
    const int32_t H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k;
    if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || d->group_size <= 0)
        return -1;
    if (d->has_shared && !shared)
        return -1;
    if (T == 0)
        return 0;
    if (!xhat || !residual || !w_router || !experts || !out || !idx || !w)
        return -1;
    double *x = malloc(sizeof(double) * (size_t)H);
    double *y = malloc(sizeof(double) * (size_t)H);
    if (!x || !y) {
        free(x); free(y);
        return -3;
    }
    int rc = 0;
    for (int32_t t = 0; t < T && !rc; ++t) {
        for (int32_t j = 0; j < H; ++j)
            x[j] = oracle_bf16_to_f64(xhat[(int64_t)t * H + j]);
        double *o = out + (int64_t)t * H;
        for (int32_t j = 0; j < H; ++j)
            o[j] = oracle_bf16_to_f64(residual[(int64_t)t * H + j]);
        rc = oracle_route(E, H, k, x, w_router, router_is_f32,
                          logit_bias ? logit_bias + (int64_t)t * E : NULL,
                          NULL, idx + (int64_t)t * k, w + (int64_t)t * k);
        /* routed experts, weighted */
        for (int32_t i = 0; i < k && !rc; ++i) {
            rc = oracle_expert_ffn(d->bits, d->group_size, H, I,
                                   &experts[idx[(int64_t)t * k + i]], x, NULL, y);
            for (int32_t j = 0; j < H && !rc; ++j)
                o[j] += w[(int64_t)t * k + i] * y[j];
        }
        /* shared expert, gated */
        double gam = 1.0;
        if (!rc && d->has_shared) {
            if (shared_gate) {
                double z = 0.0;
                for (int32_t j = 0; j < H; ++j)
                    z += oracle_bf16_to_f64(shared_gate[j]) * x[j];
                gam = 1.0 / (1.0 + exp(-z));
            }
            rc = oracle_expert_ffn(d->bits, d->group_size, H, I, shared, x, NULL, y);
            for (int32_t j = 0; j < H && !rc; ++j)
                o[j] += gam * y[j];
        }
        if (gamma)
            gamma[t] = d->has_shared ? gam : 0.0;
    }
    free(x); free(y);
    return rc;
}

void oracle_rmsnorm(int32_t H, const double *x, double eps, double *out)
{
    double ss = 0.0;
    for (int32_t j = 0; j < H; ++j)
        ss += x[j] * x[j];
    double inv = 1.0 / sqrt(ss / (double)H + eps);
    for (int32_t j = 0; j < H; ++j)
        out[j] = x[j] * inv;
}
