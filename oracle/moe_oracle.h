/*
 * moe_oracle.h -- plain, slow fp64 CPU oracle for one decoder layer's
 * quantised MoE expert FFN (router softmax/top-k, gate/up/down mat-vecs over
 * 4-bit or 2-bit affine group-quantised experts, SwiGLU, routing-weighted
 * combine with the shared expert and the residual).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this library.  It shares no
 * code, header, table or helper with the CUDA library; the product path never
 * calls it.
 *
 * Sources (web pages, cited by title and section):
 *   [FlashMoE]  "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres
 *               sur un ordinateur portable" (fr.news.hada.io, topic 27758):
 *               sections "Architecture du modèle", "Technologies clés" >
 *               "SSD Expert Streaming", "Noyau de déquantification optimisé
 *               FMA", "Shaders de calcul Metal", "Deferred GPU Expert Compute".
 *   [PagedMoE]  "Qwen3.5-397B MoE fonctionne avec 14 Go de RAM via un
 *               chargement d'expert paginé sur M1 Ultra" (openclawradar.com),
 *               opening paragraph (512 experts, top-10 routing).
 *
 * Every function below is pinned by CPU tests against facts fixed outside the
 * oracle itself (worked examples, closed forms, brute force, library
 * routines); none is "parity unpinned".
 *
 * Conventions (readings of the pages where they are silent):
 *   - codes: each row is a little-endian bit stream of uint32 words; element
 *     j takes stream bits [b*j, b*j + b) (word w holds stream bits
 *     [32w, 32w + 32)), low bits first, b in {2, 3, 4}.  For b = 2 or 4 this
 *     is bits [b*(j % (32/b)), ...) of word j / (32/b); 3-bit codes may
 *     straddle two words.  Every row starts on a word boundary.
 *   - weight of element j of row r: q * scale[r][j/G] + bias[r][j/G]
 *     ([FlashMoE] "Noyau de déquantification optimisé FMA": nibble*scale+bias).
 *   - gate/up matrices are [inter][hidden], down is [hidden][inter] (out x in).
 *   - top-k: k largest logits, ties to the lower expert index, returned in
 *     that order; weights = softmax over the selected logits (sum to 1).
 *   - h = silu(gate) * up, silu(z) = z / (1 + exp(-z)).
 *   - out = residual + sum_i w_i y_{e_i} + gamma * y_shared,
 *     gamma = sigmoid(shared_gate . xhat) when a shared gate is given, else 1.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 bit patterns <-> double.  bf16 -> double is exact.  double -> bf16 is
 * one round-to-nearest-even step straight from the double (no double
 * rounding through float). */
double   oracle_bf16_to_f64(uint16_t h);
uint16_t oracle_f64_to_bf16(double v);

/* Pack/unpack `rows` x `cols` codes (each in [0, 2^bits)) to/from words,
 * bits in {2, 3, 4}; cols * bits must be a multiple of 32.  Returns 0, or -1 on a
 * bad argument. */
int oracle_pack(int bits, const uint8_t *q, int64_t rows, int64_t cols, uint32_t *words);
int oracle_unpack(int bits, const uint32_t *words, int64_t rows, int64_t cols, uint8_t *q);

/* Materialise the fp64 weight matrix W[rows][cols] = q*s + b of one
 * quantised matrix (codes words, bf16 scale/bias [rows][cols/group]). */
int oracle_dequant(int bits, int group, int64_t rows, int64_t cols,
                   const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                   double *W);

/* y = W v for a quantised matrix, by materialising W (literal form). */
int oracle_qmatvec(int bits, int group, int64_t rows, int64_t cols,
                   const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                   const double *v, double *y);

/* The same product in the rewritten form y_r = sum_g [ s_rg * sum_{j in g} q_j v_j
 * + b_rg * sum_{j in g} v_j ], the algebra of [FlashMoE] "Noyau de
 * déquantification optimisé FMA".  A second formulation used to pin the
 * first. */
int oracle_qmatvec_grouped(int bits, int group, int64_t rows, int64_t cols,
                           const uint32_t *codes, const uint16_t *scale, const uint16_t *bias,
                           const double *v, double *y);

/* One quantised matrix: codes, bf16 scale, bf16 bias (host pointers). */
typedef struct {
    const uint32_t *codes;
    const uint16_t *scale;
    const uint16_t *bias;
} oracle_qmat;

/* One expert: gate [I][H], up [I][H], down [H][I]. */
typedef struct {
    oracle_qmat gate, up, down;
} oracle_qexpert;

typedef struct {
    int32_t hidden, inter, n_experts, top_k, group_size, bits, has_shared;
} oracle_desc;

/* Router: logits[e] = sum_h Wr[e][h] xhat[h] (+ logit_bias[e] if given),
 * router_is_f32 selects fp32 or bf16 Wr [E][H].  Top-k as described above;
 * idx[k], w[k] out.  logits may be NULL. */
int oracle_route(int32_t E, int32_t H, int32_t k, const double *xhat,
                 const void *w_router, int router_is_f32, const double *logit_bias,
                 double *logits, int32_t *idx, double *w);

/* One expert's FFN: y = W_down (silu(W_gate xhat) * (W_up xhat)).  h (length
 * I) may be NULL; when given it receives the SwiGLU activations. */
int oracle_expert_ffn(int bits, int group, int32_t H, int32_t I, const oracle_qexpert *ex,
                      const double *xhat, double *h, double *y);

/* Whole layer for T tokens.
 *   xhat      bf16 [T][H]  normalised layer input
 *   residual  bf16 [T][H]  residual added to the output
 *   experts   E entries (entries of unselected experts may hold NULL pointers)
 *   shared    NULL or the shared expert (used iff desc->has_shared)
 *   shared_gate NULL or bf16 [H]
 *   logit_bias NULL or fp64 [T][E]
 * Out: out fp64 [T][H]; idx [T][k]; w fp64 [T][k]; gamma fp64 [T] (may be NULL).
 * Returns 0, -1 on a bad argument, -2 if a selected expert has NULL pointers. */
int oracle_layer_forward(const oracle_desc *d, int32_t T,
                         const uint16_t *xhat, const uint16_t *residual,
                         const void *w_router, int router_is_f32, const double *logit_bias,
                         const oracle_qexpert *experts, const oracle_qexpert *shared,
                         const uint16_t *shared_gate,
                         double *out, int32_t *idx, double *w, double *gamma);

/* RMSNorm with unit weight: out = x / sqrt(mean(x^2) + eps). */
void oracle_rmsnorm(int32_t H, const double *x, double eps, double *out);

#ifdef __cplusplus
}
#endif
#endif /* MOE_ORACLE_H */
