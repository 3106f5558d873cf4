/*
 * Flint MoE block oracle: a plain, slow fp64 CPU statement of what the block
 * computes.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
 * benchmark's CPU-baseline leg call it; the CUDA library never does, and the
 * two share no code.
 *
 * Definitions followed (page titles and sections of the source pages):
 *  - "How to Run Flint Locally", section "The architecture, from config.json":
 *    256 routed experts per MoE layer, 6 per token, expert size 512, a sigmoid
 *    router with normalized top-k; one shared expert of size 1,024 that runs
 *    for every token; each routed expert is three 2,048 x 512 matrices.
 *  - TandemLLM "21 Flint", section 21.1 "The model": experts "routed by
 *    sigmoid score with a bias"; SwiGLU MLPs.  Section 21.2 "The packs": the
 *    engine multiplies the routing weights back onto the expert outputs.
 *  - The quantization format (symmetric int4, codes in [-8, 7], one bf16 scale
 *    per 128 consecutive elements along K) and the stack recipe (RMSNorm with
 *    eps 1e-6 and unit weight, residual add in fp32) are the workload's own
 *    definitions; the pages ship other 4-bit formats, which the layer's
 *    `format` also states: group-64 affine int4 ("How to Run Flint Locally",
 *    section "Every build and its size") and NVFP4 weight-only (section "What
 *    vLLM changed").
 *
 * Readings where the pages are silent: the bias is added to sigmoid(z) and is
 * used for selection only; the combine weights are the unbiased sigmoid
 * scores of the chosen experts divided by their sum; equal biased scores are
 * broken toward the lower expert index; the shared expert is ungated (weight
 * 1); no routed scaling factor; no group-limited routing.
 *
 * Packed layout read here (its own unpacker): row n of a [N, K] matrix is K/2
 * bytes, byte j holding element 2j in the low nibble and 2j+1 in the high
 * nibble, each a two's-complement 4-bit code; scales are [N, K/128] bf16 bits.
 */
#ifndef FLINT_ORACLE_H
#define FLINT_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int n_experts, top_k, hidden, expert_i, shared_i;
  const uint16_t *router_w; /* [E][H] bf16 bits */
  const float *router_b;    /* [E] */
  const uint8_t *w13_q;     /* [E][2I][H/2]  rows 0..I-1 gate, I..2I-1 up */
  const uint16_t *w13_s;    /* [E][2I][H/128] */
  const uint8_t *w2_q;      /* [E][H][I/2] */
  const uint16_t *w2_s;     /* [E][H][I/128] */
  const uint8_t *sh13_q;    /* [2Is][H/2] */
  const uint16_t *sh13_s;   /* [2Is][H/128] */
  const uint8_t *sh2_q;     /* [H][Is/2] */
  const uint16_t *sh2_s;    /* [H][Is/128] */
  /* Routed up projections stored divided by this (TandemLLM "21 Flint",
   * section 21.2 "The packs": expert_interm_div, the routing weights
   * multiplied back in the combine); 0 or 1: not divided. */
  double expert_interm_div;
  /* Format of the expert matrices (the router is bf16 in both): 0 the
   * symmetric int4 above; 1 group-64 affine int4 ("How to Run Flint Locally",
   * section "Every build and its size": the MLX int4 build, the Q4_1 GGUF):
   * unsigned codes 0..15 in the same nibble order, the *_s arrays fp16 scales
   * [rows][K/64] and the *_m arrays fp16 offsets [rows][K/64],
   * weight = code * scale + offset.  2 NVFP4 weight-only ("How to Run Flint
   * Locally", section "What vLLM changed": the NVFP4 checkpoint runs with BF16
   * activations): the *_q arrays FP4 E2M1 codes in the same nibble order, the
   * *_s arrays (read as bytes) FP8 E4M3 scales [rows][K/16], and one fp32
   * global scale per expert matrix in the *_g arrays (w13_g [E] for an
   * expert's gate and up rows, w2_g [E], sh13_g [1], sh2_g [1]);
   * weight = e2m1(code) * e4m3(scale) * global. */
  int format;
  const uint16_t *w13_m, *w2_m, *sh13_m, *sh2_m;
  const float *w13_g, *w2_g, *sh13_g, *sh2_g;
} oracle_layer;

void oracle_set_threads(int n);
int oracle_get_threads(void);

/* codes[i] = the int4 code of element i of a packed row of n elements */
void oracle_unpack_int4(const uint8_t *q, int64_t n, int8_t *codes);
/* W[n][k] = code * scale, exactly, for an [N, K] packed matrix */
void oracle_dequant(const uint8_t *q, const uint16_t *s, int64_t N, int64_t K, double *W);
double oracle_bf16_to_double(uint16_t v);
uint16_t oracle_double_to_bf16(double v); /* round to nearest, ties to even */

/* y[b][n] = sum_k W[n][k] x[b][k]; argmax[b] lowest index of the row maximum;
 * gap[b] = top-1 minus top-2 value (argmax/gap may be NULL). */
void oracle_int4_gemv(const uint8_t *q, const uint16_t *s, int64_t N, int64_t K,
                      const uint16_t *x, int B, double *y, int32_t *argmax, double *gap);

/* Group-64 affine int4 ("How to Run Flint Locally", section "Every build and
 * its size": the MLX int4 build quantizes to group-64 affine int4; the Q4_1
 * GGUF stores the same codes with FP16 scales and offsets).  Row n of an
 * [N, K] matrix: q as above but each nibble an UNSIGNED code 0..15, s and m
 * [N, K/64] fp16 bits; weight = code * s + m, exactly, in fp64. */
double oracle_fp16_to_double(uint16_t v);
void oracle_dequant_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t N,
                           int64_t K, double *W);
void oracle_int4_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t N,
                             int64_t K, const uint16_t *x, int B, double *y, int32_t *argmax,
                             double *gap);

/* NVFP4 weight-only ("How to Run Flint Locally", section "What vLLM changed":
 * the NVFP4 checkpoint runs weight-only with BF16 activations; FP4 E2M1
 * elements, one FP8 E4M3 scale per 16 elements, one FP32 scale per tensor).
 * Row n of an [N, K] matrix: q packed as above, each nibble an E2M1 code
 * (sign bit 3, exponent bits 2-1 with bias 1, mantissa bit 0); s [N, K/16]
 * E4M3 codes (sign bit 7, exponent bits 6-3 with bias 7, mantissa bits 2-0;
 * 0x7F / 0xFF NaN); weight = e2m1 * e4m3 * global, exactly, in fp64. */
double oracle_e2m1_to_double(uint8_t v);
double oracle_e4m3_to_double(uint8_t v);
void oracle_dequant_nvfp4(const uint8_t *q, const uint8_t *s, float global, int64_t N, int64_t K,
                          double *W);
void oracle_int4_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float global, int64_t N,
                            int64_t K, const uint16_t *x, int B, double *y, int32_t *argmax,
                            double *gap);

/* Router for B rows.  z, sig, biased: [B][E] (any may be NULL); idx, w: [B][k];
 * gap[b] = k-th minus (k+1)-th biased score in selection order. */
void oracle_route(const oracle_layer *L, const uint16_t *x, int B, double *z, double *sig,
                  double *biased, int32_t *idx, double *w, double *gap);

/* One SwiGLU expert on one fp64 input row: y = W2 (silu(W1 x) * (W3 x)). */
void oracle_swiglu_expert(const uint8_t *q13, const uint16_t *s13, const uint8_t *q2,
                          const uint16_t *s2, int hidden, int inter, const double *x, double *y);

/* The MoE block for B rows of bf16 input: out[b] = sum_j w_j y_j + y_shared.
 * idx, w, gap as in oracle_route (may be NULL). */
void oracle_moe_layer(const oracle_layer *L, const uint16_t *x, int B, double *out,
                      int32_t *idx, double *w, double *gap);

/* The terms of the block from the routed experts e_lo <= e < e_hi and (with
 * with_shared) the shared expert: one rank's share under expert parallelism;
 * the sum over a partition of the experts is the block output.  Routing is
 * over all experts. */
void oracle_moe_layer_partial(const oracle_layer *L, const uint16_t *x, int B, int e_lo, int e_hi,
                              int with_shared, double *out);

/* x = bf16(h / sqrt(mean(h^2) + eps)) for B rows of length H (unit weight). */
void oracle_rmsnorm_bf16(const float *h, int B, int H, double eps, uint16_t *x);

/* One stacked decode layer: x = rmsnorm(h); h <- fp32(h + bf16(moe(x))).
 * h is [B][H] fp32, updated in place.  idx/w/gap as above (may be NULL). */
void oracle_stack_layer(const oracle_layer *L, float *h, int B, double eps, int32_t *idx,
                        double *w, double *gap);

#ifdef __cplusplus
}
#endif
#endif
