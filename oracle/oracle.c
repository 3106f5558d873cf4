/*
 * Flint MoE block oracle, fp64 CPU.  TEST INFRASTRUCTURE ONLY (tests, smoke
 * check, benchmark CPU baseline); see oracle.h for the definitions followed and
 * the readings taken where the pages are silent.  Every sum is a plain
 * left-to-right fp64 loop; threads only split independent output rows.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------ threading */
static int g_threads = 1;
void oracle_set_threads(int n) { g_threads = n < 1 ? 1 : n; }
int oracle_get_threads(void) { return g_threads; }

typedef void (*range_fn)(void *ctx, int64_t i);
typedef struct {
  range_fn fn;
  void *ctx;
  int64_t lo, hi;
} chunk;

/* set inside a worker: a par_for called from one runs its loop itself */
static __thread int t_in_worker = 0;

static void *run_chunk(void *p) {
  chunk *c = (chunk *)p;
  t_in_worker = 1;
  for (int64_t i = c->lo; i < c->hi; ++i) c->fn(c->ctx, i);
  return NULL;
}

/* fn(ctx, i) for i in [0, n): contiguous chunks, one per thread. */
static void par_for(int64_t n, range_fn fn, void *ctx) {
  int t = t_in_worker ? 1 : g_threads;
  if (t > n) t = (int)n;
  if (t <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(ctx, i);
    return;
  }
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * t);
  chunk *ch = (chunk *)malloc(sizeof(chunk) * t);
  for (int i = 0; i < t; ++i) {
    ch[i].fn = fn;
    ch[i].ctx = ctx;
    ch[i].lo = n * i / t;
    ch[i].hi = n * (i + 1) / t;
    pthread_create(&th[i], NULL, run_chunk, &ch[i]);
  }
  for (int i = 0; i < t; ++i) pthread_join(th[i], NULL);
  free(th);
  free(ch);
}

/* ------------------------------------------------------------ numbers */
double oracle_bf16_to_double(uint16_t v) {
  uint32_t u = (uint32_t)v << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

uint16_t oracle_double_to_bf16(double v) {
  /* v = m * 2^e with 0.5 <= |m| < 1; keep 8 significant bits of m, rounding
   * to nearest with ties to even (nearbyint under the default mode). */
  int e;
  double m = frexp(v, &e);
  double r = ldexp(nearbyint(m * 256.0), e - 8);
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

static float round_to_float(double v) { return (float)v; } /* IEEE nearest-even */

/* The int4 code of element k of a packed row (low nibble = even element). */
static int code_of(const uint8_t *row, int64_t k) {
  uint8_t byte = row[k / 2];
  int nib = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
  return nib >= 8 ? nib - 16 : nib;
}

void oracle_unpack_int4(const uint8_t *q, int64_t n, int8_t *codes) {
  for (int64_t k = 0; k < n; ++k) codes[k] = (int8_t)code_of(q, k);
}

/* Weight element (n, k) of a packed [N, K] matrix: code * its group's scale. */
static double weight(const uint8_t *q, const uint16_t *s, int64_t K, int64_t n, int64_t k) {
  const uint8_t *row = q + n * (K / 2);
  double scale = oracle_bf16_to_double(s[n * (K / 128) + k / 128]);
  return (double)code_of(row, k) * scale;
}

void oracle_dequant(const uint8_t *q, const uint16_t *s, int64_t N, int64_t K, double *W) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) W[n * K + k] = weight(q, s, K, n, k);
}

/* sum_k W[n][k] x[k], left to right */
static double row_dot(const uint8_t *q, const uint16_t *s, int64_t K, int64_t n, const double *x) {
  double acc = 0.0;
  for (int64_t k = 0; k < K; ++k) acc += weight(q, s, K, n, k) * x[k];
  return acc;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ------------------------------------------------------------ group-64 affine int4 */
/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_double(uint16_t v) {
  const int sign = v >> 15, e = (v >> 10) & 31, f = v & 1023;
  double mag;
  if (e == 0) mag = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
  else if (e == 31) mag = f ? NAN : INFINITY;
  else mag = ldexp((double)(1024 + f), e - 25);            /* (1 + f/1024) * 2^(e-15) */
  return sign ? -mag : mag;
}

/* The unsigned code of element k of a packed row (low nibble = even element). */
static int ucode_of(const uint8_t *row, int64_t k) {
  uint8_t byte = row[k / 2];
  return (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
}

/* Weight element (n, k): code * scale + offset of its 64-element group. */
static double weight_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t K,
                            int64_t n, int64_t k) {
  const int64_t g = n * (K / 64) + k / 64;
  return (double)ucode_of(q + n * (K / 2), k) * oracle_fp16_to_double(s[g]) +
         oracle_fp16_to_double(m[g]);
}

static double row_dot_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t K,
                             int64_t n, const double *x) {
  double acc = 0.0;
  for (int64_t k = 0; k < K; ++k) acc += weight_affine(q, s, m, K, n, k) * x[k];
  return acc;
}

void oracle_dequant_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t N,
                           int64_t K, double *W) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) W[n * K + k] = weight_affine(q, s, m, K, n, k);
}

/* ------------------------------------------------------------ int4 GEMV */
typedef struct {
  const uint8_t *q;
  const uint16_t *s;
  int64_t N, K;
  const double *x; /* [K] */
  double *y;       /* [N] */
} gemv_ctx;

static void gemv_row(void *p, int64_t n) {
  gemv_ctx *c = (gemv_ctx *)p;
  c->y[n] = row_dot(c->q, c->s, c->K, n, c->x);
}

static void to_double(const uint16_t *x, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_double(x[i]);
}

/* argmax[b] = lowest index of the row maximum; gap[b] = top-1 minus top-2 */
static void argmax_row(const double *yb, int64_t N, int32_t *argmax, double *gap) {
  int64_t best = 0;
  for (int64_t n = 1; n < N; ++n)
    if (yb[n] > yb[best]) best = n;
  double second = -INFINITY;
  for (int64_t n = 0; n < N; ++n)
    if (n != best && yb[n] > second) second = yb[n];
  if (argmax) *argmax = (int32_t)best;
  if (gap) *gap = yb[best] - second;
}

void oracle_int4_gemv(const uint8_t *q, const uint16_t *s, int64_t N, int64_t K,
                      const uint16_t *x, int B, double *y, int32_t *argmax, double *gap) {
  double *xd = (double *)malloc(sizeof(double) * K);
  for (int b = 0; b < B; ++b) {
    to_double(x + (int64_t)b * K, K, xd);
    gemv_ctx c = {q, s, N, K, xd, y + (int64_t)b * N};
    par_for(N, gemv_row, &c);
    argmax_row(y + (int64_t)b * N, N, argmax ? argmax + b : NULL, gap ? gap + b : NULL);
  }
  free(xd);
}

/* ------------------------------------------------------------ NVFP4 */
double oracle_e2m1_to_double(uint8_t v) {
  const int sign = (v >> 3) & 1, e = (v >> 1) & 3, m = v & 1;
  const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

double oracle_e4m3_to_double(uint8_t v) {
  const int sign = v >> 7, e = (v >> 3) & 15, m = v & 7;
  double mag;
  if (e == 15 && m == 7) mag = NAN;
  else if (e == 0) mag = ldexp((double)m, -9);            /* subnormal: m/8 * 2^-6 */
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Weight element (n, k): its E2M1 code times its 16-block's E4M3 scale times the global scale. */
static double weight_nvfp4(const uint8_t *q, const uint8_t *s, double global, int64_t K, int64_t n,
                           int64_t k) {
  return oracle_e2m1_to_double((uint8_t)ucode_of(q + n * (K / 2), k)) *
         oracle_e4m3_to_double(s[n * (K / 16) + k / 16]) * global;
}

void oracle_dequant_nvfp4(const uint8_t *q, const uint8_t *s, float global, int64_t N, int64_t K,
                          double *W) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) W[n * K + k] = weight_nvfp4(q, s, (double)global, K, n, k);
}

typedef struct {
  const uint8_t *q, *s;
  double global;
  int64_t K;
  const double *x;
  double *y;
} gemv_nvfp4_ctx;

static void gemv_nvfp4_row(void *p, int64_t n) {
  gemv_nvfp4_ctx *c = (gemv_nvfp4_ctx *)p;
  double acc = 0.0;
  for (int64_t k = 0; k < c->K; ++k) acc += weight_nvfp4(c->q, c->s, c->global, c->K, n, k) * c->x[k];
  c->y[n] = acc;
}

typedef struct {
  const uint8_t *q;
  const uint16_t *s, *m;
  int64_t K;
  const double *x;
  double *y;
} gemv_affine_ctx;

static void gemv_affine_row(void *p, int64_t n) {
  gemv_affine_ctx *c = (gemv_affine_ctx *)p;
  double acc = 0.0;
  for (int64_t k = 0; k < c->K; ++k) acc += weight_affine(c->q, c->s, c->m, c->K, n, k) * c->x[k];
  c->y[n] = acc;
}

void oracle_int4_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int64_t N,
                             int64_t K, const uint16_t *x, int B, double *y, int32_t *argmax,
                             double *gap) {
  double *xd = (double *)malloc(sizeof(double) * K);
  for (int b = 0; b < B; ++b) {
    to_double(x + (int64_t)b * K, K, xd);
    gemv_affine_ctx c = {q, s, m, K, xd, y + (int64_t)b * N};
    par_for(N, gemv_affine_row, &c);
    argmax_row(y + (int64_t)b * N, N, argmax ? argmax + b : NULL, gap ? gap + b : NULL);
  }
  free(xd);
}

void oracle_int4_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float global, int64_t N,
                            int64_t K, const uint16_t *x, int B, double *y, int32_t *argmax,
                            double *gap) {
  double *xd = (double *)malloc(sizeof(double) * K);
  for (int b = 0; b < B; ++b) {
    to_double(x + (int64_t)b * K, K, xd);
    gemv_nvfp4_ctx c = {q, s, (double)global, K, xd, y + (int64_t)b * N};
    par_for(N, gemv_nvfp4_row, &c);
    argmax_row(y + (int64_t)b * N, N, argmax ? argmax + b : NULL, gap ? gap + b : NULL);
  }
  free(xd);
}

/* ------------------------------------------------------------ router */
/* Selection order: larger biased score first, lower expert index on ties. */
static int ranks_before(double bi, int i, double bj, int j) { return bi > bj || (bi == bj && i < j); }

static void route_row(const oracle_layer *L, const double *x, double *z, double *sig,
                      double *biased, int32_t *idx, double *w, double *gap) {
  const int E = L->n_experts, H = L->hidden, k = L->top_k;
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h)
      acc += oracle_bf16_to_double(L->router_w[(int64_t)e * H + h]) * x[h];
    z[e] = acc;
    sig[e] = sigmoid(acc);
    biased[e] = sig[e] + (double)L->router_b[e];
  }
  /* k picks by repeated scan (selection sort), then the (k+1)-th for the gap */
  char *taken = (char *)calloc(E, 1);
  int order[64];
  int npick = k + 1 <= E ? k + 1 : E;
  for (int p = 0; p < npick; ++p) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || ranks_before(biased[e], e, biased[best], best)) best = e;
    }
    taken[best] = 1;
    order[p] = best;
  }
  free(taken);
  double ssum = 0.0;
  for (int j = 0; j < k; ++j) ssum += sig[order[j]];
  for (int j = 0; j < k; ++j) {
    idx[j] = order[j];
    w[j] = sig[order[j]] / ssum;
  }
  *gap = (k < E) ? biased[order[k - 1]] - biased[order[k]] : INFINITY;
}

void oracle_route(const oracle_layer *L, const uint16_t *x, int B, double *z, double *sig,
                  double *biased, int32_t *idx, double *w, double *gap) {
  const int E = L->n_experts, H = L->hidden, k = L->top_k;
  double *xd = (double *)malloc(sizeof(double) * H);
  double *zz = (double *)malloc(sizeof(double) * E * 3);
  for (int b = 0; b < B; ++b) {
    to_double(x + (int64_t)b * H, H, xd);
    double g;
    route_row(L, xd, zz, zz + E, zz + 2 * E, idx + b * k, w + b * k, &g);
    if (z) memcpy(z + (int64_t)b * E, zz, sizeof(double) * E);
    if (sig) memcpy(sig + (int64_t)b * E, zz + E, sizeof(double) * E);
    if (biased) memcpy(biased + (int64_t)b * E, zz + 2 * E, sizeof(double) * E);
    if (gap) gap[b] = g;
  }
  free(xd);
  free(zz);
}

/* ------------------------------------------------------------ experts */
/* Several matrix-vector products whose output rows are numbered one after
 * the other, so that one par_for covers them all; each output element is the
 * plain left-to-right row_dot. */
/* A matrix of the set in one of the layer formats: fmt 0 symmetric int4
 * (s bf16), 1 group-64 affine (s fp16 scales, m fp16 offsets), 2 NVFP4 (s
 * E4M3 bytes, g the global scale). */
typedef struct {
  int n;
  const uint8_t *q[16];
  const void *s[16];
  const uint16_t *m[16];
  int fmt[16];
  double g[16];
  int64_t K[16], rows[16];
  const double *x[16];
  double *y[16];
} matvec_set;

static double row_dot_nvfp4(const uint8_t *q, const uint8_t *s, double global, int64_t K,
                            int64_t n, const double *x) {
  double acc = 0.0;
  for (int64_t k = 0; k < K; ++k) acc += weight_nvfp4(q, s, global, K, n, k) * x[k];
  return acc;
}

static void matvec_set_row(void *p, int64_t i) {
  matvec_set *m = (matvec_set *)p;
  int j = 0;
  while (i >= m->rows[j]) i -= m->rows[j++];
  if (m->fmt[j] == 2)
    m->y[j][i] = row_dot_nvfp4(m->q[j], (const uint8_t *)m->s[j], m->g[j], m->K[j], i, m->x[j]);
  else if (m->fmt[j] == 1)
    m->y[j][i] = row_dot_affine(m->q[j], (const uint16_t *)m->s[j], m->m[j], m->K[j], i, m->x[j]);
  else
    m->y[j][i] = row_dot(m->q[j], (const uint16_t *)m->s[j], m->K[j], i, m->x[j]);
}

static void matvec_set_add(matvec_set *m, int fmt, const uint8_t *q, const void *s,
                           const uint16_t *off, double global, int64_t rows, int64_t K,
                           const double *x, double *y) {
  m->q[m->n] = q, m->s[m->n] = s, m->m[m->n] = off, m->fmt[m->n] = fmt, m->g[m->n] = global;
  m->rows[m->n] = rows, m->K[m->n] = K, m->x[m->n] = x, m->y[m->n] = y;
  ++m->n;
}

static void matvec_set_run(matvec_set *m) {
  int64_t total = 0;
  for (int j = 0; j < m->n; ++j) total += m->rows[j];
  par_for(total, matvec_set_row, m);
}

/* h[r] = silu(gate[r]) * up[r], with gate rows 0..I-1 and up rows I..2I-1 of g */
static void swiglu_mid(const double *g, int inter, double *hmid) {
  for (int r = 0; r < inter; ++r) hmid[r] = g[r] * sigmoid(g[r]) * g[inter + r];
}

void oracle_swiglu_expert(const uint8_t *q13, const uint16_t *s13, const uint8_t *q2,
                          const uint16_t *s2, int hidden, int inter, const double *x, double *y) {
  double *g = (double *)malloc(sizeof(double) * 2 * inter);
  double *hmid = (double *)malloc(sizeof(double) * inter);
  matvec_set m = {0};
  matvec_set_add(&m, 0, q13, s13, NULL, 0.0, 2 * inter, hidden, x, g);
  matvec_set_run(&m);
  swiglu_mid(g, inter, hmid);
  matvec_set m2 = {0};
  matvec_set_add(&m2, 0, q2, s2, NULL, 0.0, hidden, inter, hmid, y);
  matvec_set_run(&m2);
  free(g);
  free(hmid);
}

typedef struct {
  const oracle_layer *L;
  const uint16_t *x;
  double *out;
  int32_t *idx;
  double *w, *gap;
  int e_lo, e_hi, with_shared; /* the experts whose terms are summed */
} moe_ctx;

static void moe_row(void *p, int64_t b) {
  moe_ctx *c = (moe_ctx *)p;
  const oracle_layer *L = c->L;
  const int E = L->n_experts, H = L->hidden, k = L->top_k, I = L->expert_i, Is = L->shared_i;
  double *xd = (double *)malloc(sizeof(double) * H);
  double *scr = (double *)malloc(sizeof(double) * 3 * E);
  int32_t idx[64];
  double w[64], gap;
  to_double(c->x + b * H, H, xd);
  route_row(L, xd, scr, scr + E, scr + 2 * E, idx, w, &gap);
  double *out = c->out + b * H;
  /* the k chosen experts and the shared expert (slot k), each
   * y = W2 (silu(W1 x) * (W3 x)): all gate/up rows in one set of products,
   * then all down rows in another */
  double *g = (double *)malloc(sizeof(double) * (2 * (size_t)I * k + 2 * (size_t)Is));
  double *hmid = (double *)malloc(sizeof(double) * ((size_t)I * k + Is));
  double *ys = (double *)malloc(sizeof(double) * (size_t)H * (k + 1));
  matvec_set m13 = {0}, m2 = {0};
  for (int j = 0; j <= k; ++j) {
    const int64_t e = j < k ? idx[j] : 0;
    const int inter = j < k ? I : Is;
    const size_t go = 2 * (size_t)I * j, ho = (size_t)I * j;
    if (j < k ? (e < c->e_lo || e >= c->e_hi) : !c->with_shared) continue; /* term not summed */
    /* scales (and affine offsets) per 128 (symmetric), 64 (affine) or 16
     * (NVFP4: one E4M3 byte each) elements; NVFP4 adds a global scale */
    const int fmt = L->format, aff = fmt == 1, nv = fmt == 2;
    const int gs = aff ? 64 : (nv ? 16 : 128), sb = nv ? 1 : 2; /* scale bytes */
    const char *s13b = (const char *)L->w13_s, *s2b = (const char *)L->w2_s;
    const uint8_t *q13 = j < k ? L->w13_q + e * (2 * I) * (H / 2) : L->sh13_q;
    const int64_t g13 = j < k ? e * (2 * I) * (H / gs) : 0;
    const char *s13 = (j < k ? s13b : (const char *)L->sh13_s) + sb * g13;
    if (nv) {
      /* NVFP4: the gate rows and the up rows have global scales of their own
       * (w13_g[e][0], w13_g[e][1]; sh13_g[0], sh13_g[1]) */
      const float *gl = j < k ? L->w13_g + 2 * e : L->sh13_g;
      matvec_set_add(&m13, fmt, q13, s13, NULL, (double)gl[0], inter, H, xd, g + go);
      matvec_set_add(&m13, fmt, q13 + (int64_t)inter * (H / 2), s13 + (int64_t)inter * (H / gs),
                     NULL, (double)gl[1], inter, H, xd, g + go + inter);
    } else {
      matvec_set_add(&m13, fmt, q13, s13,
                     aff ? (j < k ? L->w13_m + g13 : L->sh13_m) : NULL, 0.0, 2 * inter, H, xd,
                     g + go);
    }
    if (j < k) {
      const int64_t g2 = e * H * (I / gs);
      matvec_set_add(&m2, fmt, L->w2_q + e * H * (I / 2), s2b + sb * g2,
                     aff ? L->w2_m + g2 : NULL, nv ? (double)L->w2_g[e] : 0.0, H, inter,
                     hmid + ho, ys + (size_t)H * j);
    } else {
      matvec_set_add(&m2, fmt, L->sh2_q, L->sh2_s, aff ? L->sh2_m : NULL,
                     nv ? (double)L->sh2_g[0] : 0.0, H, inter, hmid + ho, ys + (size_t)H * j);
    }
  }
  matvec_set_run(&m13);
  for (int j = 0; j <= k; ++j)
    swiglu_mid(g + 2 * (size_t)I * j, j < k ? I : Is, hmid + (size_t)I * j);
  matvec_set_run(&m2);
  /* routing weight times the divisor of the stored up projections */
  const double div = L->expert_interm_div > 1.0 ? L->expert_interm_div : 1.0;
  for (int n = 0; n < H; ++n) out[n] = 0.0;
  for (int j = 0; j < k; ++j) {
    if (idx[j] < c->e_lo || idx[j] >= c->e_hi) continue;
    for (int n = 0; n < H; ++n) out[n] += (w[j] * div) * ys[(size_t)H * j + n];
  }
  if (c->with_shared)
    for (int n = 0; n < H; ++n) out[n] += ys[(size_t)H * k + n];
  free(g);
  free(hmid);
  free(ys);
  if (c->idx) memcpy(c->idx + b * k, idx, sizeof(int32_t) * k);
  if (c->w) memcpy(c->w + b * k, w, sizeof(double) * k);
  if (c->gap) c->gap[b] = gap;
  free(xd);
  free(scr);
}

static void moe_rows(const oracle_layer *L, const uint16_t *x, int B, double *out, int32_t *idx,
                     double *w, double *gap, int e_lo, int e_hi, int with_shared) {
  moe_ctx c = {L, x, out, idx, w, gap, e_lo, e_hi, with_shared};
  if (B >= g_threads) {
    par_for(B, moe_row, &c); /* one row per worker, its products in turn */
  } else {
    for (int b = 0; b < B; ++b) moe_row(&c, b); /* rows in turn, their products threaded */
  }
}

void oracle_moe_layer(const oracle_layer *L, const uint16_t *x, int B, double *out,
                      int32_t *idx, double *w, double *gap) {
  moe_rows(L, x, B, out, idx, w, gap, 0, L->n_experts, 1);
}

void oracle_moe_layer_partial(const oracle_layer *L, const uint16_t *x, int B, int e_lo, int e_hi,
                              int with_shared, double *out) {
  moe_rows(L, x, B, out, NULL, NULL, NULL, e_lo, e_hi, with_shared);
}

/* ------------------------------------------------------------ stack layer */
void oracle_rmsnorm_bf16(const float *h, int B, int H, double eps, uint16_t *x) {
  for (int b = 0; b < B; ++b) {
    const float *hb = h + (int64_t)b * H;
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += (double)hb[i] * (double)hb[i];
    double inv = 1.0 / sqrt(ss / H + eps);
    for (int i = 0; i < H; ++i) x[(int64_t)b * H + i] = oracle_double_to_bf16((double)hb[i] * inv);
  }
}

void oracle_stack_layer(const oracle_layer *L, float *h, int B, double eps, int32_t *idx,
                        double *w, double *gap) {
  const int H = L->hidden;
  uint16_t *x = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)B * H);
  double *out = (double *)malloc(sizeof(double) * (size_t)B * H);
  oracle_rmsnorm_bf16(h, B, H, eps, x);
  oracle_moe_layer(L, x, B, out, idx, w, gap);
  for (int64_t i = 0; i < (int64_t)B * H; ++i) {
    double o = oracle_bf16_to_double(oracle_double_to_bf16(out[i])); /* block output is bf16 */
    h[i] = round_to_float((double)h[i] + o);                         /* residual add in fp32 */
  }
  free(x);
  free(out);
}
