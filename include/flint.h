/*
 * flint.h: C ABI of the Flint int4 MoE block library for NVIDIA B200 (sm_100a).
 *
 * The block is the per-token mixture-of-experts layer of Flint, as described
 * on "How to Run Flint Locally", section "The architecture, from config.json"
 * (hidden 2,048; 256 routed experts of size 512 with 6 chosen per token by a
 * sigmoid router with normalized top-k; one shared expert of size 1,024 that
 * runs for every token) and on TandemLLM "21 Flint", section 21.1 "The model"
 * (experts routed by sigmoid score with a bias, SwiGLU experts).  The same
 * int4 GEMV serves the 150,144 x 2,048 output head ("How to Run Flint
 * Locally", section "One decode step in bytes": the head is read in full for
 * every token and was quantized to 4 bits).
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers to memory the caller owns; the
 *    library never allocates, frees or keeps them past the call.  Every
 *    pointer must be 16-byte aligned.  Layouts are dense, row-major.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t).
 *  - Packed int4 matrix [N, K]: q is N rows of K/2 bytes; byte j of a row
 *    holds element 2j in its low nibble and element 2j+1 in its high nibble,
 *    each a two's-complement code in [-8, 7].  s is [N, K/128] bf16: the scale
 *    of elements 128g .. 128g+127 of the row.  Weight = code * scale.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *    asynchronous; errors in arguments are reported before anything is
 *    launched, by the return code.  Device-side errors are recorded in the
 *    workspace's status word and read with flint_read_status.
 *  - Workspace: `ws` is caller-owned device scratch of at least
 *    flint_workspace_bytes(op, n) bytes.  Calls that share a workspace must
 *    be ordered on one stream.  The first use of a workspace must be preceded
 *    by flint_workspace_init (which zeroes its counters and status word).
 *  - Return value: FLINT_OK or a FLINT_E* code; never aborts the process.
 */
#ifndef FLINT_H
#define FLINT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLINT_API __attribute__((visibility("default")))
#else
#define FLINT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define FLINT_HIDDEN 2048
#define FLINT_EXPERTS 256
#define FLINT_TOPK 6
#define FLINT_EXPERT_I 512
#define FLINT_SHARED_I 1024
#define FLINT_GROUP 128
#define FLINT_MAX_DECODE_B 8
/* The decode calls on a layer in the group-64 affine or the NVFP4 format
 * take B <= 7: each of the 128 down-projection CTAs holds up to 6B experts'
 * rows with their scales (and offsets), and 48 of them do not fit its shared
 * memory.  (flint_moe_route takes B <= 8 in every format.) */
#define FLINT_MAX_DECODE_B_AFFINE 7
#define FLINT_MAX_PREFILL_T (1 << 20)
#define FLINT_MAX_STACK_LAYERS 256
#define FLINT_RMS_EPS 1e-6

enum {
  FLINT_OK = 0,
  FLINT_EINVAL = 1,   /* bad pointer, alignment, size or workspace */
  FLINT_ECUDA = 2,    /* a CUDA runtime call or launch failed */
  FLINT_ETIMEOUT = 3, /* a bounded device-side wait gave up (status word) */
  FLINT_EDEVICE = 4   /* a device-side check failed (status word) */
};
/* FLINT_EDEVICE comes from the bounds-checked build of this library
 * (libflint_debug.so, the same sources compiled with FLINT_DEBUG): its kernels
 * check every index they read back from device memory (slot words, expert
 * indices, sorted token rows, grouped-GEMM tile descriptors) before it
 * addresses memory, skip the access when a check fails and record
 * FLINT_EDEVICE in the call's status word (flint_read_status).  The release
 * build compiles the checks away.  Both export this same ABI. */

/* Workspace kinds for flint_workspace_bytes. */
enum { FLINT_OP_ROUTE = 0, FLINT_OP_DECODE = 1, FLINT_OP_PREFILL = 2, FLINT_OP_GEMV = 3 };

/*
 * One MoE layer's weights (all device pointers, read only).
 *  router_w  bf16 [256][2048]        z = router_w . x
 *  router_b  fp32 [256]              selection bias
 *  w13_q/s   packed [256][1024][2048]: per expert, rows 0..511 are the gate
 *            projection W1, rows 512..1023 the up projection W3
 *  w2_q/s    packed [256][2048][512]: per expert, the down projection W2
 *  sh13_q/s  packed [2048][2048]: shared expert, rows 0..1023 gate, 1024..2047 up
 *  sh2_q/s   packed [2048][1024]: shared expert down projection
 * Expert e's block starts at e * rows * row_bytes; the struct holds only base
 * pointers (and the up-projection divisor below).
 */
typedef struct {
  const uint16_t *router_w;
  const float *router_b;
  const uint8_t *w13_q;
  const uint16_t *w13_s;
  const uint8_t *w2_q;
  const uint16_t *w2_s;
  const uint8_t *sh13_q;
  const uint16_t *sh13_s;
  const uint8_t *sh2_q;
  const uint16_t *sh2_s;
  /* Routed experts' up projections stored divided by this power of two (the
   * packs' expert_interm_div of TandemLLM "21 Flint", section 21.2 "The
   * packs": the up projection / 128 keeps SwiGLU intermediates in fp16 range;
   * the engine multiplies the routing weights back).  0 or 1: not divided;
   * otherwise 2^n with 1 <= n <= 16.  The block computes the same function
   * either way: outputs equal those of the undivided weights. */
  int expert_interm_div;
  /* Weight format of the routed and shared experts (the router is bf16 in
   * both).  FLINT_FMT_SYM_INT4 (0): the layout above.  FLINT_FMT_AFFINE_INT4
   * (1): group-64 affine int4 ("How to Run Flint Locally", section "Every
   * build and its size": the MLX int4 build, and the Q4_1 GGUF's codes with
   * FP16 scales and offsets): the *_q arrays as above but each nibble an
   * unsigned code 0..15; the *_s arrays fp16 scales and the *_m arrays fp16
   * offsets, one per 64 elements along K: w13_s / w13_m [E][2I][H/64],
   * w2_s / w2_m [E][H][I/64], sh13_s / sh13_m [2Is][H/64], sh2_s / sh2_m
   * [H][Is/64]; weight = code * scale + offset.  The *_m pointers are read
   * only for format 1 (16-byte aligned there).
   * FLINT_FMT_NVFP4 (2): NVFP4 weight-only ("How to Run Flint Locally",
   * section "What vLLM changed": the NVFP4 checkpoint runs with BF16
   * activations): the *_q arrays FP4 E2M1 codes in the same nibble order
   * (the lower nibble is the even element); the *_s arrays FP8 E4M3 scales,
   * one byte per 16 elements along K (w13_s [E][2I][H/16], w2_s [E][H][I/16],
   * sh13_s [2Is][H/16], sh2_s [H][Is/16]); and fp32 global scales in the *_g
   * arrays: w13_g [E][2] (an expert's gate rows, then its up rows), w2_g [E],
   * sh13_g [2] (gate, up), sh2_g [1]; weight = e2m1(code) * e4m3(scale) *
   * global.  The *_g pointers are read only for format 2 (4-byte aligned
   * there).
   * Every call takes every format (formats 1 and 2 decode up to
   * FLINT_MAX_DECODE_B_AFFINE rows). */
  int format;
  const uint16_t *w13_m;
  const uint16_t *w2_m;
  const uint16_t *sh13_m;
  const uint16_t *sh2_m;
  const float *w13_g;
  const float *w2_g;
  const float *sh13_g;
  const float *sh2_g;
} flint_moe_layer;

#define FLINT_FMT_SYM_INT4 0
#define FLINT_FMT_AFFINE_INT4 1
#define FLINT_FMT_NVFP4 2

/* Library version (major*10000 + minor*100 + patch). */
FLINT_API int flint_version(void);

/* Name of the CUDA error behind the calling thread's last FLINT_ECUDA
 * ("none" if there was none); static string. */
FLINT_API const char *flint_last_cuda_error(void);

/* Human-readable name of a FLINT_* code (static string). */
FLINT_API const char *flint_strerror(int code);

/* Bytes of workspace `op` needs for n rows (B for decode and gemv, T for
 * route and prefill); for FLINT_OP_GEMV, n = B and the size also depends on
 * N via flint_gemv_workspace_bytes.  Returns 0 for an unsupported n. */
FLINT_API size_t flint_workspace_bytes(int op, int n);
FLINT_API size_t flint_gemv_workspace_bytes(int N, int B);

/* Zero a whole workspace (async on `stream`), counters and status word
 * included. */
FLINT_API int flint_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Copy the workspace's device status word to *status (synchronizes `stream`).
 * *status is FLINT_OK unless a device-side check or bounded wait failed. */
FLINT_API int flint_read_status(const void *ws, int *status, void *stream);

/* Test hook for the failure path: the poll bound of the decode kernels'
 * (flint_moe_route, flint_moe_decode, flint_moe_decode_residual) and the
 * int4 GEMV's (flint_int4_gemv and its allocation-free variant) first wait
 * on each shared-memory barrier.  The default is 1 << 26 polls (seconds); a
 * small value, 0 included, makes those waits give up at once, so the call
 * records FLINT_ETIMEOUT in the workspace status word and returns without a
 * result (the outputs are left as they were).  Every wait on that error path
 * keeps the default bound, so copies already in flight land before a CTA
 * exits.  polls = 0xFFFFFFFF restores the default.  Applies to the current
 * device; synchronous.  Not for production use: a lowered bound turns
 * ordinary latency into timeouts. */
FLINT_API int flint_debug_set_wait_polls(uint32_t polls);

/* Measurement hook: while enabled (enable != 0), flint_moe_prefill records a
 * CUDA event on its stream before and after each of its six stages (routing;
 * sort; operand scaling and token gather; grouped GEMM 1; grouped GEMM 2;
 * combine).  flint_debug_prefill_stage_ms waits for the last call's final
 * event and writes the six stage times in milliseconds to ms[0..5] (n >= 6).
 * The events belong to the device that was current at the first enable; one
 * call at a time; not for production use. */
FLINT_API int flint_debug_prefill_events(int enable);
FLINT_API int flint_debug_prefill_stage_ms(float *ms, int n);

/*
 * Router for B rows ("How to Run Flint Locally", section "The architecture,
 * from config.json": sigmoid router over 256 experts, top 6 kept, weights
 * normalized; TandemLLM "21 Flint" section 21.1: selection by sigmoid score
 * with a bias).
 *   z = router_w . x  (bf16 products, accumulated in fp64, rounded to fp32)
 *   s = sigmoid(z) (fp32);  b = s + router_b (fp32)
 *   idx[r][0..5] = the 6 largest b, largest first; equal b -> lower index
 *   w[r][j] = s[idx[r][j]] / sum_j s[idx[r][j]]   (fp32)
 *   x    bf16 [B][2048];  idx int32 [B][6];  w fp32 [B][6];  1 <= B <= 2^20
 *   ws   workspace of flint_workspace_bytes(FLINT_OP_ROUTE, B)
 * B <= 8 uses the decode router; larger B the prefill router (tensor-core
 * tiles over tokens); both sum bf16 products in fp32 per 128-wide k-group and
 * the groups in fp64, so they select the same experts up to near-ties.
 */
FLINT_API int flint_moe_route(const flint_moe_layer *layer, const uint16_t *x, int B, int32_t *idx,
                    float *w, void *ws, size_t ws_bytes, void *stream);

/*
 * Decode step of the MoE block for B in [1, 8] rows (B in [1, 7] for a layer in
 * the affine or NVFP4 format, FLINT_MAX_DECODE_B_AFFINE):
 *   out[r] = sum_j w[r][j] * W2_e (silu(W1_e x) * (W3_e x))  (j over the 6
 *            chosen experts e, in ascending expert order)
 *          + W2_sh (silu(W1_sh x) * (W3_sh x))               (shared expert)
 * with routing as in flint_moe_route.  fp32 accumulation throughout, fp32
 * SwiGLU intermediates (they can exceed the fp16 range: TandemLLM "21 Flint",
 * section 21.2 "The packs"), bf16 output.  Each output row is bit-identical
 * to running that row alone (batch invariance, as the Strix Halo engine
 * states in "Flint preview", section "What is in it").
 *   x   bf16 [B][2048];  out bf16 [B][2048] (may not alias x)
 *   ws  workspace of flint_workspace_bytes(FLINT_OP_DECODE, B)
 */
FLINT_API int flint_moe_decode(const flint_moe_layer *layer, const uint16_t *x, int B, uint16_t *out,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * One stacked decode layer on an fp32 residual stream h [B][2048], B in [1, 8]
 * (B in [1, 7] for the affine and NVFP4 formats):
 *   x = bf16(h / sqrt(mean(h^2) + 1e-6))   (RMSNorm, unit weight, fp64 inside)
 *   h = h + bf16(moe(x))                   (residual add in fp32, in place)
 * Optional outputs (NULL to skip): idx int32 [B][6], w fp32 [B][6] in
 * selection order, as flint_moe_route returns them.
 */
FLINT_API int flint_moe_decode_residual(const flint_moe_layer *layer, float *h, int B, int32_t *idx,
                              float *w, void *ws, size_t ws_bytes, void *stream);

/*
 * One rank's share of the decode block under expert parallelism (experts
 * sharded by index across ranks, routing replicated; the split is the next
 * step the workload's scope names for this path):
 *   partial[r] = sum over row r's chosen experts e with expert_lo <= e <
 *                expert_hi of w[r][j] * W2_e (silu(W1_e x) * (W3_e x)), in the
 *                row's ascending expert order
 *              + (with_shared != 0) W2_sh (silu(W1_sh x) * (W3_sh x))
 * in fp32, before any rounding.  Routing is computed over all 256 experts (as
 * flint_moe_route), so every rank agrees on it.  The block output is the sum
 * of the ranks' partials (an all-reduce), finished by
 * flint_moe_combine_partials.  Exactly one of the inputs is given: x bf16
 * [B][2048] (the block input, as flint_moe_decode) or h fp32 [B][2048] (the
 * residual stream, read only: x = its RMSNorm, as flint_moe_decode_residual).
 * Only the shard's experts' weights are read, so a rank may hold only those:
 * the layer's routed base pointers may be offset so that expert expert_lo's
 * block sits at the rank's first shard byte (they must stay 16-byte aligned).
 *   partial fp32 [B][2048];  0 <= expert_lo < expert_hi <= 256;  B in [1, 8]
 *   ws  workspace of flint_workspace_bytes(FLINT_OP_DECODE, B)
 */
FLINT_API int flint_moe_decode_partial(const flint_moe_layer *layer, const uint16_t *x,
                                       const float *h, int B, int expert_lo, int expert_hi,
                                       int with_shared, float *partial, void *ws,
                                       size_t ws_bytes, void *stream);

/*
 * The last step of a block whose output was summed from partials:
 *   out[i] = bf16(sum[i])            (if out != NULL)
 *   h[i]   = h[i] + bf16(sum[i])     (if h != NULL; the residual add in fp32)
 * sum fp32 [B][2048]; out bf16 [B][2048]; h fp32 [B][2048]; at least one of
 * out and h.
 */
FLINT_API int flint_moe_combine_partials(const float *sum, int B, uint16_t *out, float *h,
                                         void *stream);

/*
 * L stacked decode layers on an fp32 residual stream h [B][2048], B in
 * [1, 8], 1 <= L <= FLINT_MAX_STACK_LAYERS: flint_moe_decode_residual applied
 * with layers[0], then layers[1], ..., in one call (three programmatic-
 * dependent kernels per layer on `stream`: each layer's router and shared
 * expert weights are fetched while the previous kernel runs).  Bitwise equal
 * to L calls of flint_moe_decode_residual.
 *   layers   HOST array of L layer structs (read during the call only)
 *   h        fp32 [B][2048], updated in place
 *   idx, w   optional outputs (NULL to skip): int32 / fp32 [L][B][6], each
 *            layer's selection as flint_moe_route returns it
 *   h_trace  optional output (NULL to skip): fp32 [L][B][2048], the residual
 *            h entering each layer (for layer-by-layer checks; one
 *            device-to-device copy per layer)
 *   ws       workspace of flint_workspace_bytes(FLINT_OP_DECODE, B)
 */
FLINT_API int flint_moe_decode_stack(const flint_moe_layer *layers, int L, float *h, int B,
                                     int32_t *idx, float *w, float *h_trace, void *ws,
                                     size_t ws_bytes, void *stream);

/*
 * Prefill of the MoE block for T >= 1 tokens: the same function as
 * flint_moe_decode row by row, computed as routing for T tokens, a stable
 * token-by-expert sort, grouped GEMMs on the tensor cores and a fixed-order
 * combine.  The GEMMs multiply exact fp16 operands (code x scale with a
 * power-of-two shift per weight matrix; token rows with one per token) in one
 * fp32 accumulation per output; the SwiGLU intermediate is rounded once, to
 * fp16 after a per-token power-of-two shift from a bound it cannot exceed.
 * Group-64 affine experts (format 1): each weight code x scale + offset
 * (times the matrix's power of two) is rounded once to fp16, a relative
 * error of at most 2^-11 per weight; the rest is as above.  NVFP4 experts
 * (format 2): each E2M1 value times its E4M3 block scale is an exact fp16
 * weight (no shift); the global scales multiply the GEMMs' read-out.
 *   x bf16 [T][2048];  out bf16 [T][2048] (may not alias x);  1 <= T <= 2^20
 *   ws workspace of flint_workspace_bytes(FLINT_OP_PREFILL, T) (about 67 KB
 *      per token, 70 KB up to T = 4,608 where the router keeps two fp64
 *      partial logits per token and expert: routing tables, the fp16 token
 *      rows, the SwiGLU and expert outputs)
 */
FLINT_API int flint_moe_prefill(const flint_moe_layer *layer, const uint16_t *x, int T, uint16_t *out,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * Int4 GEMV for B in [1, 8] rows (the output head: N = 150,144, K = 2,048):
 *   y[r][n] = sum_k W[n][k] x[r][k]  (fp32 accumulation)
 *   argmax[r] = the lowest n with the largest y[r][n]   (argmax may be NULL)
 *   q, s  packed int4 [N][K], K a multiple of 128 and at most 8192
 *   x bf16 [B][K];  y fp32 [B][N]
 *   ws workspace of flint_gemv_workspace_bytes(N, B)
 * Rows are batch-invariant like flint_moe_decode.
 */
FLINT_API int flint_int4_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x, int B,
                    float *y, int32_t *argmax, void *ws, size_t ws_bytes, void *stream);

/*
 * Int4 GEMV on group-64 affine weights, the format of the MLX int4 build and
 * of the Q4_1 GGUF ("How to Run Flint Locally", section "Every build and its
 * size": group-64 affine int4; the same int4 codes with FP16 scales and
 * offsets), for B in [1, 8] rows:
 *   W[n][k] = code(n, k) * s[n][k/64] + m[n][k/64]   (code unsigned, 0..15)
 *   y[r][n] = sum_k W[n][k] x[r][k]  (fp32 accumulation: per 64-group
 *             scale * (codes . x) + offset * sum(x over the group))
 *   argmax[r] = the lowest n with the largest y[r][n]   (argmax may be NULL)
 *   q packed [N][K/2] (byte j: element 2j low nibble, 2j+1 high nibble, each
 *     an unsigned code); s, m fp16 bits [N][K/64]; K a multiple of 128, at
 *     most 8192
 *   x bf16 [B][K];  y fp32 [B][N];  ws as for flint_int4_gemv
 * Rows are batch-invariant; errors as flint_int4_gemv.
 */
FLINT_API int flint_int4_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int N,
                                     int K, const uint16_t *x, int B, float *y, int32_t *argmax,
                                     void *ws, size_t ws_bytes, void *stream);

/*
 * GEMV on NVFP4 weights run weight-only with bf16 activations (the checkpoint
 * the vLLM path of "How to Run Flint Locally", section "What vLLM changed",
 * benchmarks: NVIDIA's NVFP4 format, repacked losslessly and run W4A16), for B
 * in [1, 8] rows:
 *   W[n][k] = e2m1(code(n, k)) * e4m3(s[n][k/16]) * global_scale
 *   y[r][n] = sum_k W[n][k] x[r][k]  (fp32 accumulation)
 *   argmax[r] = the lowest n with the largest y[r][n]   (argmax may be NULL)
 *   q packed [N][K/2] (byte j: element 2j in the low nibble, 2j+1 in the high
 *     nibble, each an FP4 E2M1 code: sign bit 3, exponent bits 2-1, mantissa
 *     bit 0); s [N][K/16] FP8 E4M3 block scales (one byte each); K a multiple
 *     of 128, at most 8192; global_scale a finite fp32
 *   x bf16 [B][K];  y fp32 [B][N];  ws as for flint_int4_gemv
 * Every code times its block scale is exact in fp16 and is multiplied on the
 * tensor cores with x as fp16 scaled by a power of two per row (exact for
 * elements down to 2^-24 of the row's largest); errors as flint_int4_gemv.
 */
FLINT_API int flint_int4_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float global_scale, int N,
                                    int K, const uint16_t *x, int B, float *y, int32_t *argmax,
                                    void *ws, size_t ws_bytes, void *stream);

/*
 * flint_int4_gemv without a workspace, for callers that cannot allocate
 * device memory themselves: code embedded in a host program that owns every
 * device allocation (and forbids cudaMalloc from libraries), or a hot path
 * whose memory budget is fixed up front and that must not fail or stall on an
 * allocation.  The pages have no counterpart: this entry point is an
 * integration convenience, not part of the method.
 *
 * Same arguments and results as flint_int4_gemv, minus `ws`; argument errors
 * are returned the same way, and a device-side timeout is recorded in the
 * array's status word, read with flint_int4_gemv_noalloc_status.  The scratch
 * (a counter, a status word and per-CTA argmax partials) is a 65,792-byte
 * array inside the library, one per GPU that loads it, kept until the process
 * exits; calls whose scratch would not fit are rejected with FLINT_EINVAL
 * (none with B <= 8 do; B = 8 fills it).  Nothing is allocated: the call
 * clears the counter and status word with an asynchronous memset on
 * `stream`, then launches.  Outside a stream capture every call looks the
 * array's device address up (cudaGetSymbolAddress, with the device current)
 * and keeps it per device; inside a capture the kept address is used, so the
 * first call on a device must be made before any capture (a capture without
 * it returns FLINT_ECUDA).  All calls on a device share the one array and it
 * keeps the last call's contents, so calls that may overlap on the GPU
 * (different streams without ordering between them) race and must not be
 * issued; order them on one stream.
 */
FLINT_API int flint_int4_gemv_noalloc(const uint8_t *q, const uint16_t *s, int N, int K,
                                      const uint16_t *x, int B, float *y, int32_t *argmax,
                                      void *stream);

/*
 * Status word of the allocation-free GEMV's array on the current device:
 * FLINT_OK, or FLINT_ETIMEOUT if a bounded wait of the last
 * flint_int4_gemv_noalloc call on this device gave up (its y and argmax are
 * then incomplete).  Copies the word to *status and synchronizes `stream`
 * (use the stream of that call, outside any stream capture).  The next
 * flint_int4_gemv_noalloc call clears the word.  Allocates nothing.
 */
FLINT_API int flint_int4_gemv_noalloc_status(int *status, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* FLINT_H */
