// C ABI entry points: argument checks (before anything is launched), workspace
// sizing, status read-back.  All compute is in the kernels of decode.cu,
// gemv.cu and prefill.cu.
#include <cuda_runtime.h>
#include <stdio.h>

#include "../../include/flint.h"
#include "internal.h"

using namespace flint;

namespace {

bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// the NVFP4 global-scale arrays are read one float at a time (and an expert
// shard may offset them by its first expert)
bool aligned4(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// 0 or 1 (not divided), or a power of two from 2 to 2^16
bool div_ok(int d) { return d == 0 || (d > 0 && d <= 65536 && (d & (d - 1)) == 0); }

bool layer_ok(const flint_moe_layer *l) {
  if (!l || (l->format != FLINT_FMT_SYM_INT4 && l->format != FLINT_FMT_AFFINE_INT4 &&
             l->format != FLINT_FMT_NVFP4))
    return false;
  if (l->format == FLINT_FMT_AFFINE_INT4 &&
      !(aligned16(l->w13_m) && aligned16(l->w2_m) && aligned16(l->sh13_m) && aligned16(l->sh2_m)))
    return false;
  if (l->format == FLINT_FMT_NVFP4 &&
      !(aligned4(l->w13_g) && aligned4(l->w2_g) && aligned4(l->sh13_g) && aligned4(l->sh2_g)))
    return false;
  return div_ok(l->expert_interm_div) && aligned16(l->router_w) && aligned16(l->router_b) &&
         aligned16(l->w13_q) &&
         aligned16(l->w13_s) && aligned16(l->w2_q) && aligned16(l->w2_s) && aligned16(l->sh13_q) &&
         aligned16(l->sh13_s) && aligned16(l->sh2_q) && aligned16(l->sh2_s);
}

// the decode calls' batch limit for a layer: K3 stages up to 6B experts'
// down rows of its 16 output rows; the affine format's fp16 scales and
// offsets, and the NVFP4 format's E4M3 scales per 16 (4.5 KB a slot instead
// of 4.1 KB), fit 42 slots, not 48
bool decode_batch_ok(const flint_moe_layer *l, int B) {
  return B >= 1 && B <= (l->format != FLINT_FMT_SYM_INT4 ? FLINT_MAX_DECODE_B_AFFINE
                                                         : FLINT_MAX_DECODE_B);
}

thread_local cudaError_t g_last_cuda = cudaSuccess;
thread_local const char *g_last_where = "";
thread_local const char *g_step = "";
thread_local char g_msg[160];

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FLINT_OK;
  g_last_cuda = e;
  g_last_where = g_step;
  return FLINT_ECUDA;
}

}  // namespace

int flint_from_cuda(cudaError_t e) { return from_cuda(e); }

namespace flint {
void note_step(const char *where) { g_step = where; }
cudaError_t noted(cudaError_t e, const char *where) {
  g_step = where;
  return e;
}
}  // namespace flint

extern "C" {

int flint_version(void) { return 100; }

const char *flint_last_cuda_error(void) {
  if (g_last_cuda == cudaSuccess) return "none";
  snprintf(g_msg, sizeof(g_msg), "%s at %s", cudaGetErrorName(g_last_cuda), g_last_where);
  return g_msg;
}

const char *flint_strerror(int code) {
  switch (code) {
    case FLINT_OK: return "ok";
    case FLINT_EINVAL: return "invalid argument (pointer, alignment, size or workspace)";
    case FLINT_ECUDA: return "CUDA runtime or launch error";
    case FLINT_ETIMEOUT: return "a bounded device-side wait gave up";
    case FLINT_EDEVICE: return "a device-side check failed";
    default: return "unknown flint status";
  }
}

size_t flint_workspace_bytes(int op, int n) {
  if (n < 1) return 0;
  switch (op) {
    case FLINT_OP_ROUTE:
      return n <= FLINT_MAX_DECODE_B ? decode_layout(n).total : prefill_layout(n).route_total;
    case FLINT_OP_DECODE:
      return n <= FLINT_MAX_DECODE_B ? decode_layout(n).total : 0;
    case FLINT_OP_PREFILL:
      return n <= FLINT_MAX_PREFILL_T ? prefill_layout(n).total : 0;
    case FLINT_OP_GEMV:
      return 0;  // depends on N: flint_gemv_workspace_bytes
    default:
      return 0;
  }
}

size_t flint_gemv_workspace_bytes(int N, int B) {
  if (N < 1 || B < 1 || B > FLINT_MAX_DECODE_B) return 0;
  return gemv_ws_bytes(N, B);
}

int flint_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!aligned16(ws) || ws_bytes < 256) return FLINT_EINVAL;
  return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int flint_read_status(const void *ws, int *status, void *stream) {
  if (!aligned16(ws) || !status) return FLINT_EINVAL;
  uint32_t ctrl[2] = {0, 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ctrl, ws, sizeof(ctrl), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return from_cuda(e);
  *status = static_cast<int>(ctrl[1]);
  return FLINT_OK;
}

int flint_debug_prefill_events(int enable) {
  return from_cuda(noted(prefill_set_stage_events(enable), "prefill stage events"));
}

int flint_debug_prefill_stage_ms(float *ms, int n) {
  if (!ms) return FLINT_EINVAL;
  return from_cuda(noted(prefill_stage_times(ms, n), "prefill stage times"));
}

int flint_debug_set_wait_polls(uint32_t polls) {
  cudaError_t e = noted(decode_set_wait_polls(polls), "debug wait bound (decode)");
  if (e == cudaSuccess) e = noted(gemv_set_wait_polls(polls), "debug wait bound (gemv)");
  return from_cuda(e);
}

int flint_moe_route(const flint_moe_layer *layer, const uint16_t *x, int B, int32_t *idx,
                    float *w, void *ws, size_t ws_bytes, void *stream) {
  if (!layer_ok(layer) || !aligned16(x) || !idx || !w || B < 1 || B > FLINT_MAX_PREFILL_T ||
      !aligned16(ws) || ws_bytes < flint_workspace_bytes(FLINT_OP_ROUTE, B))
    return FLINT_EINVAL;
  if (B > FLINT_MAX_DECODE_B)
    return from_cuda(launch_route_many(layer_args(layer), x, B, idx, w, static_cast<char *>(ws),
                                       static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_decode(layer_args(layer), x, nullptr, nullptr, B, nullptr, idx, w,
                                 static_cast<char *>(ws), static_cast<cudaStream_t>(stream),
                                 true));
}

int flint_moe_decode(const flint_moe_layer *layer, const uint16_t *x, int B, uint16_t *out,
                     void *ws, size_t ws_bytes, void *stream) {
  if (!layer_ok(layer) || !aligned16(x) || !aligned16(out) || !decode_batch_ok(layer, B) ||
      !aligned16(ws) || ws_bytes < flint_workspace_bytes(FLINT_OP_DECODE, B) ||
      static_cast<const void *>(x) == static_cast<const void *>(out))
    return FLINT_EINVAL;
  return from_cuda(launch_decode(layer_args(layer), x, nullptr, nullptr, B, out, nullptr, nullptr,
                                 static_cast<char *>(ws), static_cast<cudaStream_t>(stream),
                                 false));
}

int flint_moe_decode_residual(const flint_moe_layer *layer, float *h, int B, int32_t *idx,
                              float *w, void *ws, size_t ws_bytes, void *stream) {
  if (!layer_ok(layer) || !aligned16(h) || !decode_batch_ok(layer, B) || !aligned16(ws) ||
      ws_bytes < flint_workspace_bytes(FLINT_OP_DECODE, B))
    return FLINT_EINVAL;
  return from_cuda(launch_decode(layer_args(layer), nullptr, h, h, B, nullptr, idx, w,
                                 static_cast<char *>(ws), static_cast<cudaStream_t>(stream),
                                 false));
}

int flint_moe_decode_partial(const flint_moe_layer *layer, const uint16_t *x, const float *h, int B,
                             int expert_lo, int expert_hi, int with_shared, float *partial, void *ws,
                             size_t ws_bytes, void *stream) {
  if (!layer_ok(layer) || (x == nullptr) == (h == nullptr) || (x && !aligned16(x)) ||
      (h && !aligned16(h)) || !aligned16(partial) || !decode_batch_ok(layer, B) ||
      expert_lo < 0 || expert_hi > FLINT_EXPERTS || expert_lo >= expert_hi || !aligned16(ws) ||
      ws_bytes < flint_workspace_bytes(FLINT_OP_DECODE, B))
    return FLINT_EINVAL;
  DecodeShard sh;
  sh.e_lo = expert_lo, sh.e_hi = expert_hi, sh.with_shared = with_shared != 0, sh.partial = partial;
  return from_cuda(launch_decode(layer_args(layer), x, h, nullptr, B, nullptr, nullptr, nullptr,
                                 static_cast<char *>(ws), static_cast<cudaStream_t>(stream), false,
                                 sh));
}

int flint_moe_combine_partials(const float *sum, int B, uint16_t *out, float *h, void *stream) {
  if (!aligned16(sum) || B < 1 || B > FLINT_MAX_DECODE_B || (!out && !h) ||
      (out && !aligned16(out)) || (h && !aligned16(h)))
    return FLINT_EINVAL;
  return from_cuda(launch_combine_partials(sum, B, out, h, static_cast<cudaStream_t>(stream)));
}

int flint_moe_decode_stack(const flint_moe_layer *layers, int L, float *h, int B, int32_t *idx,
                           float *w, float *h_trace, void *ws, size_t ws_bytes, void *stream) {
  if (!layers || L < 1 || L > FLINT_MAX_STACK_LAYERS || !aligned16(h) || B < 1 ||
      B > FLINT_MAX_DECODE_B || !aligned16(ws) ||
      ws_bytes < flint_workspace_bytes(FLINT_OP_DECODE, B) ||
      (h_trace && !aligned16(h_trace)))
    return FLINT_EINVAL;
  for (int l = 0; l < L; ++l)
    if (!layer_ok(&layers[l]) || !decode_batch_ok(&layers[l], B)) return FLINT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int l = 0; l < L; ++l) {
    cudaError_t e = cudaSuccess;
    if (h_trace)
      e = noted(cudaMemcpyAsync(h_trace + (size_t)l * B * FLINT_HIDDEN, h,
                                sizeof(float) * (size_t)B * FLINT_HIDDEN, cudaMemcpyDeviceToDevice,
                                st),
                "stack trace copy");
    if (e == cudaSuccess)
      e = launch_decode(layer_args(&layers[l]), nullptr, h, h, B, nullptr,
                        idx ? idx + (size_t)l * B * FLINT_TOPK : nullptr,
                        w ? w + (size_t)l * B * FLINT_TOPK : nullptr, static_cast<char *>(ws), st,
                        false);
    if (e != cudaSuccess) return from_cuda(e);
  }
  return FLINT_OK;
}

int flint_int4_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x, int B,
                    float *y, int32_t *argmax, void *ws, size_t ws_bytes, void *stream) {
  if (!aligned16(q) || !aligned16(s) || !aligned16(x) || !aligned16(y) || N < 1 || K < 128 ||
      K % 128 || K > 8192 || B < 1 || B > FLINT_MAX_DECODE_B || !aligned16(ws) ||
      ws_bytes < flint_gemv_workspace_bytes(N, B))
    return FLINT_EINVAL;
  // rows of scales are K/128 bf16 = K/64 bytes; 16-byte alignment of each
  // row's start is not needed (scales are read one at a time)
  return from_cuda(launch_gemv(q, s, N, K, x, B, y, argmax, static_cast<char *>(ws),
                               static_cast<cudaStream_t>(stream)));
}

int flint_int4_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int N, int K,
                           const uint16_t *x, int B, float *y, int32_t *argmax, void *ws,
                           size_t ws_bytes, void *stream) {
  if (!aligned16(q) || !aligned16(s) || !aligned16(m) || !aligned16(x) || !aligned16(y) ||
      N < 1 || K < 128 || K % 128 || K > 8192 || B < 1 || B > FLINT_MAX_DECODE_B ||
      !aligned16(ws) || ws_bytes < flint_gemv_workspace_bytes(N, B))
    return FLINT_EINVAL;
  return from_cuda(launch_gemv_affine(q, s, m, N, K, x, B, y, argmax, static_cast<char *>(ws),
                                      static_cast<cudaStream_t>(stream)));
}

int flint_int4_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float global_scale, int N, int K,
                          const uint16_t *x, int B, float *y, int32_t *argmax, void *ws,
                          size_t ws_bytes, void *stream) {
  if (!aligned16(q) || !aligned16(s) || !aligned16(x) || !aligned16(y) || N < 1 || K < 128 ||
      K % 128 || K > 8192 || B < 1 || B > FLINT_MAX_DECODE_B || !aligned16(ws) ||
      ws_bytes < flint_gemv_workspace_bytes(N, B) || !(global_scale == global_scale))
    return FLINT_EINVAL;
  return from_cuda(launch_gemv_nvfp4(q, s, global_scale, N, K, x, B, y, argmax,
                                     static_cast<char *>(ws), static_cast<cudaStream_t>(stream)));
}

int flint_moe_prefill(const flint_moe_layer *layer, const uint16_t *x, int T, uint16_t *out,
                      void *ws, size_t ws_bytes, void *stream) {
  if (!layer_ok(layer) || !aligned16(x) ||
      !aligned16(out) || T < 1 || T > FLINT_MAX_PREFILL_T || !aligned16(ws) ||
      ws_bytes < flint_workspace_bytes(FLINT_OP_PREFILL, T) ||
      static_cast<const void *>(x) == static_cast<const void *>(out))
    return FLINT_EINVAL;
  return from_cuda(launch_prefill(layer_args(layer), x, T, out, static_cast<char *>(ws),
                                  static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
