// Host-side internals shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/flint.h"

namespace flint {

// Offsets (bytes) of one decode workspace for B rows; every region 256-aligned.
// ctrl words: [0] route completion counter, [1] status, [2] number of slots.
// Slot word u: expert (bits 0-7) | row mask (bits 8-15) | number of slots
// (bits 16-24) for u < number of slots, else all ones.
struct DecodeLayout {
  size_t ctrl, zpart, sel_idx, sel_w, asc_slot, asc_w, slot_word, hfr, hfs, total;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline DecodeLayout decode_layout(int B) {
  DecodeLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.ctrl = take(256);
  L.zpart = take(sizeof(double) * 2 * B * 256);        // router partial sums, two k-halves
  L.sel_idx = take(sizeof(int32_t) * B * 6);
  L.sel_w = take(sizeof(float) * B * 6);
  L.asc_slot = take(sizeof(int32_t) * B * 6);
  L.asc_w = take(sizeof(float) * B * 6);
  L.slot_word = take(sizeof(uint32_t) * 256);          // slot table, see kSlotInvalid
  L.hfr = take(sizeof(uint16_t) * B * 6 * 2 * 512);    // routed SwiGLU hi/lo images
  L.hfs = take(sizeof(uint16_t) * B * 2 * 1024);       // shared SwiGLU hi/lo images
  L.total = o;
  return L;
}

struct LayerArgs {
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
};

inline LayerArgs layer_args(const flint_moe_layer *l) {
  return LayerArgs{l->router_w, l->router_b, l->w13_q, l->w13_s, l->w2_q,
                   l->w2_s,     l->sh13_q,   l->sh13_s, l->sh2_q, l->sh2_s};
}

// Where the calling thread's last failing CUDA call was made (for
// flint_last_cuda_error); launchers note each step before making it.
void note_step(const char *where);
cudaError_t noted(cudaError_t e, const char *where);

}  // namespace flint

// FLINT_OK, or FLINT_ECUDA after recording e for flint_last_cuda_error.
int flint_from_cuda(cudaError_t e);

namespace flint {

// Launchers (return a cudaError_t from the launches).
cudaError_t launch_decode(const LayerArgs &L, const uint16_t *x, const float *h_in, float *h_out,
                          int B, uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                          cudaStream_t st, bool route_only);
cudaError_t launch_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x,
                        int B, float *y, int32_t *argmax, char *ws, cudaStream_t st);
size_t gemv_ws_bytes(int N, int B);

}  // namespace flint
