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
  size_t ctrl, zpart, sel_idx, sel_w, asc_slot, asc_w, slot_word, hfr, hfs, xfrag, total;
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
  L.xfrag = take((size_t)16 * 4 * B * 64);             // block input as a compact fragment image
  L.total = o;
  return L;
}

// Prefill workspace for T tokens.  The 6T routed rows are sorted by expert
// with no padding; the token tiles of GEMM 1 (kPfN1 tokens) and GEMM 2
// (kPfN2) read past a group's end into the next group or, at the end, the
// zero fill of the TMA box, and those columns are never stored.
// ctrl words: [1] status, [3] GEMM1 tile count, [4] GEMM2 tile count,
// [5] routed rows.
constexpr int kPfN1 = 256;
constexpr int kPfN2 = 256;
constexpr int kPfChunk = 256;
struct PrefillLayout {
  size_t ctrl, z, sel_idx, sel_w, asc_e, asc_w, route_total;
  size_t pos, chunk_cnt, chunk_off, ebase, ecount, tiles1, tiles2, wst, wsg, wbound,
      rsc, rm3, xp, hr, hs, yw, ys, total;
  int mr, max_tiles1, max_tiles2, nchunks;
};

// Up to this many tokens the prefill router splits every tile's K between two
// CTAs (the tiles alone would leave most SMs idle) and publishes the two
// k-half partial logits in fp64; above it, one CTA per tile publishes fp32.
constexpr int kRouteSplitMaxT = 4608;
inline int route_split(int T) { return T <= kRouteSplitMaxT ? 2 : 1; }

inline PrefillLayout prefill_layout(int T) {
  PrefillLayout L{};
  L.nchunks = (T + kPfChunk - 1) / kPfChunk;
  // at most min(256, 6T) experts hold tokens; each adds at most one partial tile
  const int busy = 6 * T < 256 ? 6 * T : 256;
  L.mr = 6 * T;
  // tiles of 256 weight rows (a CTA pair) by one token tile
  L.max_tiles1 = 4 * ((6 * T) / kPfN1 + busy) + 8 * ((T + kPfN1 - 1) / kPfN1);
  L.max_tiles2 = 8 * ((6 * T) / kPfN2 + busy) + 8 * ((T + kPfN2 - 1) / kPfN2);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.ctrl = take(256);
  L.z = take((route_split(T) == 2 ? 2 * sizeof(double) : sizeof(float)) * (size_t)T * 256);
  L.sel_idx = take(sizeof(int32_t) * (size_t)T * 6);
  L.sel_w = take(sizeof(float) * (size_t)T * 6);
  L.asc_e = take(sizeof(int32_t) * (size_t)T * 6);
  L.asc_w = take(sizeof(float) * (size_t)T * 6);
  L.route_total = o;
  L.pos = take(sizeof(int32_t) * (size_t)T * 6);
  L.chunk_cnt = take(sizeof(int32_t) * (size_t)L.nchunks * 256);
  L.chunk_off = take(sizeof(int32_t) * (size_t)L.nchunks * 256);
  L.ebase = take(sizeof(int32_t) * 257);
  L.ecount = take(sizeof(int32_t) * 256);
  L.tiles1 = take(sizeof(uint32_t) * 2 * (size_t)L.max_tiles1);  // tile descriptors (2 words)
  L.tiles2 = take(sizeof(uint32_t) * 2 * (size_t)L.max_tiles2);
  L.wst = take(sizeof(float) * 4 * 257);   // per expert matrix pair: power-of-two shifts
  L.wsg = take(sizeof(float) * 4 * 257);   // per expert: NVFP4 global scales gate, up, down
  L.wbound = take(sizeof(float) * 257);    // per expert: bound factor of the SwiGLU output
  L.rsc = take(sizeof(uint32_t) * (size_t)7 * T);    // per row: F | E << 16
  L.rm3 = take(sizeof(float) * (size_t)7 * T);       // per row: 2^E x routing weight
  L.xp = take(sizeof(uint16_t) * (size_t)7 * T * 2048);  // fp16 token rows: routed, then all T
  L.hr = take(sizeof(uint16_t) * (size_t)L.mr * 512);    // fp16 SwiGLU intermediate, routed
  L.hs = take(sizeof(uint16_t) * (size_t)T * 1024);      // fp16 SwiGLU intermediate, shared
  L.yw = take(sizeof(uint16_t) * (size_t)L.mr * 2048);
  L.ys = take(sizeof(uint16_t) * (size_t)T * 2048);
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
  float interm_div;  // routed up projections stored divided by this (a power of two, >= 1)
  int fmt;           // FLINT_FMT_SYM_INT4, _AFFINE_INT4 or _NVFP4 (experts)
  const uint16_t *w13_m;  // affine offsets (fmt 1)
  const uint16_t *w2_m;
  const uint16_t *sh13_m;
  const uint16_t *sh2_m;
  const float *w13_g;  // NVFP4 global scales (fmt 2): [E][2], [E], [2], [1]
  const float *w2_g;
  const float *sh13_g;
  const float *sh2_g;
};

inline LayerArgs layer_args(const flint_moe_layer *l) {
  const int d = l->expert_interm_div > 1 ? l->expert_interm_div : 1;
  const bool aff = l->format == FLINT_FMT_AFFINE_INT4, nv = l->format == FLINT_FMT_NVFP4;
  return LayerArgs{l->router_w, l->router_b, l->w13_q,  l->w13_s, l->w2_q,
                   l->w2_s,     l->sh13_q,   l->sh13_s, l->sh2_q, l->sh2_s, (float)d,
                   l->format,
                   aff ? l->w13_m : nullptr, aff ? l->w2_m : nullptr,
                   aff ? l->sh13_m : nullptr, aff ? l->sh2_m : nullptr,
                   nv ? l->w13_g : nullptr, nv ? l->w2_g : nullptr,
                   nv ? l->sh13_g : nullptr, nv ? l->sh2_g : nullptr};
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
// The experts a decode call computes: [e_lo, e_hi) of the routed ones and,
// with with_shared, the shared expert; with `partial` set, K3 writes that
// share of the block output in fp32 instead of the bf16 output or residual.
struct DecodeShard {
  int e_lo = 0, e_hi = 256;
  bool with_shared = true;
  float *partial = nullptr;
};
cudaError_t launch_decode(const LayerArgs &L, const uint16_t *x, const float *h_in, float *h_out,
                          int B, uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                          cudaStream_t st, bool route_only, const DecodeShard &sh = DecodeShard());
cudaError_t launch_combine_partials(const float *sum, int B, uint16_t *out, float *h,
                                    cudaStream_t st);
cudaError_t launch_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x,
                        int B, float *y, int32_t *argmax, char *ws, cudaStream_t st);
cudaError_t launch_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int N,
                               int K, const uint16_t *x, int B, float *y, int32_t *argmax,
                               char *ws, cudaStream_t st);
cudaError_t launch_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float gsc, int N, int K,
                              const uint16_t *x, int B, float *y, int32_t *argmax, char *ws,
                              cudaStream_t st);
size_t gemv_ws_bytes(int N, int B);
cudaError_t decode_set_wait_polls(uint32_t polls);
cudaError_t gemv_set_wait_polls(uint32_t polls);
cudaError_t prefill_set_stage_events(int enable);
cudaError_t prefill_stage_times(float *ms, int n);
cudaError_t launch_prefill(const LayerArgs &L, const uint16_t *x, int T, uint16_t *out, char *ws,
                           cudaStream_t st);
cudaError_t launch_route_many(const LayerArgs &L, const uint16_t *x, int T, int32_t *idx, float *w,
                              char *ws, cudaStream_t st);

}  // namespace flint
