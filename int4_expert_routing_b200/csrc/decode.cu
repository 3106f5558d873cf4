// Decode step of the Flint MoE block: three kernels chained with programmatic
// dependent launch (PDL), each loading the weights it can before waiting on
// its predecessor.
//
//   K1  router (bf16 W_r, fp64 sum of fp32 group partials, fp32 sigmoid,
//       + bias, top-6 with the lower index winning ties, normalized weights)
//       and, in other CTAs, the shared expert's gate/up GEMV + SwiGLU, which
//       does not depend on routing.  The last router CTA to finish picks the
//       experts and builds the slot table (the union of chosen experts, in
//       ascending expert order).
//   K2  gate/up int4 GEMV + SwiGLU for every slot, weighted by the routing
//       weight of each row that chose it; writes the fp32 intermediate as an
//       exact-enough hi/lo bf16 pair image for K3's tensor-core fragments.
//   K3  down-projection GEMV of every slot and of the shared expert, with the
//       weights staged in shared memory by bulk copies issued before the PDL
//       wait; combine per row in a fixed order (the row's experts in
//       ascending index, then the shared expert).
//
// Model structure: "How to Run Flint Locally", section "The architecture,
// from config.json" (256 routed experts, 6 per token, expert size 512,
// sigmoid router with normalized top-k, shared expert of size 1,024 for every
// token); TandemLLM "21 Flint" section 21.1 (routing by sigmoid score with a
// bias) and section 21.2 (fp32 intermediates: routed SwiGLU activations reach
// 2.6e5, past fp16).  The kernel structure follows the low-latency decode
// path described under "What vLLM changed" (routing and combine folded into
// the neighbouring GEMVs, every kernel launched as a programmatic dependent).
//
// Batch invariance: every output element of row b is computed by the same
// lanes, in the same order, from row b's data alone, whatever B is; the
// combine walks row b's own experts.
#include "common.cuh"
#include "internal.h"

namespace flint {

constexpr int kRouterCtas = 64;  // 256 router items: 16 expert tiles x 16 k-groups
constexpr int kSharedCtas = 32;  // 128 shared gate/up items of 8 intermediate rows
constexpr int kK1Threads = 128;
constexpr int kK2Threads = 128;
constexpr int kK3Threads = 256;
constexpr int kXFragBytes = 16 * 128 * 16;  // 16 groups, 128 uint4 each
constexpr int kNPre = 4;                    // groups of weights in flight per warp

FLINT_DEV float silu_f(float v) { return v / (1.f + expf(-v)); }

FLINT_DEV void write_hilo(uint16_t *img_hi, uint16_t *img_lo, int k, float v) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
  const int s = frag_slot(k);
  img_hi[s] = __bfloat16_as_ushort(hi);
  img_lo[s] = __bfloat16_as_ushort(lo);
}

// Gate/up GEMV of one 8-row item: tile rows g = gate row, g + 8 = up row.
// Returns acc[0..1] = gate (cols 2t, 2t+1), acc[2..3] = up.
struct GateUpPtrs {
  const uint8_t *gate;
  const uint8_t *up;
  const uint16_t *gate_s;
  const uint16_t *up_s;
};

FLINT_DEV void gateup_prefetch(const GateUpPtrs &p, uint4 (&pg)[kNPre], uint4 (&pu)[kNPre],
                               uint32_t (&sg)[kNPre], uint32_t (&su)[kNPre]) {
#pragma unroll
  for (int G = 0; G < kNPre; ++G) {
    pg[G] = ld_stream(p.gate + 64 * G);
    pu[G] = ld_stream(p.up + 64 * G);
    sg[G] = ld_nc_u16(p.gate_s + G);
    su[G] = ld_nc_u16(p.up_s + G);
  }
}

FLINT_DEV void gateup_compute(const GateUpPtrs &p, uint4 (&pg)[kNPre], uint4 (&pu)[kNPre],
                              uint32_t (&sg)[kNPre], uint32_t (&su)[kNPre], const uint4 *xfrag,
                              int lane, float (&acc)[4]) {
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
  for (int G = 0; G < kH / kG; ++G) {
    const int sl = G % kNPre;
    const uint4 wg = pg[sl], wu = pu[sl];
    const float sgf = bf16_bits_to_f32(sg[sl]), suf = bf16_bits_to_f32(su[sl]);
    if (G + kNPre < kH / kG) {
      pg[sl] = ld_stream(p.gate + 64 * (G + kNPre));
      pu[sl] = ld_stream(p.up + 64 * (G + kNPre));
      sg[sl] = ld_nc_u16(p.gate_s + G + kNPre);
      su[sl] = ld_nc_u16(p.up_s + G + kNPre);
    }
    uint32_t ra[16], rb[16], xb[16];
    int4x32_to_bf16x2(wg, ra);
    int4x32_to_bf16x2(wu, rb);
    load_frag(xfrag + (G * 32 + lane) * 4, xb);
    float d[4];
    group_mma(ra, rb, xb, d);
    acc[0] = fmaf(d[0], sgf, acc[0]);
    acc[1] = fmaf(d[1], sgf, acc[1]);
    acc[2] = fmaf(d[2], suf, acc[2]);
    acc[3] = fmaf(d[3], suf, acc[3]);
  }
}

// x fragment of the block's input rows into shared memory.  Plain decode
// reads the bf16 input; the residual form computes RMSNorm of the fp32
// residual (fp64 inside) and rounds to bf16, and CTA `writer` also stores the
// normalized rows for the next kernel.
template <bool kResidual>
FLINT_DEV void stage_input(uint4 *xfrag, const uint16_t *x_in, const float *h, int B,
                           const double *inv, uint16_t *xn_out, bool writer, int tid,
                           int nthreads) {
  for (int task = tid; task < 16 * 128; task += nthreads) {
    const int G = task >> 7, ln = (task >> 2) & 31, q = task & 3;
    const int gg = ln >> 2, tt = ln & 3;
    const int k0 = 128 * G + 32 * tt + 8 * q;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (gg < B) {
      if (kResidual) {
        const uint4 a = ld_cg_v4(h + (size_t)gg * kH + k0);
        const uint4 c = ld_cg_v4(h + (size_t)gg * kH + k0 + 4);
        const double s = inv[gg];
        const uint32_t f[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        uint32_t bits[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) bits[i] = f64_to_bf16_bits((double)__uint_as_float(f[i]) * s);
        v = make_uint4(bits[0] | (bits[1] << 16), bits[2] | (bits[3] << 16),
                       bits[4] | (bits[5] << 16), bits[6] | (bits[7] << 16));
        if (writer) *reinterpret_cast<uint4 *>(xn_out + (size_t)gg * kH + k0) = v;
      } else {
        v = ld_cg_v4(x_in + (size_t)gg * kH + k0);
      }
    }
    xfrag[task] = bf16x8_to_pairs(v);
  }
}

// RMSNorm scale 1/sqrt(mean(h^2) + eps) per row, fp64, fixed reduction order.
FLINT_DEV void rms_inv(const float *h, int B, double *s_red /*[nwarps][kMaxB]*/, double *inv,
                       int tid, int nthreads) {
  const int warp = tid >> 5, lane = tid & 31, nw = nthreads >> 5;
  for (int b = 0; b < B; ++b) {
    double ss = 0.0;
    for (int i = tid; i < kH; i += nthreads) {
      const double v = (double)ld_cg_f32(h + (size_t)b * kH + i);
      ss = fma(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_red[warp * kMaxB + b] = ss;
  }
  __syncthreads();
  if (tid < B) {
    double ss = 0.0;
    for (int w = 0; w < nw; ++w) ss += s_red[w * kMaxB + tid];
    inv[tid] = 1.0 / sqrt(ss / kH + FLINT_RMS_EPS);
  }
  __syncthreads();
}

// ============================================================== K1
template <bool kResidual>
__global__ void __launch_bounds__(kK1Threads)
    k1_route_shared(LayerArgs L, const uint16_t *__restrict__ x_in, const float *__restrict__ h,
                    int B, char *__restrict__ ws, DecodeLayout lay, int32_t *__restrict__ idx_out,
                    float *__restrict__ w_out) {
  extern __shared__ uint4 xfrag[];
  __shared__ double s_red[4 * kMaxB];
  __shared__ double s_inv[kMaxB];
  __shared__ int s_last;
  __shared__ int s_asc_e[kMaxB][kTopK];
  __shared__ float s_asc_w[kMaxB][kTopK];
  __shared__ int s_slot_of[kE];
  __shared__ uint32_t s_mask[kE];
  __shared__ int s_wcount[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + lay.ctrl);
  const bool router = blockIdx.x < kRouterCtas;
  const int item = (router ? (int)blockIdx.x : (int)blockIdx.x - kRouterCtas) * 4 + warp;

  // ---- weights first: nothing here depends on the previous kernel
  uint4 wa[4], wb[4];
  uint4 pg[kNPre], pu[kNPre];
  uint32_t sg[kNPre], su[kNPre];
  GateUpPtrs gp{};
  if (router) {
    const int et = item >> 4, G = item & 15;
    const uint16_t *ra = L.router_w + (size_t)(16 * et + g) * kH + 128 * G + 32 * t;
    const uint16_t *rb = ra + 8 * kH;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wa[q] = ld_stream(ra + 8 * q);
      wb[q] = ld_stream(rb + 8 * q);
    }
  } else {
    const int r = 8 * item + g;
    gp.gate = L.sh13_q + (size_t)r * (kH / 2) + 16 * t;
    gp.up = L.sh13_q + (size_t)(kIs + r) * (kH / 2) + 16 * t;
    gp.gate_s = L.sh13_s + (size_t)r * (kH / kG);
    gp.up_s = L.sh13_s + (size_t)(kIs + r) * (kH / kG);
    gateup_prefetch(gp, pg, pu, sg, su);
  }

  pdl_wait();
  pdl_trigger();

  // ---- input rows -> activation fragment
  if (kResidual) rms_inv(h, B, s_red, s_inv, tid, kK1Threads);
  stage_input<kResidual>(xfrag, x_in, h, B, s_inv, reinterpret_cast<uint16_t *>(ws + lay.xn),
                         blockIdx.x == 0, tid, kK1Threads);
  __syncthreads();

  if (!router) {
    float acc[4];
    gateup_compute(gp, pg, pu, sg, su, xfrag, lane, acc);
    uint16_t *hfs = reinterpret_cast<uint16_t *>(ws + lay.hfs);
    const int r = 8 * item + g;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int b = 2 * t + c;
      if (b < B) {
        const float v = silu_f(acc[c]) * acc[2 + c];
        write_hilo(hfs + (size_t)(2 * b) * kIs, hfs + (size_t)(2 * b + 1) * kIs, r, v);
      }
    }
    return;
  }

  // ---- router item: 16 experts x one 128-wide group, fp32 group partials
  {
    const int et = item >> 4, G = item & 15;
    uint32_t ra[16], rb[16], xb[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 a = bf16x8_to_pairs(wa[q]), c = bf16x8_to_pairs(wb[q]);
      ra[4 * q] = a.x, ra[4 * q + 1] = a.y, ra[4 * q + 2] = a.z, ra[4 * q + 3] = a.w;
      rb[4 * q] = c.x, rb[4 * q + 1] = c.y, rb[4 * q + 2] = c.z, rb[4 * q + 3] = c.w;
    }
    load_frag(xfrag + (G * 32 + lane) * 4, xb);
    float d[4];
    group_mma(ra, rb, xb, d);
    float *zp = reinterpret_cast<float *>(ws + lay.zpart);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int b = 2 * t + c;
      if (b < B) {
        zp[((size_t)G * B + b) * kE + 16 * et + g] = d[c];
        zp[((size_t)G * B + b) * kE + 16 * et + g + 8] = d[2 + c];
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&ctrl[0], 1u);
    s_last = (prev == (uint32_t)(kRouterCtas - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last router CTA: scores, top-6, weights, slot table
  const float *zp = reinterpret_cast<const float *>(ws + lay.zpart);
  int32_t *sel_idx = reinterpret_cast<int32_t *>(ws + lay.sel_idx);
  float *sel_w = reinterpret_cast<float *>(ws + lay.sel_w);
  for (int b = warp; b < B; b += 4) {
    float sv[8];
    uint32_t key[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      double z = 0.0;
      for (int G = 0; G < 16; ++G) z += (double)ld_cg_f32(zp + ((size_t)G * B + b) * kE + e);
      const float zf = (float)z;
      const float s = 1.f / (1.f + expf(-zf));
      sv[i] = s;
      key[i] = float_key(s + L.router_b[e]);
    }
    uint32_t taken = 0;
    int sel_e[kTopK];
    float sel_s[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
      uint32_t best = 0;
      int bi = -1;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (!((taken >> i) & 1u) && key[i] > best) best = key[i], bi = i;
      const uint32_t m = __reduce_max_sync(0xffffffffu, best);
      const uint32_t cand = (bi >= 0 && best == m) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
      float mys = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i == bi) mys = sv[i];
      sel_s[j] = __shfl_sync(0xffffffffu, mys, (int)(win & 31));
      sel_e[j] = (int)win;
      if (lane == (int)(win & 31)) taken |= 1u << (win >> 5);
    }
    float ssum = 0.f;
#pragma unroll
    for (int j = 0; j < kTopK; ++j) ssum += sel_s[j];
    if (lane == 0) {
      float wj[kTopK];
#pragma unroll
      for (int j = 0; j < kTopK; ++j) {
        wj[j] = sel_s[j] / ssum;
        sel_idx[b * kTopK + j] = sel_e[j];
        sel_w[b * kTopK + j] = wj[j];
        if (idx_out) idx_out[b * kTopK + j] = sel_e[j];
        if (w_out) w_out[b * kTopK + j] = wj[j];
      }
      // ascending expert order for the combine
      int ae[kTopK];
      float aw[kTopK];
      for (int j = 0; j < kTopK; ++j) {
        int p = j;
        while (p > 0 && ae[p - 1] > sel_e[j]) {
          ae[p] = ae[p - 1];
          aw[p] = aw[p - 1];
          --p;
        }
        ae[p] = sel_e[j];
        aw[p] = wj[j];
      }
      for (int j = 0; j < kTopK; ++j) s_asc_e[b][j] = ae[j], s_asc_w[b][j] = aw[j];
    }
  }
  __syncthreads();
  for (int e = tid; e < kE; e += kK1Threads) {
    uint32_t m = 0;
    for (int b = 0; b < B; ++b)
      for (int j = 0; j < kTopK; ++j)
        if (s_asc_e[b][j] == e) m |= 1u << b;
    s_mask[e] = m;
  }
  __syncthreads();
  int32_t *slot_e = reinterpret_cast<int32_t *>(ws + lay.slot_e);
  uint32_t *slot_rows = reinterpret_cast<uint32_t *>(ws + lay.slot_rows);
  int base = 0;
  for (int round = 0; round < kE / kK1Threads; ++round) {
    const int e = round * kK1Threads + tid;
    const bool used = s_mask[e] != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, used);
    if (lane == 0) s_wcount[warp] = __popc(bal);
    __syncthreads();
    int off = base, total = 0;
    for (int w = 0; w < 4; ++w) {
      if (w < warp) off += s_wcount[w];
      total += s_wcount[w];
    }
    if (used) {
      const int slot = off + __popc(bal & ((1u << lane) - 1u));
      s_slot_of[e] = slot;
      slot_e[slot] = e;
      slot_rows[slot] = s_mask[e];
    }
    base += total;
    __syncthreads();
  }
  int32_t *asc_slot = reinterpret_cast<int32_t *>(ws + lay.asc_slot);
  float *asc_w = reinterpret_cast<float *>(ws + lay.asc_w);
  if (tid < B * kTopK) {
    const int b = tid / kTopK, j = tid % kTopK;
    asc_slot[tid] = s_slot_of[s_asc_e[b][j]];
    asc_w[tid] = s_asc_w[b][j];
  }
  if (tid == 0) {
    ctrl[2] = (uint32_t)base;
    ctrl[0] = 0;  // ready for the next call on this workspace
  }
}

// ============================================================== K2
template <bool kResidual>
__global__ void __launch_bounds__(kK2Threads)
    k2_routed_gateup(LayerArgs L, const uint16_t *__restrict__ x_in, int B,
                     char *__restrict__ ws, DecodeLayout lay) {
  extern __shared__ uint4 xfrag[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  pdl_wait();
  pdl_trigger();
  const uint32_t *ctrl = reinterpret_cast<const uint32_t *>(ws + lay.ctrl);
  const int n_slots = (int)ld_cg_u32(ctrl + 2);
  const int item0 = blockIdx.x * 4;
  if (item0 >= n_slots * 64) return;

  const uint16_t *src = kResidual ? reinterpret_cast<const uint16_t *>(ws + lay.xn) : x_in;
  stage_input<false>(xfrag, src, nullptr, B, nullptr, nullptr, false, tid, kK2Threads);
  __syncthreads();

  const int item = item0 + warp;
  if (item >= n_slots * 64) return;
  const int u = item >> 6, r0 = 8 * (item & 63);
  const int e = (int)ld_cg_u32(reinterpret_cast<const uint32_t *>(ws + lay.slot_e) + u);
  const size_t row = (size_t)e * (2 * kI) + r0 + g;
  GateUpPtrs gp;
  gp.gate = L.w13_q + row * (kH / 2) + 16 * t;
  gp.up = L.w13_q + (row + kI) * (kH / 2) + 16 * t;
  gp.gate_s = L.w13_s + row * (kH / kG);
  gp.up_s = L.w13_s + (row + kI) * (kH / kG);
  uint4 pg[kNPre], pu[kNPre];
  uint32_t sg[kNPre], su[kNPre];
  gateup_prefetch(gp, pg, pu, sg, su);
  float acc[4];
  gateup_compute(gp, pg, pu, sg, su, xfrag, lane, acc);

  const uint32_t mask = ld_cg_u32(reinterpret_cast<const uint32_t *>(ws + lay.slot_rows) + u);
  const int32_t *asc_slot = reinterpret_cast<const int32_t *>(ws + lay.asc_slot);
  const float *asc_w = reinterpret_cast<const float *>(ws + lay.asc_w);
  uint16_t *hfr = reinterpret_cast<uint16_t *>(ws + lay.hfr);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int b = 2 * t + c;
    if (b < B && ((mask >> b) & 1u)) {
      int j = 0;
      for (int jj = 0; jj < kTopK; ++jj)
        if ((int)ld_cg_u32(asc_slot + b * kTopK + jj) == u) j = jj;
      const float w = ld_cg_f32(asc_w + b * kTopK + j);
      const float v = w * (silu_f(acc[c]) * acc[2 + c]);
      uint16_t *img = hfr + (size_t)((b * kTopK + j) * 2) * kI;
      write_hilo(img, img + kI, r0 + g, v);
    }
  }
}

// ============================================================== K3
template <bool kResidual>
__global__ void __launch_bounds__(kK3Threads)
    k3_down_combine(LayerArgs L, int B, uint16_t *__restrict__ out, float *__restrict__ h,
                    char *__restrict__ ws, DecodeLayout lay, int umax) {
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char *wsm = sm;                   // [umax][16 rows][256 B]
  unsigned char *ssm = wsm + umax * 4096;    // [umax][16 rows][4] bf16
  unsigned char *shm = ssm + umax * 128;     // [16 rows][512 B]
  unsigned char *shs = shm + 8192;           // [16 rows][8] bf16
  float *ysel = reinterpret_cast<float *>(shs + 256);  // [8 rows b][7][16]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_slots;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * 16;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + lay.ctrl);

  // Routing is final here (K2 triggered this launch after its own wait on
  // K1), so the chosen experts' down rows can be fetched before the wait.
  if (tid == 0) {
    const int ns = (int)ld_cg_u32(ctrl + 2);
    s_slots = ns;
    mbar_init(&bar, 1);
    mbar_expect_tx(&bar, (uint32_t)ns * (4096u + 128u) + 8192u + 256u);
    const uint32_t *slot_e = reinterpret_cast<const uint32_t *>(ws + lay.slot_e);
    for (int u = 0; u < ns; ++u) {
      const size_t e = ld_cg_u32(slot_e + u);
      bulk_g2s(wsm + u * 4096, L.w2_q + (e * kH + n0) * (kI / 2), 4096, &bar);
      bulk_g2s(ssm + u * 128, L.w2_s + (e * kH + n0) * (kI / kG), 128, &bar);
    }
    bulk_g2s(shm, L.sh2_q + (size_t)n0 * (kIs / 2), 8192, &bar);
    bulk_g2s(shs, L.sh2_s + (size_t)n0 * (kIs / kG), 256, &bar);
  }
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int ns = s_slots;
  const bool arrived = mbar_wait(&bar, 0);
  if (__syncthreads_or(!arrived)) {
    if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
    if (!arrived) mbar_wait(&bar, 0);  // copies still in flight get one more bounded wait
    return;
  }

  const int32_t *asc_slot = reinterpret_cast<const int32_t *>(ws + lay.asc_slot);
  const uint32_t *slot_rows = reinterpret_cast<const uint32_t *>(ws + lay.slot_rows);
  const uint16_t *hfr = reinterpret_cast<const uint16_t *>(ws + lay.hfr);
  const uint16_t *hfs = reinterpret_cast<const uint16_t *>(ws + lay.hfs);

  for (int task = warp; task <= ns; task += kK3Threads / 32) {
    const bool sh = (task == ns);
    const int ngroups = sh ? kIs / kG : kI / kG;
    const int rowbytes = sh ? kIs / 2 : kI / 2;
    const unsigned char *wbase = sh ? shm : wsm + task * 4096;
    const unsigned char *sbase = sh ? shs : ssm + task * 128;
    const uint32_t mask = sh ? ((1u << B) - 1u) : ld_cg_u32(slot_rows + task);
    // this lane supplies activation column g
    const uint16_t *img = nullptr;
    int imgstride = 0;
    if (g < B && ((mask >> g) & 1u)) {
      if (sh) {
        img = hfs + (size_t)(2 * g) * kIs;
        imgstride = kIs;
      } else {
        int j = 0;
        for (int jj = 0; jj < kTopK; ++jj)
          if (ld_cg_u32(asc_slot + g * kTopK + jj) == (uint32_t)task) j = jj;
        img = hfr + (size_t)((g * kTopK + j) * 2) * kI;
        imgstride = kI;
      }
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int G = 0; G < ngroups; ++G) {
      uint32_t xh[16], xl[16];
      if (img) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 a = ld_cg_v4(img + ((G * 4 + t) * 16 + 4 * i) * 2);
          const uint4 b = ld_cg_v4(img + imgstride + ((G * 4 + t) * 16 + 4 * i) * 2);
          xh[4 * i] = a.x, xh[4 * i + 1] = a.y, xh[4 * i + 2] = a.z, xh[4 * i + 3] = a.w;
          xl[4 * i] = b.x, xl[4 * i + 1] = b.y, xl[4 * i + 2] = b.z, xl[4 * i + 3] = b.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = xl[i] = 0u;
      }
      const uint4 w0 = *reinterpret_cast<const uint4 *>(wbase + g * rowbytes + 64 * G + 16 * t);
      const uint4 w1 =
          *reinterpret_cast<const uint4 *>(wbase + (g + 8) * rowbytes + 64 * G + 16 * t);
      uint32_t ra[16], rb[16];
      int4x32_to_bf16x2(w0, ra);
      int4x32_to_bf16x2(w1, rb);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      group_mma_acc(ra, rb, xh, d);
      group_mma_acc(ra, rb, xl, d);
      const uint16_t *sc = reinterpret_cast<const uint16_t *>(sbase);
      const float s0 = bf16_bits_to_f32(sc[g * ngroups + G]);
      const float s1 = bf16_bits_to_f32(sc[(g + 8) * ngroups + G]);
      acc[0] = fmaf(d[0], s0, acc[0]);
      acc[1] = fmaf(d[1], s0, acc[1]);
      acc[2] = fmaf(d[2], s1, acc[2]);
      acc[3] = fmaf(d[3], s1, acc[3]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int b = 2 * t + c;
      if (b < B && ((mask >> b) & 1u)) {
        int j = kTopK;
        if (!sh)
          for (int jj = 0; jj < kTopK; ++jj)
            if (ld_cg_u32(asc_slot + b * kTopK + jj) == (uint32_t)task) j = jj;
        ysel[(b * 7 + j) * 16 + g] = acc[c];
        ysel[(b * 7 + j) * 16 + g + 8] = acc[2 + c];
      }
    }
  }
  __syncthreads();
  if (tid < 16 * B) {
    const int n = tid & 15, b = tid >> 4;
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < 7; ++j) y += ysel[(b * 7 + j) * 16 + n];
    const size_t o = (size_t)b * kH + n0 + n;
    if (kResidual) {
      const float yb = __bfloat162float(__float2bfloat16_rn(y));
      h[o] = ld_cg_f32(h + o) + yb;
    } else {
      out[o] = f32_to_bf16_bits(y);
    }
  }
}

// ============================================================== host
static size_t k3_smem_bytes(int umax) { return (size_t)umax * (4096 + 128) + 8192 + 256 + 8 * 7 * 16 * 4; }

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <bool kResidual>
static cudaError_t set_attrs_once() {
  static bool done = false;  // per process; the attribute is per device function
  static cudaError_t err = cudaSuccess;
  if (!done) {
    err = cudaFuncSetAttribute(k3_down_combine<kResidual>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)k3_smem_bytes(kTopK * kMaxB));
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(k1_route_shared<kResidual>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kXFragBytes);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(k2_routed_gateup<kResidual>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kXFragBytes);
    done = true;
  }
  return err;
}

template <bool kResidual>
static cudaError_t launch_decode_t(const LayerArgs &L, const uint16_t *x, float *h, int B,
                                   uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                                   cudaStream_t st, bool route_only) {
  cudaError_t err = set_attrs_once<kResidual>();
  if (err != cudaSuccess) return err;
  const DecodeLayout lay = decode_layout(B);
  const int k1_grid = route_only ? kRouterCtas : kRouterCtas + kSharedCtas;
  err = launch_pdl(k1_route_shared<kResidual>, k1_grid, kK1Threads, kXFragBytes, st, L, x,
                   (const float *)h, B, ws, lay, idx_out, w_out);
  if (err != cudaSuccess || route_only) return err;
  const int umax = kTopK * B < kE ? kTopK * B : kE;
  err = launch_pdl(k2_routed_gateup<kResidual>, umax * 16, kK2Threads, kXFragBytes, st, L, x, B,
                   ws, lay);
  if (err != cudaSuccess) return err;
  return launch_pdl(k3_down_combine<kResidual>, kH / 16, kK3Threads, k3_smem_bytes(umax), st, L,
                    B, out, h, ws, lay, umax);
}

cudaError_t launch_decode(const LayerArgs &L, const uint16_t *x, const float *h_in, float *h_out,
                          int B, uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                          cudaStream_t st, bool route_only) {
  (void)h_in;
  if (h_out)
    return launch_decode_t<true>(L, nullptr, h_out, B, nullptr, idx_out, w_out, ws, st, false);
  return launch_decode_t<false>(L, x, nullptr, B, out, idx_out, w_out, ws, st, route_only);
}

}  // namespace flint
