// Prefill of the Flint MoE block for T tokens.
//
// The block is defined per token ("How to Run Flint Locally", section "The
// architecture, from config.json"); for many tokens it is computed as
//   1. router logits for all tokens (bf16 products on the tcgen05 tensor
//      cores, fp32 partials of each 128-wide k-group summed in fp64; for
//      small T in two k-halves on two CTAs, added as decode adds them) and a
//      per-token top-6 with the same selection rule as decode;
//   2. a stable token-by-expert counting sort: per-chunk bitmask counts, one
//      scan over (expert, chunk), then positions in token order inside every
//      expert, and the GEMM tile lists;
//   3. power-of-two shifts that make both GEMM operands exact fp16 values,
//      and the fp16 token rows (each token's shared row and its six routed
//      rows in sorted order);
//   4. grouped GEMM 1 (gate/up + SwiGLU) and grouped GEMM 2 (down, scaled by
//      the routing weight) on the tcgen05 tensor cores, by pairs of CTAs: the
//      int4 codes land in shared memory by TMA and four warps per CTA turn
//      them into the fp16 weight tile in tensor memory, the token tile is
//      loaded by TMA in two halves (one per CTA), and one MMA instruction
//      covers 256 weight rows; the fp32 accumulator lives in tensor memory.
//      The shared expert is one more group that covers every token;
//   5. a fixed-order combine per token (its experts in ascending index, then
//      the shared expert).
// "What vLLM changed" on the same page: the small-batch MoE kernels that read
// only the selected experts were also the largest prefill gain.  The SwiGLU
// intermediate is fp16 after a per-token shift from a bound it cannot exceed
// (TandemLLM "21 Flint", section 21.2 reports routed activations up to 2.6e5,
// past the unscaled fp16 range).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace flint {

// ============================================================== top-6 (T tokens)
// One warp per token: sigmoid, bias, top-6 (lower index wins ties), weights;
// selection order to sel_*, ascending expert order to asc_*.  The logits are
// fp32 z[T][256], or (zh non-null) two fp64 k-half partials zh[2][T][256]
// added here, half 0 + half 1, as the decode router adds its halves.
__global__ void __launch_bounds__(256)
    k_pf_topk(const float *__restrict__ router_b, const float *__restrict__ z,
              const double *__restrict__ zh, int T,
              int32_t *__restrict__ sel_idx, float *__restrict__ sel_w, int32_t *__restrict__ asc_e,
              float *__restrict__ asc_w) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = blockIdx.x * 8 + warp;
  if (tok >= T) return;
  float sv[8];
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const size_t zi = (size_t)tok * kE + lane + 32 * i;
    const float zf = zh ? (float)(zh[zi] + zh[(size_t)T * kE + zi]) : z[zi];
    const float s = 1.f / (1.f + expf(-zf));
    sv[i] = s;
    key[i] = float_key(s + router_b[lane + 32 * i]);
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
  if (lane < kTopK) {
    int e_me = sel_e[0];
    float s_me = sel_s[0];
#pragma unroll
    for (int j = 1; j < kTopK; ++j)
      if (lane == j) e_me = sel_e[j], s_me = sel_s[j];
    const float w_me = s_me / ssum;
    sel_idx[(size_t)tok * kTopK + lane] = e_me;
    sel_w[(size_t)tok * kTopK + lane] = w_me;
    int rank = 0;
#pragma unroll
    for (int j = 0; j < kTopK; ++j) rank += sel_e[j] < e_me;
    if (asc_e) {
      asc_e[(size_t)tok * kTopK + rank] = e_me;
      asc_w[(size_t)tok * kTopK + rank] = w_me;
    }
  }
}

// ============================================================== stable sort by expert
// Per chunk of 256 tokens (one per thread), bits[e][w] has bit `lane` set when
// token 32w + lane of the chunk chose expert e.
FLINT_DEV void chunk_bits(const int32_t *asc_e, int T, int c, uint32_t (*bits)[8],
                          uint32_t *status) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kE * 8; i += 256) bits[i >> 3][i & 7] = 0u;
  __syncthreads();
  const int tok = c * kPfChunk + tid;
  if (tok < T)
    for (int j = 0; j < kTopK; ++j) {
      const int e = asc_e[(size_t)tok * kTopK + j];
      if (FLINT_CHECK((unsigned)e < (unsigned)kE, status)) atomicOr(&bits[e][warp], 1u << lane);
    }
  __syncthreads();
}

__global__ void __launch_bounds__(256)
    k_pf_count(const int32_t *__restrict__ asc_e, int T, int32_t *__restrict__ chunk_cnt,
               uint32_t *__restrict__ status) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  __shared__ uint32_t bits[kE][8];
  chunk_bits(asc_e, T, blockIdx.x, bits, status);
  const int e = threadIdx.x;
  int n = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) n += __popc(bits[e][w]);
  chunk_cnt[(size_t)blockIdx.x * kE + e] = n;
}

// exclusive scan of one value per thread over a 256-thread block; returns the
// prefix and writes the total to *total
FLINT_DEV int block_scan(int v, int *s_warp, int *total) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int off = 0, tot = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) off += s_warp[w];
    tot += s_warp[w];
  }
  __syncthreads();
  *total = tot;
  return off + incl - v;
}

// Tile descriptor: x = expert | pair row tile << 9 | token tile << 14;
// y = first row of the token tile in the per-row tables | valid tokens << 23
// (rows < 7 * 2^20 < 2^23, valid tokens <= 256).
FLINT_DEV uint2 pack_tile(int e, int mp, int nt, int b_row, int n_valid) {
  return make_uint2((uint32_t)e | ((uint32_t)mp << 9) | ((uint32_t)nt << 14),
                    (uint32_t)b_row | ((uint32_t)n_valid << 23));
}

// One CTA of 256 threads (one per expert): chunk offsets, expert counts,
// group bases (no padding) and both GEMM tile lists.  A tile is 256 weight
// rows (two 128-row tiles, one per CTA of a pair) by one token tile; the 4 or
// 8 tiles of one token tile are adjacent, so the token tile is reused from L2.
__global__ void __launch_bounds__(256)
    k_pf_scan(int T, int nchunks, const int32_t *__restrict__ chunk_cnt,
              int32_t *__restrict__ chunk_off, int32_t *__restrict__ ebase,
              int32_t *__restrict__ ecount, uint2 *__restrict__ tiles1,
              uint2 *__restrict__ tiles2, uint32_t *__restrict__ ctrl) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  __shared__ int s_warp[8];
  const int e = threadIdx.x;
  int off = 0;
#pragma unroll 8
  for (int c = 0; c < nchunks; ++c) {
    chunk_off[(size_t)c * kE + e] = off;
    off += chunk_cnt[(size_t)c * kE + e];
  }
  ecount[e] = off;
  const int nt1 = (off + kPfN1 - 1) / kPfN1, nt2 = (off + kPfN2 - 1) / kPfN2;
  int total_rows, total1, total2;
  const int base = block_scan(off, s_warp, &total_rows);
  const int o1 = block_scan(4 * nt1, s_warp, &total1);
  const int o2 = block_scan(8 * nt2, s_warp, &total2);
  ebase[e] = base;
  if (e == 0) ebase[kE] = total_rows;
  for (int nt = 0; nt < nt1; ++nt)
    for (int mp = 0; mp < 4; ++mp)
      tiles1[o1 + nt * 4 + mp] =
          pack_tile(e, mp, nt, base + nt * kPfN1, min(kPfN1, off - nt * kPfN1));
  for (int nt = 0; nt < nt2; ++nt)
    for (int mp = 0; mp < 8; ++mp)
      tiles2[o2 + nt * 8 + mp] =
          pack_tile(e, mp, nt, base + nt * kPfN2, min(kPfN2, off - nt * kPfN2));
  // the shared expert: one group over all T tokens, rows 6T .. 7T - 1 of the tables
  const int nsh1 = (T + kPfN1 - 1) / kPfN1, nsh2 = (T + kPfN2 - 1) / kPfN2;
  for (int i = e; i < 8 * nsh1; i += kE)
    tiles1[total1 + i] =
        pack_tile(kE, i & 7, i >> 3, 6 * T + (i >> 3) * kPfN1, min(kPfN1, T - (i >> 3) * kPfN1));
  for (int i = e; i < 8 * nsh2; i += kE)
    tiles2[total2 + i] =
        pack_tile(kE, i & 7, i >> 3, 6 * T + (i >> 3) * kPfN2, min(kPfN2, T - (i >> 3) * kPfN2));
  if (e == 0) {
    ctrl[3] = (uint32_t)(total1 + 8 * nsh1);
    ctrl[4] = (uint32_t)(total2 + 8 * nsh2);
    ctrl[5] = (uint32_t)total_rows;
  }
}

// pos[t][j]: the sorted row of token t's j-th expert (ascending expert order)
__global__ void __launch_bounds__(256)
    k_pf_place(const int32_t *__restrict__ asc_e, int T, const int32_t *__restrict__ chunk_off,
               const int32_t *__restrict__ ebase, int32_t *__restrict__ pos,
               uint32_t *__restrict__ status) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  __shared__ uint32_t bits[kE][8];
  const int c = blockIdx.x;
  chunk_bits(asc_e, T, c, bits, status);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok = c * kPfChunk + tid;
  if (tok >= T) return;
  for (int j = 0; j < kTopK; ++j) {
    const int e = asc_e[(size_t)tok * kTopK + j];
    if (!FLINT_CHECK((unsigned)e < (unsigned)kE, status)) continue;  // (flagged in chunk_bits too)
    int rank = __popc(bits[e][warp] & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) rank += __popc(bits[e][w]);
    const int p = ebase[e] + chunk_off[(size_t)c * kE + e] + rank;
    pos[(size_t)tok * kTopK + j] = p;
  }
}

// ---------------------------------------------------------- fp16 operand scaling
// Both GEMM operands are fp16 holding exact values (see the GEMM below), made
// so by power-of-two shifts: per expert matrix for the weights, per token for
// the token rows and the SwiGLU intermediate.

// 2^n as a float for n in the normal range
FLINT_DEV float exp2i(int n) { return __int_as_float((n + 127) << 23); }
// a shift n such that both 2^n and 2^-n are normal floats
FLINT_DEV int clamp_shift(int n) { return min(max(n, -126), 126); }

// One CTA per expert (expert 256 = the shared one).  For the gate/up matrix
// and the down matrix the shift S puts the largest |scale| in [2^-10, 2^-9),
// so the dequantization's fp16 multipliers scale x 2^24 stay below the fp16
// maximum and every code x scale (at most 11 significant bits) is an exact
// fp16 for scales down to 2^-17 (a 256-fold spread inside one matrix);
// wst[e] = (2^-S1, 2^S1, 2^-S2, 2^S2).  wbound[e] bounds the
// SwiGLU output per unit of |x|^2: by Cauchy-Schwarz |W1 x| <= |x| |W1 row| and
// |silu(g)| <= |g|, so |silu(W1 x) (W3 x)| <= |x|^2 max|W1 row| max|W3 row|,
// with |row| <= 8 sqrt(128 sum_g scale_g^2) for 128-wide groups of codes in [-8, 7].
// Routed experts' up rows stored divided by `up_mul` (a power of two) count
// with their scales times up_mul here and in the dequantization, so the
// GEMMs see the undivided weights.
__global__ void __launch_bounds__(256)
    k_pf_wstats(const uint16_t *__restrict__ w13_s, const uint16_t *__restrict__ w2_s,
                const uint16_t *__restrict__ sh13_s, const uint16_t *__restrict__ sh2_s,
                float up_mul, float4 *__restrict__ wst, float *__restrict__ wbound) {
  // the scales are weights, not the previous kernel's output: they are read
  // before the programmatic-launch wait, which only guards the writes
  pdl_trigger();
  __shared__ float red[4][8];
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool sh = e == kE;
  const int r13 = sh ? 2 * kIs : 2 * kI;  // gate rows, then as many up rows
  const uint16_t *s13 = sh ? sh13_s : w13_s + (size_t)e * r13 * (kH / kG);
  const int g2 = (sh ? kIs : kI) / kG;
  const uint16_t *s2 = sh ? sh2_s : w2_s + (size_t)e * kH * g2;
  float mx1 = 0.f, mx2 = 0.f, bg = 0.f, bu = 0.f;
  // gate/up: a row's 16 scales are two 16-byte words; every row of the thread
  // loaded before any is used (at most 8 rows: 2,048 rows over 256 threads)
  {
    constexpr int kMaxRows = 2 * kIs / 256;
    uint4 rv[kMaxRows][2];
#pragma unroll
    for (int i = 0; i < kMaxRows; ++i) {
      const int r = tid + 256 * i;
      if (r < r13) {
        const uint4 *p = reinterpret_cast<const uint4 *>(s13 + (size_t)r * (kH / kG));
        rv[i][0] = __ldg(p), rv[i][1] = __ldg(p + 1);
      }
    }
#pragma unroll
    for (int i = 0; i < kMaxRows; ++i) {
      const int r = tid + 256 * i;
      if (r >= r13) continue;
      const float um = (!sh && r >= r13 / 2) ? up_mul : 1.f;
      float ss = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w[4] = {rv[i][h].x, rv[i][h].y, rv[i][h].z, rv[i][h].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = fabsf(__uint_as_float(w[q] << 16)) * um,
                      b = fabsf(__uint_as_float(w[q] & 0xffff0000u)) * um;
          mx1 = fmaxf(mx1, fmaxf(a, b));
          ss = fmaf(a, a, fmaf(b, b, ss));
        }
      }
      const float rb = 8.f * sqrtf(128.f * ss);
      if (r < r13 / 2) bg = fmaxf(bg, rb);
      else bu = fmaxf(bu, rb);
    }
  }
  // down: 16-byte words of scales, all of the thread's in flight at once
  // (routed: 2,048 x 4 scales = 1,024 words; shared: 2,048 x 8 = 2,048)
  {
    constexpr int kMaxWords = kH * (kIs / kG) / 8 / 256;
    const int nw = kH * g2 / 8;
    uint4 dv[kMaxWords];
#pragma unroll
    for (int i = 0; i < kMaxWords; ++i) {
      const int k = tid + 256 * i;
      if (k < nw) dv[i] = __ldg(reinterpret_cast<const uint4 *>(s2) + k);
    }
#pragma unroll
    for (int i = 0; i < kMaxWords; ++i) {
      if (tid + 256 * i >= nw) continue;
      const uint32_t w[4] = {dv[i].x, dv[i].y, dv[i].z, dv[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        mx2 = fmaxf(mx2, fmaxf(fabsf(__uint_as_float(w[q] << 16)),
                               fabsf(__uint_as_float(w[q] & 0xffff0000u))));
    }
  }
  pdl_wait();  // the previous kernel in the stream is complete before any write
  float v[4] = {mx1, mx2, bg, bu};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v[k] = fmaxf(v[k], __shfl_xor_sync(0xffffffffu, v[k], o));
    if (lane == 0) red[k][warp] = v[k];
  }
  __syncthreads();
  if (tid == 0) {
    float m[4];
    for (int k = 0; k < 4; ++k) {
      m[k] = red[k][0];
      for (int w = 1; w < 8; ++w) m[k] = fmaxf(m[k], red[k][w]);
    }
    const int S1 = m[0] > 0.f ? clamp_shift(ilogbf(m[0]) + 10) : 0;
    const int S2 = m[1] > 0.f ? clamp_shift(ilogbf(m[1]) + 10) : 0;
    wst[e] = make_float4(exp2i(-S1), exp2i(S1), exp2i(-S2), exp2i(S2));
    wbound[e] = m[2] * m[3];
  }
}

// Group-64 affine experts (unsigned codes n in 0..15, one fp16 scale s and
// offset m per 64 elements; "How to Run Flint Locally", section "Every build
// and its size"): a weight n s + m lies between m and 15 s + m, so
// W = max(|m|, |15 s + m|) bounds the group.  The shift S of a matrix puts its
// largest W in [2^-7, 2^-6): then |s| 2^-S <= 2 W 2^-S / 15 < 2^-8.9, so the
// dequant multipliers s 2^(24-S) stay below fp16's largest value, and every
// weight x 2^-S is at most 2^-6.  A row's norm is at most sqrt(64 sum_g W_g^2).
FLINT_DEV float affine_bound(uint32_t sbits, uint32_t mbits) {
  const float s = __half2float(__ushort_as_half((unsigned short)sbits));
  const float m = __half2float(__ushort_as_half((unsigned short)mbits));
  return fmaxf(fabsf(m), fabsf(fmaf(15.f, s, m)));
}

__global__ void __launch_bounds__(256)
    k_pf_wstats_aff(const uint16_t *__restrict__ w13_s, const uint16_t *__restrict__ w13_m,
                    const uint16_t *__restrict__ w2_s, const uint16_t *__restrict__ w2_m,
                    const uint16_t *__restrict__ sh13_s, const uint16_t *__restrict__ sh13_m,
                    const uint16_t *__restrict__ sh2_s, const uint16_t *__restrict__ sh2_m,
                    float up_mul, float4 *__restrict__ wst, float *__restrict__ wbound) {
  pdl_trigger();  // weights only before the wait, as in k_pf_wstats
  __shared__ float red[4][8];
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool sh = e == kE;
  constexpr int g13 = kH / 64;  // groups per gate/up row: 4 uint4 of scales, 4 of offsets
  const int r13 = sh ? 2 * kIs : 2 * kI;
  const uint16_t *s13 = sh ? sh13_s : w13_s + (size_t)e * r13 * g13;
  const uint16_t *m13 = sh ? sh13_m : w13_m + (size_t)e * r13 * g13;
  const int g2 = (sh ? kIs : kI) / 64;
  const uint16_t *s2 = sh ? sh2_s : w2_s + (size_t)e * kH * g2;
  const uint16_t *m2 = sh ? sh2_m : w2_m + (size_t)e * kH * g2;
  float mx1 = 0.f, mx2 = 0.f, bg = 0.f, bu = 0.f;
#pragma unroll 2
  for (int r = tid; r < r13; r += 256) {
    const uint4 *ps = reinterpret_cast<const uint4 *>(s13 + (size_t)r * g13);
    const uint4 *pm = reinterpret_cast<const uint4 *>(m13 + (size_t)r * g13);
    uint4 sv[4], mv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sv[i] = __ldg(ps + i), mv[i] = __ldg(pm + i);
    const float um = (!sh && r >= r13 / 2) ? up_mul : 1.f;  // both s and m were divided
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a[4] = {sv[i].x, sv[i].y, sv[i].z, sv[i].w};
      const uint32_t b[4] = {mv[i].x, mv[i].y, mv[i].z, mv[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float W = affine_bound(a[q] >> (16 * h), b[q] >> (16 * h)) * um;
          mx1 = fmaxf(mx1, W);
          ss = fmaf(W, W, ss);
        }
    }
    const float rb = 8.f * sqrtf(ss);
    if (r < r13 / 2) bg = fmaxf(bg, rb);
    else bu = fmaxf(bu, rb);
  }
  {  // down: uint4 words of 8 groups (routed 2,048 words, shared 4,096)
    const int nw = kH * g2 / 8;
    const uint4 *ps = reinterpret_cast<const uint4 *>(s2), *pm = reinterpret_cast<const uint4 *>(m2);
#pragma unroll 4
    for (int k = tid; k < nw; k += 256) {
      const uint4 sv = __ldg(ps + k), mv = __ldg(pm + k);
      const uint32_t a[4] = {sv.x, sv.y, sv.z, sv.w}, b[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        mx2 = fmaxf(mx2, fmaxf(affine_bound(a[q], b[q]), affine_bound(a[q] >> 16, b[q] >> 16)));
    }
  }
  pdl_wait();  // the previous kernel in the stream is complete before any write
  float v[4] = {mx1, mx2, bg, bu};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v[k] = fmaxf(v[k], __shfl_xor_sync(0xffffffffu, v[k], o));
    if (lane == 0) red[k][warp] = v[k];
  }
  __syncthreads();
  if (tid == 0) {
    float m[4];
    for (int k = 0; k < 4; ++k) {
      m[k] = red[k][0];
      for (int w = 1; w < 8; ++w) m[k] = fmaxf(m[k], red[k][w]);
    }
    const int S1 = m[0] > 0.f ? clamp_shift(ilogbf(m[0]) + 7) : 0;
    const int S2 = m[1] > 0.f ? clamp_shift(ilogbf(m[1]) + 7) : 0;
    wst[e] = make_float4(exp2i(-S1), exp2i(S1), exp2i(-S2), exp2i(S2));
    wbound[e] = m[2] * m[3];
  }
}

// NVFP4 experts (E2M1 codes, an E4M3 scale per 16 elements, fp32 global
// scales; "How to Run Flint Locally", section "What vLLM changed"): an E2M1
// value times an E4M3 scale is an fp16 value (at most 6 significant bits, in
// [2^-10, 2,688]), so the GEMMs take the weights unshifted (S = 0) and the
// global scales multiply the epilogues' read-out: wsg[e] = (gate, up times
// the stored divisor of a routed expert's up rows, down).  A row's norm is at
// most 6 |g| sqrt(16 sum_b s_b^2) over its blocks b.
FLINT_DEV float e4m3_to_f32(uint32_t b) {
  uint32_t h;
  asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(b));
  return __half2float(__ushort_as_half((unsigned short)(h & 0xffffu)));
}

__global__ void __launch_bounds__(256)
    k_pf_wstats_nv(const uint8_t *__restrict__ w13_s, const float *__restrict__ w13_g,
                   const float *__restrict__ w2_g, const uint8_t *__restrict__ sh13_s,
                   const float *__restrict__ sh13_g, const float *__restrict__ sh2_g,
                   float up_mul, float4 *__restrict__ wst, float4 *__restrict__ wsg,
                   float *__restrict__ wbound) {
  pdl_trigger();  // weights only before the wait, as in k_pf_wstats
  __shared__ float red[2][8];
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool sh = e == kE;
  constexpr int rb = kH / 16;  // scale bytes per gate/up row: 8 uint4
  const int r13 = sh ? 2 * kIs : 2 * kI;
  const uint8_t *s13 = sh ? sh13_s : w13_s + (size_t)e * r13 * rb;
  float bg = 0.f, bu = 0.f;
#pragma unroll 2
  for (int r = tid; r < r13; r += 256) {
    const uint4 *ps = reinterpret_cast<const uint4 *>(s13 + (size_t)r * rb);
    uint4 sv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = __ldg(ps + i);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a[4] = {sv[i].x, sv[i].y, sv[i].z, sv[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float v = e4m3_to_f32((a[q] >> (8 * k)) & 0xffu);
          ss = fmaf(v, v, ss);
        }
    }
    const float rn = 24.f * sqrtf(ss);  // 6 sqrt(16 ss), times |g| below
    if (r < r13 / 2) bg = fmaxf(bg, rn);
    else bu = fmaxf(bu, rn);
  }
  pdl_wait();  // the previous kernel in the stream is complete before any write
  float v[2] = {bg, bu};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v[k] = fmaxf(v[k], __shfl_xor_sync(0xffffffffu, v[k], o));
    if (lane == 0) red[k][warp] = v[k];
  }
  __syncthreads();
  if (tid == 0) {
    float m[2];
    for (int k = 0; k < 2; ++k) {
      m[k] = red[k][0];
      for (int w = 1; w < 8; ++w) m[k] = fmaxf(m[k], red[k][w]);
    }
    const float gg = sh ? __ldg(sh13_g) : __ldg(w13_g + 2 * e);
    const float gu = (sh ? __ldg(sh13_g + 1) : __ldg(w13_g + 2 * e + 1)) * (sh ? 1.f : up_mul);
    const float gd = sh ? __ldg(sh2_g) : __ldg(w2_g + e);
    wst[e] = make_float4(1.f, 1.f, 1.f, 1.f);
    wsg[e] = make_float4(gg, gu, gd, 0.f);
    wbound[e] = (m[0] * fabsf(gg)) * (m[1] * fabsf(gu)) * (1.f + 1.f / 1024);
  }
}

// Token rows as the fp16 operand of GEMM 1: rows [0, 6T) are the routed rows
// in sorted order, rows [6T, 7T) every token for the shared expert.  One warp
// per token (grid-stride) reads the row once and takes its shifts: F puts
// max|x| in [2^14, 2^15) (the row is stored as x 2^-F, exact), E puts the
// SwiGLU output bound |x|^2 max_e wbound[e] below 2^15.  The converted row is
// written to its shared row and its six routed rows, each 8-element block in
// the order 0,4,1,5,2,6,3,7.  Per row, rsc = (F, E) for GEMM 1's read-out
// (multipliers 2^F and 2^-E) and rm3 = 2^E x routing weight for GEMM 2's.
__global__ void __launch_bounds__(256)
    k_pf_gather(const uint16_t *__restrict__ x, int T, const int32_t *__restrict__ pos,
                const float *__restrict__ asc_w, const float *__restrict__ wbound,
                uint16_t *__restrict__ xp, uint32_t *__restrict__ rsc, float *__restrict__ rm3,
                uint32_t *__restrict__ status) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  __shared__ float s_k;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {  // the bound factor: the largest over the experts
    float k = 0.f;
    for (int i = lane; i <= kE; i += 32) k = fmaxf(k, wbound[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) k = fmaxf(k, __shfl_xor_sync(0xffffffffu, k, o));
    if (lane == 0) s_k = k;
  }
  __syncthreads();
  const int nwarps = gridDim.x * 8;
  for (int tok = blockIdx.x * 8 + (threadIdx.x >> 5); tok < T; tok += nwarps) {
    // lanes 0..5: the token's routed rows; lane 6: its shared row
    int myrow = 0;
    if (lane < kTopK) {
      myrow = __ldg(pos + (size_t)tok * kTopK + lane);
      if (!FLINT_CHECK((unsigned)myrow < (unsigned)(6 * T), status)) myrow = -1;  // not written
    } else if (lane == kTopK) {
      myrow = 6 * T + tok;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)tok * kH);
    uint4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = ld_cg_v4(src + 32 * c + lane);
    float mx = 0.f;
    double ss = 0.0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = __uint_as_float(w[q] << 16), b = __uint_as_float(w[q] & 0xffff0000u);
        mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(b)));
        ss += (double)a * a + (double)b * b;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    const int F = mx > 0.f ? clamp_shift(ilogbf(mx) - 14) : 0;
    const double bound = ss * (double)s_k * (1.0 + 1.0 / 1024);  // rounding margin
    const int E = bound > 0.0 ? clamp_shift(ilogb(bound) + 1 - 15) : 0;
    const float xs = exp2i(-F);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
      uint32_t h[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        h[2 * q] = __half_as_ushort(__float2half_rn(__uint_as_float(w[q] << 16) * xs));
        h[2 * q + 1] = __half_as_ushort(__float2half_rn(__uint_as_float(w[q] & 0xffff0000u) * xs));
      }
      // natural h[0..7] -> pairs (0,4), (1,5), (2,6), (3,7)
      v[c] = make_uint4(h[0] | (h[4] << 16), h[1] | (h[5] << 16), h[2] | (h[6] << 16),
                        h[3] | (h[7] << 16));
    }
#pragma unroll
    for (int j = 0; j <= kTopK; ++j) {
      const int row = __shfl_sync(0xffffffffu, myrow, j);
      if (row < 0) continue;  // a row the bounds-checked build refused (the same for the warp)
      uint4 *dst = reinterpret_cast<uint4 *>(xp + (size_t)row * kH);
#pragma unroll
      for (int c = 0; c < 8; ++c) dst[32 * c + lane] = v[c];
    }
    if (lane <= kTopK && myrow >= 0) {
      rsc[myrow] = ((uint32_t)F & 0xffffu) | ((uint32_t)E << 16);
      rm3[myrow] = lane < kTopK ? exp2i(E) * __ldg(asc_w + (size_t)tok * kTopK + lane) : exp2i(E);
    }
  }
}

// ============================================================== tcgen05 grouped GEMM
// One tile is 128 weight rows (the MMA's M) by kN tokens (its N), with the
// whole K summed in one fp32 accumulator in tensor memory.  Both operands are
// fp16 holding exact values:
//  - the weights as code x scale x 2^-S: a code in [-8, 7] has at most 3
//    significant bits and a bf16 scale 8, so the product fits fp16's 11, and
//    the per-matrix shift S keeps it in the normal range.  Four dequant warps
//    write the tile straight into tensor memory (tcgen05.st), and the MMA
//    takes A from there;
//  - the tokens as x 2^-F (bf16 values, exact in fp16) for GEMM 1 and as the
//    SwiGLU intermediate x 2^-E (rounded to fp16, 11 bits) for GEMM 2, loaded
//    by TMA into 128-byte-swizzled shared memory.
// The read-out multiplies by 2^(S+F) or 2^(S+E).  Inside every 8-wide k block
// both operands hold the order 0,4,1,5,2,6,3,7 (the order int4 unpacking
// yields two codes per 32-bit word); the dot products do not depend on it.
constexpr int kRawBytes = 128 * 64;  // 128 weight rows x 128 int4 codes: one k-group
// A pair of CTAs (a cluster of two on neighbouring SMs) computes one tile of
// 256 weight rows: each CTA dequantizes its 128 rows into its own tensor
// memory and loads half of the token tile into its shared memory; one thread
// of the first CTA issues tcgen05.mma.cta_group::2, which reads A from both
// CTAs' tensor memory and B from both CTAs' shared memory, and writes each
// CTA's 128 accumulator rows into that CTA's tensor memory.  Every token byte
// thus crosses L2 -> SM once per 256 weight rows.
// Four warpgroups per CTA: 0 = token-tile producer (warp 0), MMA issuer
// (warp 1, first CTA), int4-code producer (warp 2) and an idle warp; 1 = four
// dequant warps (one weight row per thread); 2-3 = eight epilogue warps (two
// per TMEM lane quarter, one per half of the tile's tokens).  The block is launched at 128 registers per thread (65,536);
// setmaxnreg moves them: 128 x 40 + 128 x 88 + 256 x 184 = 63,488.
constexpr int kGemmThreads = 512;
constexpr int kEpiThreads = 256;
constexpr int kRegCtl = 40, kRegDeq = 88, kRegEpi = 184;
static_assert(128 * kRegCtl + 128 * kRegDeq + 256 * kRegEpi <= 65536, "register split");
constexpr int kTmemCols = 512;

// kN tokens per tile, kAcc accumulators of kN columns, kNA weight tiles in
// TMEM; a stage is kKS = 2 k-groups of 128 (one wait and one commit per 16
// MMAs), with two rings in shared memory: kS half token tiles (freed when the
// MMAs that read them complete) and kR int4-code tiles (freed once the
// dequant warps have read them, so the codes run ahead of the MMAs).
template <int kMode>
struct GemmCfg {
  static constexpr int kN = kMode == 1 ? kPfN1 : kPfN2;
  static constexpr int kAcc = 1;
  static constexpr int kKS = 2;   // k-groups per stage
  static constexpr int kNA = 2;   // weight tiles (one stage each: 128 TMEM columns)
  static constexpr int kS = 3;
  static constexpr int kR = 2;
  static constexpr int kBRows = kN / 2;       // token rows per CTA (the TMA box height)
  static constexpr int kBAtom = kBRows * 128;  // kN / 2 token rows x 64 fp16
  static constexpr int kBStage = kKS * 2 * kBAtom;
  static constexpr int kRawStage = kKS * kRawBytes;
  static constexpr size_t kSmem = (size_t)kS * kBStage + (size_t)kR * kRawStage + 1024;
  static constexpr size_t b_off(int s) { return (size_t)s * kBStage; }
  static constexpr size_t raw_off(int r) { return (size_t)kS * kBStage + (size_t)r * kRawStage; }
  // TMEM columns: the accumulator 0..255, the weight tiles at 256 and 384
  static constexpr uint32_t acc_col(int b) { return (uint32_t)(256 * b); }
  static constexpr uint32_t a_col(int a) { return (uint32_t)(256 + 64 * kKS * a); }
  static_assert(kN <= 256 && kAcc == 1 && 256 + 64 * kKS * kNA <= kTmemCols, "tensor memory");
  static_assert(kBAtom % 1024 == 0 && kN % 32 == 0, "tile shape");
};

struct GemmArgs {
  const uint2 *tiles;
  const uint32_t *ctrl;
  int count_word;
  const int32_t *ebase;
  const int32_t *ecount;
  int T;
  const uint16_t *sc_r;  // scales of the routed weight tensor
  const uint16_t *sc_s;  // scales of the shared expert's tensor
  const uint16_t *mo_r;  // affine: offsets of the routed weight tensor
  const uint16_t *mo_s;  // affine: offsets of the shared expert's tensor
  const float4 *wst;     // per expert: 2^-S1, 2^S1, 2^-S2, 2^S2
  const float4 *wsg;     // per expert, NVFP4: global scales of gate, up, down
  const uint32_t *rsc;   // per row: F | E << 16 (int16 each): multipliers 2^F, 2^-E
  const float *rm3;      // per row: 2^E x routing weight
  uint16_t *out_r;       // GEMM 1: Hr fp16 [6T][512]; GEMM 2: Yw bf16 [6T][2048]
  uint16_t *out_s;       // GEMM 1: Hs fp16 [T][1024]; GEMM 2: Ys bf16 [T][2048]
  uint32_t *status;
  float up_mul;          // GEMM 1: routed up rows' scales times this (the stored divisor)
};

FLINT_DEV uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

FLINT_DEV void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// D (TMEM) += A (TMEM, 128 lanes x 8 columns of fp16 pairs) x B (shared memory),
// the same, issued for the CTA pair (M = 256: A rows 0..127 in the first
// CTA's TMEM lanes, 128..255 in the second's; B rows split in halves between
// the two CTAs' shared memory at the same offset)
FLINT_DEV void umma_f16_ts_pair(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                uint32_t accum) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, "
      "%3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accum));
}

// arrive on `bar` (same offset) in both CTAs of the pair once the pair's
// earlier MMAs have completed
FLINT_DEV void umma_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_addr(bar)),
      "h"((unsigned short)3)
      : "memory");
}

FLINT_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of `p` (this CTA's shared memory) in CTA `rank`
FLINT_DEV uint32_t cluster_addr(const void *p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
  return a;
}
FLINT_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// arrive on an mbarrier of either CTA of the pair (a shared::cluster address),
// with the default CTA-scope release: what it orders for the other CTA is
// tensor-memory or shared-memory state that this CTA's own tensor core or TMA
// reads, completed before the arrival (tcgen05.wait + tcgen05.fence); a
// cluster-scope release would also wait for this thread's global stores
FLINT_DEV void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
// Wait on a barrier that the other CTA of the pair or the pair's MMAs arrive
// on: the default (CTA-scope) acquire, as for the other barriers (what must be
// ordered is tensor-memory and shared-memory state completed before the
// arrival: tcgen05.wait / fence, TMA and MMA completion); the thread may
// suspend until the phase completes.
FLINT_DEV bool cwait_sleep(uint64_t *bar, uint32_t parity) { return mbar_wait_sleep(bar, parity); }

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar_cl`, a shared::cluster address)
FLINT_DEV void tma_load_2d_pair(void *dst, const CUtensorMap *map, int x, int y, uint32_t bar_cl) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cl)
      : "memory");
}

// Optional GEMM timeline (build with -DFLINT_TRACE): for the first kPfTrTiles
// CTAs of each GEMM, %globaltimer per k-group of the CTA's first tile for the
// producer (TMA issued), the dequant warps (tile written), the MMA warp (MMAs
// issued) and, per tile, the epilogue (accumulator read); read with
// flint_pf_trace_dump.
#ifdef FLINT_TRACE
constexpr int kPfTrTiles = 8;
static __device__ unsigned long long g_pf_tr[2][kPfTrTiles][8][64];
FLINT_DEV void pf_mark(int mode, int role, int idx) {
  if (blockIdx.x < kPfTrTiles && idx < 64) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    g_pf_tr[mode - 1][blockIdx.x][role][idx] = t;
  }
}
extern "C" FLINT_API int flint_pf_trace_dump(unsigned long long *out) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  return cudaMemcpyFromSymbol(out, g_pf_tr, sizeof(g_pf_tr)) == cudaSuccess ? 0 : -1;
}
#else
FLINT_DEV void pf_mark(int, int, int) {}
#endif

// 32 consecutive TMEM columns of this warp's 32 lanes into v[0..31]; completes
// at tmem_wait_ld().
FLINT_DEV void tmem_ld32_async(uint32_t taddr, uint32_t *v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%"
      "15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
FLINT_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// v[0..31] into 32 consecutive TMEM columns of this warp's 32 lanes
FLINT_DEV void tmem_st32(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%"
      "14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
FLINT_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// barrier `id` over the first `n` threads that reach it (a subset of warps)
FLINT_DEV void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

FLINT_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FLINT_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 8 int4 codes (one 32-bit word, code k in bits 4k..4k+3, two's complement)
// times a scale s: fp16 pairs (k, k+4) for k = 0..3, exact.  A code field
// XOR 8 is n = code + 8 in [0, 15]; left in bits 0..3 of an fp16 it is the
// subnormal n 2^-24, in bits 4..7 it is n 2^-20.  One fused multiply-add
// n 2^-24 (s 2^24) - 8 s (or with s 2^20) forms code x s exactly inside and
// rounds once, and code x s is itself an fp16, so the result is exact.
// m24 = s 2^24, m20 = s 2^20 and c8 = -8 s as fp16x2 (both halves equal).
// Unsigned codes (kSigned false, the affine format) are n itself: with c8 the
// group's offset m (times 2^-S) the same FMA forms n s + m, rounded once.
template <bool kSigned = true>
FLINT_DEV void codes8_f16(uint32_t w, uint32_t m24, uint32_t m20, uint32_t c8, uint32_t *out) {
  constexpr uint32_t x0 = kSigned ? 0x00080008u : 0u, x1 = kSigned ? 0x00800080u : 0u;
  const uint32_t w8 = w >> 8;
  const uint32_t t0 = and_xor(w, 0x000F000Fu, x0);   // codes 0, 4
  const uint32_t t1 = and_xor(w, 0x00F000F0u, x1);   // codes 1, 5
  const uint32_t t2 = and_xor(w8, 0x000F000Fu, x0);  // codes 2, 6
  const uint32_t t3 = and_xor(w8, 0x00F000F0u, x1);  // codes 3, 7
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(out[0]) : "r"(t0), "r"(m24), "r"(c8));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(out[1]) : "r"(t1), "r"(m20), "r"(c8));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(out[2]) : "r"(t2), "r"(m24), "r"(c8));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(out[3]) : "r"(t3), "r"(m20), "r"(c8));
}

// One E4M3 byte -> fp16 pair (both halves the value; exact: E4M3 has 4
// significant bits and lies in [2^-9, 448]).
FLINT_DEV uint32_t e4m3x2_dup(uint32_t b) {
  uint32_t h;
  asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(b | (b << 8)));
  return h;
}
// 8 E2M1 codes (one word, code k in bits 4k..4k+3, the lower nibble the even
// element) times a block scale s (fp16 pair): fp16 pairs (k, k+4) for k =
// 0..3 (the order of codes8_f16), exact.  Masks and a shift-or put the pairs'
// nibbles into bytes: (n0 | n4 << 4, n2 | n6 << 4) and (n1 | n5 << 4, n3 |
// n7 << 4); the hardware converts each byte to an fp16 pair.
FLINT_DEV void e2m1x8_f16_scaled(uint32_t w, uint32_t s, uint32_t *out) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t X = lo | (lo >> 12), Y = hi | (hi >> 12);
  uint32_t h0, h1, h2, h3;
  asm("{ .reg .b8 x0, x1, x2, x3, y0, y1, y2, y3;\n"
      "mov.b32 {x0, x1, x2, x3}, %4;\n"
      "mov.b32 {y0, y1, y2, y3}, %5;\n"
      "cvt.rn.f16x2.e2m1x2 %0, x0;\n"
      "cvt.rn.f16x2.e2m1x2 %1, y0;\n"
      "cvt.rn.f16x2.e2m1x2 %2, x1;\n"
      "cvt.rn.f16x2.e2m1x2 %3, y1; }"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(X), "r"(Y));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[0]) : "r"(h0), "r"(s));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[1]) : "r"(h1), "r"(s));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[2]) : "r"(h2), "r"(s));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[3]) : "r"(h3), "r"(s));
}

// 16-bit global store, skipped when `pred` is false (no branch)
FLINT_DEV void st_u16_if(uint16_t *p, uint32_t v, bool pred) {
  asm volatile("{ .reg .pred q; setp.ne.b32 q, %2, 0; @q st.global.b16 [%0], %1; }" ::"l"(p),
               "h"((unsigned short)v), "r"((int)pred));
}

// position of natural column c inside its 8-wide block: 0,4,1,5,2,6,3,7 order
FLINT_DEV int perm8(int c) { return (c & ~7) | ((c & 7) < 4 ? 2 * (c & 7) : 2 * (c & 7) - 7); }

// kMode 1: gate/up + SwiGLU -> Hr (routed rows) / Hs (shared, [T][1024]), fp16.
// kMode 2: down -> Yw (routed, weighted, [6T][2048]) / Ys ([T][2048]), bf16.
// One tile of a grouped GEMM, as every role of the CTA derives it.
struct PfTile {
  int e, mt, n0, n_valid, n_mma, b_row, row0, row1, ng;
  bool sh;
};
// The tile a descriptor names, as every role of both CTAs derives it; mt is
// this CTA's 128-row tile: 2 x (the pair's tile) + the CTA's rank.
template <int kMode>
FLINT_DEV bool pf_tile(const GemmArgs &args, uint2 w, uint32_t rank, PfTile &t) {
  constexpr int kN = GemmCfg<kMode>::kN;
  t.e = (int)(w.x & 511u);
  t.mt = 2 * (int)((w.x >> 9) & 31u) + (int)rank;
  t.n0 = (int)(w.x >> 14) * kN;
  t.b_row = (int)(w.y & ((1u << 23) - 1u));
  t.n_valid = (int)(w.y >> 23);
  t.sh = t.e == kE;
  if (t.n_valid <= 0) return false;  // guards against an N = 0 MMA
  // the bounds-checked build: the descriptor names an expert (or the shared
  // one), a weight tile inside its matrix and token rows inside the operand
  // and output arrays; every role of both CTAs refuses the same tiles
  if (!FLINT_CHECK(t.e <= kE && t.n_valid <= kN &&
                       t.mt < (kMode == 1 ? (t.sh ? kIs : kI) / 64 : kH / 128) &&
                       (t.sh ? t.n0 + t.n_valid <= args.T
                             : t.b_row + t.n_valid <= kTopK * args.T) &&
                       (!t.sh || t.b_row == kTopK * args.T + t.n0),
                   args.status))
    return false;
  t.n_mma = (t.n_valid + 31) & ~31;  // the pair MMA takes N in steps of 32
  t.ng = (kMode == 1 ? kH : (t.sh ? kIs : kI)) / kG;  // 128-wide k-groups
  if (kMode == 1) {  // weight rows: gate (tile rows 2i) / up (2i+1)
    t.row0 = t.sh ? 64 * t.mt : t.e * 2 * kI + 64 * t.mt;
    t.row1 = t.sh ? kIs + 64 * t.mt : t.e * 2 * kI + kI + 64 * t.mt;
  } else {  // tile row i is weight row row0 + i
    t.row0 = t.sh ? 128 * t.mt : t.e * kH + 128 * t.mt;
    t.row1 = t.row0;
  }
  return true;
}

// Descriptor of the pair's tile `ti` (zero past the end): each role loads the
// next one while it works on the current one.
FLINT_DEV uint2 tile_word(const GemmArgs &args, uint32_t ti, uint32_t ntiles) {
  return ti < ntiles ? __ldcg(args.tiles + ti) : make_uint2(0u, 0u);
}

// Persistent: pair c takes tiles c, c + pairs, ...  Every role of both CTAs
// walks the same tile sequence with running counters (it: k-groups, tc:
// tiles), so the stage rings, the weight tiles in TMEM and the accumulators
// carry on across tiles and one tile's epilogue overlaps the next tile's MMAs.
// Barriers that gather both CTAs (full, afull, accempty) live in the first
// CTA; the MMA commits arrive on both CTAs' copies of empty, aempty, accfull.
template <int kMode, int kFmt>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    k_pf_gemm(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
              const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
              GemmArgs args) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  constexpr bool kAff = kFmt == 1, kNv = kFmt == 2;  // FLINT_FMT_*
  using Cfg = GemmCfg<kMode>;
  constexpr int S = Cfg::kS, R = Cfg::kR, NA = Cfg::kNA, NACC = Cfg::kAcc, kN = Cfg::kN;
  constexpr int KS = Cfg::kKS;
  constexpr int kHalf = kN / 2;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[S], empty[S], rfull[R], rempty[R], afull[NA], aempty[NA],
      accfull[NACC], accempty[NACC], mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_fail, s_epi_fail;
  __shared__ uint32_t s_mul[kN];  // per token of the tile: GEMM 1 F | E << 16; GEMM 2 2^E x weight

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t ntiles = __ldcg(args.ctrl + args.count_word);
  if (pair >= ntiles) return;  // the same for both CTAs of the pair

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], 4);  // one arrival per dequant warp
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&afull[a], 8);  // one arrival per dequant warp of both CTAs
      mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 16);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(&mma_done, 1);
    s_fail = 0;
    s_epi_fail = 0;
  }
  if (warp == 1) {  // the same warp in both CTAs, the same columns in both
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // the first CTA's gathering barriers, as shared::cluster addresses
  const uint32_t full_cl = cluster_addr(&full[0], 0);
  const uint32_t afull_cl = cluster_addr(&afull[0], 0);
  const uint32_t accempty_cl = cluster_addr(&accempty[0], 0);
  if (tid == 0) pf_mark(kMode, 4, 0);

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtl));
    if (warp == 0 && lane == 0) {
      // ---- token-tile producer, by TMA
      uint32_t it = 0;
      uint2 wnext = tile_word(args, pair, ntiles);
      for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
        const uint2 w = wnext;
        wnext = tile_word(args, ti + npairs, ntiles);
        PfTile t;
        if (!pf_tile<kMode>(args, w, rank, t)) continue;
        const CUtensorMap *tB = t.sh ? &tmB_s : &tmB_r;
        // this CTA's half of the token rows (GEMM 2's shared B is Hs)
        const int brow = ((kMode == 2 && t.sh) ? t.n0 : t.b_row) + (int)rank * (t.n_mma / 2);
        for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
          const int s = it % S;
          if (it >= (uint32_t)S && !cwait_sleep(&empty[s], ((it / S) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          unsigned char *st = sm + Cfg::b_off(s);
          if (rank == 0) mbar_expect_tx(&full[s], 2 * Cfg::kBStage);  // both halves
          const uint32_t fb = full_cl + 8u * s;
#pragma unroll
          for (int j = 0; j < 2 * KS; ++j)  // (group G0 + j / 2, atom j % 2)
            tma_load_2d_pair(st + j * Cfg::kBAtom, tB, G0 * 128 + 64 * j, brow, fb);
          if (ti == pair) pf_mark(kMode, 0, G0 / KS);
        }
      }
    } else if (warp == 2 && lane == 0) {
      // ---- int4-code producer, by TMA
      uint32_t it = 0;
      uint2 wnext = tile_word(args, pair, ntiles);
      for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
        const uint2 w = wnext;
        wnext = tile_word(args, ti + npairs, ntiles);
        PfTile t;
        if (!pf_tile<kMode>(args, w, rank, t)) continue;
        const CUtensorMap *tA = t.sh ? &tmA_s : &tmA_r;
        for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
          const int r = it % R;
          if (it >= (uint32_t)R && !mbar_wait_sleep(&rempty[r], ((it / R) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          unsigned char *rw = sm + Cfg::raw_off(r);
          mbar_expect_tx(&rfull[r], Cfg::kRawStage);
#pragma unroll
          for (int g = 0; g < KS; ++g) {  // group G0 + g at rw + g * kRawBytes
            if (kMode == 1) {  // gate rows then up rows, 128 codes (64 B) each
              tma_load_2d(rw + g * kRawBytes, tA, (G0 + g) * 64, t.row0, &rfull[r]);
              tma_load_2d(rw + g * kRawBytes + 64 * 64, tA, (G0 + g) * 64, t.row1, &rfull[r]);
            } else {  // 128 rows x 128 codes
              tma_load_2d(rw + g * kRawBytes, tA, (G0 + g) * 64, t.row0, &rfull[r]);
            }
          }
        }
      }
    } else if (warp == 1 && lane == 0 && rank == 1) {
      // the pair's MMAs write this CTA's tensor memory: they complete before it is freed
      if (!cwait_sleep(&mma_done, 0)) s_fail = 1;
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer (first CTA): tile tc accumulates into buffer tc % NACC of both CTAs
      uint32_t it = 0, tc = 0;
      uint2 wnext = tile_word(args, pair, ntiles);
      for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
        const uint2 w = wnext;
        wnext = tile_word(args, ti + npairs, ntiles);
        PfTile t;
        if (!pf_tile<kMode>(args, w, rank, t)) continue;
        const int b = tc % NACC;
        if (tc >= (uint32_t)NACC && !cwait_sleep(&accempty[b], ((tc / NACC) - 1) & 1)) {
          s_fail = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + Cfg::acc_col(b);
        // kind::f16, A = B = f16, D = f32, K-major, N = n_mma, M = 256 (the pair)
        const uint32_t idesc =
            (1u << 4) | ((uint32_t)(t.n_mma >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
        bool ok = true;
        for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
          const int s = it % S, a = it % NA;
          if (!cwait_sleep(&afull[a], (it / NA) & 1) || !cwait_sleep(&full[s], (it / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_addr = smem_addr(sm + Cfg::b_off(s));
          const uint32_t a_tm = tmem + Cfg::a_col(a);
#pragma unroll
          for (int j = 0; j < 2 * KS; ++j) {  // (group G0 + j / 2, atom j % 2): 64 k each
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_f16_ts_pair(d, a_tm + 8u * (4 * j + k),
                               sw128_desc(b_addr + j * Cfg::kBAtom + 32 * k), idesc,
                               (G0 | j | k) != 0);
          }
          umma_commit_pair(&empty[s]);   // both halves of the stage are free for the producers
          umma_commit_pair(&aempty[a]);  // both weight tiles are free for the dequant warps
          if (ti == pair) pf_mark(kMode, 2, G0 / KS);
        }
        if (!ok) {
          s_fail = 1;
          break;
        }
        umma_commit_pair(&accfull[b]);  // the tile's sums are complete in accumulator b
        ++tc;
      }
      // every MMA this thread issued completes before either CTA frees tensor memory
      umma_commit_pair(&mma_done);
      if (!cwait_sleep(&mma_done, 0)) s_fail = 1;
    }  // other lanes and warp 3: idle (register donors)
  } else if (warp < 8 && kNv) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegDeq));
    // ---- dequant, NVFP4 weights: each code pair's byte through the hardware
    // E2M1 conversion (an exact fp16 pair) times its 16-element block's E4M3
    // scale (an exact fp16 product: at most 6 significant bits, in [2^-10,
    // 2,688]); no shift (S = 0), the global scales in the epilogue.  A stage
    // (two 128-groups, 16 blocks) takes 16 scale bytes of the row, one uint4:
    // a tile's first stage loaded during the previous tile, the others from L1.
    static_assert(KS == 2, "a stage's 16 blocks are one uint4 of E4M3 scales");
    const int i = tid - 128, q = warp - 4;
    const int raw_row = kMode == 1 ? ((i & 1) ? 64 + (i >> 1) : (i >> 1)) : i;
    auto row_of = [&](const PfTile &tn) {  // this thread's row of scale bytes, as uint4
      const int wrow = kMode == 1 ? ((i & 1) ? tn.row1 : tn.row0) + (i >> 1) : tn.row0 + i;
      return reinterpret_cast<const uint4 *>(
          reinterpret_cast<const uint8_t *>(tn.sh ? args.sc_s : args.sc_r) +
          (size_t)wrow * (8 * (size_t)tn.ng));  // 8 blocks of 16 per 128-group
    };
    auto fetch = [&](uint2 w, uint4 &s0) {  // a tile's first stage
      PfTile tn;
      if (!pf_tile<kMode>(args, w, rank, tn)) return;
      s0 = __ldg(row_of(tn));
    };
    uint2 wa = tile_word(args, pair, ntiles), wb = tile_word(args, pair + npairs, ntiles);
    uint4 ns = make_uint4(0u, 0u, 0u, 0u);
    fetch(wa, ns);
    uint32_t it = 0;
    for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
      const uint2 w = wa;
      wa = wb;
      wb = tile_word(args, ti + 2 * npairs, ntiles);
      PfTile t;
      const bool valid = pf_tile<kMode>(args, w, rank, t);
      uint4 cs = ns;
      fetch(wa, ns);  // the next tile's, in flight during this one
      if (!valid) continue;
      const uint4 *ps = row_of(t);
      for (int c = 0; c < t.ng / 2; c += 8) asm volatile("prefetch.global.L1 [%0];" ::"l"(ps + c));
      bool ok = true;
      for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
        if (G0 > 0) cs = __ldg(ps + G0 / 2);
        const int rr = it % R, a = it % NA;
        if (!mbar_wait_sleep(&rfull[rr], (it / R) & 1) ||
            (it >= (uint32_t)NA && !cwait_sleep(&aempty[a], ((it / NA) - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sw[4] = {cs.x, cs.y, cs.z, cs.w};  // blocks 0..15 of the stage, a byte each
#pragma unroll
        for (int g = 0; g < KS; ++g) {  // group G0 + g -> TMEM columns 64 g .. of the tile
          const unsigned char *raw = sm + Cfg::raw_off(rr) + g * kRawBytes + raw_row * 64;
          const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + Cfg::a_col(a) + 64u * g;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // columns 32 hf ..: chunks 2 hf, 2 hf + 1
            uint32_t v[32];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const int j = 2 * hf + jj;  // chunk j: blocks 8 g + 2 j, 8 g + 2 j + 1
              const uint4 wv = *reinterpret_cast<const uint4 *>(raw + 16 * (j ^ ((raw_row >> 1) & 3)));
              const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
              const int b0 = 8 * g + 2 * j;
              const uint32_t sA = e4m3x2_dup((sw[b0 >> 2] >> (8 * (b0 & 3))) & 0xffu);
              const uint32_t sB = e4m3x2_dup((sw[(b0 + 1) >> 2] >> (8 * ((b0 + 1) & 3))) & 0xffu);
#pragma unroll
              for (int wi = 0; wi < 4; ++wi)
                e2m1x8_f16_scaled(words[wi], wi < 2 ? sA : sB, v + 16 * jj + 4 * wi);
            }
            tmem_st32(tbase + 32u * hf, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rr]);  // the codes are in registers and TMEM
          mbar_arrive_cluster(afull_cl + 8u * a);
        }
      }
      if (!ok) {
        s_fail = 1;
        break;
      }
    }
  } else if (warp < 8 && kAff) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegDeq));
    // ---- dequant, group-64 affine weights: as below, but every 64 codes have
    // their own fp16 scale s and offset m, and a weight is n s + m (times
    // 2^-S) rounded once to fp16 by the FMA of codes8_f16<false>.  A stage
    // (two 128-groups) takes four scales and four offsets of the row, one
    // uint2 apiece: a tile's first stage loaded during the previous tile
    // (with the tile descriptors two ahead), the others from L1.
    static_assert(KS == 2, "a stage's four 64-groups are one uint2 of scales and one of offsets");
    const int i = tid - 128, q = warp - 4;
    const int raw_row = kMode == 1 ? ((i & 1) ? 64 + (i >> 1) : (i >> 1)) : i;
    // this thread's row of a tile: its scales and offsets as uint2 (4 groups each)
    auto row_of = [&](const PfTile &tn, const uint2 *&ps, const uint2 *&pm) {
      const int wrow = kMode == 1 ? ((i & 1) ? tn.row1 : tn.row0) + (i >> 1) : tn.row0 + i;
      const size_t g64 = 2 * (size_t)tn.ng;  // 64-groups per row
      ps = reinterpret_cast<const uint2 *>((tn.sh ? args.sc_s : args.sc_r) + (size_t)wrow * g64);
      pm = reinterpret_cast<const uint2 *>((tn.sh ? args.mo_s : args.mo_r) + (size_t)wrow * g64);
    };
    auto fetch = [&](uint2 w, uint2 &s0, uint2 &m0, float &mul) {  // a tile's first stage
      PfTile tn;
      if (!pf_tile<kMode>(args, w, rank, tn)) return;
      const uint2 *ps, *pm;
      row_of(tn, ps, pm);
      s0 = __ldg(ps);
      m0 = __ldg(pm);
      const float4 ws = __ldg(args.wst + tn.e);
      mul = kMode == 1 ? ws.x : ws.z;
      if (kMode == 1 && (i & 1) && !tn.sh) mul *= args.up_mul;  // routed up rows: undo the divisor
    };
    uint2 wa = tile_word(args, pair, ntiles), wb = tile_word(args, pair + npairs, ntiles);
    uint2 ns = make_uint2(0u, 0u), nm = make_uint2(0u, 0u);
    float muln = 0.f;
    fetch(wa, ns, nm, muln);
    uint32_t it = 0;
    for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
      const uint2 w = wa;
      wa = wb;
      wb = tile_word(args, ti + 2 * npairs, ntiles);
      PfTile t;
      const bool valid = pf_tile<kMode>(args, w, rank, t);
      uint2 cs = ns, cm = nm;
      const float smul = muln;
      fetch(wa, ns, nm, muln);  // the next tile's, in flight during this one
      if (!valid) continue;
      const uint2 *ps, *pm;
      row_of(t, ps, pm);
      // the row's scales and offsets (t.ng / 2 uint2 each) into L1; a stage's
      // are read before its wait
      for (int c = 0; c < t.ng / 2; c += 16) {
        asm volatile("prefetch.global.L1 [%0];" ::"l"(ps + c));
        asm volatile("prefetch.global.L1 [%0];" ::"l"(pm + c));
      }
      bool ok = true;
      for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
        if (G0 > 0) cs = __ldg(ps + G0 / 2), cm = __ldg(pm + G0 / 2);
        const int rr = it % R, a = it % NA;
        if (!mbar_wait_sleep(&rfull[rr], (it / R) & 1) ||
            (it >= (uint32_t)NA && !cwait_sleep(&aempty[a], ((it / NA) - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 64-groups 2 G0 .. 2 G0 + 3 of the row, in memory order
        const uint32_t sv[4] = {cs.x & 0xffffu, cs.x >> 16, cs.y & 0xffffu, cs.y >> 16};
        const uint32_t mv[4] = {cm.x & 0xffffu, cm.x >> 16, cm.y & 0xffffu, cm.y >> 16};
#pragma unroll
        for (int g = 0; g < KS; ++g) {  // group G0 + g -> TMEM columns 64 g .. of the tile
          const unsigned char *raw = sm + Cfg::raw_off(rr) + g * kRawBytes + raw_row * 64;
          const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + Cfg::a_col(a) + 64u * g;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // 64-group 2 (G0 + g) + hf: chunks 2 hf, 2 hf + 1
            // s 2^(24-S), s 2^(20-S) and m 2^-S as fp16x2: fp16 values times
            // powers of two, exact while normal (the scale's are, by the
            // choice of S; an offset far below the group's bound W may round
            // there, by less than 2^-25 against weights near 2^-7)
            const float sf = __half2float(__ushort_as_half((unsigned short)sv[2 * g + hf])) * smul;
            const float mf = __half2float(__ushort_as_half((unsigned short)mv[2 * g + hf])) * smul;
            const uint32_t h24 = __half_as_ushort(__float2half_rn(sf * 16777216.f));
            const uint32_t h20 = __half_as_ushort(__float2half_rn(sf * 1048576.f));
            const uint32_t hm = __half_as_ushort(__float2half_rn(mf));
            const uint32_t m24 = h24 | (h24 << 16), m20 = h20 | (h20 << 16), mm = hm | (hm << 16);
            uint32_t v[32];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const int j = 2 * hf + jj;  // the box is 64-byte swizzled, as below
              const uint4 wv = *reinterpret_cast<const uint4 *>(raw + 16 * (j ^ ((raw_row >> 1) & 3)));
              codes8_f16<false>(wv.x, m24, m20, mm, v + 16 * jj + 0);
              codes8_f16<false>(wv.y, m24, m20, mm, v + 16 * jj + 4);
              codes8_f16<false>(wv.z, m24, m20, mm, v + 16 * jj + 8);
              codes8_f16<false>(wv.w, m24, m20, mm, v + 16 * jj + 12);
            }
            tmem_st32(tbase + 32u * hf, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rr]);  // the codes are in registers and TMEM
          mbar_arrive_cluster(afull_cl + 8u * a);
        }
      }
      if (!ok) {
        s_fail = 1;
        break;
      }
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegDeq));
    // ---- dequant: thread i owns weight row i of every tile, TMEM lane i
    const int i = tid - 128, q = warp - 4;
    const int raw_row = kMode == 1 ? ((i & 1) ? 64 + (i >> 1) : (i >> 1)) : i;
    // the row's bf16 scales for the whole K (16, 8 or 4 groups) and the matrix
    // shift, fetched one tile ahead (tile descriptors two ahead)
    auto fetch = [&](uint2 w, uint32_t (&sc)[8], float &mul) {
      PfTile tn;
      if (!pf_tile<kMode>(args, w, rank, tn)) return;
      const int wrow = kMode == 1 ? ((i & 1) ? tn.row1 : tn.row0) + (i >> 1) : tn.row0 + i;
      const uint32_t *srow = reinterpret_cast<const uint32_t *>(
          (tn.sh ? args.sc_s : args.sc_r) + (size_t)wrow * tn.ng);
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) sc[w2] = w2 < tn.ng / 2 ? __ldg(srow + w2) : 0u;
      const float4 ws = __ldg(args.wst + tn.e);
      mul = kMode == 1 ? ws.x : ws.z;
      if (kMode == 1 && (i & 1) && !tn.sh) mul *= args.up_mul;  // routed up rows: undo the divisor
    };
    uint2 wa = tile_word(args, pair, ntiles), wb = tile_word(args, pair + npairs, ntiles);
    uint32_t scn[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    float muln = 0.f;
    fetch(wa, scn, muln);
    uint32_t it = 0;
    for (uint32_t ti = pair; ti < ntiles && !s_fail; ti += npairs) {
      const uint2 w = wa;
      wa = wb;
      wb = tile_word(args, ti + 2 * npairs, ntiles);
      PfTile t;
      const bool valid = pf_tile<kMode>(args, w, rank, t);
      uint32_t scw[8];
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) scw[w2] = scn[w2];
      const float smul = muln;
      fetch(wa, scn, muln);  // the next tile's, in flight during this one
      if (!valid) continue;
      bool ok = true;
      for (int G0 = 0; G0 < t.ng; G0 += KS, ++it) {
        const int rr = it % R, a = it % NA;
        if (!mbar_wait_sleep(&rfull[rr], (it / R) & 1) ||
            (it >= (uint32_t)NA && !cwait_sleep(&aempty[a], ((it / NA) - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < KS; ++g) {  // group G0 + g -> TMEM columns 64 g .. of the tile
          const int G = G0 + g;
          // the group's scale s x 2^-S and its multipliers as fp16x2 (exact: 8
          // significant bits; s 2^24 < 2^15 by the choice of S)
          const uint32_t sw = scw[G >> 1] >> (16 * (G & 1));
          const float sf = __uint_as_float(sw << 16) * smul;
          const uint32_t h24 = __half_as_ushort(__float2half_rn(sf * 16777216.f));
          const uint32_t h20 = __half_as_ushort(__float2half_rn(sf * 1048576.f));
          const uint32_t hc8 = __half_as_ushort(__float2half_rn(sf * -8.f));
          const uint32_t m24 = h24 | (h24 << 16), m20 = h20 | (h20 << 16),
                         c8 = hc8 | (hc8 << 16);
          const unsigned char *raw = sm + Cfg::raw_off(rr) + g * kRawBytes + raw_row * 64;
          const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + Cfg::a_col(a) + 64u * g;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // columns 32 hf .. 32 hf + 31: chunks 2 hf, 2 hf + 1
            uint32_t v[32];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              // chunk j = codes 32 j .. 32 j + 31 of the group -> columns 16 j ..;
              // the box is 64-byte swizzled: chunk j of box row r sits at
              // chunk j ^ ((r >> 1) & 3) (address bits 7-8 of a 1024-aligned box)
              const int j = 2 * hf + jj;
              const uint4 w = *reinterpret_cast<const uint4 *>(raw + 16 * (j ^ ((raw_row >> 1) & 3)));
              codes8_f16(w.x, m24, m20, c8, v + 16 * jj + 0);
              codes8_f16(w.y, m24, m20, c8, v + 16 * jj + 4);
              codes8_f16(w.z, m24, m20, c8, v + 16 * jj + 8);
              codes8_f16(w.w, m24, m20, c8, v + 16 * jj + 12);
            }
            tmem_st32(tbase + 32u * hf, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rr]);  // the codes are in registers and TMEM
          mbar_arrive_cluster(afull_cl + 8u * a);
        }
        if (tid == 128 && ti == pair) pf_mark(kMode, 1, G0 / KS);
      }
      if (!ok) {
        s_fail = 1;
        break;
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegEpi));
    // ---- epilogue warps 8..15: TMEM lane quarter (warp % 4) -> tile rows;
    // token half (warp - 8) / 4 -> tile columns kHalf h .. kHalf h + kHalf - 1
    const int q4 = warp & 3;
    const int c_lo = kHalf * ((warp - 8) >> 2);
    const int r = 32 * q4 + lane;
    // The tile's per-token multipliers pass through shared memory (thread
    // tid - 256 fetches token tid - 256 before the accumulator is ready);
    // two barriers of the 256 epilogue threads per tile guard the array, and
    // the loop ends on a flag only these threads write before the second, so
    // all eight warps leave in the same iteration.
    const int et = tid - 256;
    uint32_t tc = 0;
    uint2 wnext = tile_word(args, pair, ntiles);
    for (uint32_t ti = pair; ti < ntiles; ti += npairs) {
      const uint2 w = wnext;
      wnext = tile_word(args, ti + npairs, ntiles);
      PfTile t;
      if (!pf_tile<kMode>(args, w, rank, t)) continue;
      const int b = tc % NACC;
      const float4 ws = __ldg(args.wst + t.e);
      const float4 gsc = kNv ? __ldg(args.wsg + t.e) : make_float4(1.f, 1.f, 1.f, 1.f);
      uint32_t pre = 0u;
      if (et < t.n_valid)
        pre = kMode == 1 ? __ldg(args.rsc + t.b_row + et)
                         : __float_as_uint(__ldg(args.rm3 + t.b_row + et));
      const bool ok = cwait_sleep(&accfull[b], (tc / NACC) & 1);
      tc_fence_after();
      uint32_t acc[kHalf];
      if (ok && c_lo < t.n_mma) {  // the same for the whole warp
        const uint32_t base = tmem + Cfg::acc_col(b) + (uint32_t)c_lo + ((uint32_t)(32 * q4) << 16);
#pragma unroll
        for (int c = 0; c < kHalf / 32; ++c)
          if (c_lo + 32 * c < t.n_mma) tmem_ld32_async(base + 32u * c, acc + 32 * c);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive_cluster(accempty_cl + 8u * b);  // tile tc + NACC may start
      if (tid == 256 && ti == pair) pf_mark(kMode, 3, 0);
      ++tc;
      named_bar_sync(1, kEpiThreads);  // every warp is done with the previous tile's multipliers
      if (!ok) s_epi_fail = 1;
      if (et < kN) s_mul[et] = pre;
      named_bar_sync(1, kEpiThreads);
      if (s_epi_fail) {
        s_fail = 1;
        break;
      }
      const int nv = t.n_valid - c_lo;  // valid tokens in this half
      if (nv <= 0) continue;            // the same for the whole warp
      if (kMode == 1) {
        // lanes r (gate row) and r + 1 (up row) hold the same column: the gate
        // lane finishes the first half of the warp's tokens, the up lane the rest
        const bool up_lane = r & 1;
        const int col = perm8(64 * t.mt + (r >> 1));
        uint16_t *hb = t.sh ? args.out_s + (size_t)t.n0 * kIs + col
                            : args.out_r + (size_t)t.b_row * kI + col;
        const size_t ld = t.sh ? kIs : kI;
        const float mw = ws.y;  // 2^S1
        constexpr int kQ = kHalf / 2;
        const int j0 = up_lane ? kQ : 0;
        // branch-free arithmetic first (the tokens overlap), then predicated stores
        constexpr int kC = 16;  // tokens per pass (bounds the live registers)
#pragma unroll
        for (int c0 = 0; c0 < kQ; c0 += kC) {
          uint32_t hp[kC / 2];
#pragma unroll
          for (int u = 0; u < kC; ++u) {
            const int jj = c0 + u;
            const float mine = __uint_as_float(up_lane ? acc[kQ + jj] : acc[jj]);
            const float theirs =
                __shfl_xor_sync(0xffffffffu, __uint_as_float(up_lane ? acc[jj] : acc[kQ + jj]), 1);
            const uint32_t fe = s_mul[c_lo + j0 + jj];  // F | E << 16
            const float m = mw * exp2i((int)(int16_t)(fe & 0xffffu));
            // (NVFP4: times the gate's and the up rows' global scales)
            const float g = (up_lane ? theirs : mine) * (kNv ? m * gsc.x : m);
            const float uu = (up_lane ? mine : theirs) * (kNv ? m * gsc.y : m);
            const float h = __fdividef(g, 1.f + __expf(-g)) * uu *
                            exp2i(-(int)(int16_t)(fe >> 16));  // silu(gate) * up / 2^E
            const uint32_t hv = __half_as_ushort(__float2half_rn(h));
            hp[u >> 1] = (u & 1) ? (hp[u >> 1] | (hv << 16)) : hv;
          }
#pragma unroll
          for (int u = 0; u < kC; ++u) {
            const int jj = c0 + u;
            st_u16_if(hb + (size_t)(c_lo + j0 + jj) * ld, hp[u >> 1] >> (16 * (u & 1)), j0 + jj < nv);
          }
        }
      } else {
        const int col = 128 * t.mt + r;
        const float mw = ws.w;  // 2^S2
        uint16_t *yb = t.sh ? args.out_s + (size_t)t.n0 * kH + col
                            : args.out_r + (size_t)t.b_row * kH + col;
#pragma unroll
        for (int j = 0; j < kHalf; ++j) {
          const float m = mw * __uint_as_float(s_mul[c_lo + j]) * (kNv ? gsc.z : 1.f);
          st_u16_if(yb + (size_t)(c_lo + j) * kH, f32_to_bf16_bits(__uint_as_float(acc[j]) * m), j < nv);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still reach its memory
  if (tid == 0) pf_mark(kMode, 4, 1);
  if (s_fail && tid == 0) set_status(args.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// ============================================================== router on tcgen05
// z[t][e] = sum over the 16 k-groups of the fp32 sum of the group's 128 bf16
// products, the groups added in fp64 in order (the same rule as the decode
// router).  One tile = 128 tokens (the MMA's M: the token rows, TMA) x 128
// experts (its N: router rows, TMA), K in 128-wide groups; each group's MMAs
// write one of two TMEM slots (so the next group runs while this one is read)
// and eight epilogue warps add the slot into fp64 registers.
constexpr int kRtM = 128, kRtN = 128;
constexpr int kRtThreads = 384;  // warp 0 producer, warp 1 MMA, 2-3 idle, 4-11 epilogue
constexpr int kRtStages = 3;
constexpr int kRtAtom = 128 * 128;                 // 128 rows x 64 bf16 (one SW128 atom)
constexpr int kRtStageBytes = 4 * kRtAtom;         // x: 2 atoms, W: 2 atoms
constexpr size_t kRtSmem = (size_t)kRtStages * kRtStageBytes + 1024;
constexpr int kRtRegCtl = 40, kRtRegEpi = 232;
static_assert(128 * kRtRegCtl + 256 * kRtRegEpi <= 384 * 168, "router register split");

FLINT_DEV void umma_bf16_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                            uint32_t accum) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, "
      "%3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}
FLINT_DEV void umma_commit1(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Persistent: CTA c takes work items c, c + grid, ...; item i is tile
// i / nsplit (token tile tile / 2, expert half tile % 2) over the k-groups of
// k-part i % nsplit.  nsplit = 1: the tile's fp32 logits to z[T][256];
// nsplit = 2: the k-half's fp64 partial sums to zh[half][T][256].
__global__ void __launch_bounds__(kRtThreads, 1)
    k_pf_router_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   int T, int nsplit, float *__restrict__ z, double *__restrict__ zh,
                   uint32_t *status) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kRtStages], empty[kRtStages], sfull[2], sempty[2], done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_fail;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = 2 * ((T + kRtM - 1) / kRtM), nitems = ntiles * nsplit;
  if ((int)blockIdx.x >= nitems) return;
  if (tid == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull[b], 1);
      mbar_init(&sempty[b], 8);  // one arrival per epilogue warp
    }
    mbar_init(&done, 1);
    s_fail = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&s_tmem)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  constexpr int kG = kH / 128;  // 16 k-groups
  const int gper = kG / nsplit;  // k-groups per work item

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRtRegCtl));
    if (warp == 0 && lane == 0) {
      // ---- producer: the token rows and the router rows of each k-group
      uint32_t it = 0;
      for (int wi = blockIdx.x; wi < nitems && !s_fail; wi += gridDim.x) {
        const int ti = wi / nsplit, g0 = gper * (wi % nsplit);
        const int t0 = kRtM * (ti >> 1), e0 = kRtN * (ti & 1);
        for (int G = g0; G < g0 + gper; ++G, ++it) {
          const int s = it % kRtStages;
          if (it >= (uint32_t)kRtStages &&
              !mbar_wait_sleep(&empty[s], ((it / kRtStages) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          unsigned char *st = sm + (size_t)s * kRtStageBytes;
          mbar_expect_tx(&full[s], kRtStageBytes);
          tma_load_2d(st, &tmX, 128 * G, t0, &full[s]);
          tma_load_2d(st + kRtAtom, &tmX, 128 * G + 64, t0, &full[s]);
          tma_load_2d(st + 2 * kRtAtom, &tmW, 128 * G, e0, &full[s]);
          tma_load_2d(st + 3 * kRtAtom, &tmW, 128 * G + 64, e0, &full[s]);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer: k-group number it writes TMEM slot it % 2
      // kind::f16, A = B = bf16, D = f32, K-major, N = 128, M = 128
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRtN >> 3) << 17) |
                             ((uint32_t)(kRtM >> 4) << 24);
      uint32_t it = 0;
      for (int wi = blockIdx.x; wi < nitems && !s_fail; wi += gridDim.x) {
        bool ok = true;
        for (int G = 0; G < gper; ++G, ++it) {
          const int s = it % kRtStages, b = it & 1;
          if ((it >= 2 && !mbar_wait(&sempty[b], ((it >> 1) - 1) & 1)) ||
              !mbar_wait(&full[s], (it / kRtStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_addr(sm + (size_t)s * kRtStageBytes);
#pragma unroll
          for (int atom = 0; atom < 2; ++atom)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ss(tmem + (uint32_t)(128 * b), sw128_desc(st + atom * kRtAtom + 32 * k),
                           sw128_desc(st + (2 + atom) * kRtAtom + 32 * k), idesc, (atom | k) != 0);
          umma_commit1(&empty[s]);  // the stage is free for the producer
          umma_commit1(&sfull[b]);  // the group's fp32 partials are in slot b
        }
        if (!ok) {
          s_fail = 1;
          break;
        }
      }
      umma_commit1(&done);  // every MMA completes before tensor memory is freed
      if (!mbar_wait(&done, 0)) s_fail = 1;
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRtRegEpi));
    // ---- epilogue warps 4..11: TMEM lane quarter (warp % 4) = tokens; expert
    // half (warp - 4) / 4 of the tile's 128 experts (64 columns)
    const int q4 = warp & 3, c_lo = 64 * ((warp - 4) >> 2);
    uint32_t it = 0;
    for (int wi = blockIdx.x; wi < nitems; wi += gridDim.x) {
      const int ti = wi / nsplit, kh = wi % nsplit;
      const int t0 = kRtM * (ti >> 1), e0 = kRtN * (ti & 1);
      double acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.0;
      bool ok = true;
      for (int G = 0; G < gper; ++G, ++it) {
        const int b = it & 1;
        if (!mbar_wait_sleep(&sfull[b], (it >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = tmem + (uint32_t)(128 * b + c_lo) + ((uint32_t)(32 * q4) << 16);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          tmem_ld32_async(base + 32u * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[32 * h + j] += (double)__uint_as_float(v[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[b]);
      }
      if (!ok) {
        s_fail = 1;
        break;
      }
      const int tok = t0 + 32 * q4 + lane;
      if (tok < T && nsplit == 1) {
        float4 *zr = reinterpret_cast<float4 *>(z + (size_t)tok * kE + e0 + c_lo);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          zr[j] = make_float4((float)acc[4 * j], (float)acc[4 * j + 1], (float)acc[4 * j + 2],
                              (float)acc[4 * j + 3]);
      } else if (tok < T) {
        double2 *zr = reinterpret_cast<double2 *>(zh + ((size_t)kh * T + tok) * kE + e0 + c_lo);
#pragma unroll
        for (int j = 0; j < 32; ++j) zr[j] = make_double2(acc[2 * j], acc[2 * j + 1]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (s_fail && tid == 0) set_status(status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
  }
}

// ============================================================== combine
__global__ void __launch_bounds__(256)
    k_pf_combine(const int32_t *__restrict__ pos, const uint16_t *__restrict__ yw,
                 const uint16_t *__restrict__ ys, int T, uint16_t *__restrict__ out,
                 uint32_t *__restrict__ status) {
  pdl_wait();  // the previous kernel in the stream is complete (programmatic launch)
  pdl_trigger();
  const size_t n = (size_t)T * (kH / 8);
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
    const size_t tok = i / (kH / 8), c = i % (kH / 8);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j <= kTopK; ++j) {
      const int p = j < kTopK ? pos[tok * kTopK + j] : 0;
      if (!FLINT_CHECK(j == kTopK || (unsigned)p < (unsigned)(6 * T), status)) continue;
      const uint16_t *src = j < kTopK ? yw + (size_t)p * kH : ys + tok * kH;
      const uint4 v = ld_cg_v4(src + 8 * c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] += __uint_as_float(w[k] << 16);
        acc[2 * k + 1] += __uint_as_float(w[k] & 0xffff0000u);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o[k] = (uint32_t)f32_to_bf16_bits(acc[2 * k]) | ((uint32_t)f32_to_bf16_bits(acc[2 * k + 1]) << 16);
    *reinterpret_cast<uint4 *>(out + tok * kH + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ============================================================== host
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

cudaError_t get_encode() {
  std::lock_guard<std::mutex> lock(g_encode_mu);
  if (g_encode) return cudaSuccess;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// 2-D tile map: rows x cols (inner), row pitch in bytes.
cudaError_t make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t cols,
                     uint64_t rows, uint64_t pitch, uint32_t box_cols, uint32_t box_rows,
                     CUtensorMapSwizzle sw) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t elem[2] = {1, 1};
  const CUresult r = g_encode(m, dt, 2, const_cast<void *>(base), dims, strides, box, elem,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Every prefill kernel is launched with programmatic stream serialization: its
// CTAs may be scheduled while the previous kernel drains, and each waits
// (griddepcontrol.wait, first thing) until that kernel is complete.
template <typename... KArgs, typename... Args>
cudaError_t pf_launch(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                      Args... args) {
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

// Clusters of two GEMM CTAs that can be resident at once on this device.
cudaError_t max_pairs(const void *fn, size_t smem, int *pairs) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
  if (e != cudaSuccess) return e;
  *pairs = n > 0 ? n : 1;
  return cudaSuccess;
}

// Stage timing for measurement (flint_debug_prefill_events): events recorded
// on the call's stream between the stages of flint_moe_prefill.
constexpr int kPfStages = 6;  // routing, sort, scaling + gather, GEMM 1, GEMM 2, combine
std::mutex g_ev_mu;
bool g_ev_on = false;
int g_ev_dev = -1;
cudaEvent_t g_ev[kPfStages + 1];

void stage_mark(int i, cudaStream_t st) {
  if (g_ev_on) cudaEventRecord(g_ev[i], st);
}

}  // namespace

cudaError_t prefill_set_stage_events(int enable) {
  std::lock_guard<std::mutex> lock(g_ev_mu);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (enable && g_ev_dev != dev) {
    if (g_ev_dev >= 0) return cudaErrorInvalidDevice;  // events live on the first device used
    for (int i = 0; i <= kPfStages; ++i)
      if ((e = cudaEventCreate(&g_ev[i])) != cudaSuccess) return e;
    g_ev_dev = dev;
  }
  g_ev_on = enable != 0;
  return cudaSuccess;
}

cudaError_t prefill_stage_times(float *ms, int n) {
  std::lock_guard<std::mutex> lock(g_ev_mu);
  if (g_ev_dev < 0 || n < kPfStages) return cudaErrorInvalidValue;
  cudaError_t e = cudaEventSynchronize(g_ev[kPfStages]);
  for (int i = 0; i < kPfStages && e == cudaSuccess; ++i)
    e = cudaEventElapsedTime(ms + i, g_ev[i], g_ev[i + 1]);
  return e;
}

// The two grouped GEMMs of a prefill call, for the experts' weight format
// (FLINT_FMT_*: symmetric int4 with bf16 scales, group-64 affine with fp16
// scales and offsets, or NVFP4): persistent, as many CTA pairs as fit at once (the tile counts are
// on the device).  Stage event 4 falls between them.
template <int kFmt>
cudaError_t launch_gemms(const PrefillLayout &P, const CUtensorMap &mA1r, const CUtensorMap &mA1s,
                         const CUtensorMap &mB1, const CUtensorMap &mA2r, const CUtensorMap &mA2s,
                         const CUtensorMap &mB2r, const CUtensorMap &mB2s, const GemmArgs &a1,
                         const GemmArgs &a2, cudaStream_t st) {
  cudaError_t e;
  note_step("prefill GEMM attributes");
  if ((e = cudaFuncSetAttribute(k_pf_gemm<1, kFmt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GemmCfg<1>::kSmem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_pf_gemm<2, kFmt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GemmCfg<2>::kSmem)) != cudaSuccess)
    return e;
  int pairs1 = 0, pairs2 = 0;
  if ((e = max_pairs(reinterpret_cast<const void *>(k_pf_gemm<1, kFmt>), GemmCfg<1>::kSmem,
                     &pairs1)) ||
      (e = max_pairs(reinterpret_cast<const void *>(k_pf_gemm<2, kFmt>), GemmCfg<2>::kSmem,
                     &pairs2)))
    return e;
  note_step("prefill GEMM 1 launch");
  e = pf_launch(k_pf_gemm<1, kFmt>, 2 * min(P.max_tiles1, pairs1), kGemmThreads, GemmCfg<1>::kSmem,
                st, mA1r, mA1s, mB1, mB1, a1);
  if (e != cudaSuccess) return e;
  stage_mark(4, st);
  note_step("prefill GEMM 2 launch");
  return pf_launch(k_pf_gemm<2, kFmt>, 2 * min(P.max_tiles2, pairs2), kGemmThreads,
                   GemmCfg<2>::kSmem, st, mA2r, mA2s, mB2r, mB2s, a2);
}

cudaError_t launch_route_many(const LayerArgs &L, const uint16_t *x, int T, int32_t *idx, float *w,
                              char *ws, cudaStream_t st) {
  const PrefillLayout P = prefill_layout(T);
  float *z = reinterpret_cast<float *>(ws + P.z);
  cudaError_t e = noted(get_encode(), "cuTensorMapEncodeTiled entry point");
  if (e != cudaSuccess) return e;
  note_step("prefill router tensor maps");
  CUtensorMap mX, mW;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((e = make_map(&mX, x, BF, kH, (uint64_t)T, kH * 2, 64, kRtM, CU_TENSOR_MAP_SWIZZLE_128B)) ||
      (e = make_map(&mW, L.router_w, BF, kH, kE, kH * 2, 64, kRtN, CU_TENSOR_MAP_SWIZZLE_128B)))
    return e;
  note_step("prefill router attribute");
  if ((e = cudaFuncSetAttribute(k_pf_router_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kRtSmem)) != cudaSuccess)
    return e;
  note_step("prefill router launch");
  const int nsplit = route_split(T);
  double *zh = nsplit > 1 ? reinterpret_cast<double *>(ws + P.z) : nullptr;
  {
    const int nitems = 2 * ((T + kRtM - 1) / kRtM) * nsplit;
    e = pf_launch(k_pf_router_tc, nitems < 148 ? nitems : 148, kRtThreads, kRtSmem, st, mX, mW, T,
                  nsplit, z, zh, reinterpret_cast<uint32_t *>(ws + P.ctrl) + 1);
  }
  if (e != cudaSuccess) return e;
  note_step("prefill top-6 launch");
  return pf_launch(k_pf_topk, (T + 7) / 8, 256, 0, st, L.router_b, (const float *)z,
                   (const double *)zh, T, idx, w,
                   reinterpret_cast<int32_t *>(ws + P.asc_e), reinterpret_cast<float *>(ws + P.asc_w));
}

cudaError_t launch_prefill(const LayerArgs &L, const uint16_t *x, int T, uint16_t *out, char *ws,
                           cudaStream_t st) {
  const PrefillLayout P = prefill_layout(T);
  cudaError_t e = noted(get_encode(), "cuTensorMapEncodeTiled entry point");
  if (e != cudaSuccess) return e;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + P.ctrl);
  int32_t *asc_e = reinterpret_cast<int32_t *>(ws + P.asc_e);
  float *asc_w = reinterpret_cast<float *>(ws + P.asc_w);
  int32_t *pos = reinterpret_cast<int32_t *>(ws + P.pos);
  int32_t *cc = reinterpret_cast<int32_t *>(ws + P.chunk_cnt);
  int32_t *co = reinterpret_cast<int32_t *>(ws + P.chunk_off);
  int32_t *ebase = reinterpret_cast<int32_t *>(ws + P.ebase);
  int32_t *ecount = reinterpret_cast<int32_t *>(ws + P.ecount);
  uint2 *tiles1 = reinterpret_cast<uint2 *>(ws + P.tiles1);
  uint2 *tiles2 = reinterpret_cast<uint2 *>(ws + P.tiles2);
  float4 *wst = reinterpret_cast<float4 *>(ws + P.wst);
  float *wbound = reinterpret_cast<float *>(ws + P.wbound);
  uint32_t *rsc = reinterpret_cast<uint32_t *>(ws + P.rsc);
  float *rm3 = reinterpret_cast<float *>(ws + P.rm3);
  uint16_t *xp = reinterpret_cast<uint16_t *>(ws + P.xp);
  uint16_t *hr = reinterpret_cast<uint16_t *>(ws + P.hr);
  uint16_t *hs = reinterpret_cast<uint16_t *>(ws + P.hs);
  uint16_t *yw = reinterpret_cast<uint16_t *>(ws + P.yw);
  uint16_t *ys = reinterpret_cast<uint16_t *>(ws + P.ys);

  // 1. routing
  stage_mark(0, st);
  e = launch_route_many(L, x, T, reinterpret_cast<int32_t *>(ws + P.sel_idx),
                        reinterpret_cast<float *>(ws + P.sel_w), ws, st);
  if (e != cudaSuccess) return e;
  stage_mark(1, st);
  // 2. stable sort by expert
  note_step("prefill sort launches");
  if ((e = pf_launch(k_pf_count, P.nchunks, 256, 0, st, asc_e, T, cc, ctrl + 1)) ||
      (e = pf_launch(k_pf_scan, 1, 256, 0, st, T, P.nchunks, cc, co, ebase, ecount, tiles1, tiles2,
                     ctrl)) ||
      (e = pf_launch(k_pf_place, P.nchunks, 256, 0, st, asc_e, T, co, ebase, pos, ctrl + 1)))
    return e;
  stage_mark(2, st);
  // 3. power-of-two shifts of the fp16 operands, and the fp16 token rows
  note_step("prefill operand scaling launches");
  const int fmt = L.fmt;
  float4 *wsg = reinterpret_cast<float4 *>(ws + P.wsg);
  if (fmt == FLINT_FMT_AFFINE_INT4)
    e = pf_launch(k_pf_wstats_aff, kE + 1, 256, 0, st, L.w13_s, L.w13_m, L.w2_s, L.w2_m, L.sh13_s,
                  L.sh13_m, L.sh2_s, L.sh2_m, L.interm_div, wst, wbound);
  else if (fmt == FLINT_FMT_NVFP4)
    e = pf_launch(k_pf_wstats_nv, kE + 1, 256, 0, st, reinterpret_cast<const uint8_t *>(L.w13_s),
                  L.w13_g, L.w2_g, reinterpret_cast<const uint8_t *>(L.sh13_s), L.sh13_g, L.sh2_g,
                  L.interm_div, wst, wsg, wbound);
  else
    e = pf_launch(k_pf_wstats, kE + 1, 256, 0, st, L.w13_s, L.w2_s, L.sh13_s, L.sh2_s,
                  L.interm_div, wst, wbound);
  if (e) return e;
  {
    int blocks = (T + 7) / 8;  // 8 tokens (warps) per block
    if (blocks > 148 * 8) blocks = 148 * 8;
    if ((e = pf_launch(k_pf_gather, blocks, 256, 0, st, x, T, pos, asc_w, wbound, xp, rsc, rm3,
                       ctrl + 1)))
      return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  stage_mark(3, st);
  // 4. tensor maps and the two grouped GEMMs
  CUtensorMap mA1r, mA1s, mB1, mA2r, mA2s, mB2r, mB2s;
  note_step("prefill tensor maps");
  const auto F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16, U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  // code boxes of 64-byte rows, 64-byte swizzled: the dequant warps' row reads
  // (8 consecutive rows per 16-byte load phase) hit every bank once
  const auto SW64 = CU_TENSOR_MAP_SWIZZLE_64B;
  if ((e = make_map(&mA1r, L.w13_q, U8, kH / 2, (uint64_t)kE * 2 * kI, kH / 2, 64, 64, SW64)) ||
      (e = make_map(&mA1s, L.sh13_q, U8, kH / 2, 2 * kIs, kH / 2, 64, 64, SW64)) ||
      (e = make_map(&mB1, xp, F16, kH, (uint64_t)7 * T, kH * 2, 64, GemmCfg<1>::kBRows, SW)) ||
      (e = make_map(&mA2r, L.w2_q, U8, kI / 2, (uint64_t)kE * kH, kI / 2, 64, 128, SW64)) ||
      (e = make_map(&mA2s, L.sh2_q, U8, kIs / 2, kH, kIs / 2, 64, 128, SW64)) ||
      (e = make_map(&mB2r, hr, F16, kI, (uint64_t)P.mr, kI * 2, 64, GemmCfg<2>::kBRows, SW)) ||
      (e = make_map(&mB2s, hs, F16, kIs, (uint64_t)T, kIs * 2, 64, GemmCfg<2>::kBRows, SW)))
    return e;
  // (NVFP4: the routed up rows' divisor is in the up global scale, not the weights)
  const float up_mul = fmt == FLINT_FMT_NVFP4 ? 1.f : L.interm_div;
  GemmArgs a1{tiles1, ctrl, 3,   ebase, ecount,   T,   L.w13_s, L.sh13_s, L.w13_m,
              L.sh13_m, wst, wsg, rsc, rm3, hr,     hs, ctrl + 1, up_mul};
  GemmArgs a2{tiles2, ctrl, 4,   ebase, ecount,   T,   L.w2_s, L.sh2_s, L.w2_m,
              L.sh2_m, wst, wsg, rsc, rm3, yw,     ys, ctrl + 1, 1.f};
  if (fmt == FLINT_FMT_AFFINE_INT4)
    e = launch_gemms<FLINT_FMT_AFFINE_INT4>(P, mA1r, mA1s, mB1, mA2r, mA2s, mB2r, mB2s, a1, a2, st);
  else if (fmt == FLINT_FMT_NVFP4)
    e = launch_gemms<FLINT_FMT_NVFP4>(P, mA1r, mA1s, mB1, mA2r, mA2s, mB2r, mB2s, a1, a2, st);
  else
    e = launch_gemms<FLINT_FMT_SYM_INT4>(P, mA1r, mA1s, mB1, mA2r, mA2s, mB2r, mB2s, a1, a2, st);
  if (e != cudaSuccess) return e;
  stage_mark(5, st);
  // 5. combine
  note_step("prefill combine launch");
  {
    int blocks = (int)(((size_t)T * (kH / 8) + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if ((e = pf_launch(k_pf_combine, blocks, 256, 0, st, pos, yw, ys, T, out, ctrl + 1)))
      return e;
  }
  stage_mark(6, st);
  return cudaGetLastError();
}

}  // namespace flint
