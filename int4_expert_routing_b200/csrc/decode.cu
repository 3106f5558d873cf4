// Decode step of the Flint MoE block: three kernels chained with programmatic
// dependent launch (PDL).  Each kernel issues every load that does not depend
// on its predecessor before it waits on it.
//
//   K1  router: bf16 W_r against the input, one 128-wide k-group per warp on
//       mma.sync, group partials summed in fp64 in a fixed order; the last
//       CTA to finish takes sigmoid (fp32), adds the bias, picks the top 6
//       (lower index wins ties), normalizes the weights and builds the slot
//       table (the union of chosen experts, ascending).
//   K2  gate/up int4 GEMV + SwiGLU.  Shared-expert items need no routing and
//       run before the PDL wait, overlapping K1; routed items run after it,
//       for every slot, scaled by the routing weight of each row that chose
//       the expert, and leave the fp32 intermediate as a hi/lo bf16 pair image
//       shaped for K3's tensor-core fragments.
//   K3  down projection of every slot and of the shared expert: the weights
//       are bulk-copied into shared memory before the PDL wait; after it the
//       intermediates are staged in one round trip and each row is combined
//       in a fixed order (its experts in ascending index, then the shared
//       expert).
//
// Model structure: "How to Run Flint Locally", section "The architecture,
// from config.json" (256 routed experts, 6 per token, expert size 512,
// sigmoid router with normalized top-k, shared expert of size 1,024 for every
// token); TandemLLM "21 Flint" section 21.1 (routing by sigmoid score with a
// bias) and section 21.2 (routed SwiGLU activations reach 2.6e5, past fp16:
// intermediates stay fp32).  The kernel structure follows the low-latency
// decode path under "What vLLM changed" (routing and combine folded into the
// neighbouring GEMVs, every kernel a programmatic dependent that loads its
// weights while the previous one runs) and TandemLLM section 21.4 (the
// shared expert overlapped with the routed path, same bits either way).
//
// Batch invariance: every output element of row b is computed by the same
// lanes, in the same order, from row b's data alone, whatever B is; the
// combine walks row b's own experts.
#include "common.cuh"
#include "internal.h"

namespace flint {

// Optional timeline trace (build with -DFLINT_TRACE): thread 0 of every CTA
// records %globaltimer at marked points, read back with flint_trace_dump.
#ifdef FLINT_TRACE
constexpr unsigned kTraceCap = 1u << 18;
static __device__ unsigned long long g_trace_time[kTraceCap];
static __device__ unsigned int g_trace_tag[kTraceCap];
static __device__ unsigned int g_trace_n;
// Event 0 (kernel start) reserves the CTA's 16 records with one atomic,
// before any wait; later events are plain stores.
FLINT_DEV void trace_point(uint32_t kernel, uint32_t event, uint32_t dep = 0) {
  __shared__ unsigned s_base;
  if (threadIdx.x == 0) {
    unsigned long long t;  // dep: a value the mark must wait for
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t) : "r"(dep));
    if (event == 0) s_base = atomicAdd(&g_trace_n, 16u);
    const unsigned i = s_base + event;
    if (i < kTraceCap) {
      g_trace_time[i] = t;
      g_trace_tag[i] = (kernel << 28) | (event << 24) | blockIdx.x;
    }
  }
}
#else
FLINT_DEV void trace_point(uint32_t, uint32_t, uint32_t = 0) {}
#endif

// Poll bound of the decode kernels' first wait on each barrier (the copies a
// CTA issued).  flint_debug_set_wait_polls lowers it so that a test can drive
// the timeout path; every wait on an error path uses the fixed kWaitPolls,
// so copies still in flight land before the CTA exits.
static __device__ uint32_t g_decode_polls = kWaitPolls;
FLINT_DEV bool dwait(uint64_t *bar, uint32_t parity) {
  const uint32_t n = *reinterpret_cast<volatile uint32_t *>(&g_decode_polls);
  for (uint32_t i = 0; i < n; ++i)
    if (mbar_try(bar, parity)) return true;
  return false;
}

constexpr int kRouterCtas = 32;   // 16 expert tiles x 2 k-halves
constexpr int kK1Threads = 256;   // 8 warps: one 128-wide k-group each
static_assert(kK1Threads == kE, "the last router CTA scores one expert per thread");
constexpr int kK3Threads = 512;
constexpr int kXFragBytes = 16 * 128 * 16;  // 16 groups x 128 uint4
// Router rows sit 2064 B apart in shared memory (16 B of padding) so that the
// eight rows a fragment load touches fall in different banks.
constexpr int kRouterRowStride = 2048 + 16;

FLINT_DEV float silu_f(float v) { return v / (1.f + expf(-v)); }

FLINT_DEV void write_hilo(uint16_t *img_hi, uint16_t *img_lo, int k, float v) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
  const int s = frag_slot(k);
  img_hi[s] = __bfloat16_as_ushort(hi);
  img_lo[s] = __bfloat16_as_ushort(lo);
}

// ---------------------------------------------------------------- input
// RMSNorm scale 1/sqrt(mean(h^2) + eps) per row, fp64, in one fixed order
// whatever the block size: 128 "lanes" t each sum the squares of elements
// t, t+128, ..., t+1920 in that order, then an xor tree inside each warp of
// 32 consecutive t, then the four warps in order.  Every K1 CTA runs the
// same code on the same row, so all of them normalize to the same bits.
//
// The normalized row, rounded to bf16 (fp64 product, one rounding), goes
// straight into the compact mma fragment: for element k of row b the slot is
// 8 * ((G * 4B + 4b + tt) * 4 + q) + 2 * (e & 3) + (e >> 2) with G = k/128,
// tt = k/32 mod 4, q = k/8 mod 4, e = k mod 8 (the pair order that
// bf16x8_to_pairs produces).  Other lanes of the fragment read zeros.
FLINT_DEV int compact_slot(int b, int k, int B) {
  const int G = k >> 7, tt = (k >> 5) & 3, q = (k >> 3) & 3, e = k & 7;
  return 8 * ((G * 4 * B + 4 * b + tt) * 4 + q) + 2 * (e & 3) + (e >> 2);
}

// All kThreads threads; rows are taken kThreads/128 at a time, each thread
// holding up to kRowsPerPass rows' 16 elements in registers so that every
// load of a pass is in flight at once.  The scale needs the whole row; only
// k-groups g_lo .. g_lo+7 are converted into the fragment.
template <int kThreads, int kRowsPerPass, int kTraceK = 0>
FLINT_DEV void rms_stage(const float *h, int B, int g_lo, double *s_red /*[4 * kMaxB]*/,
                         double *s_inv, uint16_t *frag16, int tid) {
  constexpr int kPar = kThreads / 128;
  const int t = tid & 127, hv = tid >> 7, lane = tid & 31, tw = t >> 5;
  for (int p0 = 0; p0 < B; p0 += kPar * kRowsPerPass) {
    float v[kRowsPerPass][16];
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) {
      const int b = p0 + hv + kPar * r;
      if (b < B) {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[r][j] = __ldcg(h + (size_t)b * kH + t + 128 * j);
      }
    }
    if (kTraceK && p0 == 0) trace_point(kTraceK, 13, __float_as_uint(v[0][15]));
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) {
      const int b = p0 + hv + kPar * r;
      if (b < B) {  // the same b for all lanes of a warp
        double ss = 0.0;
#pragma unroll
        for (int j = 0; j < 16; ++j) ss = fma((double)v[r][j], (double)v[r][j], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) s_red[tw * kMaxB + b] = ss;
      }
    }
    __syncthreads();
    if (tid < B && tid >= p0 && tid < p0 + kPar * kRowsPerPass) {
      double ss = 0.0;
      for (int w = 0; w < 4; ++w) ss += s_red[w * kMaxB + tid];
      s_inv[tid] = 1.0 / sqrt(ss / kH + FLINT_RMS_EPS);
    }
    __syncthreads();
    if (kTraceK && p0 == 0) trace_point(kTraceK, 14);
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) {
      const int b = p0 + hv + kPar * r;
      if (b < B) {
        const double sc = s_inv[b];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if ((unsigned)(j - g_lo) < 8u)
            frag16[compact_slot(b, t + 128 * j, B)] =
                (uint16_t)f64_to_bf16_bits((double)v[r][j] * sc);
      }
    }
  }
  __syncthreads();
}

// Compact fragment of a bf16 input (plain decode), k-groups g_lo .. g_lo+7:
// frag[(G * 4B + 4g + t) * 4 + q].
FLINT_DEV void stage_x_compact(uint4 *frag, const uint16_t *x_in, int B, int g_lo, int tid,
                               int nthreads) {
  const int n = 8 * 4 * B * 4, base = g_lo * 4 * B * 4;
  for (int i = tid; i < n; i += nthreads) {
    const int task = base + i;
    const int q = task & 3, gt = (task >> 2) % (4 * B), G = (task >> 2) / (4 * B);
    const int gg = gt >> 2, tt = gt & 3;
    frag[task] = bf16x8_to_pairs(ld_cg_v4(x_in + (size_t)gg * kH + 128 * G + 32 * tt + 8 * q));
  }
  __syncthreads();
}

template <bool kResidual, int kThreads, int kRowsPerPass, int kTraceK = 0>
FLINT_DEV void stage_input(uint4 *frag, const uint16_t *x_in, const float *h, int B, int g_lo,
                           double *s_red, double *s_inv, int tid) {
  if (kResidual)
    rms_stage<kThreads, kRowsPerPass, kTraceK>(h, B, g_lo, s_red, s_inv,
                                               reinterpret_cast<uint16_t *>(frag), tid);
  else
    stage_x_compact(frag, x_in, B, g_lo, tid, kThreads);
}

FLINT_DEV void load_frag_compact(const uint4 *frag, int G, int B, int lane, uint32_t (&x)[16]) {
  const int g = lane >> 2, t = lane & 3;
  if (g < B) {
    const uint4 *p = frag + (size_t)(G * 4 * B + g * 4 + t) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = p[i];
      x[4 * i] = v.x, x[4 * i + 1] = v.y, x[4 * i + 2] = v.z, x[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = 0u;
  }
}

// ============================================================== K1: router
constexpr uint32_t kSlotInvalid = 0xffffffffu;
FLINT_DEV uint32_t slot_expert(uint32_t w) { return w & 0xffu; }
FLINT_DEV uint32_t slot_mask(uint32_t w) { return (w >> 8) & 0xffu; }
FLINT_DEV int slot_count(uint32_t w) { return (int)((w >> 16) & 0x1ffu); }
// Index of the i-th set bit (i from 0) of m; m has more than i bits set.
FLINT_DEV int nth_bit(uint32_t m, int i) {
  for (int r = 0; r < i; ++r) m &= m - 1u;
  return __ffs(m) - 1;
}

// Release-publish this CTA's results and tell whether it is the last of
// `nctas` to do so; one fence per CTA on each side of the counter.
FLINT_DEV bool last_cta(uint32_t *counter, uint32_t nctas, int *s_flag) {
  __syncthreads();  // the CTA's writes happen before thread 0's release
  if (threadIdx.x == 0) {
    uint32_t prev;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
    *s_flag = prev == nctas - 1;
  }
  __syncthreads();  // ... and the acquire happens before the CTA's reads
  return *s_flag != 0;
}

template <bool kResidual>
__global__ void __launch_bounds__(kK1Threads)
    k1_router(LayerArgs L, const uint16_t *__restrict__ x_in, const float *__restrict__ h, int B,
              char *__restrict__ ws, DecodeLayout lay, int32_t *__restrict__ idx_out,
              float *__restrict__ w_out, int e_lo, int e_hi) {
  extern __shared__ __align__(128) unsigned char sm[];  // [16 rows][2064 B] | compact x fragment
  uint4 *frag = reinterpret_cast<uint4 *>(sm + 16 * kRouterRowStride);
  __shared__ __align__(8) uint64_t bar;
  __shared__ double s_part[8][kMaxB][16];
  __shared__ double s_red[4 * kMaxB];
  __shared__ double s_inv[kMaxB];
  __shared__ int s_last;
  __shared__ int s_asc_e[kMaxB][kTopK];
  __shared__ float s_asc_w[kMaxB][kTopK];
  __shared__ int s_slot_of[kE];
  __shared__ int s_slot_e[kE];
  __shared__ uint32_t s_slot_m[kE];
  __shared__ int s_wcount[8];
  __shared__ __align__(16) uint32_t s_key[kMaxB][kE];  // selection keys, one row per warp
  __shared__ float s_sv[kMaxB][kE];
  __shared__ int s_sel_e[kMaxB][kTopK];
  __shared__ float s_sel_s[kMaxB][kTopK];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + lay.ctrl);
  const int et = blockIdx.x >> 1, kh = blockIdx.x & 1;
  trace_point(1, 0);

  // this CTA's router block: 16 experts x one k-half (2 KB per row), fetched
  // before the wait (the weights do not depend on the previous kernel)
  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_expect_tx(&bar, 16 * 2048);
  }
  __syncthreads();
  if (tid < 16)
    bulk_g2s(sm + tid * kRouterRowStride, L.router_w + (size_t)(16 * et + tid) * kH + kh * (kH / 2), 2048, &bar);
  // selection bias of expert tid for the last CTA's top-6, also a weight
  const float bias = __ldg(L.router_b + tid);
  pdl_wait();
  pdl_trigger();
  trace_point(1, 1);

  stage_input<kResidual, kK1Threads, 4, 1>(frag, x_in, h, B, 8 * kh, s_red, s_inv, tid);
  trace_point(1, 4);
  {  // publish this k-half of the fragment (the 16 CTAs of the half a share each)
    const int per = 8 * B;  // uint4: the half is 128 B uint4, split 16 ways
    const int i = (8 * kh) * 4 * B * 4 + et * per + tid;
    if (tid < per) reinterpret_cast<uint4 *>(ws + lay.xfrag)[i] = frag[i];
  }
  const bool ok = dwait(&bar, 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
    if (!ok) mbar_wait(&bar, 0);  // the router rows still in flight land first
    return;
  }
  trace_point(1, 5);
  {
    uint32_t ra[16], rb[16], xb[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 a = bf16x8_to_pairs(
          *reinterpret_cast<const uint4 *>(sm + g * kRouterRowStride + 256 * warp + 64 * t + 16 * q));
      const uint4 c = bf16x8_to_pairs(
          *reinterpret_cast<const uint4 *>(sm + (g + 8) * kRouterRowStride + 256 * warp + 64 * t + 16 * q));
      ra[4 * q] = a.x, ra[4 * q + 1] = a.y, ra[4 * q + 2] = a.z, ra[4 * q + 3] = a.w;
      rb[4 * q] = c.x, rb[4 * q + 1] = c.y, rb[4 * q + 2] = c.z, rb[4 * q + 3] = c.w;
    }
    load_frag_compact(frag, 8 * kh + warp, B, lane, xb);
    float d[4];
    group_mma(ra, rb, xb, d);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int b = 2 * t + c;
      if (b < B) {
        s_part[warp][b][g] = (double)d[c];
        s_part[warp][b][g + 8] = (double)d[2 + c];
      }
    }
  }
  __syncthreads();
  double *zp = reinterpret_cast<double *>(ws + lay.zpart);
  if (tid < B * 16) {
    const int b = tid >> 4, r = tid & 15;
    double p = 0.0;
    for (int w = 0; w < 8; ++w) p += s_part[w][b][r];
    zp[((size_t)kh * B + b) * kE + 16 * et + r] = p;
  }
  trace_point(1, 2);
  if (!last_cta(&ctrl[0], kRouterCtas, &s_last)) return;
  trace_point(1, 6);

  // ---- last CTA: scores, top-6, weights, slot table.  Thread e scores
  // expert e of every row into shared memory; warp b then picks row b's 6
  // best in 6 rounds, lane l holding experts 8l .. 8l+7: the lane's best live
  // key (ties to the lower expert), the warp's largest key, the lowest lane
  // holding it (= the lowest expert).  Rounds 0..5 give the selection order.
  int32_t *sel_idx = reinterpret_cast<int32_t *>(ws + lay.sel_idx);
  float *sel_w = reinterpret_cast<float *>(ws + lay.sel_w);
  {
    double zz[kMaxB];
#pragma unroll
    for (int b = 0; b < kMaxB; ++b)
      if (b < B) zz[b] = ld_cg_f64(zp + (size_t)b * kE + tid) + ld_cg_f64(zp + ((size_t)B + b) * kE + tid);
#pragma unroll
    for (int b = 0; b < kMaxB; ++b) {
      if (b < B) {
        const float sv = 1.f / (1.f + expf(-(float)zz[b]));
        s_key[b][tid] = float_key(sv + bias);
        s_sv[b][tid] = sv;
      }
    }
  }
  trace_point(1, 10);
  __syncthreads();
  if (warp < B) {
    const int b = warp;
    const uint4 ka = *reinterpret_cast<const uint4 *>(&s_key[b][8 * lane]);
    const uint4 kb = *reinterpret_cast<const uint4 *>(&s_key[b][8 * lane + 4]);
    const uint32_t key[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
    uint32_t live = 0xffu;
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
      uint32_t best = 0;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (((live >> i) & 1u) && key[i] > best) best = key[i], bi = i;
      const uint32_t m = __reduce_max_sync(0xffffffffu, best);
      const uint32_t win = __ballot_sync(0xffffffffu, live != 0u && best == m);
      if (lane == __ffs(win) - 1) {
        live &= ~(1u << bi);
        s_sel_e[b][j] = 8 * lane + bi;
        s_sel_s[b][j] = s_sv[b][8 * lane + bi];
      }
    }
    __syncwarp();
    trace_point(1, 11);
    if (lane < kTopK) {
      float ssum = 0.f;
#pragma unroll
      for (int j = 0; j < kTopK; ++j) ssum += s_sel_s[b][j];
      const int e_me = s_sel_e[b][lane];
      const float w_me = s_sel_s[b][lane] / ssum;
      sel_idx[b * kTopK + lane] = e_me;
      sel_w[b * kTopK + lane] = w_me;
      if (idx_out) idx_out[b * kTopK + lane] = e_me;
      if (w_out) w_out[b * kTopK + lane] = w_me;
      int rank = 0;  // ascending expert order
#pragma unroll
      for (int j = 0; j < kTopK; ++j) rank += s_sel_e[b][j] < e_me;
      s_asc_e[b][rank] = e_me;
      s_asc_w[b][rank] = w_me;
    }
  }
  __syncthreads();
  trace_point(1, 7);
  // slot table: experts of this call's range [e_lo, e_hi) used by any row,
  // ascending; one expert per thread (an expert without a slot maps to -1)
  const int e = tid;
  uint32_t m = 0;
  s_slot_of[e] = -1;
  if (e >= e_lo && e < e_hi)
    for (int b = 0; b < B; ++b)
      for (int j = 0; j < kTopK; ++j)
        if (s_asc_e[b][j] == e) m |= 1u << b;
  const uint32_t bal = __ballot_sync(0xffffffffu, m != 0);
  if (lane == 0) s_wcount[warp] = __popc(bal);
  __syncthreads();
  int off = 0, total = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) off += s_wcount[w];
    total += s_wcount[w];
  }
  if (m) {
    const int slot = off + __popc(bal & ((1u << lane) - 1u));
    s_slot_of[e] = slot;
    s_slot_e[slot] = e;
    s_slot_m[slot] = m;
  }
  __syncthreads();
  uint32_t *slot_word = reinterpret_cast<uint32_t *>(ws + lay.slot_word);
  slot_word[tid] = tid < total ? ((uint32_t)s_slot_e[tid] | (s_slot_m[tid] << 8) | ((uint32_t)total << 16))
                               : kSlotInvalid;
  int32_t *asc_slot = reinterpret_cast<int32_t *>(ws + lay.asc_slot);
  float *asc_w = reinterpret_cast<float *>(ws + lay.asc_w);
  if (tid < B * kTopK) {
    const int b = tid / kTopK, j = tid % kTopK;
    asc_slot[tid] = s_slot_of[s_asc_e[b][j]];
    asc_w[tid] = s_asc_w[b][j];
  }
  trace_point(1, 12);
  if (tid == 0) {
    ctrl[2] = (uint32_t)total;
    ctrl[0] = 0;  // ready for the next call on this workspace
  }
  trace_point(1, 3);
}

// ============================================================== K2: gate/up + SwiGLU
// One CTA per work item: 8 intermediate rows of one expert (shared expert:
// items 0..127; routed: item 128 + 64u + r/8 for slot u).  The item's bytes
// (8 gate rows, 8 up rows, their scales; 16.5 KB) arrive in shared memory by
// four bulk copies (the shared expert's before the wait on K1), the block
// input fragment K1 published by one more after it; the warps split the 16
// k-groups and their partial sums are added in warp order.
#ifndef FLINT_K2_WARPS
#define FLINT_K2_WARPS 4
#endif
constexpr int kK2Warps = FLINT_K2_WARPS;
constexpr int kK2Groups = 16 / kK2Warps;  // k-groups per warp
static_assert(kK2Warps * kK2Groups == 16, "the warps split the 16 k-groups evenly");
constexpr int kItemBytes = 16384 + 512;      // codes, bf16 scales per 128
constexpr int kItemBytesAff = 16384 + 2048;  // codes, fp16 scales and offsets per 64
                                             // (NVFP4: E4M3 scales per 16, the same size)
constexpr int kSharedItems = kIs / 8;
// expert formats (FLINT_FMT_*): symmetric int4, group-64 affine int4, NVFP4
constexpr int kFmtSym = 0, kFmtAff = 1, kFmtNv = 2;
template <int kFmt>
constexpr int item_bytes() {
  return kFmt == kFmtSym ? kItemBytes : kItemBytesAff;
}

struct ItemSrc {
  const uint8_t *gate;
  const uint8_t *up;
  const uint16_t *gate_s;
  const uint16_t *up_s;
  const uint16_t *gate_m;  // affine offsets
  const uint16_t *up_m;
};

// scale (and offset) words of 16 bits per gate/up row: 16 scales of 128, 32
// of 64, or (NVFP4) the 128 E4M3 bytes of the blocks of 16 as 64 words
template <int kFmt>
constexpr int item_groups() {
  return kFmt == kFmtAff ? kH / 64 : (kFmt == kFmtNv ? kH / 32 : kH / kG);
}
template <int kFmt>
FLINT_DEV ItemSrc shared_item(const LayerArgs &L, int it) {
  constexpr bool kAff = kFmt == kFmtAff;
  const int r = 8 * it;
  constexpr int gpr = item_groups<kFmt>();
  return ItemSrc{L.sh13_q + (size_t)r * (kH / 2), L.sh13_q + (size_t)(kIs + r) * (kH / 2),
                 L.sh13_s + (size_t)r * gpr, L.sh13_s + (size_t)(kIs + r) * gpr,
                 kAff ? L.sh13_m + (size_t)r * gpr : nullptr,
                 kAff ? L.sh13_m + (size_t)(kIs + r) * gpr : nullptr};
}
template <int kFmt>
FLINT_DEV ItemSrc routed_item(const LayerArgs &L, int e, int r0) {
  constexpr bool kAff = kFmt == kFmtAff;
  const size_t row = (size_t)e * (2 * kI) + r0;
  constexpr int gpr = item_groups<kFmt>();
  return ItemSrc{L.w13_q + row * (kH / 2), L.w13_q + (row + kI) * (kH / 2),
                 L.w13_s + row * gpr, L.w13_s + (row + kI) * gpr,
                 kAff ? L.w13_m + row * gpr : nullptr, kAff ? L.w13_m + (row + kI) * gpr : nullptr};
}
// one thread; the caller accounts the bytes on the barrier (mbar_add_tx).
// Item layout: gate codes, up codes (8 rows x 1 KB each), then the gate and
// up rows' scales (8 rows x groups) and, affine, their offsets.
template <int kFmt>
FLINT_DEV void issue_item(const ItemSrc &src, unsigned char *buf, uint64_t *bar) {
  constexpr uint32_t sb = 8 * item_groups<kFmt>() * 2;  // 256, 512 or 1,024 bytes
  bulk_g2s(buf, src.gate, 8192, bar);
  bulk_g2s(buf + 8192, src.up, 8192, bar);
  bulk_g2s(buf + 16384, src.gate_s, sb, bar);
  bulk_g2s(buf + 16384 + sb, src.up_s, sb, bar);
  if (kFmt == kFmtAff) {
    bulk_g2s(buf + 16384 + 2 * sb, src.gate_m, sb, bar);
    bulk_g2s(buf + 16384 + 3 * sb, src.up_m, sb, bar);
  }
}

// This warp's k-groups of the item: acc[0..1] gate, [2..3] up partials for
// columns 2t, 2t+1 of row r0 + g.
FLINT_DEV void item_part(const unsigned char *buf, const uint4 *frag, int B, int warp, int lane,
                         float (&acc)[4]) {
  const int g = lane >> 2, t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  const uint16_t *sg = reinterpret_cast<const uint16_t *>(buf + 16384 + g * 32);
  const uint16_t *su = reinterpret_cast<const uint16_t *>(buf + 16640 + g * 32);
#pragma unroll
  for (int k = 0; k < kK2Groups; ++k) {
    const int G = kK2Groups * warp + k;
    const uint4 wg = *reinterpret_cast<const uint4 *>(buf + g * 1024 + 64 * G + 16 * t);
    const uint4 wu = *reinterpret_cast<const uint4 *>(buf + 8192 + g * 1024 + 64 * G + 16 * t);
    uint32_t ra[16], rb[16], xb[16];
    int4x32_to_bf16x2(wg, ra);
    int4x32_to_bf16x2(wu, rb);
    load_frag_compact(frag, G, B, lane, xb);
    float d[4];
    group_mma(ra, rb, xb, d);
    const float sgf = bf16_bits_to_f32(sg[G]), suf = bf16_bits_to_f32(su[G]);
    acc[0] = fmaf(d[0], sgf, acc[0]);
    acc[1] = fmaf(d[1], sgf, acc[1]);
    acc[2] = fmaf(d[2], suf, acc[2]);
    acc[3] = fmaf(d[3], suf, acc[3]);
  }
}

// The affine item: lane t's 32 elements of a 128-group lie in its 64-group
// 2G (t < 2) or 2G + 1 (t >= 2).  Two MMAs per group on the same codes, each
// with the other half's activation lanes zeroed, give the two 64-groups'
// exact sums dA, dB; then y += s_A dA + m_A sum(x over 2G) + s_B dB + m_B
// sum(x over 2G+1) per row (xs: [32 groups][kMaxB] sums of the block input).
FLINT_DEV void item_part_aff(const unsigned char *buf, const uint4 *frag, const float *xs, int B,
                             int warp, int lane, float (&acc)[4]) {
  const int g = lane >> 2, t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  const uint16_t *sg = reinterpret_cast<const uint16_t *>(buf + 16384 + g * 64);
  const uint16_t *su = reinterpret_cast<const uint16_t *>(buf + 16384 + 512 + g * 64);
  const uint16_t *mg = reinterpret_cast<const uint16_t *>(buf + 16384 + 1024 + g * 64);
  const uint16_t *mu = reinterpret_cast<const uint16_t *>(buf + 16384 + 1536 + g * 64);
  const uint32_t mA = t < 2 ? 0xffffffffu : 0u, mB = ~mA;
  const int c0 = 2 * t, c1 = 2 * t + 1;
  auto h2f = [](uint16_t v) { return __half2float(__ushort_as_half(v)); };
#pragma unroll
  for (int k = 0; k < kK2Groups; ++k) {
    const int G = kK2Groups * warp + k, gA = 2 * G, gB = 2 * G + 1;
    const uint4 wg = *reinterpret_cast<const uint4 *>(buf + g * 1024 + 64 * G + 16 * t);
    const uint4 wu = *reinterpret_cast<const uint4 *>(buf + 8192 + g * 1024 + 64 * G + 16 * t);
    uint32_t ra[16], rb[16], xb[16], xa[16], xo[16];
    uint4x32_to_bf16x2(wg, ra);
    uint4x32_to_bf16x2(wu, rb);
    load_frag_compact(frag, G, B, lane, xb);
#pragma unroll
    for (int i = 0; i < 16; ++i) xa[i] = xb[i] & mA, xo[i] = xb[i] & mB;
    float dA[4], dB[4];
    group_mma(ra, rb, xa, dA);
    group_mma(ra, rb, xo, dB);
    const float xa0 = c0 < B ? xs[gA * kMaxB + c0] : 0.f, xa1 = c1 < B ? xs[gA * kMaxB + c1] : 0.f;
    const float xb0 = c0 < B ? xs[gB * kMaxB + c0] : 0.f, xb1 = c1 < B ? xs[gB * kMaxB + c1] : 0.f;
    const float sgA = h2f(sg[gA]), sgB = h2f(sg[gB]), suA = h2f(su[gA]), suB = h2f(su[gB]);
    const float mgA = h2f(mg[gA]), mgB = h2f(mg[gB]), muA = h2f(mu[gA]), muB = h2f(mu[gB]);
    acc[0] += fmaf(sgA, dA[0], mgA * xa0) + fmaf(sgB, dB[0], mgB * xb0);
    acc[1] += fmaf(sgA, dA[1], mgA * xa1) + fmaf(sgB, dB[1], mgB * xb1);
    acc[2] += fmaf(suA, dA[2], muA * xa0) + fmaf(suB, dB[2], muB * xb0);
    acc[3] += fmaf(suA, dA[3], muA * xa1) + fmaf(suB, dB[3], muB * xb1);
  }
}

// 32 NVFP4 codes (one 16-byte load; E2M1, the lower nibble the even element)
// -> 16 bf16 pairs {w(8q+p), w(8q+p+4)} at register 4q+p (the order of
// int4x32_to_bf16x2), each weight its code times its 16-element block's E4M3
// scale: elements 0..15 take the low byte of sw, 16..31 the high byte.  An
// E2M1 value times an E4M3 scale has at most 6 significant bits and lies in
// [2^-10, 2,688], so every weight is exact in bf16.  Per pair: the two codes
// as one byte, the hardware conversion to an fp16 pair (exact), the fp16 bits
// read as bf16 times 2^-112 (exponent and fraction moved three bits right:
// exact, zero stays zero), one bf16 multiply by the scale times 2^112 (exact).
FLINT_DEV uint32_t nv_scale_bf16x2(uint32_t e4m3) {  // the scale x 2^112, both halves
  uint32_t h;
  asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(e4m3));
  const float f = __half2float(__ushort_as_half((unsigned short)(h & 0xffffu))) * 0x1p112f;
  const uint32_t b = __float_as_uint(f) >> 16;  // exact: 4 significant bits
  return b | (b << 16);
}
FLINT_DEV void nvfp4x32_to_bf16x2(const uint4 w, uint32_t sw, uint32_t (&r)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  const uint32_t sA = nv_scale_bf16x2(sw & 0xffu), sB = nv_scale_bf16x2(sw >> 8);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // nibbles n0..n7 of the word: lo bytes (n0, n2, n4, n6), hi bytes (n1,
    // n3, n5, n7); x | x >> 12 puts (n0 | n4 << 4, n2 | n6 << 4) in bytes 0-1
    const uint32_t lo = words[q] & 0x0F0F0F0Fu, hi = (words[q] >> 4) & 0x0F0F0F0Fu;
    const uint32_t X = lo | (lo >> 12), Y = hi | (hi >> 12);
    uint32_t h[4];  // pairs p = 0, 1, 2, 3 as fp16
    asm("{ .reg .b8 x0, x1, x2, x3, y0, y1, y2, y3;\n"
        "mov.b32 {x0, x1, x2, x3}, %4;\n"
        "mov.b32 {y0, y1, y2, y3}, %5;\n"
        "cvt.rn.f16x2.e2m1x2 %0, x0;\n"
        "cvt.rn.f16x2.e2m1x2 %1, y0;\n"
        "cvt.rn.f16x2.e2m1x2 %2, x1;\n"
        "cvt.rn.f16x2.e2m1x2 %3, y1; }"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(X), "r"(Y));
    const uint32_t s2 = q < 2 ? sA : sB;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t b = and_or(h[p] >> 3, 0x0FFF0FFFu, h[p] & 0x80008000u);
      uint32_t c;
      asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(b), "r"(s2));
      r[4 * q + p] = c;
    }
  }
}

// The NVFP4 item: rows g (gate) and g + 8 (up) of the lane's 32 elements as
// exact bf16 weights, each with its two block scales; the block scales are
// inside the weights, so the k-groups' sums add up directly.  The expert's
// global scales are applied by the caller after the warps' sums.
FLINT_DEV void item_part_nv(const unsigned char *buf, const uint4 *frag, int B, int warp, int lane,
                            float (&acc)[4]) {
  const int g = lane >> 2, t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  const unsigned char *sg = buf + 16384 + g * 128, *su = buf + 16384 + 1024 + g * 128;
#pragma unroll
  for (int k = 0; k < kK2Groups; ++k) {
    const int G = kK2Groups * warp + k;
    const uint4 wg = *reinterpret_cast<const uint4 *>(buf + g * 1024 + 64 * G + 16 * t);
    const uint4 wu = *reinterpret_cast<const uint4 *>(buf + 8192 + g * 1024 + 64 * G + 16 * t);
    // blocks 8G + 2t and 8G + 2t + 1 of each row: one 16-bit load
    const uint32_t sgw = *reinterpret_cast<const uint16_t *>(sg + 8 * G + 2 * t);
    const uint32_t suw = *reinterpret_cast<const uint16_t *>(su + 8 * G + 2 * t);
    uint32_t ra[16], rb[16], xb[16];
    nvfp4x32_to_bf16x2(wg, sgw, ra);
    nvfp4x32_to_bf16x2(wu, suw, rb);
    load_frag_compact(frag, G, B, lane, xb);
    float d[4];
    group_mma(ra, rb, xb, d);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += d[i];
  }
}

constexpr int kK2Stages = 2;     // items in flight per CTA
constexpr int kK2MaxItems = 16;  // items per CTA (the host sizes the grid to keep within it)

// Item list of one call: shared items 0..sh_items-1 (128, or none when the
// shared expert is left to another call), then 64 items per routed slot.
// CTA c takes items c, c + grid, c + 2 grid, ...; a CTA's first item is
// fetched before the wait when it is a shared one.
template <int kFmt>
__global__ void __launch_bounds__(kK2Warps * 32)
    k2_gateup(LayerArgs L, int B, int n_items, int sh_items, char *__restrict__ ws,
              DecodeLayout lay) {
  extern __shared__ __align__(128) unsigned char sm[];  // stages | x fragment (compact)
  constexpr bool kAff = kFmt == kFmtAff, kNv = kFmt == kFmtNv;
  constexpr int kIB = item_bytes<kFmt>();
  uint4 *frag = reinterpret_cast<uint4 *>(sm + kK2Stages * kIB);
  __shared__ __align__(8) uint64_t bar[kK2Stages];
  __shared__ __align__(8) uint64_t fbar;
  __shared__ float s_acc[kK2Warps][32][4];
  __shared__ uint32_t s_word[kK2MaxItems];
  __shared__ int s_n;
  __shared__ int s_aslot[kMaxB * kTopK];
  __shared__ float s_aw[kMaxB * kTopK];
  __shared__ float s_xs[kAff ? 32 : 1][kMaxB];  // affine: block input summed per 64-group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int c0 = blockIdx.x, step = gridDim.x;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + lay.ctrl);
  const uint32_t *slot_word = reinterpret_cast<const uint32_t *>(ws + lay.slot_word);
  trace_point(2, 0);

  // The shared expert's rows do not depend on K1.  Every copy adds its bytes
  // before the phase's single arrival, so no phase can complete early.
  if (tid == 0) {
    for (int i = 0; i < kK2Stages; ++i) mbar_init(&bar[i], 1);
    mbar_init(&fbar, 1);
    if (c0 < sh_items) {
      mbar_add_tx(&bar[0], kIB);
      issue_item<kFmt>(shared_item<kFmt>(L, c0), sm, &bar[0]);
    }
  }
  pdl_wait();  // K1 is complete: routing and the block input fragment are final
  pdl_trigger();
  trace_point(2, 1);
  if (tid == 0) {  // every CTA takes the fragment (and waits for it, even with no item)
    const uint32_t fbytes = 16u * 4u * (uint32_t)B * 64u;
    mbar_add_tx(&fbar, fbytes);
    bulk_g2s(frag, ws + lay.xfrag, fbytes, &fbar);
    mbar_arrive(&fbar);
  }
  // this CTA's items: slot words read together (kSlotInvalid ends the list)
  if (tid < kK2MaxItems) {
    const int it = c0 + tid * step;
    uint32_t w = kSlotInvalid;
    if (it < sh_items) w = 0u;
    else if (it < n_items) w = ld_cg_u32(slot_word + ((it - sh_items) >> 6));
    // the bounds-checked build: a routed item's word counts at most 6B slots,
    // the item's slot among them, and names only rows of this call (a refused
    // word ends the CTA's list like an invalid one)
    if (it >= sh_items && w != kSlotInvalid &&
        !FLINT_CHECK(slot_count(w) <= kTopK * B && ((it - sh_items) >> 6) < slot_count(w) &&
                         (slot_mask(w) >> B) == 0u,
                     ctrl + 1))
      w = kSlotInvalid;
    s_word[tid] = w;
  } else if (tid >= 32 && tid < 32 + B * kTopK) {
    s_aslot[tid - 32] = (int)ld_cg_u32(reinterpret_cast<const uint32_t *>(ws + lay.asc_slot) + tid - 32);
    s_aw[tid - 32] = ld_cg_f32(reinterpret_cast<const float *>(ws + lay.asc_w) + tid - 32);
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    while (n < kK2MaxItems && s_word[n] != kSlotInvalid) ++n;
    s_n = n;
    if (n > 0) {
      for (int j = 0; j < n && j < kK2Stages; ++j) {
        const int it = c0 + j * step;
        if (j == 0 && it < sh_items) {
          mbar_arrive(&bar[0]);  // fetched before the wait
        } else {
          mbar_add_tx(&bar[j], kIB);
          issue_item<kFmt>(it < sh_items ? shared_item<kFmt>(L, it)
                                       : routed_item<kFmt>(L, (int)slot_expert(s_word[j]),
                                                     8 * ((it - sh_items) & 63)),
                     sm + j * kIB, &bar[j]);
          mbar_arrive(&bar[j]);
        }
      }
    }
  }
  __syncthreads();
  const int n = s_n;
  const bool fok = dwait(&fbar, 0);
  bool ok = fok;
  if (kAff && fok) {
    // sum of the block input over 64-group gg of row b, from the fragment:
    // lanes tt = 2 (gg % 2), +1 of 128-group gg / 2 hold its 64 elements;
    // read by the items after the barrier that opens each of them
    for (int task = tid; task < 32 * B; task += kK2Warps * 32) {
      const int gg = task / B, b = task % B, G = gg >> 1;
      float sx = 0.f;
      for (int tt = 2 * (gg & 1); tt < 2 * (gg & 1) + 2; ++tt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = frag[(size_t)(G * 4 * B + b * 4 + tt) * 4 + q];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            sx += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xffff0000u);
        }
      s_xs[gg][b] = sx;
    }
  }
  if (n == 0) {
    if (!fok) {
      if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
      mbar_wait(&fbar, 0);  // the fragment copy still in flight lands first
    }
    return;
  }
  for (int j = 0; j < n; ++j) {
    const int st = j % kK2Stages;
    const int it = c0 + j * step;
    const uint32_t word = s_word[j];
    unsigned char *buf = sm + st * kIB;
    ok = dwait(&bar[st], (uint32_t)((j / kK2Stages) & 1)) && ok;
    trace_point(2, 2);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
      // copies still in flight land before the CTA exits
      if (!fok) mbar_wait(&fbar, 0);
      for (int jj = j; jj < n && jj < j + kK2Stages; ++jj)
        mbar_wait(&bar[jj % kK2Stages], (uint32_t)((jj / kK2Stages) & 1));
      return;
    }
    float acc[4];
    if (kAff)
      item_part_aff(buf, frag, &s_xs[0][0], B, warp, lane, acc);
    else if (kNv)
      item_part_nv(buf, frag, B, warp, lane, acc);
    else
      item_part(buf, frag, B, warp, lane, acc);
    trace_point(2, 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) s_acc[warp][lane][i] = acc[i];
    __syncthreads();  // every warp is done with buf: refill it
    trace_point(2, 5);
    if (tid == 0 && j + kK2Stages < n) {
      const int jn = j + kK2Stages, itn = c0 + jn * step;
      mbar_add_tx(&bar[st], kIB);
      issue_item<kFmt>(itn < sh_items ? shared_item<kFmt>(L, itn)
                                    : routed_item<kFmt>(L, (int)slot_expert(s_word[jn]),
                                                  8 * ((itn - sh_items) & 63)),
                 buf, &bar[st]);
      mbar_arrive(&bar[st]);
    }
    if (warp == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = s_acc[0][lane][i];
#pragma unroll
        for (int w = 1; w < kK2Warps; ++w) a += s_acc[w][lane][i];
        acc[i] = a;
      }
      if (kNv) {  // the expert's global scales: gate rows, then up rows
        const float *gp = it < sh_items ? L.sh13_g : L.w13_g + 2 * (size_t)slot_expert(word);
        const float gg = __ldg(gp), gu = __ldg(gp + 1);
        acc[0] *= gg, acc[1] *= gg, acc[2] *= gu, acc[3] *= gu;
      }
      if (it < sh_items) {
        uint16_t *hfs = reinterpret_cast<uint16_t *>(ws + lay.hfs);
        const int r = 8 * it + g;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int b = 2 * t + c;
          if (b < B)
            write_hilo(hfs + (size_t)(2 * b) * kIs, hfs + (size_t)(2 * b + 1) * kIs, r,
                       silu_f(acc[c]) * acc[2 + c]);
        }
      } else {
        const int u = (it - sh_items) >> 6, r0 = 8 * ((it - sh_items) & 63);
        const uint32_t mask = slot_mask(word);
        uint16_t *hfr = reinterpret_cast<uint16_t *>(ws + lay.hfr);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int b = 2 * t + c;
          if (b < B && ((mask >> b) & 1u)) {
            int jj = 0;
#pragma unroll
            for (int q = 0; q < kTopK; ++q)
              if (s_aslot[b * kTopK + q] == u) jj = q;
            // the routing weight, times the divisor of the stored up rows
            // (a power of two: the product equals the undivided one exactly)
            const float w = s_aw[b * kTopK + jj] * L.interm_div;
            uint16_t *img = hfr + (size_t)((b * kTopK + jj) * 2) * kI;
            write_hilo(img, img + kI, r0 + g, w * (silu_f(acc[c]) * acc[2 + c]));
          }
        }
      }
    }
    __syncthreads();  // s_acc is read before the next item writes it
  }
  trace_point(2, 3);
}

// ============================================================== K3: down + combine
// Shared-memory plan (bytes): weights [umax][16 rows][256] | scales
// [umax][16][4] bf16 (affine: [umax] of fp16 scales [16][8] then offsets
// [16][8]; NVFP4: [umax] of E4M3 scales [16][32]) | shared down [16][512] |
// shared scales [16][8] (affine: fp16 scales [16][16] then offsets [16][16];
// NVFP4: E4M3 [16][64]) | intermediates (kStage) routed [B][6][2][512] bf16,
// shared [B][2][1024] | per-row partial results [8 rows][16 parts][16
// columns] fp32.  `wide`: the affine and NVFP4 formats (512-byte slot scales).
struct K3Smem {
  int umax, B;
  bool wide;
  __host__ __device__ int slot_sb() const { return wide ? 512 : 128; }
  __host__ __device__ int sh_sb() const { return wide ? 1024 : 256; }
  __host__ __device__ size_t w() const { return 0; }
  __host__ __device__ size_t s() const { return (size_t)umax * 4096; }
  __host__ __device__ size_t shw() const { return s() + (size_t)umax * slot_sb(); }
  __host__ __device__ size_t shs() const { return shw() + 8192; }
  __host__ __device__ size_t hr() const { return shs() + sh_sb(); }
  __host__ __device__ size_t hs() const { return hr() + (size_t)B * kTopK * 2 * kI * 2; }
  __host__ __device__ size_t ysel(bool stage) const {
    return stage ? hs() + (size_t)B * 2 * kIs * 2 : hr();
  }
  __host__ __device__ size_t total(bool stage) const { return ysel(stage) + 8 * 16 * 16 * 4; }
};

template <bool kResidual, bool kStage, int kFmt>
__global__ void __launch_bounds__(kK3Threads)
    k3_down_combine(LayerArgs L, int B, uint16_t *__restrict__ out, float *__restrict__ h,
                    float *__restrict__ pout, int with_shared, char *__restrict__ ws,
                    DecodeLayout lay, int umax) {
  extern __shared__ __align__(128) unsigned char sm[];
  constexpr bool kAff = kFmt == kFmtAff, kNv = kFmt == kFmtNv;
  const K3Smem P{umax, B, kFmt != kFmtSym};
  unsigned char *wsm = sm + P.w();
  unsigned char *ssm = sm + P.s();
  unsigned char *shm = sm + P.shw();
  unsigned char *shs = sm + P.shs();
  uint16_t *himg_r = reinterpret_cast<uint16_t *>(sm + P.hr());
  uint16_t *himg_s = reinterpret_cast<uint16_t *>(sm + P.hs());
  float *ysel = reinterpret_cast<float *>(sm + P.ysel(kStage));
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_ns;
  __shared__ uint32_t s_rows[kE];
  __shared__ int s_asc[kMaxB * kTopK];
  // slot u's i-th row (ascending) b and the slot's place j among that row's
  // experts (ascending), as b | j << 4
  __shared__ uint8_t s_rbj[kMaxB * kTopK][kMaxB];
  // affine: each intermediate image pair (hi + lo) summed over its 64-groups:
  // row b's j-th routed expert at b * 6 + j (8 groups), its shared one at
  // 48 + b (16 groups)
  __shared__ float s_hs[kAff ? kMaxB * kTopK + kMaxB : 1][16];
  // NVFP4: each slot's global scale of its down projection
  __shared__ float s_gd[kNv ? kMaxB * kTopK : 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * 16;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws + lay.ctrl);
  trace_point(3, 0);

  // Routing is final here (K2 triggered this launch after its own wait on
  // K1): fetch the chosen experts' down rows before waiting on K2.
  if (tid == 0) {
    mbar_init(&bar, 1);
    s_ns = 0;  // stays 0 if slot 0 is invalid (a routing left by a failed K1)
  }
  __syncthreads();
  float h_old = 0.f;  // this thread's residual element (final: K1 waited for it)
  if (kResidual && tid < 16 * B) h_old = ld_cg_f32(h + (size_t)(tid >> 4) * kH + n0 + (tid & 15));
  if (tid < kE) {
    const uint32_t word = ld_cg_u32(reinterpret_cast<const uint32_t *>(ws + lay.slot_word) + tid);
    // at most umax slots have room here; a routing left by a failed K1 may
    // hold more, and none of it is used after the status is set
    s_rows[tid] = 0u;  // rows of an invalid slot: none
    // the bounds-checked build: the word counts at most 6B slots, this one
    // among them, and names only rows of this call
    if (word != kSlotInvalid && tid < umax &&
        FLINT_CHECK(slot_count(word) <= kTopK * B && tid < slot_count(word) &&
                        (slot_mask(word) >> B) == 0u,
                    ctrl + 1)) {
      const size_t e = slot_expert(word);
      s_rows[tid] = slot_mask(word) & ((1u << B) - 1u);
      if (kAff) {  // fp16 scales then offsets, 8 per row
        mbar_add_tx(&bar, 4096 + 512);
        bulk_g2s(wsm + tid * 4096, L.w2_q + (e * kH + n0) * (kI / 2), 4096, &bar);
        bulk_g2s(ssm + tid * 512, L.w2_s + (e * kH + n0) * (kI / 64), 256, &bar);
        bulk_g2s(ssm + tid * 512 + 256, L.w2_m + (e * kH + n0) * (kI / 64), 256, &bar);
      } else if (kNv) {  // E4M3 scales, 32 bytes per row; the global scale
        mbar_add_tx(&bar, 4096 + 512);
        bulk_g2s(wsm + tid * 4096, L.w2_q + (e * kH + n0) * (kI / 2), 4096, &bar);
        bulk_g2s(ssm + tid * 512,
                 reinterpret_cast<const unsigned char *>(L.w2_s) + (e * kH + n0) * (kI / 16), 512,
                 &bar);
        s_gd[tid] = __ldg(L.w2_g + e);
      } else {
        mbar_add_tx(&bar, 4096 + 128);
        bulk_g2s(wsm + tid * 4096, L.w2_q + (e * kH + n0) * (kI / 2), 4096, &bar);
        bulk_g2s(ssm + tid * 128, L.w2_s + (e * kH + n0) * (kI / kG), 128, &bar);
      }
      if (tid == 0) s_ns = min(slot_count(word), umax);
    }
  } else if (tid == kE && with_shared) {
    if (kAff) {  // fp16 scales then offsets, 16 per row
      mbar_add_tx(&bar, 8192 + 1024);
      bulk_g2s(shm, L.sh2_q + (size_t)n0 * (kIs / 2), 8192, &bar);
      bulk_g2s(shs, L.sh2_s + (size_t)n0 * (kIs / 64), 512, &bar);
      bulk_g2s(shs + 512, L.sh2_m + (size_t)n0 * (kIs / 64), 512, &bar);
    } else if (kNv) {  // E4M3 scales, 64 bytes per row
      mbar_add_tx(&bar, 8192 + 1024);
      bulk_g2s(shm, L.sh2_q + (size_t)n0 * (kIs / 2), 8192, &bar);
      bulk_g2s(shs, reinterpret_cast<const unsigned char *>(L.sh2_s) + (size_t)n0 * (kIs / 16),
               1024, &bar);
    } else {
      mbar_add_tx(&bar, 8192 + 256);
      bulk_g2s(shm, L.sh2_q + (size_t)n0 * (kIs / 2), 8192, &bar);
      bulk_g2s(shs, L.sh2_s + (size_t)n0 * (kIs / kG), 256, &bar);
    }
  } else if (tid >= kE + 32 && tid < kE + 32 + B * kTopK) {
    const int i = tid - kE - 32;
    s_asc[i] = (int)ld_cg_u32(reinterpret_cast<const uint32_t *>(ws + lay.asc_slot) + i);
  }
  __syncthreads();
  if (tid == 0) mbar_arrive(&bar);
  if (tid < s_ns) {  // read by the tasks after the barrier that follows the wait
    uint32_t m = s_rows[tid];
    for (int i = 0; m != 0u; ++i, m &= m - 1u) {
      const int b = __ffs(m) - 1;
      int j = 0;
      for (int jj = 0; jj < kTopK; ++jj)
        if (s_asc[b * kTopK + jj] == tid) j = jj;
      s_rbj[tid][i] = (uint8_t)(b | (j << 4));
    }
  }

  pdl_wait();
  pdl_trigger();
  trace_point(3, 1);
  if (kStage) {
    const unsigned char *src_r = reinterpret_cast<const unsigned char *>(ws + lay.hfr);
    const unsigned char *src_s = reinterpret_cast<const unsigned char *>(ws + lay.hfs);
    const int nr = B * kTopK * 2 * kI * 2 / 16, nsh = B * 2 * kIs * 2 / 16;
    for (int i = tid; i < nr; i += kK3Threads)
      cp_async16(reinterpret_cast<unsigned char *>(himg_r) + 16 * i, src_r + 16 * i);
    for (int i = tid; i < nsh; i += kK3Threads)
      cp_async16(reinterpret_cast<unsigned char *>(himg_s) + 16 * i, src_s + 16 * i);
    cp_async_wait_all();
  }
  // parts no task writes (experts outside this call's range, the shared
  // expert when it is left out) add zero
  for (int i = tid; i < 16 * 16 * B; i += kK3Threads) ysel[i] = 0.f;
  const bool arrived = dwait(&bar, 0);
  if (__syncthreads_or(!arrived)) {
    if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
    if (!arrived) mbar_wait(&bar, 0);  // copies still in flight land before the CTA exits
    return;
  }
  const int ns = s_ns;
  trace_point(3, 2);

  const uint16_t *gr = kStage ? himg_r : reinterpret_cast<const uint16_t *>(ws + lay.hfr);
  const uint16_t *gs = kStage ? himg_s : reinterpret_cast<const uint16_t *>(ws + lay.hfs);
  if (kAff) {
    // an image's 64-group gg (of its 128-group gg / 2, lanes 2 (gg % 2) and
    // +1) is 64 contiguous bf16 in the fragment order; hi then lo per element
    for (int task = tid; task < B * (kTopK * 8 + 16); task += kK3Threads) {
      const bool shr = task >= B * kTopK * 8;
      const int tk = shr ? task - B * kTopK * 8 : task;
      const int gg = shr ? tk & 15 : tk & 7, row = shr ? tk >> 4 : tk >> 3;  // row: b*6+j or b
      const size_t len = shr ? kIs : kI;
      const uint16_t *hi = shr ? gs + (size_t)(2 * row) * kIs : gr + (size_t)(2 * row) * kI;
      const size_t off = (size_t)(gg >> 1) * 128 + (size_t)(gg & 1) * 64;
      float sx = 0.f;
      for (int e8 = 0; e8 < 8; ++e8) {
        const uint4 a = kStage ? *reinterpret_cast<const uint4 *>(hi + off + 8 * e8)
                               : ld_cg_v4(hi + off + 8 * e8);
        const uint4 c = kStage ? *reinterpret_cast<const uint4 *>(hi + len + off + 8 * e8)
                               : ld_cg_v4(hi + len + off + 8 * e8);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sx += (__uint_as_float(wa[i] << 16) + __uint_as_float(wc[i] << 16)) +
                (__uint_as_float(wa[i] & 0xffff0000u) + __uint_as_float(wc[i] & 0xffff0000u));
      }
      s_hs[shr ? kMaxB * kTopK + row : row][gg] = sx;
    }
    __syncthreads();
  }
  // tasks: two k-parts (2 groups each) of routed slots 0..ns-1, then four
  // k-parts of the shared expert; partial sums land in ysel[b][m] with
  // m = 2j + part for the row's j-th expert (ascending), 12 + part shared.
  // The MMA's columns carry the task's rows R (those that chose the expert,
  // every row for the shared one) as pairs: column 2i the hi image of row
  // R[4p + i], column 2i+1 its lo image; one pass p per 4 rows.
  for (int task = warp; task < 2 * ns + (with_shared ? 4 : 0); task += kK3Threads / 32) {
    const bool sh = task >= 2 * ns;
    const int slot = task >> 1;
    const int part = sh ? task - 2 * ns : task & 1;
    const int rowbytes = sh ? kIs / 2 : kI / 2;
    const unsigned char *wbase = sh ? shm : wsm + slot * 4096;
    const uint16_t *sc =
        reinterpret_cast<const uint16_t *>(sh ? shs : ssm + slot * (kFmt != kFmtSym ? 512 : 128));
    const int nvr = sh ? kIs / 16 : kI / 16;  // NVFP4: scale bytes per row
    // scale groups per row (affine: per 64, the offsets after the scales)
    const int spr = kAff ? (sh ? kIs / 64 : kI / 64) : (sh ? kIs / kG : kI / kG);
    const uint16_t *mo = sc + 16 * spr;
    const uint32_t mask = sh ? ((1u << B) - 1u) : s_rows[slot];
    const int nr = __popc(mask);
    // this lane's column (g) in each pass, and its output row (t)
    const uint16_t *img[2] = {nullptr, nullptr};
    int orow[2] = {-1, -1}, om[2] = {0, 0}, hrow[2] = {0, 0};
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int ic = 4 * p + (g >> 1), io = 4 * p + t;
      if (ic < nr) {  // the shared expert takes every row: its i-th row is row i
        const int hl = g & 1;
        if (sh) {
          img[p] = gs + (size_t)(2 * ic + hl) * kIs;
        } else {
          const int bj = s_rbj[slot][ic];
          img[p] = gr + (size_t)(((bj & 15) * kTopK + (bj >> 4)) * 2 + hl) * kI;
        }
      }
      if (io < nr) {
        if (sh) {
          orow[p] = io;
          om[p] = 12 + part;
          hrow[p] = kMaxB * kTopK + io;
        } else {
          const int bj = s_rbj[slot][io];
          orow[p] = bj & 15;
          om[p] = 2 * (bj >> 4) + part;
          hrow[p] = (bj & 15) * kTopK + (bj >> 4);
        }
      }
    }
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int G = 2 * part + k;
      const uint4 w0 = *reinterpret_cast<const uint4 *>(wbase + g * rowbytes + 64 * G + 16 * t);
      const uint4 w1 =
          *reinterpret_cast<const uint4 *>(wbase + (g + 8) * rowbytes + 64 * G + 16 * t);
      uint32_t ra[16], rb[16];
      if (kAff) {
        uint4x32_to_bf16x2(w0, ra);
        uint4x32_to_bf16x2(w1, rb);
      } else if (kNv) {  // rows g, g + 8: E4M3 bytes of blocks 8G + 2t, 8G + 2t + 1
        const unsigned char *sb = reinterpret_cast<const unsigned char *>(sc);
        nvfp4x32_to_bf16x2(w0, *reinterpret_cast<const uint16_t *>(sb + g * nvr + 8 * G + 2 * t),
                           ra);
        nvfp4x32_to_bf16x2(
            w1, *reinterpret_cast<const uint16_t *>(sb + (g + 8) * nvr + 8 * G + 2 * t), rb);
      } else {
        int4x32_to_bf16x2(w0, ra);
        int4x32_to_bf16x2(w1, rb);
      }
      const float s0 = kFmt != kFmtSym ? 0.f : bf16_bits_to_f32(sc[g * spr + G]);
      const float s1 = kFmt != kFmtSym ? 0.f : bf16_bits_to_f32(sc[(g + 8) * spr + G]);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        if (4 * p < nr) {  // the same for the whole warp
          uint32_t xb[16];
          if (img[p]) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int off = ((G * 4 + t) * 16 + 4 * i) * 2;
              const uint4 a = kStage ? *reinterpret_cast<const uint4 *>(img[p] + off)
                                     : ld_cg_v4(img[p] + off);
              xb[4 * i] = a.x, xb[4 * i + 1] = a.y, xb[4 * i + 2] = a.z, xb[4 * i + 3] = a.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) xb[i] = 0u;
          }
          if (kAff) {
            // lanes t < 2 hold 64-group 2G of the 128-group, t >= 2 group
            // 2G + 1: one MMA per group with the other's columns zeroed
            const uint32_t mA = t < 2 ? 0xffffffffu : 0u, mB = ~mA;
            uint32_t xa[16], xo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) xa[i] = xb[i] & mA, xo[i] = xb[i] & mB;
            float dA[4] = {0.f, 0.f, 0.f, 0.f}, dB[4] = {0.f, 0.f, 0.f, 0.f};
            group_mma_acc(ra, rb, xa, dA);
            group_mma_acc(ra, rb, xo, dB);
            const int gA = 2 * G, gB = 2 * G + 1;
            auto h2f = [](uint16_t v) { return __half2float(__ushort_as_half(v)); };
            const float hA = s_hs[hrow[p]][gA], hB = s_hs[hrow[p]][gB];
            acc[p][0] += fmaf(h2f(sc[g * spr + gA]), dA[0] + dA[1], h2f(mo[g * spr + gA]) * hA) +
                         fmaf(h2f(sc[g * spr + gB]), dB[0] + dB[1], h2f(mo[g * spr + gB]) * hB);
            acc[p][1] += fmaf(h2f(sc[(g + 8) * spr + gA]), dA[2] + dA[3],
                              h2f(mo[(g + 8) * spr + gA]) * hA) +
                         fmaf(h2f(sc[(g + 8) * spr + gB]), dB[2] + dB[3],
                              h2f(mo[(g + 8) * spr + gB]) * hB);
          } else if (kNv) {  // the block scales are inside the weights
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            group_mma_acc(ra, rb, xb, d);
            acc[p][0] += d[0] + d[1];
            acc[p][1] += d[2] + d[3];
          } else {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            group_mma_acc(ra, rb, xb, d);
            acc[p][0] = fmaf(d[0] + d[1], s0, acc[p][0]);
            acc[p][1] = fmaf(d[2] + d[3], s1, acc[p][1]);
          }
        }
      }
    }
    // NVFP4: the down projection's global scale, once per part
    const float gd = kNv ? (sh ? __ldg(L.sh2_g) : s_gd[slot]) : 1.f;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if (orow[p] >= 0) {
        ysel[(orow[p] * 16 + om[p]) * 16 + g] = kNv ? acc[p][0] * gd : acc[p][0];
        ysel[(orow[p] * 16 + om[p]) * 16 + g + 8] = kNv ? acc[p][1] * gd : acc[p][1];
      }
    }
  }
  trace_point(3, 4);
  __syncthreads();
  trace_point(3, 5);
  if (tid < 16 * B) {
    const int n = tid & 15, b = tid >> 4;
    float y = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) y += ysel[(b * 16 + m) * 16 + n];
    const size_t o = (size_t)b * kH + n0 + n;
    if (pout) {
      pout[o] = y;  // this call's share of the block output, before any rounding
    } else if (kResidual) {
      const float yb = __bfloat162float(__float2bfloat16_rn(y));
      h[o] = h_old + yb;
    } else {
      out[o] = f32_to_bf16_bits(y);
    }
  }
  trace_point(3, 3);
}

// ============================================================== host
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

static int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

// dynamic shared memory cap: the 227 KB opt-in limit minus K3's static arrays
// (1.6 KB; 5.2 KB with the affine format's intermediate group sums; the NVFP4
// format's slot global scales are 192 B)
constexpr size_t kK3MaxSmem = 224 * 1024, kK3MaxSmemAff = 220 * 1024;
constexpr int kK1Smem = 16 * kRouterRowStride + kXFragBytes;
constexpr int kK2Smem = kK2Stages * kItemBytesAff + kXFragBytes;  // ring + fragment, B <= 8
static size_t k2_smem(int B, int fmt) {
  return (size_t)kK2Stages * (fmt == kFmtSym ? kItemBytes : kItemBytesAff) + (size_t)4096 * B;
}
static size_t k3_cap(int fmt) { return fmt == kFmtSym ? kK3MaxSmem : kK3MaxSmemAff; }

template <int kFmt>
static int k2_occupancy(int B) {
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k2_gateup<kFmt>, kK2Warps * 32,
                                                k2_smem(B, kFmt));
  return occ;
}

// K2 grid: as many CTAs as fit on the device at once (at most one per item),
// but never so few that a CTA would own more than kK2MaxItems items.
static int k2_grid(int dev, int B, int n_items, int fmt) {
  static int cache[64][3][kMaxB + 1];  // 0 = not computed
  int per_sm = dev < 64 ? cache[dev][fmt][B] : 0;
  if (per_sm == 0) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int occ = fmt == kFmtAff  ? k2_occupancy<kFmtAff>(B)
                    : fmt == kFmtNv ? k2_occupancy<kFmtNv>(B)
                                    : k2_occupancy<kFmtSym>(B);
    per_sm = sms * (occ > 0 ? occ : 1);
    if (dev < 64) cache[dev][fmt][B] = per_sm;
  }
  int grid = per_sm < n_items ? per_sm : n_items;
  const int floor_grid = (n_items + kK2MaxItems - 1) / kK2MaxItems;
  return grid > floor_grid ? grid : floor_grid;
}

template <bool kResidual>
static cudaError_t set_attrs(int dev) {
  static uint64_t done = 0;  // one bit per device
  if (dev < 64 && ((done >> dev) & 1u)) return cudaSuccess;
  note_step("k1_router smem attribute");
  cudaError_t e = cudaFuncSetAttribute(k1_router<kResidual>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kK1Smem);
  auto attr = [&](const void *f, size_t bytes, const char *what) {
    if (e == cudaSuccess)
      e = noted(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes),
                what);
  };
  attr(reinterpret_cast<const void *>(k2_gateup<kFmtSym>), kK2Smem, "k2_gateup smem attribute");
  attr(reinterpret_cast<const void *>(k2_gateup<kFmtAff>), kK2Smem,
       "k2_gateup (affine) smem attribute");
  attr(reinterpret_cast<const void *>(k2_gateup<kFmtNv>), kK2Smem,
       "k2_gateup (NVFP4) smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, true, kFmtSym>), kK3MaxSmem,
       "k3 smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, false, kFmtSym>), kK3MaxSmem,
       "k3 smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, true, kFmtAff>), kK3MaxSmemAff,
       "k3 (affine) smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, false, kFmtAff>), kK3MaxSmemAff,
       "k3 (affine) smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, true, kFmtNv>), kK3MaxSmemAff,
       "k3 (NVFP4) smem attribute");
  attr(reinterpret_cast<const void *>(k3_down_combine<kResidual, false, kFmtNv>), kK3MaxSmemAff,
       "k3 (NVFP4) smem attribute");
  if (e == cudaSuccess && dev < 64) done |= uint64_t(1) << dev;
  return e;
}

// K2 and K3 of one decode call for the experts' format
template <bool kResidual, int kFmt>
static cudaError_t launch_k2_k3(const LayerArgs &L, int B, uint16_t *out, float *h, char *ws,
                                const DecodeLayout &lay, cudaStream_t st, const DecodeShard &sh,
                                int umax, int n_items, int sh_items) {
  note_step("k2_gateup launch");
  const int g2 = k2_grid(current_device(), B, n_items > 0 ? n_items : 1, kFmt);
  cudaError_t err = launch_pdl(k2_gateup<kFmt>, g2, kK2Warps * 32, k2_smem(B, kFmt), st, L, B,
                               n_items, sh_items, ws, lay);
  if (err != cudaSuccess) return err;
  const K3Smem P{umax, B, kFmt != kFmtSym};
  const int wsh = sh.with_shared ? 1 : 0;
  note_step("k3_down_combine launch");
  const bool stage = P.total(true) <= k3_cap(kFmt);
  const size_t smem = P.total(stage);
  return stage ? launch_pdl(k3_down_combine<kResidual, true, kFmt>, kH / 16, kK3Threads, smem, st,
                            L, B, out, h, sh.partial, wsh, ws, lay, umax)
               : launch_pdl(k3_down_combine<kResidual, false, kFmt>, kH / 16, kK3Threads, smem,
                            st, L, B, out, h, sh.partial, wsh, ws, lay, umax);
}

template <bool kResidual>
static cudaError_t launch_decode_t(const LayerArgs &L, const uint16_t *x, float *h, int B,
                                   uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                                   cudaStream_t st, bool route_only, const DecodeShard &sh) {
  cudaError_t err = set_attrs<kResidual>(current_device());
  if (err != cudaSuccess) return err;
  const DecodeLayout lay = decode_layout(B);
  note_step("k1_router launch");
  err = launch_pdl(k1_router<kResidual>, kRouterCtas, kK1Threads, kK1Smem, st, L, x,
                   (const float *)h, B, ws, lay, idx_out, w_out, sh.e_lo, sh.e_hi);
  if (err != cudaSuccess || route_only) return err;
  const int span = sh.e_hi - sh.e_lo;
  const int umax = kTopK * B < span ? kTopK * B : span;
  const int sh_items = sh.with_shared ? kSharedItems : 0;
  const int n_items = sh_items + 64 * umax;
  if (L.fmt == kFmtAff)
    return launch_k2_k3<kResidual, kFmtAff>(L, B, out, h, ws, lay, st, sh, umax, n_items, sh_items);
  if (L.fmt == kFmtNv)
    return launch_k2_k3<kResidual, kFmtNv>(L, B, out, h, ws, lay, st, sh, umax, n_items, sh_items);
  return launch_k2_k3<kResidual, kFmtSym>(L, B, out, h, ws, lay, st, sh, umax, n_items, sh_items);
}

cudaError_t decode_set_wait_polls(uint32_t polls) {
  if (polls == 0xFFFFFFFFu) polls = kWaitPolls;
  return cudaMemcpyToSymbol(g_decode_polls, &polls, sizeof(polls));
}

#ifdef FLINT_TRACE
extern "C" FLINT_API int flint_trace_dump(unsigned long long *t, unsigned int *tag, int cap) {
  unsigned int n = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  cudaMemcpyFromSymbol(&n, g_trace_n, sizeof(n));
  if (n > kTraceCap) n = kTraceCap;
  if ((int)n > cap) n = (unsigned)cap;  // unwritten records (events not reached) keep tag 0
  cudaMemcpyFromSymbol(t, g_trace_time, sizeof(unsigned long long) * n);
  cudaMemcpyFromSymbol(tag, g_trace_tag, sizeof(unsigned int) * n);
  const unsigned int zero = 0;
  cudaMemcpyToSymbol(g_trace_n, &zero, sizeof(zero));
  static unsigned int zeros[kTraceCap];
  cudaMemcpyToSymbol(g_trace_tag, zeros, sizeof(zeros));
  return (int)n;
}
#endif

cudaError_t launch_decode(const LayerArgs &L, const uint16_t *x, const float *h_in, float *h_out,
                          int B, uint16_t *out, int32_t *idx_out, float *w_out, char *ws,
                          cudaStream_t st, bool route_only, const DecodeShard &sh) {
  if (h_out || h_in)
    return launch_decode_t<true>(L, nullptr, h_out ? h_out : const_cast<float *>(h_in), B, nullptr,
                                 idx_out, w_out, ws, st, false, sh);
  return launch_decode_t<false>(L, x, nullptr, B, out, idx_out, w_out, ws, st, route_only, sh);
}

// out = bf16(sum) and / or h += bf16(sum): the last step of a block whose
// output was summed from partials (one thread per element)
__global__ void k_combine_partials(const float *__restrict__ sum, int n, uint16_t *__restrict__ out,
                                   float *__restrict__ h) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float y = sum[i];
  if (out) out[i] = f32_to_bf16_bits(y);
  if (h) h[i] = h[i] + __bfloat162float(__float2bfloat16_rn(y));
}

cudaError_t launch_combine_partials(const float *sum, int B, uint16_t *out, float *h,
                                    cudaStream_t st) {
  note_step("k_combine_partials launch");
  const int n = B * kH;
  return launch_pdl(k_combine_partials, (n + 255) / 256, 256, 0, st, sum, n, out, h);
}

}  // namespace flint
