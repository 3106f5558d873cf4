// Int4 GEMV with fused argmax for the output head ("How to Run Flint
// Locally", section "One decode step in bytes": lm_head is 150,144 x 2,048,
// read in full for every token; Recursive quantized it to 4 bits).
//
// Persistent kernel, one CTA per SM.  A producer warp streams whole 16-row
// tiles (16 x K/2 bytes of codes plus their 16 x K/64 bytes of scales, both
// contiguous) into a ring of shared-memory stages with 1-D bulk copies;
// consumer warps take ring slots strictly in order from a shared counter and
// run each tile against up to 8 activation columns on mma.sync (see
// common.cuh).  There are never more consumers than stages, so a consumer
// waits at most one phase ahead on a stage barrier (parity waits cannot
// alias).  A final partial tile
// (N % 16 rows) is read straight from global memory.  Each warp keeps its best
// (value, row) per column; CTAs publish partials and the last CTA to finish
// reduces them (lowest row on ties), so the call is one launch.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace flint {

constexpr int kMaxConsumers = 16;
constexpr int kGemvWarps = kMaxConsumers + 1;  // producer = the last warp launched
constexpr size_t kGemvSmemCap = 200 * 1024;
constexpr int kMaxGemvCtas = 1024;

struct ArgPartial {
  float v;
  int i;
};

// (v, i) beats the current best (bv, bi): larger value, lower row on ties;
// any non-NaN value beats an empty best (bi < 0).
FLINT_DEV bool better(float v, int i, float bv, int bi) {
  return bi < 0 ? (v == v) : (v > bv || (v == bv && i < bi));
}

// Poll bound of the GEMV's first wait on each ring barrier (a consumer's wait
// for a stage to land, the producer's wait for a stage to be released).
// flint_debug_set_wait_polls lowers it so that a test can drive the timeout
// path; the error path's waits for copies still in flight keep kWaitPolls.
static __device__ uint32_t g_gemv_polls = kWaitPolls;
FLINT_DEV bool gwait(uint64_t *bar, uint32_t parity) {
  const uint32_t n = *reinterpret_cast<volatile uint32_t *>(&g_gemv_polls);
  for (uint32_t i = 0; i < n; ++i)
    if (mbar_try(bar, parity)) return true;
  return false;
}

static int gemv_grid(int N) {
  const int tiles = (N + 15) / 16;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms > kMaxGemvCtas) sms = kMaxGemvCtas;
  return tiles < sms ? tiles : sms;
}

size_t gemv_ws_bytes(int N, int B) {
  (void)N;
  return align256(256) + align256(sizeof(ArgPartial) * (size_t)kMaxGemvCtas * B);
}

struct GemvPlan {
  size_t stage_bytes, frag_bytes, smem;
  int stages;
};

// Stage of one 16-row tile: codes (16 x K/2 bytes), then the symmetric
// format's bf16 scales (16 x K/128) or the affine format's fp16 scales and
// offsets (16 x K/64 each).  The affine fragment is followed by the per-row
// sums of x over every 64-group (fp32, [K/64][B]).
// NVFP4: codes, then the 16 rows' E4M3 block scales (16 x K/16 bytes).
enum { kFmtSym = 0, kFmtAffine = 1, kFmtNvfp4 = 2 };

static GemvPlan gemv_plan(int K, int B, int fmt) {
  const bool affine = fmt == kFmtAffine;
  GemvPlan p;
  p.stage_bytes = align256((size_t)8 * K + (fmt == kFmtSym ? (size_t)K / 4 : (size_t)K));
  p.frag_bytes = align256((size_t)(K / kG) * 4 * B * 64) +
                 (affine ? align256((size_t)(K / 64) * B * 4) : 0);
  p.stages = (int)((kGemvSmemCap - p.frag_bytes) / p.stage_bytes);
  if (p.stages > 16) p.stages = 16;
  p.smem = p.frag_bytes + (size_t)p.stages * p.stage_bytes;
  return p;
}

// Compact activation fragment: only the B live columns (lanes g < B) are
// stored, frag[(G * 4B + g * 4 + t) * 4 + q] (uint4); other lanes read zeros.
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

// Rows ra, rb (codes at row stride K/2 bytes, scales at row stride K/128)
// against the fragment: acc[0..1] row ra, acc[2..3] row rb, columns 2t, 2t+1.
template <bool kGlobal>
FLINT_DEV void rows_dot(const uint8_t *qa, const uint8_t *qb, const uint16_t *sa,
                        const uint16_t *sb, int K, int B, const uint4 *frag, int lane,
                        float (&acc)[4]) {
  const int t = lane & 3;
  const int ng = K / kG;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll 2
  for (int G = 0; G < ng; ++G) {
    uint4 w0, w1;
    uint32_t s0b, s1b;
    if (kGlobal) {
      w0 = ld_stream(qa + 64 * G + 16 * t);
      w1 = ld_stream(qb + 64 * G + 16 * t);
      s0b = ld_nc_u16(sa + G);
      s1b = ld_nc_u16(sb + G);
    } else {
      w0 = *reinterpret_cast<const uint4 *>(qa + 64 * G + 16 * t);
      w1 = *reinterpret_cast<const uint4 *>(qb + 64 * G + 16 * t);
      s0b = sa[G];
      s1b = sb[G];
    }
    uint32_t ra[16], rbv[16], xb[16];
    int4x32_to_bf16x2(w0, ra);
    int4x32_to_bf16x2(w1, rbv);
    load_frag_compact(frag, G, B, lane, xb);
    float d[4];
    group_mma(ra, rbv, xb, d);
    const float s0 = bf16_bits_to_f32(s0b), s1 = bf16_bits_to_f32(s1b);
    acc[0] = fmaf(d[0], s0, acc[0]);
    acc[1] = fmaf(d[1], s0, acc[1]);
    acc[2] = fmaf(d[2], s1, acc[2]);
    acc[3] = fmaf(d[3], s1, acc[3]);
  }
}

// 16 unsigned codes (two words) -> 8 bf16 pairs {c(8q+p), c(8q+p+4)} at
// register 4q+p, exact: (w & 0x000F000F) | 0x43004300 is bf16 128 + code.
FLINT_DEV void uint4x16_to_bf16x2(const uint2 w, uint32_t (&r)[8]) {
  const uint32_t words[2] = {w.x, w.y};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t = ((words[q] >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
      uint32_t c;
      asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(t), "r"(0x43004300u));
      r[4 * q + p] = c;
    }
  }
}

// Affine rows ra, rb: codes at row stride K/2 bytes; fp16 scales and offsets
// at row stride K/64.  Lane t takes elements 64h + 16t .. 64h + 16t + 15 of
// half h of each 128-element block, so MMAs 4h .. 4h+3 cover 64-group 2G + h
// alone: y += scale * (codes . x) + offset * sum(x over the group).
template <bool kGlobal>
FLINT_DEV void rows_dot_affine(const uint8_t *qa, const uint8_t *qb, const uint16_t *sa,
                               const uint16_t *sb, const uint16_t *ma, const uint16_t *mb, int K,
                               int B, const uint4 *frag, const float *xsum, int lane,
                               float (&acc)[4]) {
  const int t = lane & 3;
  const int ng = K / kG;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  for (int G = 0; G < ng; ++G) {
    uint32_t xb[16];
    load_frag_compact(frag, G, B, lane, xb);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int off = 64 * G + 32 * h + 8 * t, grp = 2 * G + h;
      uint2 w0, w1;
      uint32_t s0b, s1b, m0b, m1b;
      if (kGlobal) {
        w0 = __ldg(reinterpret_cast<const uint2 *>(qa + off));
        w1 = __ldg(reinterpret_cast<const uint2 *>(qb + off));
        s0b = ld_nc_u16(sa + grp), s1b = ld_nc_u16(sb + grp);
        m0b = ld_nc_u16(ma + grp), m1b = ld_nc_u16(mb + grp);
      } else {
        w0 = *reinterpret_cast<const uint2 *>(qa + off);
        w1 = *reinterpret_cast<const uint2 *>(qb + off);
        s0b = sa[grp], s1b = sb[grp], m0b = ma[grp], m1b = mb[grp];
      }
      uint32_t ra[8], rb[8];
      uint4x16_to_bf16x2(w0, ra);
      uint4x16_to_bf16x2(w1, rb);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_bf16_16816(d, ra[2 * j], rb[2 * j], ra[2 * j + 1], rb[2 * j + 1], xb[8 * h + 2 * j],
                       xb[8 * h + 2 * j + 1]);
      const float s0 = __half2float(__ushort_as_half((unsigned short)s0b));
      const float s1 = __half2float(__ushort_as_half((unsigned short)s1b));
      const float m0 = __half2float(__ushort_as_half((unsigned short)m0b));
      const float m1 = __half2float(__ushort_as_half((unsigned short)m1b));
      const int c0 = 2 * t, c1 = 2 * t + 1;
      const float x0 = c0 < B ? xsum[grp * B + c0] : 0.f, x1 = c1 < B ? xsum[grp * B + c1] : 0.f;
      acc[0] = fmaf(m0, x0, fmaf(d[0], s0, acc[0]));
      acc[1] = fmaf(m0, x1, fmaf(d[1], s0, acc[1]));
      acc[2] = fmaf(m1, x0, fmaf(d[2], s1, acc[2]));
      acc[3] = fmaf(m1, x1, fmaf(d[3], s1, acc[3]));
    }
  }
}

// 8 E2M1 codes (one word; byte j = elements 2j, 2j+1 of the word's bytes)
// -> 4 f16 pairs, exact (hardware conversion, the lower nibble to the lower
// half).
FLINT_DEV void e2m1x8_to_f16x2(uint32_t w, uint32_t *r) {
  asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %4;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      "cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(w));
}
// two E4M3 codes (the lower byte first) -> f16 pair, exact
FLINT_DEV uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t d;
  asm("{ .reg .b16 h; cvt.u16.u32 h, %1; cvt.rn.f16x2.e4m3x2 %0, h; }" : "=r"(d) : "r"(v));
  return d;
}
FLINT_DEV uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
FLINT_DEV void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                             uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NVFP4 rows ra, rb: codes at row stride K/2 bytes, E4M3 block scales at row
// stride K/16 bytes.  Lane t's 32 elements of a 128-block are two 16-element
// scale blocks (2t, 2t+1); every code times its block scale is exact in fp16
// (at most 5 significant bits, magnitudes 2^-10 .. 2,688), so the f16 MMAs
// accumulate the exact products of the weights and the f16 activations in
// fp32, block after block, with no per-block step (the fragment holds x in
// natural order: pair j = elements 2j, 2j+1 of the lane's slice).
template <bool kGlobal>
FLINT_DEV void rows_dot_nvfp4(const uint8_t *qa, const uint8_t *qb, const uint8_t *sa,
                              const uint8_t *sb, int K, int B, const uint4 *frag, int lane,
                              float (&acc)[4]) {
  const int t = lane & 3;
  const int ng = K / kG;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  for (int G = 0; G < ng; ++G) {
    uint4 w0, w1;
    uint32_t s0b, s1b;
    if (kGlobal) {
      w0 = ld_stream(qa + 64 * G + 16 * t);
      w1 = ld_stream(qb + 64 * G + 16 * t);
      s0b = ld_nc_u16(sa + 8 * G + 2 * t);
      s1b = ld_nc_u16(sb + 8 * G + 2 * t);
    } else {
      w0 = *reinterpret_cast<const uint4 *>(qa + 64 * G + 16 * t);
      w1 = *reinterpret_cast<const uint4 *>(qb + 64 * G + 16 * t);
      s0b = *reinterpret_cast<const uint16_t *>(sa + 8 * G + 2 * t);
      s1b = *reinterpret_cast<const uint16_t *>(sb + 8 * G + 2 * t);
    }
    uint32_t ra[16], rb[16], xb[16];
    e2m1x8_to_f16x2(w0.x, ra), e2m1x8_to_f16x2(w0.y, ra + 4);
    e2m1x8_to_f16x2(w0.z, ra + 8), e2m1x8_to_f16x2(w0.w, ra + 12);
    e2m1x8_to_f16x2(w1.x, rb), e2m1x8_to_f16x2(w1.y, rb + 4);
    e2m1x8_to_f16x2(w1.z, rb + 8), e2m1x8_to_f16x2(w1.w, rb + 12);
    const uint32_t sa2 = e4m3x2_to_f16x2(s0b), sb2 = e4m3x2_to_f16x2(s1b);
    const uint32_t sa_lo = __byte_perm(sa2, 0, 0x1010), sa_hi = __byte_perm(sa2, 0, 0x3232);
    const uint32_t sb_lo = __byte_perm(sb2, 0, 0x1010), sb_hi = __byte_perm(sb2, 0, 0x3232);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ra[j] = hmul2(ra[j], sa_lo), ra[8 + j] = hmul2(ra[8 + j], sa_hi);
      rb[j] = hmul2(rb[j], sb_lo), rb[8 + j] = hmul2(rb[8 + j], sb_hi);
    }
    load_frag_compact(frag, G, B, lane, xb);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2)
      mma_f16_16816(acc, ra[2 * s2], rb[2 * s2], ra[2 * s2 + 1], rb[2 * s2 + 1], xb[2 * s2],
                    xb[2 * s2 + 1]);
  }
}

FLINT_DEV void rows_store(const float (&acc)[4], int n_a, int n_b, int N, int B, float *y, int t,
                          float (&best_v)[2], int (&best_i)[2]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int b = 2 * t + c;
    if (b < B) {
      if (n_a < N) {
        y[(size_t)b * N + n_a] = acc[c];
        if (better(acc[c], n_a, best_v[c], best_i[c])) best_v[c] = acc[c], best_i[c] = n_a;
      }
      if (n_b < N) {
        y[(size_t)b * N + n_b] = acc[2 + c];
        if (better(acc[2 + c], n_b, best_v[c], best_i[c])) best_v[c] = acc[2 + c], best_i[c] = n_b;
      }
    }
  }
}

// NVFP4 read-out: column c's sums times the global scale and 2^F of row c
FLINT_DEV void nv_scale(float (&acc)[4], int t, int B, const float *ymul) {
  const int c0 = 2 * t, c1 = 2 * t + 1;
  const float m0 = c0 < B ? ymul[c0] : 0.f, m1 = c1 < B ? ymul[c1] : 0.f;
  acc[0] *= m0, acc[1] *= m1, acc[2] *= m0, acc[3] *= m1;
}

template <int kFmt>
__global__ void __launch_bounds__(kGemvWarps * 32, 1)
    k_int4_gemv(const uint8_t *__restrict__ q, const uint16_t *__restrict__ s,
                const uint16_t *__restrict__ moff, float gsc, int N, int K,
                const uint16_t *__restrict__ x, int B, float *__restrict__ y,
                int32_t *__restrict__ argmax, char *__restrict__ ws, int stages,
                uint32_t stage_bytes, uint32_t frag_bytes) {
  constexpr bool kAffine = kFmt == kFmtAffine, kNv = kFmt == kFmtNvfp4;
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ unsigned int s_xmax[kMaxB];  // NVFP4: max |x| of each row (float bits)
  __shared__ float s_ymul[kMaxB];         // NVFP4: global scale x 2^F of each row
  uint4 *frag = reinterpret_cast<uint4 *>(sm);
  // affine: per-row sums of x over every 64-group, after the fragment
  float *xsum = reinterpret_cast<float *>(sm + align256((size_t)(K / kG) * 4 * B * 64));
  unsigned char *ring = sm + frag_bytes;
  __shared__ __align__(8) uint64_t full[16], empty[16];
  __shared__ ArgPartial s_part[kGemvWarps][kMaxB];
  __shared__ int s_last;
  __shared__ int s_next;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int ncons = (int)(blockDim.x >> 5) - 1, nthreads = (int)blockDim.x;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws);
  ArgPartial *parts = reinterpret_cast<ArgPartial *>(ws + align256(256));
  const int full_tiles = N / 16;
  const size_t rbytes = (size_t)K / 2;
  const int ng = K / kG, ng64 = K / 64;
  // per tile: codes, then scales (and, affine, offsets) of its 16 rows
  const uint32_t wbytes = (uint32_t)(8 * K),
                 sbytes = (uint32_t)(kAffine ? K / 2 : (kNv ? K : K / 4));

  if (tid < kMaxB) s_xmax[tid] = 0u;
  if (tid == 0) {
    s_next = 0;
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);  // each stage is released by the one warp that consumed it
    }
  }
  __syncthreads();
  bool failed = false;
  int issued = 0;  // producer lane: tiles whose copies it issued
  float best_v[2] = {0.f, 0.f};
  int best_i[2] = {-1, -1};

  if (warp == ncons) {
    // ---- producer: the weights do not depend on the previous kernel
    if (lane == 0) {
      int k = 0;
      for (int tile = blockIdx.x; tile < full_tiles; tile += gridDim.x, ++k) {
        const int st = k % stages;
        if (k >= stages && !gwait(&empty[st], ((k / stages) - 1) & 1)) {
          failed = true;
          break;
        }
        issued = k + 1;
        unsigned char *dst = ring + (size_t)st * stage_bytes;
        mbar_expect_tx(&full[st], wbytes + (kAffine ? 2 : 1) * sbytes);
        bulk_g2s(dst, q + (size_t)tile * wbytes, wbytes, &full[st]);
        bulk_g2s(dst + wbytes, reinterpret_cast<const unsigned char *>(s) + (size_t)tile * sbytes,
                 sbytes, &full[st]);
        if (kAffine)
          bulk_g2s(dst + wbytes + sbytes,
                   reinterpret_cast<const unsigned char *>(moff) + (size_t)tile * sbytes, sbytes,
                   &full[st]);
      }
    }
    pdl_wait();
    pdl_trigger();
  } else {
    // ---- consumers
    pdl_wait();
    pdl_trigger();
    const int nfrag = ng * 4 * B * 4;
    if (kNv) {
      // f16 activations: row b as x 2^-F_b with F_b putting max |x| in
      // [2^14, 2^15) (exact down to 2^-24 of the row's largest element);
      // the output is scaled back by 2^F_b and the global scale
      for (int task = tid; task < B * (K / 8); task += ncons * 32) {
        const int b = task / (K / 8), c = task % (K / 8);
        const uint4 v = ld_cg_v4(x + (size_t)b * K + 8 * c);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[i] << 16)),
                             fabsf(__uint_as_float(wv[i] & 0xffff0000u))));
        atomicMax(&s_xmax[b], __float_as_uint(m));
      }
      asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");
      if (tid < B) {
        const float m = __uint_as_float(s_xmax[tid]);
        const int F = m > 0.f ? min(max(ilogbf(m) - 14, -100), 100) : 0;
        s_ymul[tid] = gsc * ldexpf(1.f, F);
        s_xmax[tid] = (unsigned)(F + 128);  // reused: the shift, offset by 128
      }
      asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");
    }
    for (int task = tid; task < nfrag; task += ncons * 32) {
      const int q4 = task & 3, gt = (task >> 2) % (4 * B), G = (task >> 2) / (4 * B);
      const int gg = gt >> 2, tt = gt & 3;
      // symmetric: lane tt's 32 elements 32 tt ..; affine: 16 elements of each
      // 64-half, 64 (q4 / 2) + 16 tt + 8 (q4 % 2); NVFP4: 32 tt .. in natural
      // order, as f16
      const int e0 = kAffine ? 64 * (q4 >> 1) + 16 * tt + 8 * (q4 & 1) : 32 * tt + 8 * q4;
      const uint4 v = ld_cg_v4(x + (size_t)gg * K + 128 * G + e0);
      if (kNv) {
        const float sc = ldexpf(1.f, 128 - (int)s_xmax[gg]);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        uint32_t h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half lo = __float2half_rn(__uint_as_float(wv[i] << 16) * sc);
          const __half hi = __float2half_rn(__uint_as_float(wv[i] & 0xffff0000u) * sc);
          h[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        }
        frag[task] = make_uint4(h[0], h[1], h[2], h[3]);
      } else {
        frag[task] = bf16x8_to_pairs(v);
      }
    }
    if (kAffine) {  // sum of x over 64-group j of row b, elements in ascending order
      for (int task = tid; task < ng64 * B; task += ncons * 32) {
        const int j = task / B, b = task % B;
        const uint16_t *xr = x + (size_t)b * K + 64 * j;
        float sx = 0.f;
        for (int k = 0; k < 64; ++k)
          sx += bf16_bits_to_f32((uint32_t)__ldcg(reinterpret_cast<const unsigned short *>(xr + k)));
        xsum[task] = sx;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");  // consumers only
    const int my_tiles = full_tiles > (int)blockIdx.x
                             ? (full_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                             : 0;
    for (;;) {
      int k = 0;
      if (lane == 0) k = atomicAdd(&s_next, 1);
      k = __shfl_sync(0xffffffffu, k, 0);
      if (k >= my_tiles) break;
      const int tile = (int)blockIdx.x + k * (int)gridDim.x;
      const int st = k % stages;
      if (!gwait(&full[st], (k / stages) & 1)) {
        failed = true;
        break;
      }
      const unsigned char *src = ring + (size_t)st * stage_bytes;
      const uint16_t *sc = reinterpret_cast<const uint16_t *>(src + wbytes);
      float acc[4];
      if (kAffine) {
        const uint16_t *mo = reinterpret_cast<const uint16_t *>(src + wbytes + sbytes);
        rows_dot_affine<false>(src + g * rbytes, src + (g + 8) * rbytes, sc + g * ng64,
                               sc + (g + 8) * ng64, mo + g * ng64, mo + (g + 8) * ng64, K, B, frag,
                               xsum, lane, acc);
      } else if (kNv) {
        const uint8_t *sc8 = src + wbytes;
        rows_dot_nvfp4<false>(src + g * rbytes, src + (g + 8) * rbytes, sc8 + g * (K / 16),
                              sc8 + (g + 8) * (K / 16), K, B, frag, lane, acc);
        nv_scale(acc, t, B, s_ymul);
      } else {
        rows_dot<false>(src + g * rbytes, src + (g + 8) * rbytes, sc + g * ng, sc + (g + 8) * ng,
                        K, B, frag, lane, acc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      rows_store(acc, tile * 16 + g, tile * 16 + g + 8, N, B, y, t, best_v, best_i);
    }
    // the partial last tile (N % 16 rows), straight from global memory
    if (!failed && (N % 16) && warp == 0 && (int)blockIdx.x == full_tiles % (int)gridDim.x) {
      const int n_a = full_tiles * 16 + g, n_b = n_a + 8;
      const size_t ra = n_a < N ? (size_t)n_a : 0, rb = n_b < N ? (size_t)n_b : 0;
      float acc[4];
      if (kAffine) {
        rows_dot_affine<true>(q + ra * rbytes, q + rb * rbytes, s + ra * ng64, s + rb * ng64,
                              moff + ra * ng64, moff + rb * ng64, K, B, frag, xsum, lane, acc);
      } else if (kNv) {
        const uint8_t *s8 = reinterpret_cast<const uint8_t *>(s);
        rows_dot_nvfp4<true>(q + ra * rbytes, q + rb * rbytes, s8 + ra * (K / 16),
                             s8 + rb * (K / 16), K, B, frag, lane, acc);
        nv_scale(acc, t, B, s_ymul);
      } else
        rows_dot<true>(q + ra * rbytes, q + rb * rbytes, s + ra * ng, s + rb * ng, K, B, frag,
                       lane, acc);
      rows_store(acc, n_a, n_b, N, B, y, t, best_v, best_i);
    }
  }
  // lanes sharing t hold the same columns: reduce over g (xor 4, 8, 16)
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best_v[c], o);
      const int oi = __shfl_xor_sync(0xffffffffu, best_i[c], o);
      if (oi >= 0 && better(ov, oi, best_v[c], best_i[c])) best_v[c] = ov, best_i[c] = oi;
    }
    const int b = 2 * t + c;
    if (g == 0 && b < B) s_part[warp][b] = ArgPartial{best_v[c], best_i[c]};
  }
  if (__syncthreads_or(failed)) {
    if (tid == 0) set_status(ctrl + 1, kStatusTimeout);
    // copies still in flight land before the CTA exits: the last phase issued
    // on each stage (a completed phase passes at once)
    if (warp == ncons && lane == 0)
      for (int k = issued > stages ? issued - stages : 0; k < issued; ++k)
        mbar_wait(&full[k % stages], (uint32_t)((k / stages) & 1));
    return;
  }
  if (!argmax) return;
  if (tid < B) {
    ArgPartial p{0.f, -1};
    for (int w = 0; w <= ncons; ++w) {
      const ArgPartial o = s_part[w][tid];
      if (o.i >= 0 && better(o.v, o.i, p.v, p.i)) p = o;
    }
    parts[(size_t)blockIdx.x * B + tid] = p;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&ctrl[0], 1u);
    const bool last = prev == gridDim.x - 1;
    if (last) __threadfence();
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  // last CTA: every thread scans a strided share of the CTA partials, then
  // warps and the CTA reduce (order-free: lowest row wins ties).
  for (int b = 0; b < B; ++b) {
    ArgPartial p{0.f, -1};
    for (int cta = tid; cta < (int)gridDim.x; cta += nthreads) {
      const float ov = ld_cg_f32(&parts[(size_t)cta * B + b].v);
      const int oi = (int)ld_cg_u32(&parts[(size_t)cta * B + b].i);
      if (oi >= 0 && better(ov, oi, p.v, p.i)) p = ArgPartial{ov, oi};
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, p.v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, p.i, o);
      if (oi >= 0 && better(ov, oi, p.v, p.i)) p = ArgPartial{ov, oi};
    }
    if (lane == 0) s_part[warp][b] = p;
  }
  __syncthreads();
  if (tid < B) {
    ArgPartial p{0.f, -1};
    for (int w = 0; w <= ncons; ++w) {
      const ArgPartial o = s_part[w][tid];
      if (o.i >= 0 && better(o.v, o.i, p.v, p.i)) p = o;
    }
    argmax[tid] = p.i;
  }
  if (tid == 0) ctrl[0] = 0;
}

cudaError_t gemv_set_wait_polls(uint32_t polls) {
  if (polls == 0xFFFFFFFFu) polls = kWaitPolls;
  return cudaMemcpyToSymbol(g_gemv_polls, &polls, sizeof(polls));
}

template <int kFmt>
static cudaError_t launch_gemv_t(const uint8_t *q, const uint16_t *s, const uint16_t *m,
                                 float gsc, int N, int K, const uint16_t *x, int B, float *y,
                                 int32_t *argmax, char *ws, cudaStream_t st) {
  const GemvPlan p = gemv_plan(K, B, kFmt);
  note_step("k_int4_gemv plan");
  if (p.stages < 2) return cudaErrorInvalidValue;
  note_step("k_int4_gemv smem attribute");
  cudaError_t e = cudaFuncSetAttribute(k_int4_gemv<kFmt>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGemvSmemCap);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gemv_grid(N));
  const int ncons = p.stages < kMaxConsumers ? p.stages : kMaxConsumers;
  cfg.blockDim = dim3((ncons + 1) * 32);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_step("k_int4_gemv launch");
  return cudaLaunchKernelEx(&cfg, k_int4_gemv<kFmt>, q, s, m, gsc, N, K, x, B, y, argmax, ws,
                            p.stages, (uint32_t)p.stage_bytes, (uint32_t)p.frag_bytes);
}

cudaError_t launch_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x,
                        int B, float *y, int32_t *argmax, char *ws, cudaStream_t st) {
  return launch_gemv_t<kFmtSym>(q, s, nullptr, 0.f, N, K, x, B, y, argmax, ws, st);
}

cudaError_t launch_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int N,
                               int K, const uint16_t *x, int B, float *y, int32_t *argmax,
                               char *ws, cudaStream_t st) {
  return launch_gemv_t<kFmtAffine>(q, s, m, 0.f, N, K, x, B, y, argmax, ws, st);
}

cudaError_t launch_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float gsc, int N, int K,
                              const uint16_t *x, int B, float *y, int32_t *argmax, char *ws,
                              cudaStream_t st) {
  return launch_gemv_t<kFmtNvfp4>(q, reinterpret_cast<const uint16_t *>(s), nullptr, gsc, N, K, x,
                                  B, y, argmax, ws, st);
}

}  // namespace flint

// ------------------------------------------------------------------------
// Allocation-free variant.  The scratch the GEMV needs (completion counter,
// status word, one argmax partial per CTA and row) lives in this file-scope
// device array instead of a caller workspace.  Every GPU that loads the
// library holds it until the process exits.  In host code the array's name is
// only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, with the device current: on every call made outside a
// stream capture (so a context torn down by cudaDeviceReset and rebuilt gets
// the new address), and taken from the per-device cache inside a capture,
// where only a device that already made an uncaptured call can be used.
namespace {

constexpr size_t kNoAllocScratchBytes = 256 + 8 * 1024 * 8;  // counter/status + 1024 CTAs x 8 rows
static __device__ __align__(256) unsigned char g_gemv_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[64] = {};

// Device address of g_gemv_scratch on the current device.
cudaError_t scratch_address(cudaStream_t st, void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_gemv_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  } else if (!g_scratch_ptr[dev]) {
    return cudaErrorStreamCaptureUnsupported;  // no uncaptured call on this device yet
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" FLINT_API int flint_int4_gemv_noalloc(const uint8_t *q, const uint16_t *s, int N,
                                                  int K, const uint16_t *x, int B, float *y,
                                                  int32_t *argmax, void *stream) {
  auto aligned16 = [](const void *p) {
    return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
  };
  if (!aligned16(q) || !aligned16(s) || !aligned16(x) || !aligned16(y) || N < 1 || K < 128 ||
      K % 128 || K > 8192 || B < 1 || B > FLINT_MAX_DECODE_B)
    return FLINT_EINVAL;
  if (flint::gemv_ws_bytes(N, B) > kNoAllocScratchBytes) return FLINT_EINVAL;  // cannot happen for B <= 8
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *scratch = nullptr;
  cudaError_t e = flint::noted(scratch_address(st, &scratch), "no-alloc scratch address");
  // the counter and status word must start at zero; the partials need not
  if (e == cudaSuccess) e = flint::noted(cudaMemsetAsync(scratch, 0, 256, st), "no-alloc scratch clear");
  if (e == cudaSuccess)
    e = flint::launch_gemv(q, s, N, K, x, B, y, argmax, static_cast<char *>(scratch), st);
  return flint_from_cuda(e);
}

extern "C" FLINT_API int flint_int4_gemv_noalloc_status(int *status, void *stream) {
  if (!status) return FLINT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *scratch = nullptr;
  cudaError_t e = flint::noted(scratch_address(st, &scratch), "no-alloc scratch address");
  uint32_t ctrl[2] = {0, 0};
  if (e == cudaSuccess)
    e = flint::noted(cudaMemcpyAsync(ctrl, scratch, sizeof(ctrl), cudaMemcpyDeviceToHost, st),
                     "no-alloc status copy");
  if (e == cudaSuccess) e = flint::noted(cudaStreamSynchronize(st), "no-alloc status sync");
  if (e != cudaSuccess) return flint_from_cuda(e);
  *status = static_cast<int>(ctrl[1]);
  return FLINT_OK;
}
