// Int4 GEMV with fused argmax for the output head ("How to Run Flint
// Locally", section "One decode step in bytes": lm_head is 150,144 x 2,048,
// read in full for every token; Recursive quantized it to 4 bits).
//
// Persistent kernel, one CTA per SM.  A producer warp streams whole 16-row
// tiles (16 x K/2 bytes of codes plus their scales, both contiguous in global
// memory) into a ring of shared-memory stages with a few large 1-D bulk
// copies, in order.  Consumer warps work in groups of four: the groups take
// the CTA's tiles round-robin and the four warps of a group split each tile's
// K into quarters, so a stage is held for a quarter of a tile's work and the
// ring keeps more stages in flight than there are groups.  The warps run
// their rows against up to 8 activation columns on mma.sync; the quarter-0
// warp adds the other quarters' partial sums in quarter order.  A final
// partial tile (N % 16 rows) is read straight from global memory.  Each warp
// keeps its best (value, row) per column; CTAs publish partials and the last
// CTA to finish reduces them (lowest row on ties), so the call is one launch.
//
// The symmetric and NVFP4 formats run the MMAs on fp16: the activations enter
// as fp16 times a power of two per row (the row's largest element in
// [2^14, 2^15)), which the read-out multiplies back.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace flint {

constexpr int kMaxConsumers = 16;
constexpr int kGemvWarps = kMaxConsumers + 1;  // producer = the last warp launched
constexpr int kTileWarps = 4;                   // consumer warps sharing one tile, split along K
constexpr int kRegWarps = 3 * kTileWarps + 1;   // register-fragment kernel: 3 groups + producer
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

// The wait of the consumers of ring unit k: fill k has been issued (so the
// fill before it on the same stage has landed and the parity cannot alias),
// then its stage barrier passes the parity of fill k; bounded like gwait.
FLINT_DEV bool gwait_unit(uint64_t *bar, uint32_t parity, const int *issued, int k) {
  const uint32_t n = *reinterpret_cast<volatile uint32_t *>(&g_gemv_polls);
  for (uint32_t i = 0; i < n; ++i)
    if (*reinterpret_cast<const volatile int *>(issued) > k && mbar_try(bar, parity)) return true;
  return false;
}

// Named barrier `id` over `n` threads that also ORs a predicate across them.
FLINT_DEV bool bar_or(uint32_t id, uint32_t n, bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 q, %1, 0; bar.red.or.pred p, %2, %3, q; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0u;
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

// Stage of one 16-row tile: the rows' codes in 2 parts (symmetric, NVFP4) or
// 4 parts (affine) of consecutive rows, part c shifted by c x 64 (or c x 32)
// bytes so that the rows one shared-memory load phase reads (2 rows of a
// 16-byte load, 4 of an 8-byte load) come from different parts and so from
// different banks (gemv_tile_row assigns the MMA rows); then the symmetric
// format's bf16 scales (16 x K/128) or the affine format's fp16 scales and
// offsets (16 x K/64 each) or the NVFP4 E4M3 block scales (16 x K/16 bytes),
// unshifted.  The activation fragment comes first in shared memory, then the
// symmetric format's -8 x (sum of x over every 128-group) ([K/128][8] fp32) or
// the affine format's sums of x over every 64-group ([K/64][B] fp32).
enum { kFmtSym = 0, kFmtAffine = 1, kFmtNvfp4 = 2 };

// tile row held by MMA row m (0..15): rows g and g + 8 of lanes 8p..8p+7
// (16-byte loads) or 16p..16p+15 (8-byte loads) fall in different parts
template <int kFmt>
FLINT_DEV int gemv_tile_row(int m) {
  if (kFmt == kFmtAffine) return 4 * (m & 3) + ((m >> 2) & 1) + 2 * (m >> 3);
  return ((m >> 1) & 3) + 4 * (m >> 3) + 8 * (m & 1);
}
// byte offset of tile row r inside the stage (row bytes rb = K/2)
template <int kFmt>
FLINT_DEV size_t gemv_row_off(int r, size_t rb) {
  return (size_t)r * rb + (kFmt == kFmtAffine ? 32 * (r >> 2) : 64 * (r >> 3));
}
constexpr int kCodesPad = 128;  // room for the parts' shifts

static GemvPlan gemv_plan(int K, int B, int fmt) {
  GemvPlan p;
  const size_t sbytes = fmt == kFmtSym ? (size_t)K / 4 : (size_t)K;
  p.stage_bytes = align256((size_t)8 * K + kCodesPad + sbytes);
  p.frag_bytes = align256((size_t)(K / kG) * 4 * B * 64);
  if (fmt == kFmtAffine) p.frag_bytes += align256((size_t)(K / 64) * B * 4);
  if (fmt == kFmtSym) p.frag_bytes += align256((size_t)(K / kG) * 8 * 4);
  p.stages = (int)((kGemvSmemCap - p.frag_bytes) / p.stage_bytes);
  if (p.stages > 16) p.stages = 16;
  p.smem = p.frag_bytes + (size_t)p.stages * p.stage_bytes;
  return p;
}

// The lane's 16 fragment registers of k-group G for the live columns (lanes
// g < B); lanes g >= B keep what they hold (zeros from the caller): their MMA
// columns are never stored.
FLINT_DEV void load_frag_live(const uint4 *frag, int G, int B, int lane, uint32_t (&x)[16]) {
  const int g = lane >> 2, t = lane & 3;
  if (g < B) {
    const uint4 *p = frag + (size_t)(G * 4 * B + g * 4 + t) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = p[i];
      x[4 * i] = v.x, x[4 * i + 1] = v.y, x[4 * i + 2] = v.z, x[4 * i + 3] = v.w;
    }
  }
}

// The eight 4-bit fields of one word (field k in bits 4k..4k+3) as four fp16
// pairs read as subnormals, exactly: register p holds fields (p, p + 4);
// fields 0, 2, 4, 6 sit in bits 0..3 of their half and read n 2^-24, fields
// 1, 3, 5, 7 in bits 4..7 and read n 2^-20, where n is the field XOR kFlip
// (8 turns a two's-complement code c into n = c + 8; 0 keeps an unsigned
// code).  One shift and four logic operations for 8 codes.
template <uint32_t kFlip>
FLINT_DEV void fields8_f16sub(uint32_t w, uint32_t *r) {
  const uint32_t w8 = w >> 8;
  r[0] = and_xor(w, 0x000F000Fu, kFlip * 0x00010001u);
  r[1] = and_xor(w, 0x00F000F0u, kFlip * 0x00100010u);
  r[2] = and_xor(w8, 0x000F000Fu, kFlip * 0x00010001u);
  r[3] = and_xor(w8, 0x00F000F0u, kFlip * 0x00100010u);
}

FLINT_DEV void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                             uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Symmetric rows ra, rb (codes, scales at row stride K/128) against the f16
// fragment: acc[0..1] row ra, acc[2..3] row rb, columns 2t, 2t+1, in the
// activations' shifted units.  Per 128-group the f16 MMAs sum the exact
// products (c + 8) 2^-24 x (the x entries of fields 1, 3, 5, 7 carry 2^-4 to
// match their 2^-20 reading), so 2^24 d - 8 sum(x) = sum(c x), and the group's
// scale multiplies it into the fp32 accumulator.  xsn: -8 sum(x) of each
// group and column ([K/128][8]).
template <bool kGlobal>
FLINT_DEV void rows_dot(const uint8_t *qa, const uint8_t *qb, const uint16_t *sa,
                        const uint16_t *sb, int G0, int G1, int B, const uint4 *frag,
                        const float *xsn, int lane, float (&acc)[4]) {
  const int t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  uint32_t xb[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) xb[i] = 0u;
#pragma unroll 2
  for (int G = G0; G < G1; ++G) {
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
    uint32_t ra[16], rbv[16];
    fields8_f16sub<8>(w0.x, ra), fields8_f16sub<8>(w0.y, ra + 4);
    fields8_f16sub<8>(w0.z, ra + 8), fields8_f16sub<8>(w0.w, ra + 12);
    fields8_f16sub<8>(w1.x, rbv), fields8_f16sub<8>(w1.y, rbv + 4);
    fields8_f16sub<8>(w1.z, rbv + 8), fields8_f16sub<8>(w1.w, rbv + 12);
    load_frag_live(frag, G, B, lane, xb);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j)
      mma_f16_16816(d, ra[2 * j], rbv[2 * j], ra[2 * j + 1], rbv[2 * j + 1], xb[2 * j],
                    xb[2 * j + 1]);
    const float2 xn = *reinterpret_cast<const float2 *>(xsn + 8 * G + 2 * t);
    const float s0 = bf16_bits_to_f32(s0b), s1 = bf16_bits_to_f32(s1b);
    acc[0] = fmaf(s0, fmaf(d[0], 0x1p24f, xn.x), acc[0]);
    acc[1] = fmaf(s0, fmaf(d[1], 0x1p24f, xn.y), acc[1]);
    acc[2] = fmaf(s1, fmaf(d[2], 0x1p24f, xn.x), acc[2]);
    acc[3] = fmaf(s1, fmaf(d[3], 0x1p24f, xn.y), acc[3]);
  }
}

// The same with the warp's kGW k-groups G0 .. G0 + kGW - 1 fully unrolled and
// their fragment (xr) and -8 sum(x) (xn, columns 2t, 2t+1) held in registers
// for the whole kernel.
template <int kGW>
FLINT_DEV void rows_dot_reg(const uint8_t *qa, const uint8_t *qb, const uint16_t *sa,
                            const uint16_t *sb, const uint32_t (&xr)[kGW][16],
                            const float2 (&xn)[kGW], int lane, float (&acc)[4]) {
  const int t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
  for (int j = 0; j < kGW; ++j) {
    const uint4 w0 = *reinterpret_cast<const uint4 *>(qa + 64 * j + 16 * t);
    const uint4 w1 = *reinterpret_cast<const uint4 *>(qb + 64 * j + 16 * t);
    const float s0 = bf16_bits_to_f32(sa[j]), s1 = bf16_bits_to_f32(sb[j]);
    const uint32_t wa[4] = {w0.x, w0.y, w0.z, w0.w}, wb[4] = {w1.x, w1.y, w1.z, w1.w};
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // word q: fields (p, p + 4) in register p
      uint32_t ra[4], rb[4];
      fields8_f16sub<8>(wa[q], ra);
      fields8_f16sub<8>(wb[q], rb);
      mma_f16_16816(d, ra[0], rb[0], ra[1], rb[1], xr[j][4 * q], xr[j][4 * q + 1]);
      mma_f16_16816(d, ra[2], rb[2], ra[3], rb[3], xr[j][4 * q + 2], xr[j][4 * q + 3]);
    }
    acc[0] = fmaf(s0, fmaf(d[0], 0x1p24f, xn[j].x), acc[0]);
    acc[1] = fmaf(s0, fmaf(d[1], 0x1p24f, xn[j].y), acc[1]);
    acc[2] = fmaf(s1, fmaf(d[2], 0x1p24f, xn[j].x), acc[2]);
    acc[3] = fmaf(s1, fmaf(d[3], 0x1p24f, xn[j].y), acc[3]);
  }
}

// Affine rows ra, rb: codes at row stride K/2 bytes; fp16 scales and offsets
// at row stride K/64.  Lane t takes elements 64h + 16t .. 64h + 16t + 15 of
// half h of each 128-element block, so MMAs 4h .. 4h+3 cover 64-group 2G + h
// alone: the f16 MMAs sum the exact products n 2^-24 x of the unsigned codes
// n (fields read as subnormals, as in the symmetric path), and
// y += scale * 2^24 d + offset * sum(x over the group), in the activations'
// shifted units.  xsum: [K/64][B] sums of the shifted x.
template <bool kGlobal>
FLINT_DEV void rows_dot_affine(const uint8_t *qa, const uint8_t *qb, const uint16_t *sa,
                               const uint16_t *sb, const uint16_t *ma, const uint16_t *mb, int G0,
                               int G1, int B, const uint4 *frag, const float *xsum, int lane,
                               float (&acc)[4]) {
  const int t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  uint32_t xb[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) xb[i] = 0u;
  for (int G = G0; G < G1; ++G) {
    load_frag_live(frag, G, B, lane, xb);
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
      fields8_f16sub<0>(w0.x, ra), fields8_f16sub<0>(w0.y, ra + 4);
      fields8_f16sub<0>(w1.x, rb), fields8_f16sub<0>(w1.y, rb + 4);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_f16_16816(d, ra[2 * j], rb[2 * j], ra[2 * j + 1], rb[2 * j + 1], xb[8 * h + 2 * j],
                      xb[8 * h + 2 * j + 1]);
      const float s0 = __half2float(__ushort_as_half((unsigned short)s0b)) * 0x1p24f;
      const float s1 = __half2float(__ushort_as_half((unsigned short)s1b)) * 0x1p24f;
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

// NVFP4 rows ra, rb: codes at row stride K/2 bytes, E4M3 block scales at row
// stride K/16 bytes.  Lane t's 32 elements of a 128-block are two 16-element
// scale blocks (2t, 2t+1); every code times its block scale is exact in fp16
// (at most 6 significant bits, magnitudes 2^-10 .. 2,688), so the f16 MMAs
// accumulate the exact products of the weights and the f16 activations in
// fp32, block after block, with no per-block step (the fragment holds x in
// natural order: pair j = elements 2j, 2j+1 of the lane's slice).
template <bool kGlobal>
FLINT_DEV void rows_dot_nvfp4(const uint8_t *qa, const uint8_t *qb, const uint8_t *sa,
                              const uint8_t *sb, int G0, int G1, int B, const uint4 *frag,
                              int lane, float (&acc)[4]) {
  const int t = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  uint32_t xb[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) xb[i] = 0u;
  for (int G = G0; G < G1; ++G) {
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
    uint32_t ra[16], rb[16];
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
    load_frag_live(frag, G, B, lane, xb);
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

// f16-activation read-out: column c's sums times 2^F of row c (NVFP4: and the
// global scale)
FLINT_DEV void col_scale(float (&acc)[4], int t, int B, const float *ymul) {
  const int c0 = 2 * t, c1 = 2 * t + 1;
  const float m0 = c0 < B ? ymul[c0] : 0.f, m1 = c1 < B ? ymul[c1] : 0.f;
  acc[0] *= m0, acc[1] *= m1, acc[2] *= m0, acc[3] *= m1;
}

// kGW > 0 (symmetric format, K = 512 kGW): every consumer warp holds its
// K-quarter's activation fragment in registers; kGW = 0: the general path.
template <int kFmt, int kGW>
__global__ void __launch_bounds__((kGW ? kRegWarps : kGemvWarps) * 32, 1)
    k_int4_gemv(const uint8_t *__restrict__ q, const uint16_t *__restrict__ s,
                const uint16_t *__restrict__ moff, float gsc, int N, int K,
                const uint16_t *__restrict__ x, int B, float *__restrict__ y,
                int32_t *__restrict__ argmax, char *__restrict__ ws, int stages,
                uint32_t stage_bytes, uint32_t frag_bytes) {
  constexpr bool kAffine = kFmt == kFmtAffine, kNv = kFmt == kFmtNvfp4, kSym = kFmt == kFmtSym;
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ unsigned int s_xmax[kMaxB];  // max |x| of each row (float bits), then its shift
  __shared__ float s_ymul[kMaxB];         // 2^F of each row (NVFP4: times the global scale)
  uint4 *frag = reinterpret_cast<uint4 *>(sm);
  // after the fragment: affine, the sums of x over every 64-group ([K/64][B]);
  // symmetric, -8 x the sums of x over every 128-group ([K/128][8])
  float *xsum = reinterpret_cast<float *>(sm + align256((size_t)(K / kG) * 4 * B * 64));
  unsigned char *ring = sm + frag_bytes;
  __shared__ __align__(8) uint64_t full[16], empty[16];
  __shared__ ArgPartial s_part[kGemvWarps][kMaxB];
  __shared__ int s_last;
  __shared__ int s_issued;  // ring units whose copies the producer has issued
  // partial sums of the tile's K-quarters 1..3 for its quarter-0 warp
  __shared__ float4 s_red[kMaxConsumers / kTileWarps][2][kTileWarps - 1][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int ncons = (int)(blockDim.x >> 5) - 1, nthreads = (int)blockDim.x;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws);
  ArgPartial *parts = reinterpret_cast<ArgPartial *>(ws + align256(256));
  const int full_tiles = N / 16;
  const size_t rbytes = (size_t)K / 2, cbytes = (size_t)8 * K + kCodesPad;
  const int ng = K / kG, ng64 = K / 64;
  // per tile: codes, then scales (and, affine, offsets) of its 16 rows
  const uint32_t wbytes = (uint32_t)(8 * K),
                 sbytes = (uint32_t)(kAffine ? K / 2 : (kNv ? K : K / 4));

  if (tid < kMaxB) s_xmax[tid] = 0u;
  if (tid == 0) {
    s_issued = 0;
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);  // released by the quarter-0 warp of the group that read it
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
        unsigned char *dst = ring + (size_t)st * stage_bytes;
        mbar_expect_tx(&full[st], wbytes + (kAffine ? 2 : 1) * sbytes);
        constexpr int kParts = kAffine ? 4 : 2, kRows = 16 / kParts;
#pragma unroll
        for (int c = 0; c < kParts; ++c)
          bulk_g2s(dst + gemv_row_off<kFmt>(c * kRows, rbytes),
                   q + (size_t)tile * wbytes + (size_t)c * kRows * rbytes,
                   (uint32_t)(kRows * rbytes), &full[st]);
        bulk_g2s(dst + cbytes,
                 reinterpret_cast<const unsigned char *>(s) + (size_t)tile * sbytes, sbytes,
                 &full[st]);
        if (kAffine)
          bulk_g2s(dst + cbytes + sbytes,
                   reinterpret_cast<const unsigned char *>(moff) + (size_t)tile * sbytes, sbytes,
                   &full[st]);
        issued = k + 1;
        *reinterpret_cast<volatile int *>(&s_issued) = issued;
      }
    }
    pdl_wait();
    pdl_trigger();
  } else {
    // ---- consumers
    pdl_wait();
    pdl_trigger();
    const int nfrag = ng * 4 * B * 4;
    if (kSym)
      for (int i = tid; i < ng * 8; i += ncons * 32) xsum[i] = 0.f;
    {
      // f16 activations: row b as x 2^-F_b with F_b putting max |x| in
      // [2^14, 2^15) (exact down to 2^-24 of the row's largest element);
      // the output is scaled back by 2^F_b (NVFP4: and the global scale).
      // One 16-byte chunk per thread, a maximum over each half-warp (16
      // consecutive chunks of one row, K/8 being a multiple of 16), then one
      // shared atomic per half-warp
      for (int task = tid; task < B * (K / 8); task += ncons * 32) {
        const int b = task / (K / 8), c = task % (K / 8);
        const uint4 v = ld_cg_v4(x + (size_t)b * K + 8 * c);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[i] << 16)),
                             fabsf(__uint_as_float(wv[i] & 0xffff0000u))));
        const unsigned hmask = 0xFFFFu << (lane & 16);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(hmask, m, o));
        if ((lane & 15) == 0) atomicMax(&s_xmax[b], __float_as_uint(m));
      }
      asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");
      if (tid < B) {
        const float m = __uint_as_float(s_xmax[tid]);
        const int F = m > 0.f ? min(max(ilogbf(m) - 14, -100), 100) : 0;
        s_ymul[tid] = (kNv ? gsc : 1.f) * ldexpf(1.f, F);
        s_xmax[tid] = (unsigned)(F + 128);  // reused: the shift, offset by 128
      }
      asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");
    }
#pragma unroll 2
    for (int task = tid; task < nfrag; task += ncons * 32) {
      const int q4 = task & 3, gt = (task >> 2) % (4 * B), G = (task >> 2) / (4 * B);
      const int gg = gt >> 2, tt = gt & 3;
      // symmetric and NVFP4: lane tt's 32 elements 32 tt .. of the group;
      // affine: 16 elements of each 64-half, 64 (q4 / 2) + 16 tt + 8 (q4 % 2)
      const int e0 = kAffine ? 64 * (q4 >> 1) + 16 * tt + 8 * (q4 & 1) : 32 * tt + 8 * q4;
      const uint4 v = ld_cg_v4(x + (size_t)gg * K + 128 * G + e0);
      const float sc = ldexpf(1.f, 128 - (int)s_xmax[gg]);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t h[4];
      float part = 0.f;  // sum of the 8 shifted values, in element order
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (kNv) {  // natural order: pair i = elements 2i, 2i+1
          const __half lo = __float2half_rn(__uint_as_float(wv[i] << 16) * sc);
          const __half hi = __float2half_rn(__uint_as_float(wv[i] & 0xffff0000u) * sc);
          h[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        } else {    // symmetric, affine: pair i = elements i, i + 4; odd i carry 2^-4
          const uint32_t wl = wv[i >> 1], wh = wv[(i >> 1) + 2];
          const float xl = __uint_as_float((i & 1) ? (wl & 0xffff0000u) : (wl << 16)) * sc;
          const float xh = __uint_as_float((i & 1) ? (wh & 0xffff0000u) : (wh << 16)) * sc;
          const float m = (i & 1) ? 0.0625f : 1.f;
          const __half lo = __float2half_rn(xl * m), hi = __float2half_rn(xh * m);
          h[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        }
      }
      if (!kNv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t we = wv[e >> 1];
          part += __half2float(__float2half_rn(
              __uint_as_float((e & 1) ? (we & 0xffff0000u) : (we << 16)) * sc));
        }
        // the 16 tasks of one (group, row) are consecutive and share a
        // half-warp, lane (tt, q4) at 4 tt + q4: a fixed tree over them;
        // affine keeps the 64-groups q4 / 2 = 0, 1 apart (no xor 2)
        const unsigned hmask = 0xFFFFu << (lane & 16);
        part += __shfl_xor_sync(hmask, part, 1);
        if (kSym) part += __shfl_xor_sync(hmask, part, 2);
        part += __shfl_xor_sync(hmask, part, 4);
        part += __shfl_xor_sync(hmask, part, 8);
        if (kSym && (task & 15) == 0) xsum[G * 8 + gg] = -8.f * part;
        if (kAffine && (task & 13) == 0) xsum[(2 * G + (q4 >> 1)) * B + gg] = part;
      }
      frag[task] = make_uint4(h[0], h[1], h[2], h[3]);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(ncons * 32) : "memory");  // consumers only
    const int my_tiles = full_tiles > (int)blockIdx.x
                             ? (full_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                             : 0;
    const int ra_t = gemv_tile_row<kFmt>(g), rb_t = gemv_tile_row<kFmt>(g + 8);
    // groups of kTileWarps warps take the CTA's tiles round-robin; warp wq of
    // a group takes k-groups [G0, G1) of every tile, and its quarter-0 warp
    // adds the others' partial sums in quarter order, stores the rows and
    // releases the stage once the group's barrier shows every warp done.
    const int ngroups = ncons / kTileWarps, grp = warp / kTileWarps, wq = warp % kTileWarps;
    const int G0 = wq * ng / kTileWarps, G1 = (wq + 1) * ng / kTileWarps;
    constexpr int kR = kGW > 0 ? kGW : 1;
    uint32_t xr[kR][16];
    float2 xn[kR];
    if (kGW > 0) {
#pragma unroll
      for (int j = 0; j < kR; ++j) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xr[j][i] = 0u;
        load_frag_live(frag, G0 + j, B, lane, xr[j]);
        xn[j] = *reinterpret_cast<const float2 *>(xsum + 8 * (G0 + j) + 2 * t);
      }
    }
    for (int i = 0;; ++i) {
      const int k = grp + i * ngroups;
      if (k >= my_tiles) break;
      const int tile = (int)blockIdx.x + k * (int)gridDim.x;
      const int st = k % stages;
      const bool ok = __all_sync(0xffffffffu, gwait_unit(&full[st], (k / stages) & 1, &s_issued, k));
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) {
        const unsigned char *src = ring + (size_t)st * stage_bytes;
        const uint16_t *sc = reinterpret_cast<const uint16_t *>(src + cbytes);
        const unsigned char *qa = src + gemv_row_off<kFmt>(ra_t, rbytes),
                            *qb = src + gemv_row_off<kFmt>(rb_t, rbytes);
        if (kAffine) {
          const uint16_t *mo = reinterpret_cast<const uint16_t *>(src + cbytes + sbytes);
          rows_dot_affine<false>(qa, qb, sc + ra_t * ng64, sc + rb_t * ng64, mo + ra_t * ng64,
                                 mo + rb_t * ng64, G0, G1, B, frag, xsum, lane, acc);
        } else if (kNv) {
          const uint8_t *sc8 = src + cbytes;
          rows_dot_nvfp4<false>(qa, qb, sc8 + ra_t * (K / 16), sc8 + rb_t * (K / 16), G0, G1, B,
                                frag, lane, acc);
        } else if (kGW > 0) {
          rows_dot_reg<kR>(qa + 64 * G0, qb + 64 * G0, sc + ra_t * ng + G0, sc + rb_t * ng + G0, xr,
                           xn, lane, acc);
        } else {
          rows_dot<false>(qa, qb, sc + ra_t * ng, sc + rb_t * ng, G0, G1, B, frag, xsum, lane,
                          acc);
        }
      }
      if (wq != 0) s_red[grp][i & 1][wq - 1][lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (bar_or(2 + grp, kTileWarps * 32, !ok)) {
        failed = true;
        break;
      }
      if (wq == 0) {
#pragma unroll
        for (int j = 0; j < kTileWarps - 1; ++j) {
          const float4 o = s_red[grp][i & 1][j][lane];
          acc[0] += o.x, acc[1] += o.y, acc[2] += o.z, acc[3] += o.w;
        }
        col_scale(acc, t, B, s_ymul);
        if (lane == 0) mbar_arrive(&empty[st]);
        rows_store(acc, tile * 16 + ra_t, tile * 16 + rb_t, N, B, y, t, best_v, best_i);
      }
    }
    // the partial last tile (N % 16 rows), straight from global memory
    if (!failed && (N % 16) && warp == 0 && (int)blockIdx.x == full_tiles % (int)gridDim.x) {
      const int n_a = full_tiles * 16 + g, n_b = n_a + 8;
      const size_t ra = n_a < N ? (size_t)n_a : 0, rb = n_b < N ? (size_t)n_b : 0;
      float acc[4];
      if (kAffine) {
        rows_dot_affine<true>(q + ra * rbytes, q + rb * rbytes, s + ra * ng64, s + rb * ng64,
                              moff + ra * ng64, moff + rb * ng64, 0, ng, B, frag, xsum, lane,
                              acc);
        col_scale(acc, t, B, s_ymul);
      } else if (kNv) {
        const uint8_t *s8 = reinterpret_cast<const uint8_t *>(s);
        rows_dot_nvfp4<true>(q + ra * rbytes, q + rb * rbytes, s8 + ra * (K / 16),
                             s8 + rb * (K / 16), 0, ng, B, frag, lane, acc);
        col_scale(acc, t, B, s_ymul);
      } else {
        rows_dot<true>(q + ra * rbytes, q + rb * rbytes, s + ra * ng, s + rb * ng, 0, ng, B, frag,
                       xsum, lane, acc);
        col_scale(acc, t, B, s_ymul);
      }
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

template <int kFmt, int kGW>
static cudaError_t launch_gemv_t(const uint8_t *q, const uint16_t *s, const uint16_t *m,
                                 float gsc, int N, int K, const uint16_t *x, int B, float *y,
                                 int32_t *argmax, char *ws, cudaStream_t st) {
  const GemvPlan p = gemv_plan(K, B, kFmt);
  note_step("k_int4_gemv plan");
  if (p.stages < 2) return cudaErrorInvalidValue;
  note_step("k_int4_gemv smem attribute");
  cudaError_t e = cudaFuncSetAttribute(k_int4_gemv<kFmt, kGW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGemvSmemCap);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gemv_grid(N));
  // whole groups of kTileWarps consumers, at least one stage more than groups
  const int max_groups = (kGW ? kRegWarps - 1 : kMaxConsumers) / kTileWarps;
  int ngroups = p.stages - 1;
  if (ngroups > max_groups) ngroups = max_groups;
  if (ngroups < 1) ngroups = 1;
  const int ncons = ngroups * kTileWarps;
  cfg.blockDim = dim3((ncons + 1) * 32);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_step("k_int4_gemv launch");
  return cudaLaunchKernelEx(&cfg, k_int4_gemv<kFmt, kGW>, q, s, m, gsc, N, K, x, B, y, argmax,
                            ws, p.stages, (uint32_t)p.stage_bytes, (uint32_t)p.frag_bytes);
}

cudaError_t launch_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x,
                        int B, float *y, int32_t *argmax, char *ws, cudaStream_t st) {
  // K = 512, 1024, 2048: the register-fragment kernel (a K-quarter of 1, 2, 4 groups per warp)
  if (K == 2048) return launch_gemv_t<kFmtSym, 4>(q, s, nullptr, 0.f, N, K, x, B, y, argmax, ws, st);
  if (K == 1024) return launch_gemv_t<kFmtSym, 2>(q, s, nullptr, 0.f, N, K, x, B, y, argmax, ws, st);
  if (K == 512) return launch_gemv_t<kFmtSym, 1>(q, s, nullptr, 0.f, N, K, x, B, y, argmax, ws, st);
  return launch_gemv_t<kFmtSym, 0>(q, s, nullptr, 0.f, N, K, x, B, y, argmax, ws, st);
}

cudaError_t launch_gemv_affine(const uint8_t *q, const uint16_t *s, const uint16_t *m, int N,
                               int K, const uint16_t *x, int B, float *y, int32_t *argmax,
                               char *ws, cudaStream_t st) {
  return launch_gemv_t<kFmtAffine, 0>(q, s, m, 0.f, N, K, x, B, y, argmax, ws, st);
}

cudaError_t launch_gemv_nvfp4(const uint8_t *q, const uint8_t *s, float gsc, int N, int K,
                              const uint16_t *x, int B, float *y, int32_t *argmax, char *ws,
                              cudaStream_t st) {
  return launch_gemv_t<kFmtNvfp4, 0>(q, reinterpret_cast<const uint16_t *>(s), nullptr, gsc, N, K, x,
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
