// Device helpers shared by the Flint MoE kernels (sm_100a).
//
// Packed int4 rows (the library's weight format): byte j of a row holds
// element 2j in its low nibble and element 2j+1 in its high nibble, each a
// two's-complement code in [-8, 7]; one bf16 scale per 128 elements.
//
// The int4 x bf16 inner products run on mma.sync.m16n8k16 (bf16 in, fp32
// accumulate) used as a batch-wide multiply-accumulate engine: a warp holds a
// 16-row weight tile (rows g and g+8 per lane group g) against up to 8
// activation columns (the decode batch).  Decoding a 16-byte chunk of 32 codes
// into exact bf16 pairs takes 11 integer/bf16x2 instructions; the MMA then
// covers all columns at once, so the per-weight instruction cost does not grow
// with the batch and stays below the HBM delivery rate.
//
// k-order inside a lane's 32-element slice of a 128-element group: pair
// register r = 4q + p holds elements (8q + p, 8q + p + 4) of the slice (low
// half, high half).  Activation fragments are built in the same order, so
// the sum over k is the ordinary dot product, in a fixed order.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define FLINT_DEV __device__ __forceinline__

namespace flint {

constexpr int kH = 2048;
constexpr int kE = 256;
constexpr int kTopK = 6;
constexpr int kI = 512;
constexpr int kIs = 1024;
constexpr int kG = 128;
constexpr int kMaxB = 8;

// Device status codes (mirror FLINT_ETIMEOUT / FLINT_EDEVICE).
constexpr uint32_t kStatusTimeout = 3;
constexpr uint32_t kStatusDevice = 4;
// Bound on mbarrier polls before a wait is declared failed (~ seconds).
constexpr uint32_t kWaitPolls = 1u << 26;

FLINT_DEV void set_status(uint32_t *st, uint32_t code) { atomicCAS(st, 0u, code); }

// The bounds-checked build (FLINT_DEBUG, libflint_debug.so): FLINT_CHECK(ok,
// status) records a failed check as kStatusDevice in the call's status word
// (the first error recorded wins) and yields ok, so the caller skips the
// access it guards.  Every index a kernel reads back from device memory (slot
// words, expert indices, sorted rows, tile descriptors) passes one before it
// addresses memory.  In the release build it is the constant true and the
// check compiles away.
#ifdef FLINT_DEBUG
FLINT_DEV bool check_or_flag(bool ok, uint32_t *st) {
  if (!ok) set_status(st, kStatusDevice);
  return ok;
}
#define FLINT_CHECK(ok, st) ::flint::check_or_flag((ok), (st))
#else
#define FLINT_CHECK(ok, st) true
#endif

// ------------------------------------------------------------------ loads
// Weights: read once, never written while a kernel runs; keep them out of L1.
FLINT_DEV uint4 ld_stream(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
FLINT_DEV uint32_t ld_nc_u16(const void *p) {
  unsigned short v;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
// Data written by an earlier kernel of the chain (or by other CTAs of this
// one before a fence + counter): read at L2, never from a possibly stale L1
// line.  Plain (non-volatile) loads, so independent ones overlap.
FLINT_DEV uint4 ld_cg_v4(const void *p) { return __ldcg(reinterpret_cast<const uint4 *>(p)); }
FLINT_DEV uint32_t ld_cg_u32(const void *p) {
  return __ldcg(reinterpret_cast<const unsigned int *>(p));
}
FLINT_DEV float ld_cg_f32(const void *p) { return __ldcg(reinterpret_cast<const float *>(p)); }
FLINT_DEV double ld_cg_f64(const void *p) { return __ldcg(reinterpret_cast<const double *>(p)); }

FLINT_DEV uint32_t smem_addr_(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ PDL
FLINT_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
FLINT_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ numbers
FLINT_DEV float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
FLINT_DEV uint16_t f32_to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
// fp64 -> bf16, round to nearest even, without double rounding: truncate to
// fp32, fold any discarded bits into the fp32 sticky (lowest) bit ("round to
// odd", Boldo & Melquiond), then round the fp32 to bf16.
FLINT_DEV uint16_t f64_to_bf16_bits(double v) {
  float t = __double2float_rz(v);
  uint32_t u = __float_as_uint(t);
  if ((double)t != v) u |= 1u;
  uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(r >> 16);
}
// Order-preserving map of fp32 to uint32 (larger float -> larger key).
FLINT_DEV uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 32 int4 codes -> 16 bf16 pairs {c(8q+p), c(8q+p+4)} at register 4q+p, exact.
// (w & 0x000F000F) ^ 0x43084308 is bf16 128 + (nibble ^ 8) = 136 + code in
// each half; subtracting 136 (bf16 0x4308) leaves the code.
// (a & b) ^ c and (a & b) | c as one three-input logic operation each
// (truth tables 0x6A and 0xEA); written out because the compiler does not
// always fuse the pair
FLINT_DEV uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
FLINT_DEV uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

FLINT_DEV void int4x32_to_bf16x2(const uint4 w, uint32_t (&r)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t = and_xor(words[q] >> (4 * p), 0x000F000Fu, 0x43084308u);
      uint32_t c;
      asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(t), "r"(0x43084308u));
      r[4 * q + p] = c;
    }
  }
}

// The same for unsigned codes 0..15 (the affine format): (w & 0x000F000F) |
// 0x43004300 is the bf16 pair 128 + code, less 128 exact.
FLINT_DEV void uint4x32_to_bf16x2(const uint4 w, uint32_t (&r)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t = and_or(words[q] >> (4 * p), 0x000F000Fu, 0x43004300u);
      uint32_t c;
      asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(t), "r"(0x43004300u));
      r[4 * q + p] = c;
    }
  }
}

// 8 consecutive bf16 (one 16-byte load, 4 words) -> pairs {v[p], v[p+4]}.
FLINT_DEV uint4 bf16x8_to_pairs(const uint4 v) {
  uint4 o;
  o.x = __byte_perm(v.x, v.z, 0x5410);  // (v0, v4)
  o.y = __byte_perm(v.x, v.z, 0x7632);  // (v1, v5)
  o.z = __byte_perm(v.y, v.w, 0x5410);  // (v2, v6)
  o.w = __byte_perm(v.y, v.w, 0x7632);  // (v3, v7)
  return o;
}

FLINT_DEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 128-element group of a 16-row tile against an 8-column fragment:
// d = W[rows g, g+8][group] . X[group][cols 2t, 2t+1], fp32, from zero.
// ra/rb: the lane's 16 pair registers of rows g and g+8; xb: the lane's 16
// pair registers of the activation fragment.
FLINT_DEV void group_mma(const uint32_t (&ra)[16], const uint32_t (&rb)[16],
                         const uint32_t (&xb)[16], float (&d)[4]) {
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int s = 0; s < 8; ++s)
    mma_bf16_16816(d, ra[2 * s], rb[2 * s], ra[2 * s + 1], rb[2 * s + 1], xb[2 * s], xb[2 * s + 1]);
}
FLINT_DEV void group_mma_acc(const uint32_t (&ra)[16], const uint32_t (&rb)[16],
                             const uint32_t (&xb)[16], float (&d)[4]) {
#pragma unroll
  for (int s = 0; s < 8; ++s)
    mma_bf16_16816(d, ra[2 * s], rb[2 * s], ra[2 * s + 1], rb[2 * s + 1], xb[2 * s], xb[2 * s + 1]);
}

// Position of element k (0 <= k < K) of a column inside a hi/lo fragment
// image laid out [G][t][16 words] (one column): returns the bf16 slot index.
FLINT_DEV int frag_slot(int k) {
  const int G = k >> 7, t = (k >> 5) & 3, i = k & 31;
  const int q = i >> 3, p = i & 3, half = (i >> 2) & 1;
  return (((G * 4 + t) * 16) + 4 * q + p) * 2 + half;
}

// ------------------------------------------------------------------ cp.async (16 B, L2 only)
FLINT_DEV void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr_(dst)), "l"(src)
               : "memory");
}
FLINT_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ------------------------------------------------------------------ mbarrier / bulk copy
FLINT_DEV uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
FLINT_DEV void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Raise the expected transaction bytes of the current phase without arriving.
FLINT_DEV void mbar_add_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
FLINT_DEV void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
FLINT_DEV void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory; 16-byte aligned, size % 16 == 0.
FLINT_DEV void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// One poll of phase `parity` of `bar`.
FLINT_DEV bool mbar_try(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for phase `parity` of `bar`; false if it did not complete.
FLINT_DEV bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitPolls; ++i) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// The same wait for threads off the critical issue path: each poll may
// suspend the thread (up to the hint, in ns) until the phase completes, so
// waiting warps leave the issue slots to the warps that have work.
constexpr uint32_t kSleepPolls = 1u << 22;
FLINT_DEV bool mbar_wait_sleep(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSleepPolls; ++i) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (done) return true;
  }
  return false;
}

}  // namespace flint
