// Prefill of the Flint MoE block for T tokens.
//
// The block is defined per token ("How to Run Flint Locally", section "The
// architecture, from config.json"); for many tokens it is computed as
//   1. router logits for all tokens (bf16 products on mma.sync, fp32
//      partials of each 128-wide k-group summed in fp64) and a per-token
//      top-6 with the same selection rule as decode;
//   2. a stable token-by-expert counting sort: per-chunk bitmask counts, one
//      scan over (expert, chunk), then positions in token order inside every
//      expert; each expert's group is padded to the 128-token tile;
//   3. a gather of the routed token rows;
//   4. grouped GEMM 1 (gate/up + SwiGLU) and grouped GEMM 2 (down, scaled by
//      the routing weight) on the tcgen05 tensor cores: the weights are the
//      128-row A operand, their int4 codes land in shared memory by TMA and
//      four warps dequantize them to bf16 tiles in the 128-byte-swizzled
//      K-major layout the MMA reads; the tokens are the N operand, loaded by
//      TMA; the fp32 accumulator lives in tensor memory.  The shared expert
//      is one more group that covers every token;
//   5. a fixed-order combine per token (its experts in ascending index, then
//      the shared expert).
// "What vLLM changed" on the same page: the small-batch MoE kernels that read
// only the selected experts were also the largest prefill gain.  SwiGLU
// intermediates travel as hi/lo bf16 pairs: bf16 range (TandemLLM "21 Flint",
// section 21.2 reports routed activations up to 2.6e5, past fp16) with about
// 16 significant bits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace flint {

// ============================================================== router (T tokens)
constexpr int kRtTok = 64;  // tokens per CTA (8 column blocks of 8)

// 16 warps: warp w multiplies experts 16w .. 16w+15 against the CTA's 64 tokens.
__global__ void __launch_bounds__(512)
    k_pf_router(LayerArgs L, const uint16_t *__restrict__ x, int T, float *__restrict__ z) {
  // fragment of one k-half: [8 groups][8 blocks][4 words q][32 lanes] (uint4),
  // so the 32 lanes of a load read 512 consecutive bytes
  extern __shared__ __align__(128) unsigned char sm[];
  uint4 *frag = reinterpret_cast<uint4 *>(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int t0 = blockIdx.x * kRtTok, e0 = 16 * warp;
  double acc[8][4];
#pragma unroll
  for (int nb = 0; nb < 8; ++nb)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nb][i] = 0.0;

  for (int half = 0; half < 2; ++half) {
    __syncthreads();
    for (int task = tid; task < 8 * 8 * 32 * 4; task += 512) {
      const int ln = task & 31, q = (task >> 5) & 3, nb = (task >> 7) & 7, Gl = task >> 10;
      const int tok = t0 + 8 * nb + (ln >> 2);
      const int k0 = 128 * (8 * half + Gl) + 32 * (ln & 3) + 8 * q;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (tok < T) v = ld_cg_v4(x + (size_t)tok * kH + k0);
      frag[task] = bf16x8_to_pairs(v);
    }
    __syncthreads();
#pragma unroll 1
    for (int Gl = 0; Gl < 8; ++Gl) {
      const int G = 8 * half + Gl;
      const uint16_t *ra = L.router_w + (size_t)(e0 + g) * kH + 128 * G + 32 * t;
      uint32_t a[16], b[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 p0 = bf16x8_to_pairs(ld_stream(ra + 8 * q));
        const uint4 p1 = bf16x8_to_pairs(ld_stream(ra + 8 * kH + 8 * q));
        a[4 * q] = p0.x, a[4 * q + 1] = p0.y, a[4 * q + 2] = p0.z, a[4 * q + 3] = p0.w;
        b[4 * q] = p1.x, b[4 * q + 1] = p1.y, b[4 * q + 2] = p1.z, b[4 * q + 3] = p1.w;
      }
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
        uint32_t xb[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = frag[((Gl * 8 + nb) * 4 + q) * 32 + lane];
          xb[4 * q] = v.x, xb[4 * q + 1] = v.y, xb[4 * q + 2] = v.z, xb[4 * q + 3] = v.w;
        }
        float d[4];
        group_mma(a, b, xb, d);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nb][i] += (double)d[i];
      }
    }
  }
#pragma unroll
  for (int nb = 0; nb < 8; ++nb)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int tok = t0 + 8 * nb + 2 * t + c;
      if (tok < T) {
        z[(size_t)tok * kE + e0 + g] = (float)acc[nb][c];
        z[(size_t)tok * kE + e0 + g + 8] = (float)acc[nb][2 + c];
      }
    }
}

// One warp per token: sigmoid, bias, top-6 (lower index wins ties), weights;
// selection order to sel_*, ascending expert order to asc_*.
__global__ void __launch_bounds__(256)
    k_pf_topk(const float *__restrict__ router_b, const float *__restrict__ z, int T,
              int32_t *__restrict__ sel_idx, float *__restrict__ sel_w, int32_t *__restrict__ asc_e,
              float *__restrict__ asc_w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = blockIdx.x * 8 + warp;
  if (tok >= T) return;
  float sv[8];
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float zf = z[(size_t)tok * kE + lane + 32 * i];
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
FLINT_DEV void chunk_bits(const int32_t *asc_e, int T, int c, uint32_t (*bits)[8]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kE * 8; i += 256) bits[i >> 3][i & 7] = 0u;
  __syncthreads();
  const int tok = c * kPfChunk + tid;
  if (tok < T)
    for (int j = 0; j < kTopK; ++j) atomicOr(&bits[asc_e[(size_t)tok * kTopK + j]][warp], 1u << lane);
  __syncthreads();
}

__global__ void __launch_bounds__(256)
    k_pf_count(const int32_t *__restrict__ asc_e, int T, int32_t *__restrict__ chunk_cnt) {
  __shared__ uint32_t bits[kE][8];
  chunk_bits(asc_e, T, blockIdx.x, bits);
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

FLINT_DEV uint32_t pack_tile(int e, int mt, int nt) {
  return (uint32_t)e | ((uint32_t)mt << 9) | ((uint32_t)nt << 14);
}

// One CTA of 256 threads (one per expert): chunk offsets, expert counts,
// padded bases, padding rows of the permutation, and both GEMM tile lists
// (the 16 or 8 row tiles of one token tile are adjacent, so the token tile is
// reused from L2).
__global__ void __launch_bounds__(256)
    k_pf_scan(int T, int nchunks, const int32_t *__restrict__ chunk_cnt,
              int32_t *__restrict__ chunk_off, int32_t *__restrict__ ebase,
              int32_t *__restrict__ ecount, int32_t *__restrict__ perm,
              uint32_t *__restrict__ tiles1, uint32_t *__restrict__ tiles2,
              uint32_t *__restrict__ ctrl) {
  __shared__ int s_warp[8];
  const int e = threadIdx.x;
  int off = 0;
#pragma unroll 8
  for (int c = 0; c < nchunks; ++c) {
    chunk_off[(size_t)c * kE + e] = off;
    off += chunk_cnt[(size_t)c * kE + e];
  }
  ecount[e] = off;
  const int ntile = (off + kPfTile - 1) / kPfTile;
  int total_rows, total1, total2;
  const int base = block_scan(ntile * kPfTile, s_warp, &total_rows);
  const int o1 = block_scan(8 * ntile, s_warp, &total1);
  const int o2 = block_scan(16 * ntile, s_warp, &total2);
  ebase[e] = base;
  if (e == 0) ebase[kE] = total_rows;
  for (int p = base + off; p < base + ntile * kPfTile; ++p) perm[p] = -1;
  for (int nt = 0; nt < ntile; ++nt) {
    for (int mt = 0; mt < 8; ++mt) tiles1[o1 + nt * 8 + mt] = pack_tile(e, mt, nt);
    for (int mt = 0; mt < 16; ++mt) tiles2[o2 + nt * 16 + mt] = pack_tile(e, mt, nt);
  }
  // the shared expert: one group over all T tokens
  const int nsh = (T + kPfTile - 1) / kPfTile;
  for (int i = e; i < 16 * nsh; i += kE) {
    tiles1[total1 + i] = pack_tile(kE, i & 15, i >> 4);
    tiles2[total2 + i] = pack_tile(kE, i & 15, i >> 4);
  }
  if (e == 0) {
    ctrl[3] = (uint32_t)(total1 + 16 * nsh);
    ctrl[4] = (uint32_t)(total2 + 16 * nsh);
    ctrl[5] = (uint32_t)total_rows;
  }
}

__global__ void __launch_bounds__(256)
    k_pf_place(const int32_t *__restrict__ asc_e, const float *__restrict__ asc_w, int T,
               const int32_t *__restrict__ chunk_off, const int32_t *__restrict__ ebase,
               int32_t *__restrict__ pos, int32_t *__restrict__ perm, float *__restrict__ pw) {
  __shared__ uint32_t bits[kE][8];
  const int c = blockIdx.x;
  chunk_bits(asc_e, T, c, bits);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok = c * kPfChunk + tid;
  if (tok >= T) return;
  for (int j = 0; j < kTopK; ++j) {
    const int e = asc_e[(size_t)tok * kTopK + j];
    int rank = __popc(bits[e][warp] & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) rank += __popc(bits[e][w]);
    const int p = ebase[e] + chunk_off[(size_t)c * kE + e] + rank;
    pos[(size_t)tok * kTopK + j] = p;
    perm[p] = tok;
    pw[p] = asc_w[(size_t)tok * kTopK + j];
  }
}

// Routed token rows in sorted order; padding rows are zero.
__global__ void __launch_bounds__(256)
    k_pf_gather(const uint16_t *__restrict__ x, const int32_t *__restrict__ perm,
                const uint32_t *__restrict__ ctrl, uint16_t *__restrict__ xp) {
  const size_t rows = __ldcg(ctrl + 5);
  const size_t n = rows * (kH / 8);
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
    const size_t row = i / (kH / 8), c = i % (kH / 8);
    const int tok = perm[row];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok >= 0) v = ld_cg_v4(x + (size_t)tok * kH + 8 * c);
    *reinterpret_cast<uint4 *>(xp + row * kH + 8 * c) = v;
  }
}

// ============================================================== tcgen05 grouped GEMM
// Tile: 128 weight rows (A) x 128 tokens (N), K in stages of 64.  A holds the
// int4 codes as exact bf16 values; the bf16 scale of each (row, 128-wide
// k-group) is applied in fp32 when the group's partial sum is read out of
// tensor memory, so the weights enter the product exactly.  Two TMEM
// accumulator buffers let the MMAs of group G+1 run while group G is read.
// GEMM 2's token operand is the SwiGLU intermediate as a hi/lo bf16 pair (two
// MMA passes over the same A tile), ~16 significant bits.
constexpr int kABytes = 128 * 128;      // 128 weight rows x 64 bf16
constexpr int kBBytes = kPfTile * 128;  // 128 token rows x 64 bf16
constexpr int kRawBytes = 128 * 32;     // 128 weight rows x 64 int4
// Four warpgroups: 0 = producer, MMA issuer and two idle warps; 1 = four
// dequant warps (one weight row per thread); 2-3 = eight epilogue warps (two
// per TMEM lane quarter, one per 64-token half of the tile).  The block is
// launched at 128 registers per thread (65,536); setmaxnreg then moves them:
// 128 x 40 + 128 x 64 + 256 x 200 = 64,512.
constexpr int kGemmThreads = 512;
constexpr int kDeqThreads = 128;
constexpr int kEpiThreads = 256;
constexpr int kRegCtl = 40, kRegDeq = 64, kRegEpi = 200;
static_assert(128 * kRegCtl + 128 * kRegDeq + 256 * kRegEpi <= 65536, "register split");
constexpr int kTmemCols = 512;          // four 128-column fp32 accumulators (one CTA per SM)
constexpr int kTmemBufs = kTmemCols / 128;

template <int kMode>
struct GemmCfg {
  static constexpr int kNB = kMode == 1 ? 1 : 2;  // token operands per stage (hi, lo)
  static constexpr int kAtoms = 2;                // 64-wide k atoms per stage: one k-group
  // stage: A atoms | token atoms (operand-major) | int4 codes of the atoms
  static constexpr int kStageBytes = kAtoms * (kABytes + kNB * kBBytes + kRawBytes);
  static constexpr int kStages = kMode == 1 ? 3 : 2;
  static constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024;
  static constexpr uint32_t a_off(int atom) { return (uint32_t)(atom * kABytes); }
  static constexpr uint32_t b_off(int nb, int atom) {
    return (uint32_t)(kAtoms * kABytes + (nb * kAtoms + atom) * kBBytes);
  }
  static constexpr uint32_t raw_off() { return (uint32_t)(kAtoms * (kABytes + kNB * kBBytes)); }
};

struct GemmArgs {
  const uint32_t *tiles;
  const uint32_t *ctrl;
  int count_word;
  const int32_t *ebase;
  const int32_t *ecount;
  int T;
  const uint16_t *sc_r;  // scales of the routed weight tensor
  const uint16_t *sc_s;  // scales of the shared expert's tensor
  uint16_t *out_r;       // GEMM 1: H hi (lo follows at out_r_lo); GEMM 2: Yw
  uint16_t *out_r_lo;
  uint16_t *out_s;       // GEMM 1: Hs hi; GEMM 2: Ys
  uint16_t *out_s_lo;
  const float *pw;
  uint32_t *status;
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

FLINT_DEV void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accum) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, "
      "%3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}

FLINT_DEV void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Optional GEMM timeline (build with -DFLINT_TRACE): for the first kPfTrTiles
// CTAs of each GEMM, %globaltimer per k-stage for the producer (TMA issued),
// the dequant warps (tile written), the MMA warp (MMAs issued), and per
// k-group for the epilogue (group read out); read with flint_pf_trace_dump.
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

// 32 consecutive TMEM columns of this warp's 32 lanes; completes at tmem_wait_ld().
FLINT_DEV void tmem_ld32_async(uint32_t taddr, uint32_t (&v)[32]) {
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

FLINT_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FLINT_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 int4 codes (one 16-byte chunk of a raw row) -> four 16-byte chunks of
// exact bf16 codes in natural element order.
FLINT_DEV void codes32(uint4 w, uint4 (&out)[4]) {
  uint32_t r[16];
  int4x32_to_bf16x2(w, r);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    out[q] = make_uint4(__byte_perm(r[4 * q + 0], r[4 * q + 1], 0x5410),   // (c0, c1)
                        __byte_perm(r[4 * q + 2], r[4 * q + 3], 0x5410),   // (c2, c3)
                        __byte_perm(r[4 * q + 0], r[4 * q + 1], 0x7632),   // (c4, c5)
                        __byte_perm(r[4 * q + 2], r[4 * q + 3], 0x7632));  // (c6, c7)
}

FLINT_DEV void split_hilo(float v, uint16_t &hi, uint16_t &lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi = __bfloat16_as_ushort(h);
  lo = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(h)));
}

// kMode 1: gate/up + SwiGLU -> H hi/lo (routed [rows][512], shared [T][1024]).
// kMode 2: down -> Yw (routed, weighted, [rows][2048]) / Ys (shared, [T][2048]).
// One tile of a grouped GEMM, as every role of the CTA derives it.
template <int kMode>
struct PfTile {
  int e, mt, n0, n_valid, n_mma, b_row, row0, row1, ks, ng;
  bool sh;
};
template <int kMode>
FLINT_DEV bool pf_tile(const GemmArgs &args, uint32_t idx, PfTile<kMode> &t) {
  using Cfg = GemmCfg<kMode>;
  const uint32_t packed = __ldcg(args.tiles + idx);
  t.e = (int)(packed & 511u);
  t.mt = (int)((packed >> 9) & 31u);
  const int nt = (int)(packed >> 14);
  t.sh = t.e == kE;
  t.n0 = nt * kPfTile;
  t.n_valid = min(kPfTile, (t.sh ? args.T : __ldcg(args.ecount + t.e)) - t.n0);
  if (t.n_valid <= 0) return false;  // not produced by the scan; guards against an N = 0 MMA
  t.n_mma = (t.n_valid + 15) & ~15;
  t.b_row = t.sh ? t.n0 : __ldcg(args.ebase + t.e) + t.n0;
  t.ks = (kMode == 1 ? kH : (t.sh ? kIs : kI)) / (64 * Cfg::kAtoms);  // k stages = k-groups
  t.ng = t.ks;
  if (kMode == 1) {  // weight rows: gate (tile rows 2i) / up (2i+1)
    t.row0 = t.sh ? 64 * t.mt : t.e * 2 * kI + 64 * t.mt;
    t.row1 = t.sh ? kIs + 64 * t.mt : t.e * 2 * kI + kI + 64 * t.mt;
  } else {  // tile row i is weight row row0 + i
    t.row0 = t.sh ? 128 * t.mt : t.e * kH + 128 * t.mt;
    t.row1 = t.row0;
  }
  return true;
}

// Persistent: CTA c takes tiles c, c + grid, ...  Every role walks the same
// tile sequence; the stage ring and the two TMEM accumulator buffers carry
// on across tiles (running counters it, gc), so one tile's epilogue and the
// next tile's loads and MMAs overlap.
template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_pf_gemm(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
              const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
              const __grid_constant__ CUtensorMap tmB_r_lo,
              const __grid_constant__ CUtensorMap tmB_s_lo, GemmArgs args) {
  using Cfg = GemmCfg<kMode>;
  constexpr int S = Cfg::kStages;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[S], afull[S], empty[S], gfull[kTmemBufs],
      gempty[kTmemBufs];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_fail;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ntiles = __ldcg(args.ctrl + args.count_word);
  if (blockIdx.x >= ntiles) return;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], kDeqThreads);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kTmemBufs; ++b) {
      mbar_init(&gfull[b], 1);
      mbar_init(&gempty[b], kEpiThreads);
    }
    s_fail = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (tid == 0) pf_mark(kMode, 4, 0);

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtl));
    if (warp == 0 && lane == 0) {
      // ---- producer: int4 codes of the weight tile and the token tile(s), by TMA
      uint32_t it = 0;
      for (uint32_t ti = blockIdx.x; ti < ntiles && !s_fail; ti += gridDim.x) {
        PfTile<kMode> t;
        if (!pf_tile<kMode>(args, ti, t)) continue;
        const CUtensorMap *tA = t.sh ? &tmA_s : &tmA_r;
        const CUtensorMap *tB = t.sh ? &tmB_s : &tmB_r;
        const CUtensorMap *tBl = t.sh ? &tmB_s_lo : &tmB_r_lo;
        for (int kb = 0; kb < t.ks; ++kb, ++it) {
          const int s = it % S;
          if (it >= (uint32_t)S && !mbar_wait_sleep(&empty[s], ((it / S) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          unsigned char *st = sm + (size_t)s * Cfg::kStageBytes;
          unsigned char *raw = st + Cfg::raw_off();
          mbar_expect_tx(&full[s], Cfg::kAtoms * (kRawBytes + Cfg::kNB * kBBytes));
          if (kMode == 1) {  // gate rows then up rows, 128 codes (64 B) each
            tma_load_2d(raw, tA, kb * 64, t.row0, &full[s]);
            tma_load_2d(raw + 64 * 64, tA, kb * 64, t.row1, &full[s]);
            tma_load_2d(st + Cfg::b_off(0, 0), tB, kb * 128, t.b_row, &full[s]);
            tma_load_2d(st + Cfg::b_off(0, 1), tB, kb * 128 + 64, t.b_row, &full[s]);
          } else {  // 128 rows x 128 codes; hi and lo token atoms
            tma_load_2d(raw, tA, kb * 64, t.row0, &full[s]);
            for (int atom = 0; atom < 2; ++atom) {
              tma_load_2d(st + Cfg::b_off(0, atom), tB, kb * 128 + 64 * atom, t.b_row, &full[s]);
              tma_load_2d(st + Cfg::b_off(1, atom), tBl, kb * 128 + 64 * atom, t.b_row, &full[s]);
            }
          }
          if (ti == blockIdx.x) pf_mark(kMode, 0, kb);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer: group gc accumulates into TMEM buffer gc % kTmemBufs
      uint32_t it = 0, gc = 0;
      for (uint32_t ti = blockIdx.x; ti < ntiles && !s_fail; ti += gridDim.x) {
        PfTile<kMode> t;
        if (!pf_tile<kMode>(args, ti, t)) continue;
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                               ((uint32_t)(t.n_mma >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
        for (int G = 0; G < t.ng && !s_fail; ++G, ++gc) {
          const int b = gc % kTmemBufs;
          if (gc >= kTmemBufs && !mbar_wait(&gempty[b], ((gc / kTmemBufs) - 1) & 1)) {
            s_fail = 1;
            break;
          }
          if (ti == blockIdx.x) pf_mark(kMode, 5, G);
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(128 * b);
          {  // the group's single stage
            const int s = it % S;
            const uint32_t ph = (it / S) & 1;
            // afull implies full: the dequant warps arrive on afull only after
            // they have waited on full (the stage's TMA bytes) themselves
            if (!mbar_wait(&afull[s], ph)) {
              s_fail = 1;
              break;
            }
            tc_fence_after();
            const uint32_t st_addr = smem_addr(sm + (size_t)s * Cfg::kStageBytes);
#pragma unroll
            for (int atom = 0; atom < Cfg::kAtoms; ++atom) {
              const uint32_t a_addr = st_addr + Cfg::a_off(atom);
              const uint32_t b_addr = st_addr + Cfg::b_off(0, atom);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                umma_bf16(d, sw128_desc(a_addr + 32 * k), sw128_desc(b_addr + 32 * k), idesc,
                          (atom | k) != 0);
                if (kMode == 2)
                  umma_bf16(d, sw128_desc(a_addr + 32 * k),
                            sw128_desc(st_addr + Cfg::b_off(1, atom) + 32 * k), idesc, 1u);
              }
            }
            umma_commit(&empty[s]);    // the stage is free for the producer
            umma_commit(&gfull[b]);    // group gc is complete in TMEM buffer b
            if (ti == blockIdx.x) pf_mark(kMode, 2, G);
            ++it;
          }
        }
      }
    }  // other lanes and warps 2-3: idle (register donors)
  } else if (warp < 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegDeq));
    // ---- dequant: thread i owns weight row i of every tile (exact codes)
    const int i = tid - 128;
    const int raw_row = kMode == 1 ? ((i & 1) ? 64 + (i >> 1) : (i >> 1)) : i;
    uint32_t it = 0;
    for (uint32_t ti = blockIdx.x; ti < ntiles && !s_fail; ti += gridDim.x) {
      PfTile<kMode> t;
      if (!pf_tile<kMode>(args, ti, t)) continue;
      for (int kb = 0; kb < t.ks; ++kb, ++it) {
        const int s = it % S;
        if (!mbar_wait_sleep(&full[s], (it / S) & 1)) {
          s_fail = 1;
          break;
        }
        unsigned char *st = sm + (size_t)s * Cfg::kStageBytes;
        // the row's codes: 32 B per atom; chunk j (32 codes) -> atom j / 2, 16-byte
        // slots 4 (j % 2) .. +3 of the row, XOR-swizzled by the row (SW128)
        const unsigned char *raw = st + Cfg::raw_off() + raw_row * (32 * Cfg::kAtoms);
#pragma unroll
        for (int j = 0; j < 2 * Cfg::kAtoms; ++j) {
          const uint4 w = *reinterpret_cast<const uint4 *>(raw + 16 * j);
          uint4 c[4];
          codes32(w, c);
          unsigned char *arow = st + Cfg::a_off(j >> 1) + i * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(arow + ((((j & 1) * 4 + q) ^ (i & 7)) * 16)) = c[q];
        }
        fence_proxy_async();
        mbar_arrive(&afull[s]);
        if (tid == 128 && ti == blockIdx.x) pf_mark(kMode, 1, kb);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegEpi));
    // ---- epilogue warps 8..15: TMEM lane quarter (warp % 4) -> tile rows;
    // token half (warp - 8) / 4 -> tile columns 64 h .. 64 h + 63
    const int q4 = warp & 3;
    const int c_lo = 64 * ((warp - 8) >> 2);
    const int r = 32 * q4 + lane;
    uint32_t gc = 0;
    for (uint32_t ti = blockIdx.x; ti < ntiles && !s_fail; ti += gridDim.x) {
      PfTile<kMode> t;
      if (!pf_tile<kMode>(args, ti, t)) continue;
      const int wrow = kMode == 1 ? ((r & 1) ? t.row1 : t.row0) + (r >> 1) : t.row0 + r;
      const int gpr = kMode == 1 ? kH / kG : (t.sh ? kIs / kG : kI / kG);
      const uint16_t *srow = (t.sh ? args.sc_s : args.sc_r) + (size_t)wrow * gpr;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      bool ok = true;
      for (int G = 0; G < t.ng; ++G, ++gc) {
        const int b = gc % kTmemBufs;
        const float sc = bf16_bits_to_f32(ld_nc_u16(srow + G));
        if (!mbar_wait_sleep(&gfull[b], (gc / kTmemBufs) & 1)) {
          ok = false;
          break;
        }
        if (tid == 256 && ti == blockIdx.x) pf_mark(kMode, 4, 2 + G);
        tc_fence_after();
        const uint32_t base = tmem + (uint32_t)(128 * b + c_lo) + ((uint32_t)(32 * q4) << 16);
        if (c_lo < t.n_mma) {  // the same for the whole warp
          uint32_t v0[32], v1[32];
          tmem_ld32_async(base, v0);
          if (c_lo + 32 < t.n_mma) tmem_ld32_async(base + 32u, v1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = fmaf(__uint_as_float(v0[j]), sc, acc[j]);
          if (c_lo + 32 < t.n_mma) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              acc[32 + j] = fmaf(__uint_as_float(v1[j]), sc, acc[32 + j]);
          }
        }
        tc_fence_before();
        mbar_arrive(&gempty[b]);
        if (tid == 256 && ti == blockIdx.x) pf_mark(kMode, 3, G);
        if (tid == 480 && ti == blockIdx.x) pf_mark(kMode, 3, 20 + G);
      }
      if (!ok) {
        s_fail = 1;
        break;
      }
      if (kMode == 1) {
        const int col = 64 * t.mt + (r >> 1);
        const size_t ld = t.sh ? kIs : kI;
        uint16_t *hi = t.sh ? args.out_s + (size_t)t.n0 * kIs + col
                            : args.out_r + (size_t)t.b_row * kI + col;
        uint16_t *lo = t.sh ? args.out_s_lo + (size_t)t.n0 * kIs + col
                            : args.out_r_lo + (size_t)t.b_row * kI + col;
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
          const int j = c_lo + jj;
          const float other = __shfl_xor_sync(0xffffffffu, acc[jj], 1);
          if (!(r & 1) && j < t.n_valid) {
            const float hv = acc[jj] / (1.f + expf(-acc[jj])) * other;  // silu(gate) * up
            uint16_t h16, l16;
            split_hilo(hv, h16, l16);
            hi[(size_t)j * ld] = h16;
            lo[(size_t)j * ld] = l16;
          }
        }
      } else {
        const int col = 128 * t.mt + r;
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
          const int j = c_lo + jj;
          if (j < t.n_valid) {
            if (t.sh) {
              args.out_s[(size_t)(t.n0 + j) * kH + col] = f32_to_bf16_bits(acc[jj]);
            } else {
              args.out_r[(size_t)(t.b_row + j) * kH + col] =
                  f32_to_bf16_bits(acc[jj] * args.pw[t.b_row + j]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) pf_mark(kMode, 4, 1);
  if (s_fail && tid == 0) set_status(args.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// ============================================================== combine
__global__ void __launch_bounds__(256)
    k_pf_combine(const int32_t *__restrict__ pos, const uint16_t *__restrict__ yw,
                 const uint16_t *__restrict__ ys, int T, uint16_t *__restrict__ out) {
  const size_t n = (size_t)T * (kH / 8);
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
    const size_t tok = i / (kH / 8), c = i % (kH / 8);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j <= kTopK; ++j) {
      const uint16_t *src = j < kTopK ? yw + (size_t)pos[tok * kTopK + j] * kH : ys + tok * kH;
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

}  // namespace

cudaError_t launch_route_many(const LayerArgs &L, const uint16_t *x, int T, int32_t *idx, float *w,
                              char *ws, cudaStream_t st) {
  const PrefillLayout P = prefill_layout(T);
  float *z = reinterpret_cast<float *>(ws + P.z);
  note_step("prefill router attribute");
  cudaError_t e = cudaFuncSetAttribute(k_pf_router, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       8 * 8 * 32 * 64);
  if (e != cudaSuccess) return e;
  note_step("prefill router launch");
  k_pf_router<<<(T + kRtTok - 1) / kRtTok, 512, 8 * 8 * 32 * 64, st>>>(L, x, T, z);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  note_step("prefill top-6 launch");
  k_pf_topk<<<(T + 7) / 8, 256, 0, st>>>(L.router_b, z, T, idx, w,
                                          reinterpret_cast<int32_t *>(ws + P.asc_e),
                                          reinterpret_cast<float *>(ws + P.asc_w));
  return cudaGetLastError();
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
  int32_t *perm = reinterpret_cast<int32_t *>(ws + P.perm);
  float *pw = reinterpret_cast<float *>(ws + P.pw);
  uint32_t *tiles1 = reinterpret_cast<uint32_t *>(ws + P.tiles1);
  uint32_t *tiles2 = reinterpret_cast<uint32_t *>(ws + P.tiles2);
  uint16_t *xp = reinterpret_cast<uint16_t *>(ws + P.xp);
  uint16_t *hr = reinterpret_cast<uint16_t *>(ws + P.hr);          // hi
  uint16_t *hr_lo = hr + (size_t)P.mr_max * kI;                     // lo
  uint16_t *hs = reinterpret_cast<uint16_t *>(ws + P.hs);
  uint16_t *hs_lo = hs + (size_t)T * kIs;
  uint16_t *yw = reinterpret_cast<uint16_t *>(ws + P.yw);
  uint16_t *ys = reinterpret_cast<uint16_t *>(ws + P.ys);

  // 1. routing
  e = launch_route_many(L, x, T, reinterpret_cast<int32_t *>(ws + P.sel_idx),
                        reinterpret_cast<float *>(ws + P.sel_w), ws, st);
  if (e != cudaSuccess) return e;
  // 2. stable sort by expert
  note_step("prefill sort launches");
  k_pf_count<<<P.nchunks, 256, 0, st>>>(asc_e, T, cc);
  k_pf_scan<<<1, 256, 0, st>>>(T, P.nchunks, cc, co, ebase, ecount, perm, tiles1, tiles2, ctrl);
  k_pf_place<<<P.nchunks, 256, 0, st>>>(asc_e, asc_w, T, co, ebase, pos, perm, pw);
  // 3. gather
  {
    int blocks = (int)(((size_t)P.mr_max * (kH / 8) + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_pf_gather<<<blocks, 256, 0, st>>>(x, perm, ctrl, xp);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 4. tensor maps and the two grouped GEMMs
  CUtensorMap mA1r, mA1s, mB1r, mB1s, mA2r, mA2s, mB2r, mB2s, mB2rl, mB2sl;
  note_step("prefill tensor maps");
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B, NS = CU_TENSOR_MAP_SWIZZLE_NONE;
  if ((e = make_map(&mA1r, L.w13_q, U8, kH / 2, (uint64_t)kE * 2 * kI, kH / 2, 64, 64, NS)) ||
      (e = make_map(&mA1s, L.sh13_q, U8, kH / 2, 2 * kIs, kH / 2, 64, 64, NS)) ||
      (e = make_map(&mB1r, xp, BF, kH, (uint64_t)P.mr_max, kH * 2, 64, kPfTile, SW)) ||
      (e = make_map(&mB1s, x, BF, kH, (uint64_t)T, kH * 2, 64, kPfTile, SW)) ||
      (e = make_map(&mA2r, L.w2_q, U8, kI / 2, (uint64_t)kE * kH, kI / 2, 64, 128, NS)) ||
      (e = make_map(&mA2s, L.sh2_q, U8, kIs / 2, kH, kIs / 2, 64, 128, NS)) ||
      (e = make_map(&mB2r, hr, BF, kI, (uint64_t)P.mr_max, kI * 2, 64, kPfTile, SW)) ||
      (e = make_map(&mB2rl, hr_lo, BF, kI, (uint64_t)P.mr_max, kI * 2, 64, kPfTile, SW)) ||
      (e = make_map(&mB2s, hs, BF, kIs, (uint64_t)T, kIs * 2, 64, kPfTile, SW)) ||
      (e = make_map(&mB2sl, hs_lo, BF, kIs, (uint64_t)T, kIs * 2, 64, kPfTile, SW)))
    return e;
  note_step("prefill GEMM attributes");
  if ((e = cudaFuncSetAttribute(k_pf_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GemmCfg<1>::kSmem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_pf_gemm<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GemmCfg<2>::kSmem)) != cudaSuccess)
    return e;
  // persistent GEMMs: one CTA per SM at most (the tile counts are on the device)
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 1;
  GemmArgs a1{tiles1, ctrl, 3,  ebase, ecount, T,       L.w13_s, L.sh13_s,
              hr,     hr_lo, hs, hs_lo, nullptr, ctrl + 1};
  note_step("prefill GEMM 1 launch");
  k_pf_gemm<1><<<min(P.max_tiles1, sms), kGemmThreads, GemmCfg<1>::kSmem, st>>>(
      mA1r, mA1s, mB1r, mB1s, mB1r, mB1s, a1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  GemmArgs a2{tiles2, ctrl, 4, ebase, ecount, T, L.w2_s, L.sh2_s, yw, nullptr, ys, nullptr, pw,
              ctrl + 1};
  note_step("prefill GEMM 2 launch");
  k_pf_gemm<2><<<min(P.max_tiles2, sms), kGemmThreads, GemmCfg<2>::kSmem, st>>>(
      mA2r, mA2s, mB2r, mB2s, mB2rl, mB2sl, a2);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 5. combine
  note_step("prefill combine launch");
  {
    int blocks = (int)(((size_t)T * (kH / 8) + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_pf_combine<<<blocks, 256, 0, st>>>(pos, yw, ys, T, out);
  }
  return cudaGetLastError();
}

}  // namespace flint
