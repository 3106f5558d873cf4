// Int4 GEMV with fused argmax for the output head ("How to Run Flint
// Locally", section "One decode step in bytes": lm_head is 150,144 x 2,048
// and is read in full for every token; Recursive quantized it to 4 bits).
//
// One warp computes a 16-row tile against up to 8 activation columns with
// mma.sync (see common.cuh); weights stream through registers with a few
// groups in flight; the activation fragment sits in shared memory.  Each
// warp keeps its best (value, row) per column; CTAs publish partials and the
// last CTA to finish reduces them (lowest row on ties), so the whole call is
// one launch.
#include "common.cuh"
#include "internal.h"

namespace flint {

constexpr int kGemvThreads = 256;
constexpr int kGemvNPre = 4;

struct ArgPartial {
  float v;
  int i;
};

// (v, i) beats the current best (bv, bi): larger value, lower row on ties;
// any non-NaN value beats an empty best (bi < 0).
FLINT_DEV bool better(float v, int i, float bv, int bi) {
  return bi < 0 ? (v == v) : (v > bv || (v == bv && i < bi));
}

size_t gemv_ws_bytes(int N, int B) {
  const int tiles = (N + 15) / 16;
  int grid = (tiles + 7) / 8;
  if (grid > 148 * 4) grid = 148 * 4;
  return align256(256) + align256(sizeof(ArgPartial) * (size_t)grid * B);
}

static int gemv_grid(int N) {
  const int tiles = (N + 15) / 16;
  int grid = (tiles + 7) / 8;
  return grid > 148 * 4 ? 148 * 4 : grid;
}

__global__ void __launch_bounds__(kGemvThreads)
    k_int4_gemv(const uint8_t *__restrict__ q, const uint16_t *__restrict__ s, int N, int K,
                const uint16_t *__restrict__ x, int B, float *__restrict__ y,
                int32_t *__restrict__ argmax, char *__restrict__ ws) {
  extern __shared__ uint4 xfrag[];
  __shared__ ArgPartial s_part[kGemvThreads / 32][kMaxB];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int ngroups = K / kG;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(ws);
  ArgPartial *parts = reinterpret_cast<ArgPartial *>(ws + align256(256));

  pdl_wait();
  pdl_trigger();
  build_x_frag(xfrag, ngroups, B, [&](int r) { return x + (size_t)r * K; }, tid, kGemvThreads);
  __syncthreads();

  float best_v[2] = {0.f, 0.f};
  int best_i[2] = {-1, -1};
  const int tiles = (N + 15) / 16;
  const size_t rb = (size_t)K / 2;
  for (int tile = blockIdx.x * 8 + warp; tile < tiles; tile += gridDim.x * 8) {
    const int n_a = tile * 16 + g, n_b = n_a + 8;
    const bool va = n_a < N, vb = n_b < N;
    const uint8_t *pa = q + (size_t)(va ? n_a : 0) * rb + 16 * t;
    const uint8_t *pb = q + (size_t)(vb ? n_b : 0) * rb + 16 * t;
    const uint16_t *sa = s + (size_t)(va ? n_a : 0) * ngroups;
    const uint16_t *sb = s + (size_t)(vb ? n_b : 0) * ngroups;
    uint4 wa[kGemvNPre], wb[kGemvNPre];
    uint32_t sva[kGemvNPre], svb[kGemvNPre];
#pragma unroll
    for (int G = 0; G < kGemvNPre; ++G) {
      if (G < ngroups) {
        wa[G] = ld_stream(pa + 64 * G);
        wb[G] = ld_stream(pb + 64 * G);
        sva[G] = ld_nc_u16(sa + G);
        svb[G] = ld_nc_u16(sb + G);
      }
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int G0 = 0; G0 < ngroups; G0 += kGemvNPre) {
#pragma unroll
      for (int k = 0; k < kGemvNPre; ++k) {
        const int G = G0 + k;
        if (G < ngroups) {
          const uint4 w0 = wa[k], w1 = wb[k];
          const float s0 = bf16_bits_to_f32(sva[k]), s1 = bf16_bits_to_f32(svb[k]);
          if (G + kGemvNPre < ngroups) {
            wa[k] = ld_stream(pa + 64 * (G + kGemvNPre));
            wb[k] = ld_stream(pb + 64 * (G + kGemvNPre));
            sva[k] = ld_nc_u16(sa + G + kGemvNPre);
            svb[k] = ld_nc_u16(sb + G + kGemvNPre);
          }
          uint32_t ra[16], rbv[16], xb[16];
          int4x32_to_bf16x2(w0, ra);
          int4x32_to_bf16x2(w1, rbv);
          load_frag(xfrag + (G * 32 + lane) * 4, xb);
          float d[4];
          group_mma(ra, rbv, xb, d);
          acc[0] = fmaf(d[0], s0, acc[0]);
          acc[1] = fmaf(d[1], s0, acc[1]);
          acc[2] = fmaf(d[2], s1, acc[2]);
          acc[3] = fmaf(d[3], s1, acc[3]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int b = 2 * t + c;
      if (b < B) {
        if (va) {
          y[(size_t)b * N + n_a] = acc[c];
          if (better(acc[c], n_a, best_v[c], best_i[c])) best_v[c] = acc[c], best_i[c] = n_a;
        }
        if (vb) {
          y[(size_t)b * N + n_b] = acc[2 + c];
          if (better(acc[2 + c], n_b, best_v[c], best_i[c])) best_v[c] = acc[2 + c], best_i[c] = n_b;
        }
      }
    }
  }
  if (!argmax) return;

  // lanes sharing t hold the same columns: reduce over g (xor 4, 8, 16)
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best_v[c], o);
      const int oi = __shfl_xor_sync(0xffffffffu, best_i[c], o);
      if (oi >= 0 && better(ov, oi, best_v[c], best_i[c]))
        best_v[c] = ov, best_i[c] = oi;
    }
    const int b = 2 * t + c;
    if (g == 0 && b < B) s_part[warp][b] = ArgPartial{best_v[c], best_i[c]};
  }
  __syncthreads();
  if (tid < B) {
    ArgPartial p{0.f, -1};
    for (int w = 0; w < kGemvThreads / 32; ++w) {
      const ArgPartial o = s_part[w][tid];
      if (o.i >= 0 && better(o.v, o.i, p.v, p.i)) p = o;
    }
    parts[(size_t)blockIdx.x * B + tid] = p;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&ctrl[0], 1u);
    s_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid < B) {
    ArgPartial p{0.f, -1};
    for (int cta = 0; cta < (int)gridDim.x; ++cta) {
      const float ov = ld_cg_f32(&parts[(size_t)cta * B + tid].v);
      const int oi = (int)ld_cg_u32(&parts[(size_t)cta * B + tid].i);
      if (oi >= 0 && better(ov, oi, p.v, p.i)) p = ArgPartial{ov, oi};
    }
    argmax[tid] = p.i;
  }
  if (tid == 0) ctrl[0] = 0;
}

cudaError_t launch_gemv(const uint8_t *q, const uint16_t *s, int N, int K, const uint16_t *x,
                        int B, float *y, int32_t *argmax, char *ws, cudaStream_t st) {
  const size_t smem = (size_t)(K / kG) * 128 * 16;
  static int configured = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(k_int4_gemv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (8192 / kG) * 128 * 16);
    if (e != cudaSuccess) return e;
    configured = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gemv_grid(N));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_int4_gemv, q, s, N, K, x, B, y, argmax, ws);
}

}  // namespace flint
