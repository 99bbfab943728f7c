// k_calibrate.cuh -- Calibration (page "Revolutionizing LLM Inference: The Power of Efficient
// Low-Bit Communication", section "The Hybrid Quantization Algorithm", bullet "Calibration"):
// per rank and feature, the min and max of one calibration batch folded into moving averages.
//
// Layout: x bf16 [P][T][H]; one CTA per (64-feature slab, rank).  256 threads = 32 row lanes x
// 8 groups of 8 features; each thread streams rows t = lane, lane+32, ... with 16-byte loads
// and keeps packed bf16x2 min/max (min/max are exact, so the reduction order is free; the
// bf16x2 min/max instructions skip a NaN operand).  The 32 row lanes are combined with warp
// shuffles and shared memory, then one thread per group finalises 8 features: -0 -> +0 and the
// moving-average update ema = beta*ema + (1-beta)*b in explicit fp32 steps.
//
// Roofline: HBM-bound, 2 bytes read per element, no scratch memory.
#pragma once

#include <cuda_bf16.h>

#include "hq_common.cuh"

namespace hq {

constexpr int kCalThreads = 256;
constexpr int kCalCols = 64;   // features per CTA
constexpr int kCalLanes = 32;  // row lanes per CTA

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t w) {
  return *reinterpret_cast<__nv_bfloat162*>(&w);
}
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kCalThreads) calibrate_kernel(
    const uint16_t* __restrict__ x, int ldx, int T, int H, float beta, float one_minus_beta, int first_batch,
    float* __restrict__ ema_min, float* __restrict__ ema_max) {
  __shared__ uint32_t s_min[kCalThreads / 32][32];  // [warp][group*4 + pair]
  __shared__ uint32_t s_max[kCalThreads / 32][32];

  const int r = blockIdx.y;
  const int g = threadIdx.x & 7;      // group within the slab
  const int lane_row = threadIdx.x >> 3;
  const int h0 = blockIdx.x * kCalCols + g * 8;

  const uint32_t kPosInf2 = 0x7F807F80u, kNegInf2 = 0xFF80FF80u;
  __nv_bfloat162 mn[4], mx[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    mn[p] = as_bf162(kPosInf2);
    mx[p] = as_bf162(kNegInf2);
  }

  if (h0 < H) {
    const size_t row_stride = (size_t)ldx;
    const uint16_t* base = x + (size_t)r * T * row_stride + h0;
    int t = lane_row;
#pragma unroll 1
    for (; t + 3 * kCalLanes < T; t += 4 * kCalLanes) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_stream16(base + (size_t)(t + u * kCalLanes) * row_stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          mn[p] = __hmin2(mn[p], as_bf162(w[p]));
          mx[p] = __hmax2(mx[p], as_bf162(w[p]));
        }
      }
    }
    for (; t < T; t += kCalLanes) {
      const uint4 v = ld_stream16(base + (size_t)t * row_stride);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        mn[p] = __hmin2(mn[p], as_bf162(w[p]));
        mx[p] = __hmax2(mx[p], as_bf162(w[p]));
      }
    }
  }

  // A warp holds 4 row lanes of the 8 groups (lanes g, g+8, g+16, g+24).
#pragma unroll
  for (int p = 0; p < 4; ++p) {
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
      mn[p] = __hmin2(mn[p], as_bf162(__shfl_xor_sync(0xFFFFFFFFu, as_u32(mn[p]), off)));
      mx[p] = __hmax2(mx[p], as_bf162(__shfl_xor_sync(0xFFFFFFFFu, as_u32(mx[p]), off)));
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < 8) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      s_min[warp][lane * 4 + p] = as_u32(mn[p]);
      s_max[warp][lane * 4 + p] = as_u32(mx[p]);
    }
  }
  __syncthreads();
  if (threadIdx.x < 8 && h0 < H) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      mn[p] = as_bf162(s_min[0][g * 4 + p]);
      mx[p] = as_bf162(s_max[0][g * 4 + p]);
    }
    for (int wv = 1; wv < kCalThreads / 32; ++wv) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        mn[p] = __hmin2(mn[p], as_bf162(s_min[wv][g * 4 + p]));
        mx[p] = __hmax2(mx[p], as_bf162(s_max[wv][g * 4 + p]));
      }
    }
    float bmin[8], bmax[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t a = as_u32(mn[p]), b = as_u32(mx[p]);
      bmin[2 * p] = __fadd_rn(bf16_lo(a), 0.0f);  // -0 -> +0
      bmin[2 * p + 1] = __fadd_rn(bf16_hi(a), 0.0f);
      bmax[2 * p] = __fadd_rn(bf16_lo(b), 0.0f);
      bmax[2 * p + 1] = __fadd_rn(bf16_hi(b), 0.0f);
    }
    float* pmin = ema_min + (size_t)r * H + h0;
    float* pmax = ema_max + (size_t)r * H + h0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (first_batch) {
        pmin[i] = bmin[i];
        pmax[i] = bmax[i];
      } else {
        pmin[i] = __fadd_rn(__fmul_rn(beta, pmin[i]), __fmul_rn(one_minus_beta, bmin[i]));
        pmax[i] = __fadd_rn(__fmul_rn(beta, pmax[i]), __fmul_rn(one_minus_beta, bmax[i]));
      }
    }
  }
}

}  // namespace hq
