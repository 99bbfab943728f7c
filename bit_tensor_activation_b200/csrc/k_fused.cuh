// k_fused.cuh -- Fused compress-reduce (page "Revolutionizing LLM Inference: The Power of
// Efficient Low-Bit Communication", sections "Combating Quantization Errors with Tensor
// Parallelism" and "The Hybrid Quantization Algorithm"): every rank's partial sum is quantized
// and immediately dequantized and summed, without a wire buffer.  Bit-identical to
// quantize-pack followed by dequant-reduce:
//   non-kept:  c = clamp(rint(x*inv_scale), -zero, 15-zero)   ( = q - zero )
//              acc = fma(float(c), scale, acc)
//   kept:      acc = fma(x, 1, acc) = acc + x  (exact equivalent of the fp32 add)
// float(c) is formed without a conversion instruction: the bits c + 0x4B400000 are the float
// 1.5*2^23 + c, from which 1.5*2^23 is subtracted exactly.
//
// Work decomposition as in dequant-reduce: a CTA covers a slice of kFuGroups groups of 8
// features and kFuThreads/kFuGroups row lanes; a thread owns one group and kFuRows rows and walks
// the ranks in order, loading that rank's parameters for its 8 features once per row block.
//
// Roofline: HBM-bound, P*2 bytes read + 2 (or 4) bytes written per output element.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr int kFuThreads = 256;
constexpr int kFuGroups = 64;
constexpr int kFuRows = 2;

template <typename OutT>
__global__ void __launch_bounds__(kFuThreads) compress_reduce_kernel(
    const uint16_t* __restrict__ x, int P, int T, int H, int k, const int32_t* __restrict__ keep_idx,
    const float* __restrict__ scale, const float* __restrict__ inv_scale,
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int S, int NB,
    long long units_per_cta) {
  constexpr int RL = kFuThreads / kFuGroups;
  const int tid = threadIdx.x;
  const int gi = tid % kFuGroups, lane_row = tid / kFuGroups;
  const int rows_per_block = RL * kFuRows;
  const long long U = (long long)S * NB;

  long long u = (long long)blockIdx.x * units_per_cta;
  const long long u_end = min(U, u + units_per_cta);
  int cur_slice = -1;
  int h0 = 0;
  bool active = false;
  uint32_t kmask = 0;

  for (; u < u_end; ++u) {
    const int s = (int)(u / NB);
    const int b = (int)(u - (long long)s * NB);
    if (s != cur_slice) {
      cur_slice = s;
      h0 = 8 * (s * kFuGroups + gi);
      active = h0 < H;
      kmask = active ? group_layout(keep_idx, k, H, h0).kmask : 0u;
    }
    if (!active) continue;

    const int t_blk = b * rows_per_block;
    float acc[kFuRows][8];
#pragma unroll
    for (int m = 0; m < kFuRows; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[m][i] = 0.0f;

    for (int r = 0; r < P; ++r) {
      const size_t p = (size_t)r * H + h0;
      const float4 i0 = *reinterpret_cast<const float4*>(inv_scale + p);
      const float4 i1 = *reinterpret_cast<const float4*>(inv_scale + p + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(scale + p);
      const float4 s1 = *reinterpret_cast<const float4*>(scale + p + 4);
      const uint2 zz = *reinterpret_cast<const uint2*>(zero + p);
      const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
      float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      int lo[8], hi[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int z = (int)(((i < 4 ? zz.x : zz.y) >> (8 * (i & 3))) & 0xFFu);
        lo[i] = -z;
        hi[i] = 15 - z;
        if ((kmask >> i) & 1u) sc[i] = 1.0f;
      }
      uint4 xv[kFuRows];
#pragma unroll
      for (int m = 0; m < kFuRows; ++m) {
        const int t = t_blk + lane_row + m * RL;
        if (t < T) xv[m] = ld_stream16(x + ((size_t)r * T + t) * H + h0);
        else xv[m] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int m = 0; m < kFuRows; ++m) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float f = bf16_at(xv[m], i);
          int c = __float2int_rn(__fmul_rn(f, inv[i]));
          c = min(max(c, lo[i]), hi[i]);
          const float d = __fadd_rn(__int_as_float(c + 0x4B400000), -12582912.0f);
          const float v = ((kmask >> i) & 1u) ? f : d;
          acc[m][i] = __fmaf_rn(v, sc[i], acc[m][i]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kFuRows; ++m) {
      const int t = t_blk + lane_row + m * RL;
      if (t < T) store_row8<OutT>(out + (size_t)t * H + h0, acc[m]);
    }
  }
}

}  // namespace hq
