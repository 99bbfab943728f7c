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
// Work decomposition as in dequant-reduce: the 8 warps of a CTA share one slice of 256 features
// (one group of 8 per lane) and its per-(rank, feature) constants in shared memory, and split
// the CTA's row range in blocks of kFuR rows.  A warp walks the ranks in order; each lane stages
// its own 16 bytes of the kFuR rows of upcoming ranks into shared memory with cp.async, kFuD - 1
// tiles ahead, and reads back only what it copied (its own wait_group is the only sync needed).
//
// Roofline: HBM-bound, P*2 bytes read + 2 (or 4) bytes written per output element.
#pragma once

#include "hq_common.cuh"
#include "k_dequant.cuh"

namespace hq {

constexpr int kFuWarps = 8;
constexpr int kFuThreads = 32 * kFuWarps;
constexpr int kFuR = 4;
constexpr int kFuD = 3;  // tiles staged per warp
constexpr int kFuSliceGroups = 32;

inline size_t fu_smem_bytes(int P) {
  return (size_t)P * 5 * 32 * 16 + (size_t)kFuWarps * kFuD * kFuR * 32 * 16;
}

template <typename OutT>
__global__ void __launch_bounds__(kFuThreads) compress_reduce_kernel(
    const uint16_t* __restrict__ x, int P, int T, int H, int k, const int32_t* __restrict__ keep_idx,
    const float* __restrict__ scale, const float* __restrict__ inv_scale,
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int S, int chunks, int rows_per_chunk) {
  extern __shared__ float4 s_dyn[];
  float4* s_const = s_dyn;  // [P][5][32]: inv 0-3, inv 4-7, scale 0-3, scale 4-7, (zero bytes, kmask)

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = blockIdx.x / chunks, chunk = blockIdx.x - s * chunks;
  const int t_first = chunk * rows_per_chunk, t_last = min(T, t_first + rows_per_chunk);
  const int h0 = 8 * (s * kFuSliceGroups + lane);
  const bool active = h0 < H;

  for (int idx = threadIdx.x; idx < P * 32; idx += kFuThreads) {
    const int r = idx >> 5, g = idx & 31;
    const int hg = 8 * (s * kFuSliceGroups + g);
    float iv[8], sc[8];
    uint32_t zlo = 0, zhi = 0, km = 0;
    if (hg < H) {
      km = group_layout(keep_idx, k, H, hg).kmask;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const size_t p = (size_t)r * H + hg + i;
        iv[i] = inv_scale[p];
        sc[i] = ((km >> i) & 1u) ? 1.0f : scale[p];
        const uint32_t z = zero[p];
        if (i < 4) zlo |= z << (8 * i);
        else zhi |= z << (8 * (i - 4));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) iv[i] = sc[i] = 0.0f;
    }
    float4* dst = s_const + (size_t)r * 5 * 32 + g;
    dst[0] = make_float4(iv[0], iv[1], iv[2], iv[3]);
    dst[32] = make_float4(iv[4], iv[5], iv[6], iv[7]);
    dst[64] = make_float4(sc[0], sc[1], sc[2], sc[3]);
    dst[96] = make_float4(sc[4], sc[5], sc[6], sc[7]);
    dst[128] = make_float4(__uint_as_float(zlo), __uint_as_float(zhi), __uint_as_float(km), 0.0f);
  }
  __syncthreads();
  if (!active) return;

  const uint32_t kmask = __float_as_uint(s_const[128 + lane].z);
  const int nblk_total = (t_last - t_first + kFuR - 1) / kFuR;
  const int my_blocks = nblk_total > warp ? (nblk_total - warp + kFuWarps - 1) / kFuWarps : 0;
  const int n_tiles = my_blocks * P;  // tile i = (block i / P, rank i % P)
  uint4* my_rows = reinterpret_cast<uint4*>(s_const + (size_t)P * 5 * 32) + (size_t)warp * kFuD * kFuR * 32;
  const uint16_t* xl = x + h0;

  auto block_row0 = [&](int bi) { return t_first + (warp + kFuWarps * bi) * kFuR; };
  auto issue = [&](int i) {
    if (i < n_tiles) {
      const int bi = i / P, r = i - bi * P;
      const int t0 = block_row0(bi);
      const int stage = i % kFuD;
#pragma unroll
      for (int m = 0; m < kFuR; ++m)
        if (t0 + m < t_last)
          cp_async16(smem_addr(my_rows + (stage * kFuR + m) * 32 + lane), xl + ((size_t)r * T + t0 + m) * H);
    }
    cp_async_commit();
  };
  for (int i = 0; i < kFuD - 1; ++i) issue(i);

  int tile = 0;
  for (int bi = 0; bi < my_blocks; ++bi) {
    const int t0 = block_row0(bi);
    const int nrows = min(kFuR, t_last - t0);
    float acc[kFuR][8];
#pragma unroll
    for (int m = 0; m < kFuR; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[m][i] = 0.0f;

    for (int r = 0; r < P; ++r, ++tile) {
      issue(tile + kFuD - 1);
      cp_async_wait<kFuD - 1>();
      const uint4* st = my_rows + (tile % kFuD) * kFuR * 32 + lane;
      const float4* cst = s_const + (size_t)r * 5 * 32 + lane;
      const float4 i0 = cst[0], i1 = cst[32], s0 = cst[64], s1 = cst[96], zz = cst[128];
      const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
      const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const uint32_t zlo = __float_as_uint(zz.x), zhi = __float_as_uint(zz.y);
      int lo[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) lo[i] = -(int)(((i < 4 ? zlo : zhi) >> (8 * (i & 3))) & 0xFFu);
#pragma unroll
      for (int m = 0; m < kFuR; ++m) {
        if (m < nrows) {
          const uint4 xv = st[m * 32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float f = bf16_at(xv, i);
            int c = __float2int_rn(__fmul_rn(f, inv[i]));  // saturating; NaN -> 0
            c = min(max(c, lo[i]), lo[i] + 15);
            const float d = __fadd_rn(__int_as_float(c + 0x4B400000), -12582912.0f);
            const float v = ((kmask >> i) & 1u) ? f : d;
            acc[m][i] = __fmaf_rn(v, sc[i], acc[m][i]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kFuR; ++m)
      if (m < nrows) store_row8<OutT>(out + (size_t)(t0 + m) * H + h0, acc[m]);
  }
  cp_async_wait<0>();
}

}  // namespace hq
