// k_dequant.cuh -- Dequant-reduce, the receiving side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): each rank's shard is converted back and the ranks are summed
// in rank order, acc = fma(float(q_r - zero_r), scale_r, acc) for 4-bit features and
// acc = acc + side_r for kept ones.
//
// Work decomposition.  A CTA covers a slice of G groups of 8 consecutive output features
// (G = 64 for P <= 8, fewer for more ranks so that the constants below fit) and RL = 256/G row
// lanes; each thread owns one group and R rows of a row block, and keeps R x 8 fp32 sums in
// registers while it walks the ranks in order.  Work units are (slice, row block), slice-major,
// split into one contiguous run per CTA of a persistent grid.
//
// Codes of a group: its n non-kept features occupy compact positions c0..c0+n-1, i.e. at most
// two consecutive words; a funnel shift brings them to bits 0..4n-1 of v, and feature i of the
// group reads nibble j_i (its rank among the non-kept ones).  The nibble is turned into a float
// without a conversion instruction: (nibble | 0x4B000000) is the float 2^23 + q, and adding the
// constant -(2^23 + zero) gives q - zero exactly.  Per (rank, feature) the kernel needs scale
// and that offset; they are written to shared memory once per slice (a kept feature gets scale 0
// and offset -2^23, which leaves its sum untouched).
//
// Kept features are summed separately: "kept lanes" (one per (row, kept feature) pair of the
// block) add the P side values in rank order into a small shared buffer, and the owning threads
// take them from there before the bf16 (or fp32) output row is stored with 16-byte stores.
//
// Roofline: HBM-bound; per output element ~P*(H'/H*0.5 + k/H*2) bytes read + 2 (or 4) written.
// No scratch memory.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr int kDqThreads = 256;
constexpr int kDqRows = 4;          // rows per thread per block
constexpr int kDqKeptChunk = 64;    // kept features per pass of the kept lanes
constexpr int kDqMaxG = 64;

// Groups per slice for P ranks: the constants take P * G * 64 bytes (<= 32 KB).
inline int dq_groups_for(int P) {
  int g = kDqMaxG;
  while (g > 8 && P * g * 64 > 32 * 1024) g >>= 1;
  return g;
}

template <typename OutT>
__device__ __forceinline__ void store_row8(OutT* dst, const float* v);

template <>
__device__ __forceinline__ void store_row8<uint16_t>(uint16_t* dst, const float* v) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = w;
}

// fp32 output: a NaN sum is written as the canonical quiet NaN 0x7FC00000.
__device__ __forceinline__ float canonical_nan(float v) {
  return (v != v) ? __uint_as_float(0x7FC00000u) : v;
}

template <>
__device__ __forceinline__ void store_row8<float>(float* dst, const float* v) {
  reinterpret_cast<float4*>(dst)[0] =
      make_float4(canonical_nan(v[0]), canonical_nan(v[1]), canonical_nan(v[2]), canonical_nan(v[3]));
  reinterpret_cast<float4*>(dst)[1] =
      make_float4(canonical_nan(v[4]), canonical_nan(v[5]), canonical_nan(v[6]), canonical_nan(v[7]));
}

template <typename OutT>
__global__ void __launch_bounds__(kDqThreads) dequant_reduce_kernel(
    const uint32_t* __restrict__ codes, const uint16_t* __restrict__ side, int P, int T, int H,
    int k, const int32_t* __restrict__ keep_idx, const float* __restrict__ scale,
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int G, int S, int NB,
    long long units_per_cta) {
  extern __shared__ float4 s_dyn[];
  float* s_const = reinterpret_cast<float*>(s_dyn);         // [P][G][16]: scale x8, offset x8
  float* s_kept = s_const + (size_t)P * G * 16;             // [RL*R][kDqKeptChunk]

  const int tid = threadIdx.x;
  const int RL = kDqThreads / G;
  const int gi = tid % G, lane_row = tid / G;
  const int Hr = H - k, Wr = Hr / 8;
  const int rows_per_block = RL * kDqRows;
  const long long U = (long long)S * NB;

  long long u = (long long)blockIdx.x * units_per_cta;
  const long long u_end = min(U, u + units_per_cta);
  int cur_slice = -1;

  // per-thread static layout of its group in the current slice
  int h0 = 0, c0 = 0, n = 0, j0 = 0;
  uint32_t kmask = 0;
  int nib_shift[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) nib_shift[i] = 0;
  bool active = false;
  int ja = 0, jb = 0;

  for (; u < u_end; ++u) {
    const int s = (int)(u / NB);
    const int b = (int)(u - (long long)s * NB);

    if (s != cur_slice) {
      __syncthreads();  // previous users of s_const are done
      cur_slice = s;
      const int g = s * G + gi;
      h0 = 8 * g;
      active = h0 < H;
      if (active) {
        const GroupLayout L = group_layout(keep_idx, k, H, h0);
        c0 = L.c0;
        n = L.n;
        j0 = L.j0;
        kmask = L.kmask;
        int j = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const bool kept = (kmask >> i) & 1u;
          nib_shift[i] = kept ? 0 : 4 * j;
          j += kept ? 0 : 1;
        }
      } else {
        c0 = n = j0 = 0;
        kmask = 0;
      }
      const int ha = s * G * 8, hb = min(H, ha + G * 8);
      ja = lower_bound_i32(keep_idx, k, ha);
      jb = lower_bound_i32(keep_idx, k, hb);
      if (tid == 0 && ((s == 0 && ja != 0) || (s == S - 1 && jb != k))) record_error(HQ_ERR_BAD_INDEX);
      // constants of the slice: threads of row lane 0 fill their own group for all ranks
      if (lane_row == 0) {
        for (int r = 0; r < P; ++r) {
          float* dst = s_const + ((size_t)r * G + gi) * 16;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float sc = 0.0f, off = -8388608.0f;  // kept / inactive: contributes fma(q, 0, acc)
            if (active && !((kmask >> i) & 1u)) {
              const size_t p = (size_t)r * H + h0 + i;
              sc = scale[p];
              off = -__int_as_float(0x4B000000 | (int)zero[p]);  // -(2^23 + zero)
            }
            dst[i] = sc;
            dst[8 + i] = off;
          }
        }
      }
      __syncthreads();
    }

    const int t_blk = b * rows_per_block;
    float acc[kDqRows][8];
#pragma unroll
    for (int m = 0; m < kDqRows; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[m][i] = 0.0f;

    const int w0 = c0 >> 3, fsh = 4 * (c0 & 7);
    const bool has_hi = (w0 + 1) < Wr;
    if (active && n > 0) {
      for (int r = 0; r < P; ++r) {
        const float4* cst = reinterpret_cast<const float4*>(s_const + ((size_t)r * G + gi) * 16);
        const float4 s0 = cst[0], s1 = cst[1], o0 = cst[2], o1 = cst[3];
        const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const float off[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        uint32_t wlo[kDqRows], whi[kDqRows];
#pragma unroll
        for (int m = 0; m < kDqRows; ++m) {
          const int t = t_blk + lane_row + m * RL;
          wlo[m] = whi[m] = 0u;
          if (t < T) {
            const uint32_t* row = codes + ((size_t)r * T + t) * Wr;
            wlo[m] = __ldg(row + w0);
            if (has_hi) whi[m] = __ldg(row + w0 + 1);
          }
        }
#pragma unroll
        for (int m = 0; m < kDqRows; ++m) {
          const uint32_t v = __funnelshift_r(wlo[m], whi[m], fsh);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t bits = ((v >> nib_shift[i]) & 0xFu) | 0x4B000000u;
            const float d = __fadd_rn(__uint_as_float(bits), off[i]);
            acc[m][i] = __fmaf_rn(d, sc[i], acc[m][i]);
          }
        }
      }
    }

    // ---- kept features of the slice, in chunks -------------------------------------------
    const int nk = jb - ja;
    for (int kc = 0; kc < nk; kc += kDqKeptChunk) {
      const int kw = min(kDqKeptChunk, nk - kc);
      const int pairs = rows_per_block * kw;
      for (int p = tid; p < pairs; p += kDqThreads) {
        const int row = p / kw, jj = p - row * kw;
        const int t = t_blk + row;
        float a = 0.0f;
        if (t < T) {
          const int j = ja + kc + jj;
          for (int r = 0; r < P; ++r)
            a = __fadd_rn(a, __uint_as_float((uint32_t)__ldg(side + ((size_t)r * T + t) * k + j) << 16));
        }
        s_kept[row * kDqKeptChunk + jj] = a;
      }
      __syncthreads();
      if (kmask) {
        int jk = j0;  // keep_idx position of the group's next kept feature
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((kmask >> i) & 1u) {
            const int jj = jk - ja - kc;
            if (jj >= 0 && jj < kw) {
#pragma unroll
              for (int m = 0; m < kDqRows; ++m) acc[m][i] = s_kept[(lane_row + m * RL) * kDqKeptChunk + jj];
            }
            ++jk;
          }
        }
      }
      __syncthreads();
    }

    if (active) {
#pragma unroll
      for (int m = 0; m < kDqRows; ++m) {
        const int t = t_blk + lane_row + m * RL;
        if (t < T) store_row8<OutT>(out + (size_t)t * H + h0, acc[m]);
      }
    }
  }
}

}  // namespace hq
