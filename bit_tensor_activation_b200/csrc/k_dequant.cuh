// k_dequant.cuh -- Dequant-reduce, the receiving side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): each rank's shard is converted back and the ranks are summed
// in rank order, acc = fma(float(q_r - zero_r), scale_r, acc) for 4-bit features and
// acc = acc + side_r for kept ones.
//
// Work decomposition.  A warp owns a slice of 32 groups of 8 consecutive output features (256
// features, one group per lane) and a block of kDqR rows at a time; the 8 warps of a CTA share
// one slice (so they share its per-(rank, feature) constants in shared memory) and split the
// CTA's row range between them.  Nothing in the main loop synchronises more than one warp.
//
// Data movement.  For every (row block, rank) the warp stages the code words its 32 groups need
// -- at most 35 consecutive words per row -- into shared memory with 4-byte cp.async copies,
// kDqD tiles ahead of the tile it consumes (an 8-deep pipeline per warp, ~0.6 KB per tile), so
// the latency of HBM is covered without holding the data in registers.  cp.async.wait_group is a
// hardware wait: there is no spin loop.
//
// Codes of a group: its n non-kept features occupy compact positions c0..c0+n-1, i.e. at most
// two consecutive words; a funnel shift brings them to bits 0..4n-1 of v, and feature i of the
// group reads nibble j_i (its rank among the group's non-kept features).  The nibble becomes a
// float without a conversion instruction: (nibble | 0x4B000000) is the float 2^23 + q, and
// adding the per-(rank, feature) constant -(2^23 + zero) gives q - zero exactly.  A kept feature
// gets scale 0 and offset -2^23, which leaves its sum untouched; its sum over the side values is
// computed by "kept lanes" and written into the owner's registers through a small warp buffer.
//
// Roofline: HBM-bound; per output element P*(0.5*H'/H + 2*k/H) bytes read + 2 (or 4) written.
// No memory beyond the inputs and outputs is used.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr int kDqWarps = 8;
constexpr int kDqThreads = 32 * kDqWarps;
constexpr int kDqR = 4;       // rows per block
constexpr int kDqD = 8;       // cp.async tiles in flight per warp
constexpr int kDqWin = 36;    // staged words per row (>= 35)
constexpr int kDqSliceGroups = 32;

// Dynamic shared memory of one CTA for P ranks.
inline size_t dq_smem_bytes(int P) {
  return (size_t)P * 4 * 32 * 16                            // constants: [P][4][32] float4
         + (size_t)kDqWarps * kDqD * kDqR * kDqWin * 4      // staged code tiles
         + (size_t)kDqWarps * kDqR * 32 * 4;                // kept sums
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
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int S, int chunks, int rows_per_chunk) {
  extern __shared__ float4 s_dyn[];
  float4* s_const = s_dyn;                                                    // [P][4][32]
  uint32_t* s_tiles = reinterpret_cast<uint32_t*>(s_const + (size_t)P * 4 * 32);
  float* s_kept = reinterpret_cast<float*>(s_tiles + kDqWarps * kDqD * kDqR * kDqWin);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Hr = H - k, Wr = Hr / 8;
  const int s = blockIdx.x / chunks, chunk = blockIdx.x - s * chunks;
  const int t_first = chunk * rows_per_chunk, t_last = min(T, t_first + rows_per_chunk);

  // ---- this lane's group: layout and nibble positions ----------------------------------------
  const int h0 = 8 * (s * kDqSliceGroups + lane);
  const bool active = h0 < H;
  GroupLayout L{0, 0, 0u, 0};
  if (active) L = group_layout(keep_idx, k, H, h0);
  int nib_shift[8];
  {
    int j = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool kept = (L.kmask >> i) & 1u;
      nib_shift[i] = kept ? 0 : 4 * j;
      j += kept ? 0 : 1;
    }
  }
  // words the warp stages per row: [w_first, w_end), at most 35
  const int hs = 8 * s * kDqSliceGroups, he = min(H, hs + 8 * kDqSliceGroups);
  const int ja = lower_bound_i32(keep_idx, k, hs), jb = lower_bound_i32(keep_idx, k, he);
  if (threadIdx.x == 0 && ((s == 0 && ja != 0) || (s == S - 1 && jb != k))) record_error(HQ_ERR_BAD_INDEX);
  const int Ca = min(max(hs - ja, 0), Hr), Cb = min(max(he - jb, 0), Hr);
  const int w_first = Ca >> 3;
  const int n_words = max(0, min(Wr, (Cb >> 3) + 2) - w_first);
  const int my_w = (L.c0 >> 3) - w_first;  // this lane's first word inside the window
  const int fsh = 4 * (L.c0 & 7);
  const bool has_hi = (L.c0 >> 3) + 1 < Wr;

  // ---- constants of the slice for all ranks (conflict-free [P][4][32] float4 layout) ---------
  for (int idx = threadIdx.x; idx < P * 32; idx += kDqThreads) {
    const int r = idx >> 5, g = idx & 31;
    const int hg = 8 * (s * kDqSliceGroups + g);
    float sc[8], off[8];
    uint32_t km = 0;
    if (hg < H) km = group_layout(keep_idx, k, H, hg).kmask;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[i] = 0.0f;
      off[i] = -8388608.0f;
      if (hg < H && !((km >> i) & 1u)) {
        const size_t p = (size_t)r * H + hg + i;
        sc[i] = scale[p];
        off[i] = -__int_as_float(0x4B000000 | (int)zero[p]);  // -(2^23 + zero)
      }
    }
    float4* dst = s_const + (size_t)r * 4 * 32 + g;
    dst[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
    dst[32] = make_float4(sc[4], sc[5], sc[6], sc[7]);
    dst[64] = make_float4(off[0], off[1], off[2], off[3]);
    dst[96] = make_float4(off[4], off[5], off[6], off[7]);
  }
  __syncthreads();

  // ---- this warp's row blocks: rows t_first + (warp + kDqWarps*bi)*kDqR + m ------------------
  const int nblk_total = (t_last - t_first + kDqR - 1) / kDqR;
  const int my_blocks = nblk_total > warp ? (nblk_total - warp + kDqWarps - 1) / kDqWarps : 0;
  const int n_tiles = my_blocks * P;  // tile i = (block i / P, rank i % P)
  uint32_t* my_tiles = s_tiles + (size_t)warp * kDqD * kDqR * kDqWin;
  float* my_kept = s_kept + warp * kDqR * 32;
  const uint32_t tiles_saddr = smem_addr(my_tiles);

  auto block_row0 = [&](int bi) { return t_first + (warp + kDqWarps * bi) * kDqR; };
  auto issue_tile = [&](int i) {
    if (i < n_tiles) {
      const int bi = i / P, r = i - bi * P;
      const int t0 = block_row0(bi);
      const int stage = i % kDqD;
#pragma unroll
      for (int m = 0; m < kDqR; ++m) {
        const int t = t0 + m;
        if (t < t_last) {
          const uint32_t* src = codes + ((size_t)r * T + t) * Wr + w_first;
          const uint32_t dst = tiles_saddr + (uint32_t)(((stage * kDqR + m) * kDqWin) * 4);
          for (int w = lane; w < n_words; w += 32) cp_async4(dst + 4u * w, src + w);
        }
      }
    }
    cp_async_commit();  // one group per tile, empty ones included, keeps the count uniform
  };

  for (int i = 0; i < kDqD - 1; ++i) issue_tile(i);

  const int nk = jb - ja;
  int tile = 0;
  for (int bi = 0; bi < my_blocks; ++bi) {
    const int t0 = block_row0(bi);
    float acc[kDqR][8];
#pragma unroll
    for (int m = 0; m < kDqR; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[m][i] = 0.0f;

    for (int r = 0; r < P; ++r, ++tile) {
      issue_tile(tile + kDqD - 1);
      cp_async_wait<kDqD - 1>();
      __syncwarp();
      const uint32_t* st = my_tiles + (size_t)(tile % kDqD) * kDqR * kDqWin;
      const float4* cst = s_const + (size_t)r * 4 * 32 + lane;
      const float4 s0 = cst[0], s1 = cst[32], o0 = cst[64], o1 = cst[96];
      const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const float off[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
      if (active && L.n > 0) {
#pragma unroll
        for (int m = 0; m < kDqR; ++m) {
          const uint32_t wlo = st[m * kDqWin + my_w];
          const uint32_t whi = has_hi ? st[m * kDqWin + my_w + 1] : 0u;
          const uint32_t v = __funnelshift_r(wlo, whi, fsh);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t bits = ((v >> nib_shift[i]) & 0xFu) | 0x4B000000u;
            const float d = __fadd_rn(__uint_as_float(bits), off[i]);
            acc[m][i] = __fmaf_rn(d, sc[i], acc[m][i]);
          }
        }
      }
      __syncwarp();  // the stage is free for the copy issued next iteration
    }

    // ---- kept features of the warp's slice: (row, kept feature) pairs over the lanes ---------
    for (int kc = 0; kc < nk; kc += 32) {
      const int kw = min(32, nk - kc);
      for (int p = lane; p < kDqR * kw; p += 32) {
        const int m = p / kw, jj = p - m * kw;
        const int t = t0 + m;
        float a = 0.0f;
        if (t < t_last) {
          const uint16_t* sp = side + (size_t)t * k + ja + kc + jj;
          const size_t rank_stride = (size_t)T * k;
#pragma unroll 8
          for (int r = 0; r < P; ++r) a = __fadd_rn(a, __uint_as_float((uint32_t)__ldg(sp + r * rank_stride) << 16));
        }
        my_kept[m * 32 + jj] = a;
      }
      __syncwarp();
      if (L.kmask) {
        int jk = L.j0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((L.kmask >> i) & 1u) {
            const int jj = jk - ja - kc;
            if (jj >= 0 && jj < kw) {
#pragma unroll
              for (int m = 0; m < kDqR; ++m) acc[m][i] = my_kept[m * 32 + jj];
            }
            ++jk;
          }
        }
      }
      __syncwarp();
    }

    if (active) {
#pragma unroll
      for (int m = 0; m < kDqR; ++m) {
        const int t = t0 + m;
        if (t < t_last) store_row8<OutT>(out + (size_t)t * H + h0, acc[m]);
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace hq
