// k_quantize.cuh -- Quantize-pack, the sending side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): kept features are copied to the BF16 side buffer, all others
// become 4-bit codes q = clamp(rint(x*inv_scale)+zero, 0, 15) packed 8 per uint32 in rest_idx
// order.
//
// Work decomposition.  A warp owns a slice of 32 groups of 8 consecutive features (256 features,
// one group per lane).  A work unit is one row of one rank restricted to one slice; units are
// laid out rank-major, then slice, then row, and every warp of a persistent grid takes one
// contiguous run of them, so it changes (rank, slice) rarely and keeps its features' parameters
// in registers in between.  Warps never wait for one another.
//
// Data movement.  Each lane stages its own 16 bytes of kQpR rows per tile into shared memory
// with cp.async, kQpD - 1 tiles ahead of the tile it computes; a lane only reads what it copied,
// so its own cp.async.wait_group (a hardware wait) is the only synchronisation the data needs.
//
// Per lane: inv_scale, the clamp bound -zero and a nibble multiplier 16^j (0 for a kept feature,
// j = the feature's rank among the group's non-kept ones) for its 8 features.  The group's code
// word is V = sum_i (zero_i + clamp_i) * 16^j_i: every nibble stays in [0,15], so the sum is the
// packed word of the group's n non-kept codes.  Its compact position c0 is in general not a
// multiple of 8, so V is split across two words and OR-ed into a per-warp word buffer in shared
// memory.
//
// Ownership of compact words: a slice owns the words whose first nibble one of its groups
// produces; it drops nibbles that fall into the previous slice's last word and completes its own
// last word from the next <= 7 non-kept features of the next slice ("halo", read through
// rest_idx, one lane each).  So every codes word is written by exactly one warp with plain
// coalesced stores.  Kept values are taken from the owner lane's staged row with shuffles.
//
// Roofline: HBM-bound; 2 bytes read + 0.5 byte written per non-kept element, 2 + 2 per kept one.
// No memory beyond the inputs and outputs is used.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr int kQpWarps = 8;
constexpr int kQpThreads = 32 * kQpWarps;
constexpr int kQpR = 4;              // rows per tile
constexpr int kQpD = 3;              // tiles staged per warp (kQpD - 1 in flight while computing)
constexpr int kQpSliceGroups = 32;   // groups per warp slice
constexpr int kQpBufWords = 36;      // >= 33 owned words per row

struct QpWarpSmem {
  uint4 rows[kQpD][kQpR][32];        // each lane's 16 bytes of each staged row
  uint32_t halo[kQpD][kQpR][8];      // the 4-byte word holding each halo lane's feature
  uint32_t buf[kQpR][kQpBufWords];   // compact words being assembled
};

__global__ void __launch_bounds__(kQpThreads) quantize_pack_kernel(
    const uint16_t* __restrict__ x, int P, int T, int H, int k, const int32_t* __restrict__ keep_idx,
    const int32_t* __restrict__ rest_idx, const float* __restrict__ inv_scale,
    const uint8_t* __restrict__ zero, uint32_t* __restrict__ codes, uint16_t* __restrict__ side,
    int S, long long units_per_warp) {
  extern __shared__ float4 s_dyn[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  QpWarpSmem& W = reinterpret_cast<QpWarpSmem*>(s_dyn)[warp];
  const int Hr = H - k, Wr = Hr / 8, NG = H / 8;
  const long long U = (long long)P * S * T;

  for (int i = lane; i < kQpR * kQpBufWords; i += 32) (&W.buf[0][0])[i] = 0u;
  __syncwarp();

  long long u = ((long long)blockIdx.x * kQpWarps + warp) * units_per_warp;
  const long long u_end = min(U, u + units_per_warp);

  while (u < u_end) {
    const long long rs = u / T;
    const int t_begin = (int)(u - rs * T);
    const int t_stop = (int)min((long long)T, (long long)t_begin + (u_end - u));
    const int r = (int)(rs / S), s = (int)(rs - (long long)r * S);

    // ---- this lane's group: parameters in registers ----------------------------------------
    const int g = s * kQpSliceGroups + lane;
    const bool active = g < NG;
    const int h0 = 8 * g;
    GroupLayout L{0, 0, 0u, 0};
    float inv[8];
    int lo[8];
    uint32_t mul[8], zbase = 0;
    if (active) L = group_layout(keep_idx, k, H, h0);
    {
      int j = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool kept = (L.kmask >> i) & 1u;
        int z = 0;
        inv[i] = 0.0f;
        if (active) {
          const size_t p = (size_t)r * H + h0 + i;
          z = zero[p];
          inv[i] = inv_scale[p];
        }
        lo[i] = -z;
        mul[i] = (active && !kept) ? (1u << (4 * j)) : 0u;
        j += kept ? 0 : 1;
        zbase += (uint32_t)z * mul[i];
      }
    }

    // ---- slice ownership (the same values in every lane) ------------------------------------
    const int ha = 8 * s * kQpSliceGroups, hb = min(H, ha + 8 * kQpSliceGroups);
    const int ja = lower_bound_i32(keep_idx, k, ha), jb = lower_bound_i32(keep_idx, k, hb);
    if (lane == 0 && ((s == 0 && ja != 0) || (s == S - 1 && jb != k))) record_error(HQ_ERR_BAD_INDEX);
    const int Ca = min(max(ha - ja, 0), Hr), Cb = min(max(hb - jb, 0), Hr);
    const int Wb = (Ca + 7) >> 3, We = (Cb + 7) >> 3;  // owned words [Wb, We)
    const int nw = max(We - Wb, 0);                    // <= 33
    const int nhalo = (We > Wb) ? (8 * We - Cb) : 0;   // 0..7 codes from the next slice

    // halo lane: one non-kept feature after the slice
    const bool is_halo = lane < nhalo;
    float h_inv = 0.0f;
    int h_col = 0, h_lo = 0, h_z = 0, h_shift = 0;
    if (is_halo) {
      h_col = checked_col(rest_idx, Cb + lane, H);
      const size_t p = (size_t)r * H + h_col;
      h_z = zero[p];
      h_inv = inv_scale[p];
      h_lo = -h_z;
      h_shift = 4 * ((Cb + lane) & 7);
    }
    const int nk = jb - ja;
    const int w0 = (L.c0 >> 3) - Wb, sh = 4 * (L.c0 & 7);
    const uint16_t* xr = x + ((size_t)r * T) * H;
    const int n_tiles = (t_stop - t_begin + kQpR - 1) / kQpR;

    auto issue = [&](int i) {
      if (i < n_tiles) {
        const int stage = i % kQpD;
#pragma unroll
        for (int m = 0; m < kQpR; ++m) {
          const int t = t_begin + i * kQpR + m;
          if (t < t_stop) {
            if (active) cp_async16(smem_addr(&W.rows[stage][m][lane]), xr + (size_t)t * H + h0);
            if (is_halo) cp_async4(smem_addr(&W.halo[stage][m][lane]), xr + (size_t)t * H + (h_col & ~1));
          }
        }
      }
      cp_async_commit();
    };
    for (int i = 0; i < kQpD - 1; ++i) issue(i);

    for (int i = 0; i < n_tiles; ++i) {
      issue(i + kQpD - 1);
      cp_async_wait<kQpD - 1>();
      __syncwarp();  // the kept-value shuffles below read other lanes' registers, not their smem
      const int stage = i % kQpD;
      const int t = t_begin + i * kQpR;
      const int nrows = min(kQpR, t_stop - t);
#pragma unroll
      for (int m = 0; m < kQpR; ++m) {
        if (m >= nrows) break;
        const uint4 v = W.rows[stage][m][lane];
        if (active && L.n > 0) {
          uint32_t V = zbase;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = __fmul_rn(bf16_at(v, e), inv[e]);
            int c = __float2int_rn(a);  // saturating; NaN -> 0
            c = min(max(c, lo[e]), lo[e] + 15);
            V += (uint32_t)c * mul[e];
          }
          const uint32_t lo_part = V << sh;
          const uint32_t hi_part = sh ? (V >> (32 - sh)) : 0u;
          if (lo_part && w0 >= 0 && w0 < nw) atomicOr(&W.buf[m][w0], lo_part);
          if (hi_part && w0 + 1 >= 0 && w0 + 1 < nw) atomicOr(&W.buf[m][w0 + 1], hi_part);
        }
        if (is_halo) {
          const uint32_t hw = W.halo[stage][m][lane];
          const uint32_t hb16 = (h_col & 1) ? (hw & 0xFFFF0000u) : (hw << 16);
          int c = __float2int_rn(__fmul_rn(__uint_as_float(hb16), h_inv));
          c = min(max(c, h_lo), h_lo + 15) + h_z;
          if (c) atomicOr(&W.buf[m][nw - 1], (uint32_t)c << h_shift);
        }
        // kept values, one per lane (rounds of 32), from the owner lane's staged row
        for (int kc = 0; kc < nk; kc += 32) {
          const int j = ja + kc + lane;
          const bool mine = j < jb;
          const int col = mine ? checked_col(keep_idx, j, H) : ha;
          const int src = min(max((col - ha) >> 3, 0), 31), e = col & 7;
          const uint32_t a0 = __shfl_sync(0xFFFFFFFFu, v.x, src);
          const uint32_t a1 = __shfl_sync(0xFFFFFFFFu, v.y, src);
          const uint32_t a2 = __shfl_sync(0xFFFFFFFFu, v.z, src);
          const uint32_t a3 = __shfl_sync(0xFFFFFFFFu, v.w, src);
          const uint32_t w = (e < 2) ? a0 : (e < 4) ? a1 : (e < 6) ? a2 : a3;
          if (mine) side[((size_t)r * T + t + m) * k + j] = (uint16_t)((e & 1) ? (w >> 16) : (w & 0xFFFFu));
        }
      }
      __syncwarp();
      // owned words out, buffer cleared
#pragma unroll
      for (int m = 0; m < kQpR; ++m) {
        if (m < nrows) {
          uint32_t* dst = codes + ((size_t)r * T + t + m) * Wr + Wb;
          for (int q = lane; q < nw; q += 32) {
            dst[q] = W.buf[m][q];
            W.buf[m][q] = 0u;
          }
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();
    u += t_stop - t_begin;
  }
}

}  // namespace hq
