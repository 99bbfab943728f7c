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
constexpr int kQpBufWords = 36;      // >= 33 owned words + 2 guard slots per row

struct QpWarpSmem {
  uint4 rows[kQpD][kQpR][32];        // each lane's 16 bytes of each staged row
  uint32_t halo[kQpD][kQpR][8];      // the 4-byte word holding each halo feature
  uint32_t buf[kQpR][kQpBufWords];   // slot 1 + (word - Wb); slot 0 and slot nw + 1 are guards
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
    int lo[8], hi[8];
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
        hi[i] = 15 - z;
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
    const int slot = (L.c0 >> 3) - Wb + 1;             // buffer slot of the group's first word
    const int sh = 4 * (L.c0 & 7);

    // halo work of a tile: lane p < nhalo*kQpR takes halo feature p % nhalo of row p / nhalo
    const bool is_halo = lane < nhalo * kQpR;
    const int h_row = is_halo ? lane / nhalo : 0, h_idx = is_halo ? lane - h_row * nhalo : 0;
    float h_inv = 0.0f;
    int h_col = 0, h_lo = 0, h_z = 0, h_shift = 0;
    if (is_halo) {
      h_col = checked_col(rest_idx, Cb + h_idx, H);
      const size_t p = (size_t)r * H + h_col;
      h_z = zero[p];
      h_inv = inv_scale[p];
      h_lo = -h_z;
      h_shift = 4 * ((Cb + h_idx) & 7);
    }
    // kept work of a tile: pair p = jj * kQpR + m (rounds of 32 pairs)
    const int nk = jb - ja;
    const int npairs = nk * kQpR;

    const uint16_t* xr = x + ((size_t)r * T) * H;
    uint32_t* crow = codes + ((size_t)r * T) * Wr + Wb;
    uint16_t* srow = side + ((size_t)r * T) * k;
    const int n_tiles = (t_stop - t_begin + kQpR - 1) / kQpR;

    int i_next = 0;
    auto issue_next = [&]() {
      if (i_next < n_tiles) {
        const int stage = i_next % kQpD;
        const int t0 = t_begin + i_next * kQpR;
        const uint16_t* src = xr + (size_t)t0 * H;
#pragma unroll
        for (int m = 0; m < kQpR; ++m)
          if (active && t0 + m < t_stop) cp_async16(smem_addr(&W.rows[stage][m][lane]), src + (size_t)m * H + h0);
        if (is_halo && t0 + h_row < t_stop)
          cp_async4(smem_addr(&W.halo[stage][h_row][h_idx]), src + (size_t)h_row * H + (h_col & ~1));
        ++i_next;
      }
      cp_async_commit();
    };
    for (int i = 0; i < kQpD - 1; ++i) issue_next();

    for (int i = 0; i < n_tiles; ++i) {
      issue_next();
      cp_async_wait<kQpD - 1>();
      __syncwarp();
      const int stage = i % kQpD;
      const int t0 = t_begin + i * kQpR;
      const int nrows = min(kQpR, t_stop - t0);
      // codes of the lane's group, one word V per row, OR-ed into two slots
      if (active && L.n > 0) {
#pragma unroll
        for (int m = 0; m < kQpR; ++m) {
          const uint4 v = W.rows[stage][m][lane];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t V = zbase;
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float a0, a1;
            fmul2(a0, a1, __uint_as_float(w[e / 2] << 16), __uint_as_float(w[e / 2] & 0xFFFF0000u),
                  inv[e], inv[e + 1]);
            int c0 = __float2int_rn(a0), c1 = __float2int_rn(a1);  // saturating; NaN -> 0
            c0 = min(max(c0, lo[e]), hi[e]);
            c1 = min(max(c1, lo[e + 1]), hi[e + 1]);
            V += (uint32_t)c0 * mul[e] + (uint32_t)c1 * mul[e + 1];
          }
          atomicOr(&W.buf[m][slot], V << sh);
          atomicOr(&W.buf[m][slot + 1], sh ? (V >> (32 - sh)) : 0u);
        }
      }
      if (is_halo && h_row < nrows) {
        const uint32_t hw = W.halo[stage][h_row][h_idx];
        const uint32_t hb16 = (h_col & 1) ? (hw & 0xFFFF0000u) : (hw << 16);
        int c = __float2int_rn(__fmul_rn(__uint_as_float(hb16), h_inv));
        c = min(max(c, h_lo), h_lo + 15) + h_z;
        atomicOr(&W.buf[h_row][nw], (uint32_t)c << h_shift);
      }
      // kept values straight from the staged rows
      for (int p = lane; p < npairs; p += 32) {
        const int jj = p / kQpR, m = p - jj * kQpR;
        if (m < nrows) {
          const int j = ja + jj;
          const int col = checked_col(keep_idx, j, H);
          const int src = min(max((col - ha) >> 3, 0), 31);
          const uint16_t* rowp = reinterpret_cast<const uint16_t*>(&W.rows[stage][m][src]);
          srow[(size_t)(t0 + m) * k + j] = rowp[col & 7];
        }
      }
      __syncwarp();
      // owned words out (slots 1..nw).  Each lane clears exactly the slots it read (slots
      // 1..kQpBufWords-1 in all; slot 0 only ever collects nibbles of the previous slice's word
      // and is never read), so every read precedes its clear in that lane's program order.
#pragma unroll
      for (int m = 0; m < kQpR; ++m) {
        uint32_t* dst = crow + (size_t)(t0 + m) * Wr;
        const uint32_t a = W.buf[m][lane + 1];
        if (m < nrows && lane < nw) dst[lane] = a;
        W.buf[m][lane + 1] = 0u;
        if (lane + 33 < kQpBufWords) {
          const uint32_t b = W.buf[m][lane + 33];
          if (m < nrows && lane + 32 < nw) dst[lane + 32] = b;
          W.buf[m][lane + 33] = 0u;
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();
    u += t_stop - t_begin;
  }
}

}  // namespace hq
