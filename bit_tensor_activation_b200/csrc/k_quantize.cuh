// k_quantize.cuh -- Quantize-pack, the sending side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): kept features are copied to the BF16 side buffer, all others
// become 4-bit codes q = clamp(rint(x*inv_scale)+zero, 0, 15) packed 8 per uint32 in rest_idx
// order.
//
// Work decomposition.  A feature slice is kQpGroups groups of 8 consecutive features (1024
// features); a work unit is one row of one rank restricted to one slice.  The units are laid
// out rank-major, then slice, then row, and every CTA of a persistent grid takes one contiguous
// run of units, so it changes (rank, slice) at most a few times and keeps the per-feature
// parameters in registers in between.
//
// Per thread: 8 consecutive features h0..h0+7 -- one 16-byte load per row -- with inv_scale,
// the clamp bounds [-zero, 15-zero] and a per-feature nibble multiplier 16^j (0 for a kept
// feature, j = the feature's rank among the group's non-kept features) in registers.  The
// group's code word is V = sum_i (zero_i + clamp_i) * 16^j_i: every nibble stays in [0,15], so
// the sum is the packed word of the group's n non-kept codes.  Its compact position c0 is
// generally not a multiple of 8, so V is split across two words and OR-ed (shared-memory
// atomics) into a per-row word buffer.
//
// Ownership of compact words: a slice owns the words whose first nibble one of its groups
// produces; it drops nibbles that fall into the previous slice's last word and completes its own
// last word from the next <= 7 non-kept features of the next slice ("halo", read through
// rest_idx, one lane each).  So every codes word is written by exactly one CTA with plain
// coalesced stores, and no scratch memory is used.
//
// Roofline: HBM-bound; 2 bytes read + 0.5 byte written per non-kept element, 2 + 2 per kept one.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr int kQpGroups = 128;           // groups of 8 features per slice = threads per CTA
constexpr int kQpThreads = kQpGroups;
constexpr int kQpRows = 2;               // rows per iteration

struct QpThreadState {
  int h0;          // first feature of the group
  bool active;     // h0 < H
  int c0;          // compact position of the group's first non-kept feature
  int n;           // non-kept features in the group
  float inv[8];
  int lo[8], hi[8];
  uint32_t mul[8];
  uint32_t zbase;  // sum_i zero_i * mul_i
};

__global__ void __launch_bounds__(kQpThreads) quantize_pack_kernel(
    const uint16_t* __restrict__ x, int P, int T, int H, int k, const int32_t* __restrict__ keep_idx,
    const int32_t* __restrict__ rest_idx, const float* __restrict__ inv_scale,
    const uint8_t* __restrict__ zero, uint32_t* __restrict__ codes, uint16_t* __restrict__ side,
    int S, long long units_per_cta) {
  constexpr int kBufWords = kQpGroups + 1;
  __shared__ uint32_t s_buf[2][kQpRows][kBufWords];

  const int tid = threadIdx.x;
  const int Hr = H - k, Wr = Hr / 8, NG = H / 8;
  const long long U = (long long)P * S * T;

  for (int i = tid; i < 2 * kQpRows * kBufWords; i += kQpThreads) (&s_buf[0][0][0])[i] = 0u;
  __syncthreads();

  long long u = (long long)blockIdx.x * units_per_cta;
  const long long u_end = min(U, u + units_per_cta);
  int par = 0;

  while (u < u_end) {
    const long long rs = u / T;
    const int t_begin = (int)(u - rs * T);
    const int t_stop = (int)min((long long)T, (long long)t_begin + (u_end - u));
    const int r = (int)(rs / S), s = (int)(rs - (long long)r * S);

    // ---- per-thread parameters of group g --------------------------------------------------
    QpThreadState st;
    const int g = s * kQpGroups + tid;
    st.active = g < NG;
    st.h0 = 8 * g;
    st.c0 = 0;
    st.n = 0;
    st.zbase = 0;
    if (st.active) {
      const GroupLayout L = group_layout(keep_idx, k, H, st.h0);
      st.c0 = L.c0;
      st.n = L.n;
      int j = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const size_t p = (size_t)r * H + st.h0 + i;
        const int z = zero[p];
        st.inv[i] = inv_scale[p];
        st.lo[i] = -z;
        st.hi[i] = 15 - z;
        const bool kept = (L.kmask >> i) & 1u;
        st.mul[i] = kept ? 0u : (1u << (4 * j));
        j += kept ? 0 : 1;
        st.zbase += (uint32_t)z * st.mul[i];
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        st.inv[i] = 0.0f;
        st.lo[i] = 0;
        st.hi[i] = 0;
        st.mul[i] = 0u;
      }
    }

    // ---- slice ownership (same values in every thread) -------------------------------------
    const int ha = s * kQpGroups * 8, hb = min(H, ha + kQpGroups * 8);
    const int ja = lower_bound_i32(keep_idx, k, ha), jb = lower_bound_i32(keep_idx, k, hb);
    // entries below 0 or from H up belong to no slice: report them
    if (tid == 0 && ((s == 0 && ja != 0) || (s == S - 1 && jb != k))) record_error(HQ_ERR_BAD_INDEX);
    const int Ca = min(max(ha - ja, 0), Hr), Cb = min(max(hb - jb, 0), Hr);
    const int Wb = (Ca + 7) >> 3, We = (Cb + 7) >> 3;  // owned words [Wb, We)
    const int nw = max(We - Wb, 0);
    const int nhalo = (We > Wb) ? (8 * We - Cb) : 0;  // 0..7 codes from the next slice

    // halo lane: one non-kept feature after the slice
    float h_inv = 0.0f;
    int h_col = 0, h_lo = 0, h_hi = 0, h_z = 0, h_shift = 0;
    const bool is_halo = tid < nhalo;
    if (is_halo) {
      h_col = checked_col(rest_idx, Cb + tid, H);
      const size_t p = (size_t)r * H + h_col;
      h_z = zero[p];
      h_inv = inv_scale[p];
      h_lo = -h_z;
      h_hi = 15 - h_z;
      h_shift = 4 * ((Cb + tid) & 7);
    }

    const int w0 = st.c0 >> 3, sh = 4 * (st.c0 & 7);

    for (int t = t_begin; t < t_stop; t += kQpRows) {
      const int nrows = min(kQpRows, t_stop - t);
      const size_t row0 = (size_t)r * T + t;

      // ---- phase A: codes into the word buffer, side copies -------------------------------
      uint4 xv[kQpRows];
#pragma unroll
      for (int m = 0; m < kQpRows; ++m)
        if (st.active && m < nrows) xv[m] = ld_stream16(x + (row0 + m) * H + st.h0);
#pragma unroll
      for (int m = 0; m < kQpRows; ++m) {
        if (m >= nrows) break;
        if (st.active && st.n > 0) {
          uint32_t V = st.zbase;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = __fmul_rn(bf16_at(xv[m], i), st.inv[i]);
            int c = __float2int_rn(a);  // saturating; NaN -> 0
            c = min(max(c, st.lo[i]), st.hi[i]);
            V += (uint32_t)c * st.mul[i];
          }
          const uint32_t lo_part = V << sh;
          const uint32_t hi_part = sh ? (V >> (32 - sh)) : 0u;
          if (lo_part && w0 >= Wb && w0 < We) atomicOr(&s_buf[par][m][w0 - Wb], lo_part);
          if (hi_part && w0 + 1 >= Wb && w0 + 1 < We) atomicOr(&s_buf[par][m][w0 + 1 - Wb], hi_part);
        }
        if (is_halo) {
          const uint16_t b = x[(row0 + m) * H + h_col];
          const float a = __fmul_rn(__uint_as_float((uint32_t)b << 16), h_inv);
          int c = __float2int_rn(a);
          c = min(max(c, h_lo), h_hi) + h_z;
          if (c) atomicOr(&s_buf[par][m][We - 1 - Wb], (uint32_t)c << h_shift);
        }
        for (int j = ja + tid; j < jb; j += kQpThreads) {
          const int col = checked_col(keep_idx, j, H);
          side[(row0 + m) * k + j] = x[(row0 + m) * H + col];
        }
      }
      __syncthreads();

      // ---- phase B: owned words out, buffer cleared ----------------------------------------
      for (int m = 0; m < nrows; ++m) {
        uint32_t* dst = codes + (row0 + m) * Wr + Wb;
        for (int i = tid; i < nw; i += kQpThreads) {
          dst[i] = s_buf[par][m][i];
          s_buf[par][m][i] = 0u;
        }
      }
      par ^= 1;
    }
    u += t_stop - t_begin;
  }
}

}  // namespace hq
