// k_quantize.cuh -- Quantize-pack, the sending side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): kept features are copied to the BF16 side buffer, all others
// become 4-bit codes q = clamp(rint(x*inv_scale)+zero, 0, 15) packed 8 per uint32 in rest_idx
// order.
//
// Work decomposition.  A slice is 256 features; a work unit is one (rank, 64-row block) of a
// slice, numbered rank-major, u = rank * NB + block.  The grid is one wave of S slices x J CTAs:
// CTA j of every slice takes the same contiguous range of units [j*U/J, (j+1)*U/J) (U = P*NB), so
// the ranges differ by at most one unit and a CTA changes rank at most a few times.  The CTAs of
// the S slices that share j write the same rows of codes and side at about the same time: the
// 32-byte sectors those rows share at slice boundaries are completed in L2 before eviction
// instead of costing a read-modify-write in HBM each time.  Blocks are numbered slice-minor
// (blockIdx = j*S + s), so the S CTAs of one j are launched together and land in the same round
// of CTAs per SM; the first CTA resident on an SM gets more of its issue slots than the second,
// and with slice-major numbering the slices sharing rows drifted apart by up to 15%.  In a CTA, warp 8 is the producer: one lane issues, per unit, one TMA load of a
// 64-row tile of the slice's 256 features and the 8 after them (a box of 132 32-bit elements, so
// the halo features below are staged too in the common case), into a 3-stage ring.  Warps 0..7
// are consumers; warp w quantizes rows 8w..8w+7 of each tile, lane l the 8 features 8l..8l+7
// (parameters in registers, reloaded only when the unit's rank changes).
//
// Packing.  Per lane: inv_scale, the clamp bounds -zero and 15-zero and a nibble multiplier 16^j
// (0 for a kept feature, j = the feature's rank among the group's non-kept ones) for its 8
// features.  The group's code word is V = sum_i (zero_i + clamp_i) * 16^j_i: every nibble stays
// in [0,15], so the sum is the packed word of the group's n non-kept codes.  Its compact position
// c0 is in general not a multiple of 8, so V is split across two words and OR-ed into a per-warp
// word buffer in shared memory, from which whole words are stored with coalesced 32-bit stores.
//
// Ownership of compact words: a slice owns the words whose first nibble one of its groups
// produces; it drops nibbles that fall into the previous slice's last word and completes its own
// last word from the next <= 7 non-kept features of the next slice (the "halo": their columns
// come from the kept list, rest_idx being the complement of keep_idx; they are spread over the
// lanes as (row, feature) pairs and read from the staged tile when they lie within its 8 extra
// columns, else from global memory).  So every codes word is written by
// exactly one CTA.  Kept values are copied from the staged tile to the side buffer (16 bytes per
// kept feature and warp when T % 8 == 0).
//
// Roofline: HBM-bound; 2 bytes read + 0.5 byte written per non-kept element, 2 + 2 per kept one.
// No memory beyond the inputs and outputs is used.
#pragma once

#include "hq_common.cuh"
#include "hq_tma.cuh"

namespace hq {

constexpr int kQtWarps = 8;                             // consumer warps
constexpr int kQtThreads = 32 * (kQtWarps + 1);         // + one producer warp
constexpr int kQtRowsPerWarp = 8;
constexpr int kQtTileRows = kQtWarps * kQtRowsPerWarp;  // 64
constexpr int kQtStages = 3;
constexpr int kQtSlice = 256;                           // features per slice
constexpr int kQtBoxCols = kQtSlice + 8;                // staged features per row: the slice and 8 beyond
constexpr int kQtBoxU32 = kQtBoxCols / 2;               // box inner dim in 32-bit elements (<= 256)
constexpr int kQtBufWords = 36;                         // >= 33 owned words + 2 guard slots per row
constexpr int kQtHaloSlots = 2;                         // (row, halo feature) pairs per lane
constexpr int kQtKeptSlots = 4;                         // (row, kept feature) pairs per lane
constexpr int kQtHaloCand = 16;                         // features after the slice whose parameters are preloaded
constexpr int kQtStartBarrier = 2;                      // named barrier: consumers' set-up loads issued
constexpr int kQtMaxFastKept = 32 * kQtKeptSlots / kQtRowsPerWarp;  // slices with more copy in a loop
constexpr unsigned kQtTileBytes = kQtTileRows * kQtBoxCols * 2;

struct QtSmem {
  alignas(128) uint16_t tile[kQtStages][kQtTileRows][kQtBoxCols];
  uint32_t buf[kQtWarps][kQtRowsPerWarp][kQtBufWords];
  int klist[kQtSlice + kQtHaloCand];  // the slice's kept features, then those among the halo candidates
  int kcnt[3];
  uint32_t gkmask[kQtSlice / 8];  // per group of the slice: kept mask, kept features before it
  int gj0[kQtSlice / 8];
  TmaRing<kQtStages> ring;
  int abort;
};

// Slice facts of the consumers.
struct QtSlice {
  int ha, hb, ja, jb, Ca, Cb, Wb, We, nw, nhalo;
};

// ja, jb = number of kept features before ha and before hb.
__device__ __forceinline__ QtSlice qt_slice(int ja, int jb, int H, int k, int s) {
  QtSlice q;
  const int Hr = H - k;
  q.ha = s * kQtSlice;
  q.hb = min(H, q.ha + kQtSlice);
  q.ja = ja;
  q.jb = jb;
  q.Ca = min(max(q.ha - q.ja, 0), Hr);
  q.Cb = min(max(q.hb - q.jb, 0), Hr);
  q.Wb = (q.Ca + 7) >> 3;
  q.We = (q.Cb + 7) >> 3;
  q.nw = max(q.We - q.Wb, 0);
  q.nhalo = (q.We > q.Wb) ? (8 * q.We - q.Cb) : 0;
  return q;
}

// The idx-th (from 0) feature at or after hb that is not kept: compact position Cb + idx.
// cand_kept: bit d set when feature hb + d (d < kQtHaloCand) is kept.  Features beyond the
// candidates are found by walking keep_idx from jc (the first kept feature >= hb + kQtHaloCand);
// every entry read is range-checked.
__device__ __forceinline__ int qt_rest_col(int idx, int hb, uint32_t cand_kept, const int32_t* __restrict__ keep_idx,
                                           int k, int jc, int H) {
  int n = 0;
#pragma unroll
  for (int d = 0; d < kQtHaloCand; ++d) {
    if (!((cand_kept >> d) & 1u)) {
      if (n == idx) return hb + d;
      ++n;
    }
  }
  int j = jc;
  for (int c = hb + kQtHaloCand; c < H; ++c) {
    const int kj = j < k ? checked_col(keep_idx, j, H) : H;
    if (kj == c) {
      ++j;
      continue;
    }
    if (n == idx) return c;
    ++n;
  }
  record_error(HQ_ERR_BAD_INDEX);
  return H - 1;
}

// A lane's 8 parameters: inv_scale and zero of features h0 .. h0+7 of one rank.
struct QtParams {
  float4 i0, i1;
  uint2 z;
};
__device__ __forceinline__ QtParams qt_load_params(const float* __restrict__ inv_scale,
                                                   const uint8_t* __restrict__ zero, size_t p, bool on) {
  QtParams r;
  r.i0 = r.i1 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  r.z = make_uint2(0u, 0u);
  if (on) {  // p is a multiple of 8; both arrays are 16-byte aligned
    r.i0 = __ldg(reinterpret_cast<const float4*>(inv_scale + p));
    r.i1 = __ldg(reinterpret_cast<const float4*>(inv_scale + p) + 1);
    r.z = __ldg(reinterpret_cast<const uint2*>(zero + p));
  }
  return r;
}

__global__ void __launch_bounds__(kQtThreads, 2) quantize_pack_tma_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const uint16_t* __restrict__ x, int ldx, int P, int T, int H,
    int k, const int32_t* __restrict__ keep_idx, const int32_t* __restrict__ rest_idx,
    const float* __restrict__ inv_scale, const uint8_t* __restrict__ zero, uint32_t* __restrict__ codes,
    uint16_t* __restrict__ side, int S, int J, WaitLimits lim) {
  extern __shared__ __align__(128) unsigned char s_raw[];
  QtSmem& sm = *reinterpret_cast<QtSmem*>(s_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = blockIdx.x / S, s = blockIdx.x - j * S;  // slice-minor numbering
  const int NB = (T + kQtTileRows - 1) / kQtTileRows;  // 64-row blocks per rank
  const long long U = (long long)P * NB;
  const int u0 = (int)(U * j / J), u1 = (int)(U * (j + 1) / J);
  const int n_units = u1 - u0;  // unit u0 + i = (rank (u0+i) / NB, block (u0+i) % NB)

  if (threadIdx.x == 0) {
    sm.ring.init(kQtWarps);
    sm.abort = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kQtWarps * kQtRowsPerWarp * kQtBufWords; i += kQtThreads)
    (&sm.buf[0][0][0])[i] = 0u;
  __syncthreads();
  volatile int* abort = &sm.abort;

  // ---------------------------------------------------------------- producer warp
  if (warp == kQtWarps) {
    // the first tiles go out after the consumers' set-up loads (which then are not queued
    // behind them); the consumers arrive on this barrier before they wait for anything
    named_barrier_sync_id(kQtStartBarrier, kQtThreads);
    if (lane == 0) {
      prefetch_tensor_map(&tmap_x);
      producer_start_delay(lim.start_delay);
      int issued = 0;
      int r = u0 / NB, b = u0 - (u0 / NB) * NB;  // unit (rank r, row block b), advanced incrementally
      for (int i = 0; i < n_units; ++i) {
        if (i > 0 && ++b == NB) {
          b = 0;
          ++r;
        }
        if (!sm.ring.acquire(i, abort, lim.producer)) break;
        const int st = i % kQtStages;
        const int row = r * T + b * kQtTileRows;
        mbar_arrive_expect_tx(&sm.ring.full[st], kQtTileBytes);
        tma_load_2d(&sm.tile[st][0][0], &tmap_x, (s * kQtSlice) / 2, row, &sm.ring.full[st]);
        ++issued;
      }
      if (*abort) sm.ring.drain(issued, lim.producer);
    }
    return;
  }

  // ---------------------------------------------------------------- consumer warps
  const int Hr = H - k, Wr = Hr / 8, NG = H / 8;
  int r = u0 / NB, b = u0 - (u0 / NB) * NB;
  constexpr int kConsumers = 32 * kQtWarps;
  const int ha0 = s * kQtSlice, hb0 = min(H, ha0 + kQtSlice);
  const int g = s * (kQtSlice / 8) + lane;  // this lane's group
  const bool active = g < NG;
  // Set-up loads first, independent of one another so that they cost one round trip together:
  // this lane's parameters for the first unit's rank, the parameters of the kQtHaloCand features
  // after the slice (lane d of every warp: feature hb0 + d; the halo is among them unless kept
  // features crowd the start of the next slice), and one keep_idx entry per thread.
  QtParams pr = qt_load_params(inv_scale, zero, (size_t)r * H + 8 * g, active && n_units > 0);
  float hc_inv = 0.0f;
  uint32_t hc_z = 0;
  if (lane < kQtHaloCand && hb0 + lane < H && n_units > 0) {
    hc_inv = __ldg(inv_scale + (size_t)r * H + hb0 + lane);
    hc_z = __ldg(zero + (size_t)r * H + hb0 + lane);
  }
  const int kv0 = (int)threadIdx.x < k ? __ldg(keep_idx + threadIdx.x) : 0x7FFFFFFF;
  named_barrier_arrive_id(kQtStartBarrier, kQtThreads);
  // the slice's kept features and those among the halo candidates
  const SliceKept3 sk = slice_kept3(kv0, keep_idx, k, ha0, hb0, hb0 + kQtHaloCand, sm.kcnt, sm.klist,
                                    kQtSlice + kQtHaloCand, kConsumers);
  const QtSlice q = qt_slice(sk.ja, sk.jb, H, k, s);
  if (threadIdx.x == 0 && ((s == 0 && q.ja != 0) || (s == S - 1 && q.jb != k) || q.jb - q.ja > kQtSlice))
    record_error(HQ_ERR_BAD_INDEX);
  // the groups' layouts, the same for every rank
  if (warp == 0) {
    const GroupLayout Lg = active ? group_layout_list(sm.klist, min(q.jb - q.ja, kQtSlice), q.ja, H, k, 8 * g)
                                  : GroupLayout{0, 0, 0u, 0};
    sm.gkmask[lane] = Lg.kmask;
    sm.gj0[lane] = Lg.j0;
  }
  // kept features among the halo candidates (a candidate past H counts as kept: never a halo)
  uint32_t cand_kept = (hb0 + kQtHaloCand > H) ? ~0u << max(H - hb0, 0) : 0u;
  for (int i = min(q.jb - q.ja, kQtSlice); i < min(sk.jc - sk.ja, kQtSlice + kQtHaloCand); ++i) {
    const int d = sm.klist[i] - hb0;
    if (d >= 0 && d < kQtHaloCand) cand_kept |= 1u << d;
  }
  group_sync(kConsumers);
  GroupLayout L{0, 0, 0u, 0};
  if (active) {
    L.kmask = sm.gkmask[lane];
    L.j0 = sm.gj0[lane];
    L.n = 8 - __popc(L.kmask);
    L.c0 = min(max(8 * g - L.j0, 0), Hr);
  }
  float inv[8];
  int lo[8], hi[8];
  uint32_t mul[8], zbase = 0;
  // halo work: pair p = lane + 32c (c < kQtHaloSlots) is (row p / nhalo, halo feature p % nhalo);
  // h_pack = row | shift << 4 | zero << 9 | (column - ha) << 13 (row 8: no pair)
  uint32_t h_pack[kQtHaloSlots];
  float h_inv[kQtHaloSlots];
  // Kept copies.  The side buffer is feature-major, side[r][j][t], so the warp's 8 rows of one
  // kept feature are 16 contiguous bytes (the CTA's warps fill 128 per kept feature and tile).
  // When they are 16-byte aligned (T % 8 == 0) and the slice has at most 32 kept features, lane
  // j copies kept feature j with one 16-byte store (k_vcol = its column - ha).  Otherwise, for a
  // slice with at most kQtMaxFastKept: pair p = lane + 32c (c < kQtKeptSlots) is (row lane % 8,
  // kept feature lane / 8 + 4c), present while lane / 8 + 4c < nk, byte c of k_cols = its column
  // - ha, and the pair's element counted from the unit's rank and the warp's first row is
  // k_side0 + 4c*T; more kept features are copied in a loop.
  const int nk = q.jb - q.ja;
  const bool k_generic = nk > kQtMaxFastKept;
  const int k_m = lane % kQtRowsPerWarp, k_j = lane / kQtRowsPerWarp;
  const int k_row_off = (warp * kQtRowsPerWarp + k_m) * kQtBoxCols;
  const size_t k_side0 = (size_t)(q.ja + k_j) * T + k_m;
  uint32_t k_cols = 0;
#pragma unroll
  for (int c = 0; c < kQtKeptSlots; ++c) {
    if (!k_generic && k_j + 4 * c < nk) {
      const int col = sm.klist[k_j + 4 * c];
      k_cols |= (uint32_t)min(max(col - q.ha, 0), kQtSlice - 1) << (8 * c);
    }
  }
  const bool k_vec = (T % 8) == 0 && nk <= 32;
  const int k_vcol = lane < nk ? min(max(sm.klist[lane] - q.ha, 0), kQtSlice - 1) : 0;
  // This lane's parameters for rank r: inv_scale, the clamp bounds -zero and 15-zero, the nibble
  // multipliers and the zero points' packed sum.
  auto set_rank = [&](const QtParams& pr) {
    const float pinv[8] = {pr.i0.x, pr.i0.y, pr.i0.z, pr.i0.w, pr.i1.x, pr.i1.y, pr.i1.z, pr.i1.w};
    zbase = 0;
    int j = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const bool kept = (L.kmask >> e) & 1u;
      const int z = (int)(((e < 4 ? pr.z.x : pr.z.y) >> (8 * (e & 3))) & 0xFFu);
      inv[e] = pinv[e];
      lo[e] = -z;
      hi[e] = 15 - z;
      mul[e] = (active && !kept) ? (1u << (4 * j)) : 0u;
      j += kept ? 0 : 1;
      zbase += (uint32_t)z * mul[e];
    }
  };
  set_rank(pr);
  const int slot = (L.c0 >> 3) - q.Wb + 1;
  const int sh = 4 * (L.c0 & 7);
  // Halo pairs: pair p = lane + 32c is (row p / nhalo, halo feature p % nhalo), the feature at
  // compact position Cb + p % nhalo, whose column stays fixed for the launch; the first rank's
  // parameters come from the lane that loaded that candidate (or from memory past the
  // candidates).  h_pack = row | shift << 4 | zero << 9 | (column - ha) << 13 (row 8: no pair).
  bool halo_staged = true;  // every halo feature lies in the staged columns [ha, ha + kQtBoxCols)
  if (q.nhalo > 0)
    halo_staged = qt_rest_col(q.nhalo - 1, hb0, cand_kept, keep_idx, k, sk.jc, H) < q.ha + kQtBoxCols;
#pragma unroll
  for (int c = 0; c < kQtHaloSlots; ++c) {
    const int p = lane + 32 * c;
    const bool has = p < q.nhalo * kQtRowsPerWarp;
    const int col = has ? qt_rest_col(p % q.nhalo, hb0, cand_kept, keep_idx, k, sk.jc, H) : hb0;
    const int off = min(max(col - hb0, 0), kQtHaloCand - 1);
    float c_inv = __shfl_sync(0xFFFFFFFFu, hc_inv, off);
    uint32_t c_z = __shfl_sync(0xFFFFFFFFu, hc_z, off);
    h_pack[c] = kQtRowsPerWarp;
    h_inv[c] = 0.0f;
    if (has) {
      if (col - hb0 >= kQtHaloCand) {
        const size_t pp = (size_t)r * H + col;
        c_inv = __ldg(inv_scale + pp);
        c_z = __ldg(zero + pp);
      }
      const int row = p / q.nhalo, idx = p - row * q.nhalo;
      h_inv[c] = c_inv;
      h_pack[c] = (uint32_t)row | (uint32_t)(4 * ((q.Cb + idx) & 7)) << 4 | (c_z & 15u) << 9 |
                  (uint32_t)(col - q.ha) << 13;
    }
  }
  uint32_t(*buf)[kQtBufWords] = sm.buf[warp];

  for (int i = 0; i < n_units; ++i) {
    if (i > 0 && ++b == NB) {  // a new rank: this lane's parameters, and the halo features'
      b = 0;
      ++r;
      set_rank(qt_load_params(inv_scale, zero, (size_t)r * H + 8 * g, active));
#pragma unroll
      for (int c = 0; c < kQtHaloSlots; ++c) {
        if ((h_pack[c] & 15u) < kQtRowsPerWarp) {
          const size_t pp = (size_t)r * H + q.ha + (h_pack[c] >> 13);
          h_inv[c] = __ldg(inv_scale + pp);
          h_pack[c] = (h_pack[c] & ~(15u << 9)) | ((uint32_t)__ldg(zero + pp) & 15u) << 9;
        }
      }
    }
    if (!sm.ring.wait_full(i, abort, lim.consumer)) break;
    const int st = i % kQtStages;
    const int t_base = b * kQtTileRows + warp * kQtRowsPerWarp;  // this warp's first row
    const int nrows = max(0, min(kQtRowsPerWarp, T - t_base));
    const uint16_t* tile = &sm.tile[st][0][0];

    if (active && L.n > 0) {
#pragma unroll
      for (int m = 0; m < kQtRowsPerWarp; ++m) {
        const uint4 v = reinterpret_cast<const uint4*>(tile + (warp * kQtRowsPerWarp + m) * kQtBoxCols)[lane];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t V = zbase;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float a0, a1;
          fmul2(a0, a1, __uint_as_float(w[e / 2] << 16), __uint_as_float(w[e / 2] & 0xFFFF0000u), inv[e],
                inv[e + 1]);
          int c0 = __float2int_rn(a0), c1 = __float2int_rn(a1);  // saturating; NaN -> 0
          c0 = min(max(c0, lo[e]), hi[e]);
          c1 = min(max(c1, lo[e + 1]), hi[e + 1]);
          V += (uint32_t)c0 * mul[e] + (uint32_t)c1 * mul[e + 1];
        }
        atomicOr(&buf[m][slot], V << sh);
        atomicOr(&buf[m][slot + 1], __funnelshift_l(V, 0u, sh));  // V >> (32 - sh), 0 when sh == 0
      }
    }
    // halo codes: features of the next slice completing this slice's last word
#pragma unroll
    for (int c = 0; c < kQtHaloSlots; ++c) {
      const int h_row = h_pack[c] & 15u;
      if (h_row < nrows) {
        const int h_shift = (h_pack[c] >> 4) & 31u, h_z = (h_pack[c] >> 9) & 15u, h_off = h_pack[c] >> 13;
        uint32_t hb16;
        if (halo_staged) {
          hb16 = (uint32_t)tile[(warp * kQtRowsPerWarp + h_row) * kQtBoxCols + h_off] << 16;
        } else {  // halo features spread beyond the staged columns: read them directly
          hb16 = (uint32_t)x[((size_t)r * T + t_base + h_row) * ldx + q.ha + h_off] << 16;
        }
        int cc = __float2int_rn(__fmul_rn(__uint_as_float(hb16), h_inv[c]));
        cc = min(max(cc, -h_z), 15 - h_z) + h_z;
        atomicOr(&buf[h_row][q.nw], (uint32_t)cc << h_shift);
      }
    }
    // kept values straight from the staged tile
    uint16_t* srow = side + (size_t)r * k * T + t_base;
    if (k_vec && nrows == kQtRowsPerWarp) {
      if (lane < nk) {
        const uint16_t* tc = tile + (warp * kQtRowsPerWarp) * kQtBoxCols + k_vcol;
        uint4 v;
        v.x = (uint32_t)tc[0] | (uint32_t)tc[kQtBoxCols] << 16;
        v.y = (uint32_t)tc[2 * kQtBoxCols] | (uint32_t)tc[3 * kQtBoxCols] << 16;
        v.z = (uint32_t)tc[4 * kQtBoxCols] | (uint32_t)tc[5 * kQtBoxCols] << 16;
        v.w = (uint32_t)tc[6 * kQtBoxCols] | (uint32_t)tc[7 * kQtBoxCols] << 16;
        *reinterpret_cast<uint4*>(srow + (size_t)(q.ja + lane) * T) = v;
      }
    } else if (!k_generic) {
#pragma unroll
      for (int c = 0; c < kQtKeptSlots; ++c)
        if (k_j + 4 * c < nk && k_m < nrows)
          srow[k_side0 + (size_t)(4 * c) * T] = tile[k_row_off + ((k_cols >> (8 * c)) & 255u)];
    } else {
      for (int p = lane; p < nk * kQtRowsPerWarp; p += 32) {
        const int jj = p / kQtRowsPerWarp, m = p % kQtRowsPerWarp;
        if (m < nrows) {
          const int col = checked_col(keep_idx, q.ja + jj, H);
          srow[(size_t)(q.ja + jj) * T + m] =
              tile[(warp * kQtRowsPerWarp + m) * kQtBoxCols + min(max(col - q.ha, 0), kQtSlice - 1)];
        }
      }
    }
    __syncwarp();
    if (lane == 0) sm.ring.release(i);
    // owned words out (slots 1..nw); each lane clears exactly the slots it read
    uint32_t* crow = codes + ((size_t)r * T + t_base) * Wr + q.Wb + lane;
    const bool w1 = lane < q.nw;
    if (nrows == kQtRowsPerWarp) {
#pragma unroll
      for (int m = 0; m < kQtRowsPerWarp; ++m) {
        const uint32_t a = buf[m][lane + 1];
        buf[m][lane + 1] = 0u;
        if (w1) crow[(size_t)m * Wr] = a;
      }
    } else {
#pragma unroll
      for (int m = 0; m < kQtRowsPerWarp; ++m) {
        const uint32_t a = buf[m][lane + 1];
        buf[m][lane + 1] = 0u;
        if (w1 && m < nrows) crow[(size_t)m * Wr] = a;
      }
    }
    // Slots above 32 only ever hold nonzero bits when the slice owns 33 words (a hi part or a
    // halo code goes at most to slot nw); otherwise they only receive zero ORs.
    if (q.nw > 32) {
      if (lane + 33 < kQtBufWords) {
#pragma unroll
        for (int m = 0; m < kQtRowsPerWarp; ++m) {
          const uint32_t c = buf[m][lane + 33];
          buf[m][lane + 33] = 0u;
          if (m < nrows && lane + 32 < q.nw) crow[(size_t)m * Wr + 32] = c;
        }
      }
    }
    __syncwarp();
  }
}

}  // namespace hq
