// k_dequant.cuh -- Dequant-reduce, the receiving side of bullet "Inference" (page
// "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section "The
// Hybrid Quantization Algorithm"): each rank's shard is converted back and the ranks are summed
// in rank order, acc = fma(float(q_r - zero_r), scale_r, acc) for 4-bit features and
// acc = acc + side_r for kept ones.
//
// Work decomposition (both kernels below).  A CTA covers a slice of 32 groups of 8 consecutive
// output features (256 features) and a range of rows; a warp owns the whole slice (one group per
// lane) for kDqR rows at a time and keeps kDqR x 8 fp32 sums in registers while it walks the
// ranks in order.  The CTA's warps share the slice's per-(rank, feature) constants in shared
// memory.  Two ways of staging the code words:
//   - dequant_reduce_tma_kernel (default): a producer warp loads, per (32-row block, rank), one
//     32 x 40-word TMA tile (and a 32-row x 32-feature tile of the side buffer) into a 3-stage
//     mbarrier ring whose slots hold 4 ranks; eight consumer warps take 4 rows each and a
//     kept-sum warp sums the staged side values.  Needs code rows whose byte length is a
//     multiple of 16 ((H-k) % 32 == 0).
//   - dequant_reduce_kernel (any shape): each warp stages its own rows with 4-byte cp.async
//     copies, 8 tiles ahead.
//
// Decoding a group: its n non-kept features occupy compact positions c0..c0+n-1, i.e. at most
// two consecutive words; a funnel shift brings them to bits 0..4n-1 of v.  Feature i's nibble
// is turned into a float without a conversion instruction: (v & (0xF << 4p_i)) | 0x4B000000 is
// the float 2^23 + q*16^p_i; adding the per-(rank, feature) constant -(2^23 + zero*16^p_i)
// gives (q - zero)*16^p_i exactly, and the FMA uses scale/16^p_i, so the product is exactly
// (q - zero)*scale.  p_i <= 4 is arranged by reading features 5..7 from a second view
// v2 = v >> 4b.  Scales below 2^-109 could lose bits when divided by 16^4: a slice that has one
// decodes with explicit shifts and undivided constants instead ("generic" path).  The adds are
// scalar and the FMAs go two at a time through fma.rn.f32x2 (per-lane IEEE, so bit-identical).
// A kept feature gets scale 0 (its decoded value is then multiplied by 0); its sum over the side
// values, in rank order, is formed elsewhere (the kept-sum warp, or lanes of the owning warp
// reading the side buffer) and copied over the owner's sum through shared memory.
//
// Roofline: HBM-bound; per output element P*(0.5*H'/H + 2*k/H) bytes read + 2 (or 4) written.
// No memory beyond the inputs and outputs is used.
#pragma once

#include "hq_common.cuh"
#include "hq_tma.cuh"

namespace hq {

constexpr int kDqSliceGroups = 32;
constexpr int kDqR = 4;  // rows per warp per block

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

// Nibble positions of a group with kept mask km: jpos[i] = rank of feature i among the group's
// non-kept features (its nibble sits at bits 4*jpos[i] of v); pos[i] = in-place position used by
// the fast path (features 5..7 are read from v2 = v >> 4b); returns b.
__device__ __forceinline__ int dq_positions(uint32_t km, int* pos, int* jpos) {
  int j = 0, b = -1;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool kept = (km >> i) & 1u;
    jpos[i] = j;
    if (i >= 5 && !kept && b < 0) b = j;
    j += kept ? 0 : 1;
  }
  if (b < 0) b = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) pos[i] = (i < 5) ? jpos[i] : jpos[i] - b;
  return b;
}

// What one lane needs to decode its group from a staged row of code words.
struct DqLane {
  GroupLayout L;
  int h0;
  bool active;
  bool decode;       // active and at least one non-kept feature
  int my_w;          // first word of the group inside a staged row
  int fsh;           // funnel shift bringing the group's first nibble to bit 0
  int sh2;           // fast path: v2 = v >> sh2
  uint32_t key[8];   // fast path: in-place nibble mask; generic path: nibble shift
};

// max_w: the last staged word a lane may start at (its second word must be staged too); an
// inconsistent index could only move the start, and is clamped.
__device__ __forceinline__ DqLane dq_lane_layout(const GroupLayout& L, int h0, int H, int w_base, int max_w,
                                                 bool generic) {
  DqLane D;
  D.h0 = h0;
  D.active = h0 < H;
  D.L = D.active ? L : GroupLayout{0, 0, 0u, 0};
  int pos[8], jpos[8];
  const int b = dq_positions(D.L.kmask, pos, jpos);
  D.sh2 = 4 * b;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool kept = (D.L.kmask >> i) & 1u;
    D.key[i] = generic ? (uint32_t)(4 * jpos[i]) : (kept ? 0u : (0xFu << (4 * pos[i])));
  }
  D.my_w = min(max((D.L.c0 >> 3) - w_base, 0), max_w);
  D.fsh = 4 * (D.L.c0 & 7);
  D.decode = D.active && D.L.n > 0;
  return D;
}

__device__ __forceinline__ DqLane dq_lane(const int32_t* __restrict__ keep_idx, int k, int H, int s, int lane,
                                          int w_base, int max_w, bool generic) {
  const int h0 = 8 * (s * kDqSliceGroups + lane);
  const GroupLayout L = h0 < H ? group_layout(keep_idx, k, H, h0) : GroupLayout{0, 0, 0u, 0};
  return dq_lane_layout(L, h0, H, w_base, max_w, generic);
}

// Whether this thread's share of slice s has a scale below 2^-109 (the slice then needs the
// generic path); `nthreads` threads split the slice.
__device__ __forceinline__ bool dq_has_tiny_scale(const float* __restrict__ scale, int P, int H, int s,
                                                  int nthreads) {
  const int hs = 8 * s * kDqSliceGroups;
  bool tiny = false;
  for (int idx = threadIdx.x; idx < P * 8 * kDqSliceGroups; idx += nthreads) {
    const int r = idx / (8 * kDqSliceGroups), h = hs + idx % (8 * kDqSliceGroups);
    if (h < H && scale[(size_t)r * H + h] < 0x1p-109f) tiny = true;
  }
  return tiny;
}

// Per-(rank, group) constants of slice s in a conflict-free [P][4][32] float4 layout:
// scale/16^p x8, -(2^23 + zero*16^p) x8 (p = 0 on the generic path).
// group_kmask: the 32 groups' kept masks when already known (in shared memory), else NULL.
__device__ __forceinline__ void dq_fill_constants(float4* s_const, const int32_t* __restrict__ keep_idx,
                                                  const uint32_t* group_kmask, const float* __restrict__ scale,
                                                  const uint8_t* __restrict__ zero, int P, int H, int k,
                                                  int s, bool generic, int nthreads) {
  for (int idx = threadIdx.x; idx < P * 32; idx += nthreads) {
    const int r = idx >> 5, g = idx & 31;
    const int hg = 8 * (s * kDqSliceGroups + g);
    float sc[8], off[8];
    uint32_t km = 0;
    if (hg < H) km = group_kmask ? group_kmask[g] : group_layout(keep_idx, k, H, hg).kmask;
    int pos[8], jpos[8];
    dq_positions(km, pos, jpos);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[i] = 0.0f;
      off[i] = -8388608.0f;  // kept / inactive: decodes to a small value times scale 0
      if (hg < H && !((km >> i) & 1u)) {
        const size_t p = (size_t)r * H + hg + i;
        const int e = generic ? 0 : 4 * pos[i];
        sc[i] = __fmul_rn(scale[p], __int_as_float((127 - e) << 23));  // scale / 16^p, exact
        off[i] = -__int_as_float(0x4B000000 | ((int)zero[p] << e));     // -(2^23 + zero*16^p)
      }
    }
    float4* dst = s_const + (size_t)r * 4 * 32 + g;
    dst[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
    dst[32] = make_float4(sc[4], sc[5], sc[6], sc[7]);
    dst[64] = make_float4(off[0], off[1], off[2], off[3]);
    dst[96] = make_float4(off[4], off[5], off[6], off[7]);
  }
}

// One (rank, group) pair of slice s, idx = rank * 32 + group: the scale and zero of its 8
// features, loaded ahead of the rest of the set-up (nothing in the address depends on the kept
// features).  Pairs past the tensor load nothing.
struct DqPair {
  float4 s0, s1;
  uint2 z;
};
__device__ __forceinline__ DqPair dq_load_pair(const float* __restrict__ scale, const uint8_t* __restrict__ zero,
                                               int P, int H, int s, int idx) {
  DqPair d;
  d.s0 = d.s1 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
  d.z = make_uint2(0u, 0u);
  const int r = idx >> 5, hg = 8 * (s * kDqSliceGroups + (idx & 31));
  if (r < P && hg < H) {  // r*H + hg is a multiple of 8; scale and zero are 16-byte aligned
    const size_t p = (size_t)r * H + hg;
    d.s0 = __ldg(reinterpret_cast<const float4*>(scale + p));
    d.s1 = __ldg(reinterpret_cast<const float4*>(scale + p) + 1);
    d.z = __ldg(reinterpret_cast<const uint2*>(zero + p));
  }
  return d;
}
__device__ __forceinline__ bool dq_pair_tiny(const DqPair& d) {
  return d.s0.x < 0x1p-109f || d.s0.y < 0x1p-109f || d.s0.z < 0x1p-109f || d.s0.w < 0x1p-109f ||
         d.s1.x < 0x1p-109f || d.s1.y < 0x1p-109f || d.s1.z < 0x1p-109f || d.s1.w < 0x1p-109f;
}
// dq_fill_constants() for one pair from its loaded parameters (group_kmask in shared memory).
__device__ __forceinline__ void dq_fill_pair(float4* s_const, const uint32_t* group_kmask, const DqPair& d, int H,
                                             int s, int idx, bool generic) {
  const int r = idx >> 5, g = idx & 31;
  const int hg = 8 * (s * kDqSliceGroups + g);
  const uint32_t km = hg < H ? group_kmask[g] : 0u;
  int pos[8], jpos[8];
  dq_positions(km, pos, jpos);
  const float scv[8] = {d.s0.x, d.s0.y, d.s0.z, d.s0.w, d.s1.x, d.s1.y, d.s1.z, d.s1.w};
  float sc[8], off[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sc[i] = 0.0f;
    off[i] = -8388608.0f;  // kept / inactive: decodes to a small value times scale 0
    if (hg < H && !((km >> i) & 1u)) {
      const int e = generic ? 0 : 4 * pos[i];
      const uint32_t z = ((i < 4 ? d.z.x : d.z.y) >> (8 * (i & 3))) & 0xFFu;
      sc[i] = __fmul_rn(scv[i], __int_as_float((127 - e) << 23));  // scale / 16^p, exact
      off[i] = -__int_as_float(0x4B000000 | ((int)z << e));         // -(2^23 + zero*16^p)
    }
  }
  float4* dst = s_const + (size_t)r * 4 * 32 + g;
  dst[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
  dst[32] = make_float4(sc[4], sc[5], sc[6], sc[7]);
  dst[64] = make_float4(off[0], off[1], off[2], off[3]);
  dst[96] = make_float4(off[4], off[5], off[6], off[7]);
}

// Adds one rank's contribution for R staged rows (row m at st + m * stride words).  kShard: the
// literal reading of the reduction, in which the rank's dequantized value (q - zero) * scale is
// first rounded to bf16 and then added (the default adds the exact product with one FMA).
template <bool kFast, int R, bool kShard>
__device__ __forceinline__ void dq_decode_rows(const DqLane& D, const uint32_t* __restrict__ st, int stride,
                                               const float4* __restrict__ cst, float (&acc)[R][8]) {
  const float4 s0 = cst[0], s1 = cst[32], o0 = cst[64], o1 = cst[96];
  const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const float off[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
  for (int m = 0; m < R; ++m) {
    const uint32_t wlo = st[m * stride + D.my_w];
    // The next word is always inside the staged row (zero past the last code word of a row, or
    // unused words of the staging window); its bits only reach v above the group's nibbles
    // when the group fits in wlo.
    const uint32_t whi = st[m * stride + D.my_w + 1];
    const uint32_t v = __funnelshift_r(wlo, whi, D.fsh);
    float q[8];
    if (kFast) {
      const uint32_t v2 = v >> D.sh2;
      const uint32_t magic = 0x4B000000u;
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __uint_as_float(and_or(i < 5 ? v : v2, D.key[i], magic));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __uint_as_float(((v >> D.key[i]) & 0xFu) | 0x4B000000u);
    }
    // Scalar adds (exact: (q - zero) * 16^p) write their results straight into the register pair
    // the packed FMA reads; a packed add would need its two LOP3 inputs moved into a pair first.
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float d0 = __fadd_rn(q[i], off[i]), d1 = __fadd_rn(q[i + 1], off[i + 1]);
      if (kShard) {
        // (q - zero)*16^p times scale/16^p: the exact (q - zero)*scale, rounded once to fp32,
        // then to bf16
        float v0, v1;
        fmul2(v0, v1, d0, d1, sc[i], sc[i + 1]);
        const uint32_t b = round_bf16x2(v0, v1);
        acc[m][i] = __fadd_rn(acc[m][i], __uint_as_float(b << 16));
        acc[m][i + 1] = __fadd_rn(acc[m][i + 1], __uint_as_float(b & 0xFFFF0000u));
      } else {
        ffma2_acc(acc[m][i], acc[m][i + 1], d0, d1, sc[i], sc[i + 1]);
      }
    }
  }
}

// Owners of kept features ja+kc .. ja+kc+kw-1 take their sums from kept[m * 32 + (j - ja - kc)].
template <int R>
__device__ __forceinline__ void dq_patch_kept(const DqLane& D, float (&acc)[R][8], const float* kept, int ja,
                                              int kc, int kw) {
  if (D.L.kmask) {
    int jk = D.L.j0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((D.L.kmask >> i) & 1u) {
        const int jj = jk - ja - kc;
        if (jj >= 0 && jj < kw) {
#pragma unroll
          for (int m = 0; m < R; ++m) acc[m][i] = kept[m * 32 + jj];
        }
        ++jk;
      }
    }
  }
}

template <typename OutT, int R>
__device__ __forceinline__ void dq_store_rows(const DqLane& D, const float (&acc)[R][8], int ldo, int t0,
                                              int t_last, OutT* __restrict__ out) {
  if (D.active) {
#pragma unroll
    for (int m = 0; m < R; ++m) {
      const int t = t0 + m;
      if (t < t_last) store_row8<OutT>(out + (size_t)t * ldo + D.h0, acc[m]);
    }
  }
}

// Kept features of the warp's slice for rows t0..t0+R-1, read from global memory: each kept
// feature's R side values summed over the P ranks in rank order; owners copy them into their
// sums; then the rows are stored.  When the R rows are whole and 8-byte aligned (R == 4,
// T % 4 == 0) lane l takes kept feature kc + l and reads its 4 rows with one 8-byte load per
// rank (kVec; the TMA kernel, whose register budget is tighter and which stages the side values of
// all but crowded slices, leaves it out); otherwise the lanes take (row, kept feature) pairs,
// 4 rows of 8 features per warp load.  Warp-level only (uses `kept`, R x 32 floats of shared
// memory per warp).
template <typename OutT, int R, bool kVec>
__device__ __forceinline__ void dq_finish_block(const DqLane& D, float (&acc)[R][8],
                                                const uint16_t* __restrict__ side,
                                                const uint16_t* const* side_ranks, float* kept, int P,
                                                int T, int H, int k, int ja, int jb, int t0, int t_last,
                                                OutT* __restrict__ out, int ldo) {
  const int lane = threadIdx.x & 31;
  const int nk = jb - ja;
  const size_t rank_stride = (size_t)k * T;
  // rank r's side buffer: r*k*T into the stacked one, or its own (side_ranks[r])
  auto rank_side = [&](int r) { return side_ranks ? side_ranks[r] : side + r * rank_stride; };
  const bool vec = kVec && R == 4 && (T & 3) == 0 && t0 + R <= t_last;
  for (int kc = 0; kc < nk; kc += 32) {
    const int kw = min(32, nk - kc);
    if (vec) {
      if (lane < kw) {
        const size_t off = (size_t)(ja + kc + lane) * T + t0;  // side[r][j][t], feature-major
        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll 4
        for (int r = 0; r < P; ++r) {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(rank_side(r) + off));
          a0 = __fadd_rn(a0, __uint_as_float(w.x << 16));
          a1 = __fadd_rn(a1, __uint_as_float(w.x & 0xFFFF0000u));
          a2 = __fadd_rn(a2, __uint_as_float(w.y << 16));
          a3 = __fadd_rn(a3, __uint_as_float(w.y & 0xFFFF0000u));
        }
        kept[0 * 32 + lane] = a0;
        kept[1 * 32 + lane] = a1;
        kept[2 * 32 + lane] = a2;
        kept[3 * 32 + lane] = a3;
      }
    } else {
      for (int p = lane; p < R * kw; p += 32) {
        const int jj = p / R, m = p - jj * R;
        const int t = t0 + m;
        float a = 0.0f;
        if (t < t_last) {
          const size_t off = (size_t)(ja + kc + jj) * T + t;
#pragma unroll 8
          for (int r = 0; r < P; ++r)
            a = __fadd_rn(a, __uint_as_float((uint32_t)__ldg(rank_side(r) + off) << 16));
        }
        kept[m * 32 + jj] = a;
      }
    }
    __syncwarp();
    dq_patch_kept<R>(D, acc, kept, ja, kc, kw);
    __syncwarp();
  }
  dq_store_rows<OutT, R>(D, acc, ldo, t0, t_last, out);
}

// Slice bookkeeping shared by both kernels.
struct DqSlice {
  int hs, he, ja, jb, Ca, Cb, w_first, n_words;
};
__device__ __forceinline__ DqSlice dq_slice_from(int ja, int jb, int H, int k, int s, int S) {
  DqSlice q;
  const int Hr = H - k, Wr = Hr / 8;
  q.hs = 8 * s * kDqSliceGroups;
  q.he = min(H, q.hs + 8 * kDqSliceGroups);
  q.ja = ja;
  q.jb = jb;
  if (threadIdx.x == 0 && ((s == 0 && q.ja != 0) || (s == S - 1 && q.jb != k))) record_error(HQ_ERR_BAD_INDEX);
  q.Ca = min(max(q.hs - q.ja, 0), Hr);
  q.Cb = min(max(q.he - q.jb, 0), Hr);
  q.w_first = q.Ca >> 3;
  q.n_words = max(0, min(Wr, (q.Cb >> 3) + 2) - q.w_first);  // words the slice needs per row, <= 35
  return q;
}

__device__ __forceinline__ DqSlice dq_slice(const int32_t* __restrict__ keep_idx, int H, int k, int s, int S) {
  const int hs = 8 * s * kDqSliceGroups, he = min(H, hs + 8 * kDqSliceGroups);
  return dq_slice_from(lower_bound_i32(keep_idx, k, hs), lower_bound_i32(keep_idx, k, he), H, k, s, S);
}

// ======================================================================== TMA kernel (default)
// A ring slot holds the code tiles (and side tiles) of kDtG consecutive ranks for one block of
// rows, so a consumer warp waits and releases once per kDtG ranks, and the rank loop inside a
// slot has no synchronisation in it.
constexpr int kDtWarps = 8;                      // consumer warps
constexpr int kDtKeptWarp = kDtWarps + 1;        // the kept-sum warp (warp kDtWarps loads)
constexpr int kDtThreads = 32 * (kDtWarps + 2);  // + the producer warp + the kept-sum warp
constexpr int kDtR = 4;                          // rows per consumer warp per block
constexpr int kDtMinBlocks = 2;                  // CTAs per SM the register budget is set for
constexpr int kDtTileRows = kDtWarps * kDtR;     // 32
constexpr int kDtWords = 40;                     // staged words per row (box inner dim)
constexpr int kDtG = 4;                          // ranks per ring slot
constexpr int kDtStages = 3;
constexpr unsigned kDtTileBytes = kDtTileRows * kDtWords * 4;
constexpr int kDtSideCols = 32;                  // side box height: kept features staged per slice
constexpr int kDtMaxStagedKept = kDtSideCols;    // slices with more read the side buffer from HBM
constexpr unsigned kDtSideBytes = kDtTileRows * kDtSideCols * 2;
static_assert(kDtR == 4, "a consumer lane reads its rows' kept sums as one float4");
static_assert(kDtTileRows == 32, "the kept-sum warp covers a block's 32 rows with 8 lanes of 4 rows");

struct DtSmem {
  alignas(128) uint32_t tile[kDtStages][kDtG][kDtTileRows][kDtWords];
  alignas(128) uint16_t side[kDtStages][kDtG][kDtSideCols][kDtTileRows];  // [kept feature][row]
  union {
    float kept[kDtWarps][kDtR * 32];           // side read from HBM: per-warp kept sums
    float ksum[2][kDtSideCols][kDtTileRows];   // side staged: a block's kept sums, [kept feature][row]
  } k;
  uint64_t ksum_full[2];   // the kept-sum warp has written ksum[b]
  uint64_t ksum_empty[2];  // every consumer warp has read ksum[b]
  int klist[8 * kDqSliceGroups];  // the slice's kept features
  int kcnt[3];
  uint32_t gkmask[kDqSliceGroups];  // per group of the slice: kept mask and kept features before it
  int gj0[kDqSliceGroups];
  TmaRing<kDtStages> ring;
  int abort;
  // followed by the constants: float4 [P][4][32]
};

inline size_t dt_smem_bytes(int P) { return sizeof(DtSmem) + 128 + (size_t)P * 4 * 32 * 16; }

// The nr ranks of one ring slot, in rank order: 4-bit features of the warp's rows into acc
// (cst = this lane's constants of the slot's first rank).  kFull: the slot holds kDtG ranks, so
// the rank loop carries no per-rank test (worth 5% of the kernel's time).
template <bool kFast, bool kShard, bool kFull>
__device__ __forceinline__ void dt_slot(const DqLane& D, const DtSmem& sm, int st_i, int warp, int nr,
                                        const float4* __restrict__ cst, float (&acc)[kDtR][8]) {
  if (!D.decode) return;
#pragma unroll
  for (int j = 0; j < kDtG; ++j)
    if (kFull || j < nr)
      dq_decode_rows<kFast, kDtR, kShard>(D, &sm.tile[st_i][j][warp * kDtR][0], kDtWords, cst + j * 4 * 32, acc);
}

// The kept-sum warp, for slices whose side values are staged: lane l sums rows 4(l % 8) ..
// 4(l % 8) + 3 of kept features l / 8, l / 8 + 4, ... (< nk <= NK) over the ranks in order, four
// rows per 8-byte load of a side tile; the sums of block bi go to ksum[bi & 1].  It releases ring
// slots like a consumer warp.
template <int NK>
__device__ __forceinline__ void dt_kept_sums(DtSmem& sm, int nk, int P, int nblk, int n_groups,
                                             volatile int* abort, long long wait_limit) {
  constexpr int NF = NK / 4;  // kept features per lane
  const int lane = threadIdx.x & 31;
  const int m0 = 4 * (lane & 7), f0 = lane >> 3;
  int st_i = 0;
  unsigned phase = 0;
  for (int bi = 0; bi < nblk && !*abort; ++bi) {
    float a[NF][4];
#pragma unroll
    for (int i = 0; i < NF; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) a[i][m] = 0.0f;
    bool ok = true;
    for (int g = 0; g < n_groups; ++g) {
      if (!mbar_wait(&sm.ring.full[st_i], phase, abort, wait_limit)) {
        ok = false;
        break;
      }
      const int nr = min(kDtG, P - g * kDtG);
#pragma unroll
      for (int j = 0; j < kDtG; ++j) {
        if (j < nr) {
#pragma unroll
          for (int i = 0; i < NF; ++i) {
            if (f0 + 4 * i < nk) {
              const uint2 w = *reinterpret_cast<const uint2*>(&sm.side[st_i][j][f0 + 4 * i][m0]);
              fadd2(a[i][0], a[i][1], a[i][0], a[i][1], __uint_as_float(w.x << 16),
                    __uint_as_float(w.x & 0xFFFF0000u));
              fadd2(a[i][2], a[i][3], a[i][2], a[i][3], __uint_as_float(w.y << 16),
                    __uint_as_float(w.y & 0xFFFF0000u));
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ring.empty[st_i]);
      if (++st_i == kDtStages) {
        st_i = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    const int buf = bi & 1;
    if (bi >= 2 && !mbar_wait(&sm.ksum_empty[buf], ((bi >> 1) - 1) & 1, abort, wait_limit)) break;
#pragma unroll
    for (int i = 0; i < NF; ++i)
      if (f0 + 4 * i < nk)
        *reinterpret_cast<float4*>(&sm.k.ksum[buf][f0 + 4 * i][m0]) = make_float4(a[i][0], a[i][1], a[i][2], a[i][3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.ksum_full[buf]);
  }
}

// Owners of the slice's kept features take the sums of the warp's kDtR rows from one ksum buffer.
__device__ __forceinline__ void dt_patch_kept(const DqLane& D, float (&acc)[kDtR][8], const float* ksum, int ja,
                                              int nk, int warp) {
  if (D.L.kmask) {
    int jj = D.L.j0 - ja;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((D.L.kmask >> i) & 1u) {
        if (jj >= 0 && jj < nk) {
          const float4 v = reinterpret_cast<const float4*>(ksum + jj * kDtTileRows)[warp];
          acc[0][i] = v.x;
          acc[1][i] = v.y;
          acc[2][i] = v.z;
          acc[3][i] = v.w;
        }
        ++jj;
      }
    }
  }
}

// Where the P ranks' wires lie.  per_rank == 0: code[0] is one tensor map over the stacked codes
// [P*T][W] and side[0] over the stacked side buffer [P*k][T] (rank r's rows start at r*T, r*k).
// per_rank != 0: code[r] and side[r] cover rank r's own buffers, [T][W] and [k][T] -- each may be
// another GPU's memory mapped into this process, which these loads then read over the
// interconnect (TMA loads without multicast); side_ptr[r] is rank r's side buffer for the kept
// sums of slices whose side tiles are not staged.
constexpr int kMaxRankMaps = 8;
struct DqWire {
  CUtensorMap code[kMaxRankMaps];
  CUtensorMap side[kMaxRankMaps];
  const uint16_t* side_ptr[kMaxRankMaps];
  int per_rank;
};

template <typename OutT, bool kShard>
__global__ void __launch_bounds__(kDtThreads, kDtMinBlocks) dequant_reduce_tma_kernel(
    const __grid_constant__ DqWire wire, int side_tma, const uint16_t* __restrict__ side, int P, int T, int H,
    int k, const int32_t* __restrict__ keep_idx, const float* __restrict__ scale,
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int ldo, int S, int chunks, int extra, WaitLimits lim) {
  extern __shared__ __align__(128) unsigned char s_raw[];
  DtSmem& sm = *reinterpret_cast<DtSmem*>(s_raw);
  float4* s_const = reinterpret_cast<float4*>(s_raw + ((sizeof(DtSmem) + 127) & ~size_t(127)));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // Slice-minor numbering (blockIdx = chunk*S + s): the S CTAs of one chunk are launched together.
  // Slices 0..extra-1 have chunks + 1 row chunks (their last one numbered after all the others),
  // the rest `chunks`, so that the wave fills every resident slot.  Chunk c of a slice with n
  // chunks takes the 32-row blocks c, c + n, c + 2n, ..., so all CTAs sweep the rows from top to
  // bottom together and counts differ by one block at most within a slice.
  const int chunk = blockIdx.x / S, s = blockIdx.x - chunk * S;
  const int n_chunks = chunks + (s < extra ? 1 : 0);
  // Problem blockIdx.y of a batch (gridDim.y is 1 for a single problem): ranks [y*P, (y+1)*P) of
  // the stacked wire, their parameters, and its own T output rows.
  const int rank0 = blockIdx.y * P;
  scale += (size_t)rank0 * H;
  zero += (size_t)rank0 * H;
  out += (size_t)blockIdx.y * T * ldo;
  const int nb_all = (T + kDtTileRows - 1) / kDtTileRows;
  const int nblk = (nb_all - chunk + n_chunks - 1) / n_chunks;
  const int t_last = T;
  auto block_row = [&](int bi) { return (chunk + bi * n_chunks) * kDtTileRows; };
  const int n_groups = (P + kDtG - 1) / kDtG;  // ring slots per block
  const int n_slots_total = nblk * n_groups;     // slot i = (block i / n_groups, rank group i % n_groups)

  if (threadIdx.x == 0) {
    sm.ring.init(kDtWarps + 1);  // the consumer warps and the kept-sum warp release each slot
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.ksum_full[b], 1);
      mbar_init(&sm.ksum_empty[b], kDtWarps);
    }
    sm.abort = 0;
    fence_barrier_init();
  }
  // Set-up loads first, independent of one another so that they cost one round trip together:
  // each consumer thread's (rank, group) pair of parameters, and one keep_idx entry per thread.
  // The producer's first tiles need the slice's kept count, so they follow this round trip.
  const DqPair pre = warp < kDtWarps ? dq_load_pair(scale, zero, P, H, s, threadIdx.x) : DqPair{};
  const int kv0 = (int)threadIdx.x < k ? __ldg(keep_idx + threadIdx.x) : 0x7FFFFFFF;
  // the slice's kept features, counted by the whole CTA
  const int hs0 = 8 * s * kDqSliceGroups, he0 = min(H, hs0 + 8 * kDqSliceGroups);
  const SliceKept3 sk = slice_kept3(kv0, keep_idx, k, hs0, he0, he0, sm.kcnt, sm.klist, 8 * kDqSliceGroups,
                                    kDtThreads);
  const DqSlice q = dq_slice_from(sk.ja, sk.jb, H, k, s, S);
  const int w_a = q.w_first & ~3;  // 16-byte aligned x coordinate of the box
  const int nk = q.jb - q.ja;
  // the side box: rows t of the block (inner, 64 bytes) x the slice's kept features from ja on
  const bool stage_side = side_tma != 0 && nk > 0 && nk <= kDtMaxStagedKept;
  volatile int* abort = &sm.abort;

  if (warp == kDtWarps) {  // ------------------------------------------------ producer
    if (lane == 0) {
      const int n_maps = wire.per_rank ? P : 1;
      for (int r = 0; r < n_maps; ++r) {
        prefetch_tensor_map(&wire.code[r]);
        if (stage_side) prefetch_tensor_map(&wire.side[r]);
      }
      producer_start_delay(lim.start_delay);
      int issued = 0, bi = 0, g = 0;
      for (int i = 0; i < n_slots_total; ++i) {
        if (!sm.ring.acquire(i, abort, lim.producer)) break;
        const int st = i % kDtStages;
        const int r0 = g * kDtG, nr = min(kDtG, P - r0);
        mbar_arrive_expect_tx(&sm.ring.full[st], (unsigned)nr * (kDtTileBytes + (stage_side ? kDtSideBytes : 0u)));
        for (int j = 0; j < nr; ++j) {
          const int r = r0 + j, m = wire.per_rank ? r : 0;
          const int t = block_row(bi);
          tma_load_2d(&sm.tile[st][j][0][0], &wire.code[m], w_a, (wire.per_rank ? 0 : (rank0 + r) * T) + t,
                      &sm.ring.full[st]);
          if (stage_side)
            tma_load_2d(&sm.side[st][j][0][0], &wire.side[m], t, (wire.per_rank ? 0 : (rank0 + r) * k) + q.ja,
                        &sm.ring.full[st]);
        }
        ++issued;
        if (++g == n_groups) {
          g = 0;
          ++bi;
        }
      }
      if (*abort) sm.ring.drain(issued, lim.producer);
    }
    return;
  }

  if (warp == kDtKeptWarp) {  // ------------------------------------------ kept sums
    if (stage_side) {
      if (nk <= 8) dt_kept_sums<8>(sm, nk, P, nblk, n_groups, abort, lim.consumer);
      else if (nk <= 16) dt_kept_sums<16>(sm, nk, P, nblk, n_groups, abort, lim.consumer);
      else dt_kept_sums<kDtSideCols>(sm, nk, P, nblk, n_groups, abort, lim.consumer);
    } else if (lane == 0) {  // only releases the ring slots
      int st_i = 0;
      unsigned phase = 0;
      for (int i = 0; i < n_slots_total; ++i) {
        if (!mbar_wait(&sm.ring.full[st_i], phase, abort, lim.consumer)) break;
        mbar_arrive(&sm.ring.empty[st_i]);
        if (++st_i == kDtStages) {
          st_i = 0;
          phase ^= 1u;
        }
      }
    }
    return;
  }

  // ---------------------------------------------------------------------- consumers
  // (the producer is already loading while the consumers set up the slice's constants)
  constexpr int kConsumers = 32 * kDtWarps;
  if (nk > 8 * kDqSliceGroups && threadIdx.x == 0) record_error(HQ_ERR_BAD_INDEX);
  if (warp == 0) {  // the 32 groups' layouts from the kept list
    const int h0 = hs0 + 8 * lane;
    const GroupLayout L = h0 < H ? group_layout_list(sm.klist, min(nk, 8 * kDqSliceGroups), q.ja, H, k, h0)
                                 : GroupLayout{0, 0, 0u, 0};
    sm.gkmask[lane] = L.kmask;
    sm.gj0[lane] = L.j0;
  }
  // the slice's (rank, group) pairs: this thread's first one preloaded, any others (P > 8) now
  bool tiny = dq_pair_tiny(pre);
  for (int idx = threadIdx.x + kConsumers; idx < P * 32; idx += kConsumers)
    tiny = tiny || dq_pair_tiny(dq_load_pair(scale, zero, P, H, s, idx));
  const bool generic = named_barrier_or(kConsumers, tiny);
  if ((int)threadIdx.x < P * 32) dq_fill_pair(s_const, sm.gkmask, pre, H, s, threadIdx.x, generic);
  for (int idx = threadIdx.x + kConsumers; idx < P * 32; idx += kConsumers)
    dq_fill_pair(s_const, sm.gkmask, dq_load_pair(scale, zero, P, H, s, idx), H, s, idx, generic);
  GroupLayout Lg;
  Lg.kmask = sm.gkmask[lane];
  Lg.j0 = sm.gj0[lane];
  Lg.n = 8 - __popc(Lg.kmask);
  Lg.c0 = min(max(hs0 + 8 * lane - Lg.j0, 0), H - k);
  const DqLane D = dq_lane_layout(Lg, hs0 + 8 * lane, H, w_a, kDtWords - 2, generic);
  named_barrier_sync(kConsumers);
  int st_i = 0;
  unsigned phase = 0;
  // block bi starts at row t_blk = block_row(bi); the loop ends at the first block past T
  const int t_step = n_chunks * kDtTileRows;
  int bi = 0;
  for (int t_blk = block_row(0); t_blk < T && !*abort; ++bi, t_blk += t_step) {
    const int t0 = t_blk + warp * kDtR;
    float acc[kDtR][8];
#pragma unroll
    for (int m = 0; m < kDtR; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[m][e] = 0.0f;
    bool ok = true;
    for (int g = 0; g < n_groups; ++g) {
      if (!mbar_wait(&sm.ring.full[st_i], phase, abort, lim.consumer)) {
        ok = false;
        break;
      }
      const int nr = min(kDtG, P - g * kDtG);
      const float4* cst = s_const + (size_t)g * kDtG * 4 * 32 + lane;
      if (generic) dt_slot<false, kShard, false>(D, sm, st_i, warp, nr, cst, acc);
      else if (nr == kDtG) dt_slot<true, kShard, true>(D, sm, st_i, warp, nr, cst, acc);
      else dt_slot<true, kShard, false>(D, sm, st_i, warp, nr, cst, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ring.empty[st_i]);
      if (++st_i == kDtStages) {
        st_i = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    if (stage_side) {
      const int buf = bi & 1;
      if (!mbar_wait(&sm.ksum_full[buf], (bi >> 1) & 1, abort, lim.consumer)) break;
      dt_patch_kept(D, acc, &sm.k.ksum[buf][0][0], q.ja, nk, warp);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ksum_empty[buf]);
      dq_store_rows<OutT, kDtR>(D, acc, ldo, t0, t_last, out);
    } else {
      dq_finish_block<OutT, kDtR, false>(D, acc, side + (size_t)rank0 * k * T, wire.per_rank ? wire.side_ptr : nullptr,
                                         sm.k.kept[warp], P, T, H, k, q.ja, q.jb, t0, t_last, out, ldo);
    }
  }
}

// =============================================================== cp.async kernel (any shape)
constexpr int kDqWarps = 8;
constexpr int kDqThreads = 32 * kDqWarps;
constexpr int kDqD = 8;       // cp.async tiles in flight per warp
constexpr int kDqWin = 36;    // staged words per row (>= 35)

// Dynamic shared memory of one CTA for P ranks.
inline size_t dq_smem_bytes(int P) {
  return (size_t)P * 4 * 32 * 16                            // constants: [P][4][32] float4
         + (size_t)kDqWarps * kDqD * kDqR * kDqWin * 4      // staged code tiles
         + (size_t)kDqWarps * kDqR * 32 * 4;                // kept sums
}

template <typename OutT, bool kShard>
__global__ void __launch_bounds__(kDqThreads) dequant_reduce_kernel(
    const uint32_t* __restrict__ codes, const uint16_t* __restrict__ side, int P, int T, int H,
    int k, const int32_t* __restrict__ keep_idx, const float* __restrict__ scale,
    const uint8_t* __restrict__ zero, OutT* __restrict__ out, int ldo, int S, int chunks, int rows_per_chunk) {
  extern __shared__ float4 s_dyn[];
  float4* s_const = s_dyn;                                                    // [P][4][32]
  uint32_t* s_tiles = reinterpret_cast<uint32_t*>(s_const + (size_t)P * 4 * 32);
  float* s_kept = reinterpret_cast<float*>(s_tiles + kDqWarps * kDqD * kDqR * kDqWin);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Wr = (H - k) / 8;
  const int s = blockIdx.x / chunks, chunk = blockIdx.x - s * chunks;
  const int t_first = chunk * rows_per_chunk, t_last = min(T, t_first + rows_per_chunk);

  const DqSlice q = dq_slice(keep_idx, H, k, s, S);
  const bool generic = __syncthreads_or(dq_has_tiny_scale(scale, P, H, s, kDqThreads)) != 0;
  const DqLane D = dq_lane(keep_idx, k, H, s, lane, q.w_first, kDqWin - 2, generic);
  dq_fill_constants(s_const, keep_idx, nullptr, scale, zero, P, H, k, s, generic, kDqThreads);
  __syncthreads();

  // this warp's row blocks: rows t_first + (warp + kDqWarps*bi)*kDqR + m
  const int nblk_total = (t_last - t_first + kDqR - 1) / kDqR;
  const int my_blocks = nblk_total > warp ? (nblk_total - warp + kDqWarps - 1) / kDqWarps : 0;
  const int n_tiles = my_blocks * P;  // tile i = (block i / P, rank i % P)
  uint32_t* my_tiles = s_tiles + (size_t)warp * kDqD * kDqR * kDqWin;
  float* my_kept = s_kept + warp * kDqR * 32;
  const uint32_t tiles_saddr = smem_addr(my_tiles);
  const size_t rank_words = (size_t)T * Wr;

  int i_next = 0, ib = 0, ir = 0;
  auto issue_next = [&]() {
    if (i_next < n_tiles) {
      const int t0 = t_first + (warp + kDqWarps * ib) * kDqR;
      const uint32_t* src = codes + (size_t)ir * rank_words + (size_t)t0 * Wr + q.w_first;
      const uint32_t dst = tiles_saddr + (uint32_t)(((i_next % kDqD) * kDqR * kDqWin) * 4);
#pragma unroll
      for (int m = 0; m < kDqR; ++m) {
        if (t0 + m < t_last) {
          if (lane < q.n_words) cp_async4(dst + 4u * (m * kDqWin + lane), src + (size_t)m * Wr + lane);
          if (lane + 32 < q.n_words)
            cp_async4(dst + 4u * (m * kDqWin + lane + 32), src + (size_t)m * Wr + lane + 32);
        }
      }
      if (++ir == P) {
        ir = 0;
        ++ib;
      }
      ++i_next;
    }
    cp_async_commit();  // one group per tile, empty ones included, keeps the count uniform
  };
  for (int i = 0; i < kDqD - 1; ++i) issue_next();

  int tile = 0;
  for (int bi = 0; bi < my_blocks; ++bi) {
    const int t0 = t_first + (warp + kDqWarps * bi) * kDqR;
    float acc[kDqR][8];
#pragma unroll
    for (int m = 0; m < kDqR; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[m][e] = 0.0f;
    for (int r = 0; r < P; ++r, ++tile) {
      issue_next();
      cp_async_wait<kDqD - 1>();
      __syncwarp();
      const uint32_t* st = my_tiles + (size_t)(tile % kDqD) * kDqR * kDqWin;
      const float4* cst = s_const + (size_t)r * 4 * 32 + lane;
      if (D.decode) {
        if (generic) dq_decode_rows<false, kDqR, kShard>(D, st, kDqWin, cst, acc);
        else dq_decode_rows<true, kDqR, kShard>(D, st, kDqWin, cst, acc);
      }
      __syncwarp();  // the stage is free for the copy issued next iteration
    }
    dq_finish_block<OutT, kDqR, true>(D, acc, side, nullptr, my_kept, P, T, H, k, q.ja, q.jb, t0, t_last, out, ldo);
  }
  cp_async_wait<0>();
}

}  // namespace hq
