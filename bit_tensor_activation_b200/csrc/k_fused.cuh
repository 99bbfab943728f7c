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
// Work decomposition as in dequant-reduce: a CTA covers a slice of 256 features and every
// chunks-th 32-row block; its per-(rank, feature) constants live in shared memory.  Warp 8 is the producer: one
// lane loads, per (32-row block, rank), the 32 x 256 bf16 tile (16 KB) with one TMA instruction
// into a 3-stage mbarrier ring.  Warps 0..7 consume 4 rows each (lane l: features 8l..8l+7),
// walking the ranks in order with 4 x 8 fp32 sums in registers.
//
// Roofline: HBM-bound, P*2 bytes read + 2 (or 4) bytes written per output element.
// No memory beyond the inputs and outputs is used.
#pragma once

#include "hq_common.cuh"
#include "hq_tma.cuh"
#include "k_dequant.cuh"

namespace hq {

constexpr int kFuWarps = 8;                      // consumer warps
constexpr int kFuThreads = 32 * (kFuWarps + 1);  // + one producer warp
constexpr int kFuR = 4;                          // rows per consumer warp per block
constexpr int kFuTileRows = kFuWarps * kFuR;     // 32
constexpr int kFuSlice = 256;
constexpr int kFuStages = 3;
constexpr unsigned kFuTileBytes = kFuTileRows * kFuSlice * 2;

constexpr int kFuStartBarrier = 2;  // named barrier: consumers' set-up loads issued

struct FuSmem {
  alignas(128) uint16_t tile[kFuStages][kFuTileRows][kFuSlice];
  TmaRing<kFuStages> ring;
  int abort;
  int klist[kFuSlice];  // the slice's kept features
  int kcnt[3];
  uint32_t gkmask[kFuSlice / 8];
  // followed by the constants: float4 [P][5][32]
};

// One (rank, group) pair's parameters, idx = rank * 32 + group of the slice starting at hs,
// loaded ahead of the rest of the set-up (nothing in the address depends on the kept features).
struct FuPair {
  float4 i0, i1, s0, s1;
  uint2 z;
};
__device__ __forceinline__ FuPair fu_load_pair(const float* __restrict__ inv_scale, const float* __restrict__ scale,
                                               const uint8_t* __restrict__ zero, int P, int H, int hs, int idx) {
  FuPair d;
  d.i0 = d.i1 = d.s0 = d.s1 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  d.z = make_uint2(0u, 0u);
  const int r = idx >> 5, hg = hs + 8 * (idx & 31);
  if (r < P && hg < H) {  // r*H + hg is a multiple of 8; the arrays are 16-byte aligned
    const size_t p = (size_t)r * H + hg;
    d.i0 = __ldg(reinterpret_cast<const float4*>(inv_scale + p));
    d.i1 = __ldg(reinterpret_cast<const float4*>(inv_scale + p) + 1);
    d.s0 = __ldg(reinterpret_cast<const float4*>(scale + p));
    d.s1 = __ldg(reinterpret_cast<const float4*>(scale + p) + 1);
    d.z = __ldg(reinterpret_cast<const uint2*>(zero + p));
  }
  return d;
}
// The pair's constants: inv 0-3, inv 4-7, scale 0-3, scale 4-7 (1 for kept), (-zero as signed
// bytes, kmask); features past H get zeros.
__device__ __forceinline__ void fu_fill_pair(float4* s_const, const FuPair& d, uint32_t km, int H, int hs, int idx) {
  const int r = idx >> 5, g = idx & 31;
  const bool in = hs + 8 * g < H;
  const float sv[8] = {d.s0.x, d.s0.y, d.s0.z, d.s0.w, d.s1.x, d.s1.y, d.s1.z, d.s1.w};
  float sc[8];
  uint32_t zlo = 0, zhi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sc[i] = !in ? 0.0f : ((km >> i) & 1u) ? 1.0f : sv[i];
    const uint32_t zi = ((i < 4 ? d.z.x : d.z.y) >> (8 * (i & 3))) & 0xFFu;
    const uint32_t nz = (uint32_t)(-(int)zi) & 0xFFu;  // -zero as a signed byte
    if (i < 4) zlo |= nz << (8 * i);
    else zhi |= nz << (8 * (i - 4));
  }
  float4* dst = s_const + (size_t)r * 5 * 32 + g;
  dst[0] = d.i0;
  dst[32] = d.i1;
  dst[64] = make_float4(sc[0], sc[1], sc[2], sc[3]);
  dst[96] = make_float4(sc[4], sc[5], sc[6], sc[7]);
  dst[128] = make_float4(__uint_as_float(zlo), __uint_as_float(zhi), __uint_as_float(in ? km : 0u), 0.0f);
}

inline size_t fu_smem_bytes(int P) { return sizeof(FuSmem) + 128 + (size_t)P * 5 * 32 * 16; }

template <typename OutT>
__global__ void __launch_bounds__(kFuThreads, 2) compress_reduce_kernel(
    const __grid_constant__ CUtensorMap tmap_x, int P, int T, int H, int k,
    const int32_t* __restrict__ keep_idx, const float* __restrict__ scale,
    const float* __restrict__ inv_scale, const uint8_t* __restrict__ zero, OutT* __restrict__ out, int ldo, int S,
    int chunks, int extra, WaitLimits lim) {
  extern __shared__ __align__(128) unsigned char s_raw[];
  FuSmem& sm = *reinterpret_cast<FuSmem*>(s_raw);
  float4* s_const = reinterpret_cast<float4*>(s_raw + ((sizeof(FuSmem) + 127) & ~size_t(127)));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // Slice-minor numbering (blockIdx = chunk*S + s); slices 0..extra-1 have one row chunk more,
  // and chunk c of a slice with n chunks takes the 32-row blocks c, c + n, c + 2n, ...: as in
  // dequant-reduce, the wave fills every resident slot, the CTAs sweep the rows together and
  // block counts differ by one at most within a slice.
  const int chunk = blockIdx.x / S, s = blockIdx.x - chunk * S;
  const int n_chunks = chunks + (s < extra ? 1 : 0);
  const int nb_all = (T + kFuTileRows - 1) / kFuTileRows;
  const int nblk = (nb_all - chunk + n_chunks - 1) / n_chunks;
  auto block_row = [&](int bi) { return (chunk + bi * n_chunks) * kFuTileRows; };
  const int n_tiles = nblk * P;  // tile i = (block i / P, rank i % P)
  const int hs = s * kFuSlice;

  if (threadIdx.x == 0) {
    sm.ring.init(kFuWarps);
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &sm.abort;
  constexpr int kConsumers = 32 * kFuWarps;

  if (warp == kFuWarps) {  // ------------------------------------------------ producer
    // the first tiles go out after the consumers' set-up loads, which then are not queued
    // behind them; the consumers arrive on this barrier before they wait for anything
    named_barrier_sync_id(kFuStartBarrier, kFuThreads);
    if (lane == 0) {
      prefetch_tensor_map(&tmap_x);
      producer_start_delay(lim.start_delay);
      int issued = 0, bi = 0, r = 0;
      for (int i = 0; i < n_tiles; ++i) {
        if (!sm.ring.acquire(i, abort, lim.producer)) break;
        const int st = i % kFuStages;
        mbar_arrive_expect_tx(&sm.ring.full[st], kFuTileBytes);
        tma_load_2d(&sm.tile[st][0][0], &tmap_x, hs, r * T + block_row(bi), &sm.ring.full[st]);
        ++issued;
        if (++r == P) {
          r = 0;
          ++bi;
        }
      }
      if (*abort) sm.ring.drain(issued, lim.producer);
    }
    return;
  }

  // ---------------------------------------------------------------------- consumers
  // Set-up loads first, independent of one another so that they cost one round trip together:
  // each thread's (rank, group) pair of parameters and one keep_idx entry.  Then the slice's
  // kept features are counted in one coalesced pass and the groups' kept masks laid out from
  // that list, and the constants [P][5][32] filled.
  const FuPair pre = fu_load_pair(inv_scale, scale, zero, P, H, hs, threadIdx.x);
  const int kv0 = (int)threadIdx.x < k ? __ldg(keep_idx + threadIdx.x) : 0x7FFFFFFF;
  named_barrier_arrive_id(kFuStartBarrier, kFuThreads);
  const int he = min(H, hs + kFuSlice);
  const SliceKept3 sk = slice_kept3(kv0, keep_idx, k, hs, he, he, sm.kcnt, sm.klist, kFuSlice, kConsumers);
  // an index outside [0, H) belongs to no slice's groups: the end slices find it missing
  if (threadIdx.x == 0 && ((s == 0 && sk.ja != 0) || (s == S - 1 && sk.jb != k) || sk.jb - sk.ja > kFuSlice))
    record_error(HQ_ERR_BAD_INDEX);
  if (warp == 0) {
    const int hg = hs + 8 * lane;
    sm.gkmask[lane] = hg < H ? group_layout_list(sm.klist, min(sk.jb - sk.ja, kFuSlice), sk.ja, H, k, hg).kmask : 0u;
  }
  named_barrier_sync(kConsumers);
  if ((int)threadIdx.x < P * 32) fu_fill_pair(s_const, pre, sm.gkmask[threadIdx.x & 31], H, hs, threadIdx.x);
  for (int idx = threadIdx.x + kConsumers; idx < P * 32; idx += kConsumers)
    fu_fill_pair(s_const, fu_load_pair(inv_scale, scale, zero, P, H, hs, idx), sm.gkmask[idx & 31], H, hs, idx);
  named_barrier_sync(kConsumers);
  const int h0 = hs + 8 * lane;
  const bool active = h0 < H;
  const uint32_t kmask = __float_as_uint(s_const[128 + lane].z);
  int st_i = 0;  // ring stage of the next tile and the parity of its fill
  unsigned phase = 0;
  for (int bi = 0; bi < nblk && !*abort; ++bi) {
    const int t0 = block_row(bi) + warp * kFuR;
    float acc[kFuR][8];
#pragma unroll
    for (int m = 0; m < kFuR; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[m][e] = 0.0f;
    bool ok = true;
    for (int r = 0; r < P; ++r) {
      if (!mbar_wait(&sm.ring.full[st_i], phase, abort, lim.consumer)) {
        ok = false;
        break;
      }
      if (active) {
        const float4* cst = s_const + (size_t)r * 5 * 32 + lane;
        const float4 i0 = cst[0], i1 = cst[32], s0 = cst[64], s1 = cst[96], zz = cst[128];
        const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
        const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const uint32_t zlo = __float_as_uint(zz.x), zhi = __float_as_uint(zz.y);
        int lo[8], hi[8];  // clamp bounds of c: -zero and 15 - zero
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lo[e] = (int)(int8_t)(uint8_t)((e < 4 ? zlo : zhi) >> (8 * (e & 3)));  // sign-extended byte
          hi[e] = lo[e] + 15;
        }
#pragma unroll
        for (int m = 0; m < kFuR; ++m) {
          const uint4 xv = reinterpret_cast<const uint4*>(&sm.tile[st_i][warp * kFuR + m][0])[lane];
          const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float f0 = __uint_as_float(w[e / 2] << 16), f1 = __uint_as_float(w[e / 2] & 0xFFFF0000u);
            float a0, a1;
            fmul2(a0, a1, f0, f1, inv[e], inv[e + 1]);
            int c0 = __float2int_rn(a0), c1 = __float2int_rn(a1);  // saturating; NaN -> 0
            c0 = min(max(c0, lo[e]), hi[e]);
            c1 = min(max(c1, lo[e + 1]), hi[e + 1]);
            // float(c) by the 1.5 * 2^23 magic, as scalar adds: their results go straight into the
            // register pair the packed FMA reads
            const float d0 = __fadd_rn(__int_as_float(c0 + 0x4B400000), -12582912.0f);
            const float d1 = __fadd_rn(__int_as_float(c1 + 0x4B400000), -12582912.0f);
            const float v0 = ((kmask >> e) & 1u) ? f0 : d0;
            const float v1 = ((kmask >> (e + 1)) & 1u) ? f1 : d1;
            ffma2_acc(acc[m][e], acc[m][e + 1], v0, v1, sc[e], sc[e + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ring.empty[st_i]);
      if (++st_i == kFuStages) {
        st_i = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    if (active) {
#pragma unroll
      for (int m = 0; m < kFuR; ++m)
        if (t0 + m < T) store_row8<OutT>(out + (size_t)(t0 + m) * ldo + h0, acc[m]);
    }
  }
}

}  // namespace hq
