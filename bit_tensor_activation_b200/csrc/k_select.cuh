// k_select.cuh -- Selection of High Precision Features (page "Revolutionizing LLM Inference: The
// Power of Efficient Low-Bit Communication", section "The Hybrid Quantization Algorithm", bullet
// "Selection of High Precision Features"), with the 4-bit grid of bullet "Calibration".
//
// Two kernels, no memory beyond the inputs and outputs:
//   1. select_params_kernel, one thread per (feature, rank) over the whole GPU (a CTA takes 32
//      features): lo = min(ema_min,0), hi = max(ema_max,0), scale = (hi-lo)/15,
//      inv_scale = 1/scale, zero = clamp(rint(-lo*inv_scale),0,15) (degenerate scale -> 1, 0);
//      the ranges go to shared memory, and one thread per feature sums them in rank order into
//      the feature's score.  The score's fp32 bits (non-negative, so their unsigned order is the
//      numeric order; NaN ranks as +inf) are parked in the index outputs: slot h of the H slots
//      rest_idx[0..H-k) followed by keep_idx[0..k).
//   2. select_topk_kernel, one CTA of 1024 threads: reads the H keys into shared memory, then a
//      radix select, 8 bits per pass from the top, finds the k-th largest key tau and how many
//      features equal to tau are still to be taken, and a block-wide ordered scan takes every
//      feature above tau plus the lowest-indexed features equal to tau and writes keep_idx /
//      rest_idx ascending over the parked keys.
// H <= 32768 (the keys fill up to 128 KB of shared memory).
#pragma once

#include <float.h>

#include "hq_common.cuh"

namespace hq {

constexpr int kSelThreads = 1024;
constexpr int kMaxH = 32768;

// Exclusive prefix sum over the block of one value per thread; also returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += y;
    }
    s_warp[lane] = w;  // inclusive totals per warp
  }
  __syncthreads();
  total = s_warp[31];
  const int before = (warp == 0) ? 0 : s_warp[warp - 1];
  const int r = before + x - v;
  __syncthreads();
  return r;
}

constexpr int kSelParamThreads = 256;
constexpr int kSelParamFeatures = 32;                                    // features per CTA
constexpr int kSelParamRankSlots = kSelParamThreads / kSelParamFeatures;  // ranks handled at once
constexpr int kSelMaxRanks = 64;

__global__ void __launch_bounds__(kSelParamThreads) select_params_kernel(
    const float* __restrict__ ema_min, const float* __restrict__ ema_max, int P, int H, int k,
    int32_t* __restrict__ keep_idx, int32_t* __restrict__ rest_idx, float* __restrict__ scale,
    float* __restrict__ inv_scale, uint8_t* __restrict__ zero) {
  __shared__ float s_range[kSelMaxRanks][kSelParamFeatures];
  const int f = threadIdx.x % kSelParamFeatures;
  const int h = blockIdx.x * kSelParamFeatures + f;
  for (int r = threadIdx.x / kSelParamFeatures; r < P; r += kSelParamRankSlots) {
    float range = 0.0f;
    if (h < H) {
      const size_t i = (size_t)r * H + h;
      const float emin = ema_min[i], emax = ema_max[i];
      const float lo = (emin < 0.0f) ? emin : 0.0f;
      const float hi = (emax > 0.0f) ? emax : 0.0f;
      range = __fsub_rn(hi, lo);
      float s = __fdiv_rn(range, 15.0f);
      float inv = 1.0f;
      float zf = 0.0f;
      if (!(s >= FLT_MIN) || !(s <= FLT_MAX)) {
        s = 1.0f;
      } else {
        inv = __frcp_rn(s);
        zf = rintf(__fmul_rn(-lo, inv));
        zf = fminf(fmaxf(zf, 0.0f), 15.0f);
      }
      scale[i] = s;
      inv_scale[i] = inv;
      zero[i] = (uint8_t)(int)zf;
    }
    s_range[r][f] = range;
  }
  __syncthreads();
  if (threadIdx.x < kSelParamFeatures && h < H) {
    float score = 0.0f;
    for (int r = 0; r < P; ++r) score = __fadd_rn(score, s_range[r][f]);
    const uint32_t key = (score != score) ? 0x7F800000u : __float_as_uint(score);
    if (h < H - k) rest_idx[h] = (int32_t)key;
    else keep_idx[h - (H - k)] = (int32_t)key;
  }
}

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(int H, int k, int32_t* __restrict__ keep_idx,
                                                                  int32_t* __restrict__ rest_idx) {
  extern __shared__ uint32_t s_key[];  // [H]
  __shared__ int s_hist[256];
  __shared__ int s_warp[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;

  const int tid = threadIdx.x;

  // ---- 1. the parked keys -------------------------------------------------------------------
  for (int h = tid; h < H; h += kSelThreads)
    s_key[h] = (uint32_t)((h < H - k) ? rest_idx[h] : keep_idx[h - (H - k)]);
  __syncthreads();

  // ---- 2. radix select of the k-th largest key ---------------------------------------------
  if (tid == 0) {
    s_prefix = 0;
    s_remaining = k;
  }
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0 && k > 0 && k < H; shift -= 8) {
    if (tid < 256) s_hist[tid] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int h = tid; h < H; h += kSelThreads) {
      const uint32_t key = s_key[h];
      if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      int c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = s_hist[255 - 8 * tid - i];
        sum += c[i];
      }
      int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (tid >= off) incl += y;
      }
      const int above_lane = incl - sum;  // keys with a larger digit than this lane's range
      const int rem = s_remaining;
      __syncwarp();  // every lane has read s_remaining before the one owner lane rewrites it
      if (above_lane < rem && rem <= incl) {
        int above = above_lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above < rem && rem <= above + c[i]) {
            s_prefix = prefix | ((uint32_t)(255 - 8 * tid - i) << shift);
            s_remaining = rem - above;
          }
          above += c[i];
        }
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t tau = s_prefix;
  const int take_equal = s_remaining;  // features equal to tau to take, lowest index first

  // ---- 3. ordered compaction ---------------------------------------------------------------
  const int chunk = (H + kSelThreads - 1) / kSelThreads;
  const int c_begin = min(H, tid * chunk), c_end = min(H, c_begin + chunk);
  int eq = 0;
  if (k > 0 && k < H)
    for (int h = c_begin; h < c_end; ++h) eq += (s_key[h] == tau);
  int total;
  int eq_before = block_exclusive_scan(eq, s_warp, total);
  int nsel = 0;
  for (int h = c_begin; h < c_end; ++h) {
    bool sel;
    if (k == 0) sel = false;
    else if (k >= H) sel = true;
    else {
      const uint32_t key = s_key[h];
      sel = key > tau || (key == tau && eq_before < take_equal);
      eq_before += (key == tau);
    }
    nsel += sel;
  }
  int sel_before = block_exclusive_scan(nsel, s_warp, total);
  eq_before -= eq;  // back to this chunk's start
  for (int h = c_begin; h < c_end; ++h) {
    bool sel;
    if (k == 0) sel = false;
    else if (k >= H) sel = true;
    else {
      const uint32_t key = s_key[h];
      sel = key > tau || (key == tau && eq_before < take_equal);
      eq_before += (key == tau);
    }
    // The counts above make every write land inside its array; the guards keep that true even
    // if the inputs were inconsistent.
    if (sel) {
      if (sel_before < k) keep_idx[sel_before] = h;
      else record_error(HQ_ERR_BAD_INDEX);
      ++sel_before;
    } else {
      const int c = h - sel_before;
      if (c >= 0 && c < H - k) rest_idx[c] = h;
      else record_error(HQ_ERR_BAD_INDEX);
    }
  }
}

}  // namespace hq
