// hq_common.cuh -- device helpers shared by the libhq kernels (sm_100a).
//
// Floating-point discipline: every float operation on the data path is written as an explicit
// round-to-nearest intrinsic (__fmul_rn, __fadd_rn, __fmaf_rn, __fdiv_rn, __frcp_rn) and the
// library is compiled with -fmad=false and without fast-math, so that each step is exactly one
// IEEE-754 single-precision operation and denormals are kept.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hq.h"

namespace hq {

// One error word per device; the first recorded status wins.  Read and cleared by
// hq_read_device_error().
__device__ unsigned int g_error_word = 0;

__device__ __forceinline__ void record_error(hq_status s) {
  atomicCAS(&g_error_word, 0u, (unsigned)s);
}

// bf16 halves of a 32-bit word -> fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Element i (0..7) of eight bf16 values held in a uint4.
__device__ __forceinline__ float bf16_at(const uint4& v, int i) {
  const uint32_t w = (i < 2) ? v.x : (i < 4) ? v.y : (i < 6) ? v.z : v.w;
  return (i & 1) ? bf16_hi(w) : bf16_lo(w);
}

// Two fp32 -> two bf16 (round to nearest even), NaN -> 0x7FC0; a in the low half.
// cvt.rn.bf16x2.f32 writes every NaN, whatever its sign or payload, as 0x7FFF.  Read as signed
// 16-bit values, every other half it can produce is below 0x7FC0 (finite values and +inf up to
// 0x7F80, negative values below zero), so one signed 16-bit minimum with 0x7FC0 turns exactly the
// NaNs into the canonical 0x7FC0 and leaves everything else unchanged.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  asm("min.s16x2 %0, %0, %1;" : "+r"(r) : "r"(0x7FC07FC0u));
  return r;
}

// Two floats rounded to bf16 (nearest, ties to even) in one register: a in the low half, b in
// the high half.  A NaN stays a NaN (its payload is not canonicalised).
__device__ __forceinline__ uint32_t round_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// cp.async copies global -> shared (completion tracked per thread with commit/wait groups;
// cp.async.wait_group is a hardware wait, no spin loop).
__device__ __forceinline__ void cp_async4(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Packed fp32 pairs (sm_100 f32x2 instructions): each lane of __fadd2_rn / __fmul2_rn /
// __ffma2_rn is one correctly rounded IEEE operation, so results are bit-identical to the scalar
// __fadd_rn / __fmul_rn / __fmaf_rn; one instruction does two of them.
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  const float2 r = __fadd2_rn(make_float2(a0, a1), make_float2(b0, b1));
  d0 = r.x;
  d1 = r.y;
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  const float2 r = __fmul2_rn(make_float2(a0, a1), make_float2(b0, b1));
  d0 = r.x;
  d1 = r.y;
}
// (d0, d1) = (a0*b0 + d0, a1*b1 + d1), each with one rounding.
__device__ __forceinline__ void ffma2_acc(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  const float2 r = __ffma2_rn(make_float2(a0, a1), make_float2(b0, b1), make_float2(d0, d1));
  d0 = r.x;
  d1 = r.y;
}

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// (a & M) | c in one LOP3 with M as its immediate operand (c stays in a register).
template <uint32_t M>
__device__ __forceinline__ uint32_t and_or_imm(uint32_t a, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(M), "r"(c));
  return d;
}

// Number of entries of the ascending array a[0..n) that are < key (lower bound).
__device__ __forceinline__ int lower_bound_i32(const int32_t* __restrict__ a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) < key) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Kept-feature layout of one group of 8 consecutive features [h0, h0+8):
//   j0    = number of kept features before h0 (index of the group's first kept in keep_idx)
//   kmask = bit i set when feature h0+i is kept
//   c0    = compact (rest_idx) position of the group's first non-kept feature = h0 - j0
// Every keep_idx entry read is range-checked; a bad entry is recorded and ignored.
struct GroupLayout {
  int j0;
  int c0;
  uint32_t kmask;
  int n;  // non-kept features in the group
};

__device__ __forceinline__ GroupLayout group_layout(const int32_t* __restrict__ keep_idx, int k, int H,
                                                    int h0) {
  GroupLayout L;
  L.j0 = lower_bound_i32(keep_idx, k, h0);
  const int j1 = lower_bound_i32(keep_idx, k, h0 + 8);
  L.kmask = 0;
  for (int j = L.j0; j < j1 && j < L.j0 + 8; ++j) {
    const int d = __ldg(keep_idx + j) - h0;
    if (d >= 0 && d < 8) L.kmask |= 1u << d;
    else record_error(HQ_ERR_BAD_INDEX);
  }
  if (j1 - L.j0 > 8) record_error(HQ_ERR_BAD_INDEX);
  L.n = 8 - __popc(L.kmask);
  L.c0 = h0 - L.j0;
  if (L.c0 < 0 || L.c0 > H - k) {
    record_error(HQ_ERR_BAD_INDEX);
    L.c0 = min(max(L.c0, 0), H - k);
  }
  return L;
}

// The kept features of a feature range [lo, hi), for a group of threads at once: ja =
// #{keep_idx < lo} and jb = #{keep_idx < hi} (the lower bounds when keep_idx is ascending) from
// one coalesced pass over keep_idx, and keep_idx[ja .. ja + min(jb-ja, cap)) copied to list.
// Called by threads 0..nthreads-1 (whole warps), which it synchronises: with __syncthreads when
// they are the whole CTA, else with named barrier 1.
struct SliceKept {
  int ja, jb;
};
__device__ __forceinline__ void group_sync(int nthreads) {
  if (nthreads == (int)blockDim.x) __syncthreads();
  else asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}
__device__ __forceinline__ SliceKept slice_kept(const int32_t* __restrict__ keep_idx, int k, int lo, int hi,
                                                int* s_cnt, int* list, int cap, int nthreads) {
  int a = 0, b = 0;
  for (int i = threadIdx.x; i < k; i += nthreads) {
    const int v = __ldg(keep_idx + i);
    a += v < lo;
    b += v < hi;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_down_sync(0xFFFFFFFFu, a, off);
    b += __shfl_down_sync(0xFFFFFFFFu, b, off);
  }
  if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = 0;
  group_sync(nthreads);
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&s_cnt[0], a);
    atomicAdd(&s_cnt[1], b);
  }
  group_sync(nthreads);
  const SliceKept r{s_cnt[0], s_cnt[1]};
  const int n = min(r.jb - r.ja, cap);
  for (int i = threadIdx.x; i < n; i += nthreads) list[i] = __ldg(keep_idx + r.ja + i);
  group_sync(nthreads);
  return r;
}

// slice_kept() for a group of threads that has already loaded the first entry of keep_idx each
// (v0 = keep_idx[tid] for tid < k, INT_MAX otherwise), so that load can be issued together with
// the caller's other set-up loads; with a third bound hi2 >= hi: jc = #{keep_idx < hi2}, and
// list gets keep_idx[ja .. ja + min(jc - ja, cap)).  s_cnt holds 3 ints.
struct SliceKept3 {
  int ja, jb, jc;
};
__device__ __forceinline__ SliceKept3 slice_kept3(int v0, const int32_t* __restrict__ keep_idx, int k, int lo,
                                                  int hi, int hi2, int* s_cnt, int* list, int cap, int nthreads) {
  int a = v0 < lo, b = v0 < hi, c = v0 < hi2;
  for (int i = threadIdx.x + nthreads; i < k; i += nthreads) {
    const int v = __ldg(keep_idx + i);
    a += v < lo;
    b += v < hi;
    c += v < hi2;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_down_sync(0xFFFFFFFFu, a, off);
    b += __shfl_down_sync(0xFFFFFFFFu, b, off);
    c += __shfl_down_sync(0xFFFFFFFFu, c, off);
  }
  if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = s_cnt[2] = 0;
  group_sync(nthreads);
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&s_cnt[0], a);
    atomicAdd(&s_cnt[1], b);
    atomicAdd(&s_cnt[2], c);
  }
  group_sync(nthreads);
  const SliceKept3 r{s_cnt[0], s_cnt[1], s_cnt[2]};
  const int n = min(r.jc - r.ja, cap);
  const int i0 = (int)threadIdx.x - r.ja;  // this thread's own entry, already in v0
  if ((int)threadIdx.x < k && i0 >= 0 && i0 < n) list[i0] = v0;
  for (int i = r.ja + threadIdx.x; i < r.ja + n; i += nthreads)
    if (i >= nthreads) list[i - r.ja] = __ldg(keep_idx + i);
  group_sync(nthreads);
  return r;
}

// group_layout() for a group inside a range whose kept features are list[0..n) (= keep_idx[ja..),
// ascending), without touching global memory.
__device__ __forceinline__ GroupLayout group_layout_list(const int* list, int n, int ja, int H, int k, int h0) {
  GroupLayout L;
  int below = 0;
  uint32_t km = 0;
  for (int i = 0; i < n; ++i) {
    const int d = list[i] - h0;
    below += d < 0;
    if (d >= 0 && d < 8) km |= 1u << d;
  }
  L.j0 = ja + below;
  L.kmask = km;
  L.n = 8 - __popc(km);
  L.c0 = h0 - L.j0;
  if (L.c0 < 0 || L.c0 > H - k) {
    record_error(HQ_ERR_BAD_INDEX);
    L.c0 = min(max(L.c0, 0), H - k);
  }
  return L;
}

// Column index read from keep_idx / rest_idx, clamped into [0, H) with the error recorded.
__device__ __forceinline__ int checked_col(const int32_t* __restrict__ idx, int j, int H) {
  int h = __ldg(idx + j);
  if (h < 0 || h >= H) {
    record_error(HQ_ERR_BAD_INDEX);
    h = 0;
  }
  return h;
}

}  // namespace hq
