// hq_tma.cuh -- Tensor Memory Accelerator (TMA) tile loads and mbarrier pipelines (sm_100a).
//
// A producer warp (one elected lane) issues cp.async.bulk.tensor.2d tile loads into a ring of
// shared-memory stages; each stage has a "full" mbarrier (transaction-counted: completes when the
// tile's bytes have landed) and an "empty" mbarrier (completes when every consumer warp has
// released the stage).  Loads never use cluster multicast and only ever read this GPU's memory.
//
// Every wait is bounded: a waiter that sees no progress for `limit` clock cycles records
// HQ_ERR_TIMEOUT in the device error word, raises the CTA's abort flag and returns false; all
// loops then stop, and the producer waits (again bounded) for the loads it has in flight before
// the CTA exits, so no copy lands in released shared memory.
#pragma once

#include <cuda.h>

#include "hq_common.cuh"

namespace hq {

// Default bound of one wait: about one second at B200 clocks.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Bounds of a pipeline's waits, in clock cycles.  consumer: a consumer waiting for a stage to
// fill (or for another warp's hand-off); producer: the producer waiting for a stage to be
// released, and its drain after an abort.  start_delay: cycles the producer lane idles before its
// first load -- 0 in every normal launch; the abort self-test sets it above a short consumer
// bound, so that the consumers give up while the producer still has loads to issue and drain.
struct WaitLimits {
  long long consumer;
  long long producer;
  long long start_delay;
};

__device__ __forceinline__ void producer_start_delay(long long cycles) {
  if (cycles <= 0) return;
  const long long t0 = clock64();
  while (clock64() - t0 < cycles) __nanosleep(1000);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// Makes barrier initialisation visible to the async (TMA) proxy; follow with __syncthreads().
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// A try_wait whose phase is not complete yet suspends the thread until the phase completes or
// about kSuspendHintNs have passed, instead of returning at once: a waiting warp then takes no
// issue slots from the warps that have work.
constexpr unsigned kSuspendHintNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of parity `parity` of `bar`.  On timeout: HQ_ERR_TIMEOUT is
// recorded, *abort is set, false is returned.  Also returns false as soon as *abort is set.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, volatile int* abort,
                                          long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      record_error(HQ_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// 2-D tile load global -> shared, completing `bytes` of transactions on `bar`.  c0 is the
// innermost coordinate (in elements); c0 * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Barrier among the first `nthreads` threads of the CTA (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}
// Named barrier `id` among `nthreads` threads (whole warps): bar.arrive signals without waiting,
// bar.sync waits for all.  Used to order a producer's first loads after the consumers' set-up loads.
__device__ __forceinline__ void named_barrier_arrive_id(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_barrier_sync_id(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Same barrier, returning whether `pred` held in any participating thread.
__device__ __forceinline__ bool named_barrier_or(int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Ring of kStages stages shared by one producer lane and kConsumers consumer warps.
template <int kStages>
struct TmaRing {
  uint64_t full[kStages];
  uint64_t empty[kStages];

  __device__ void init(int consumers) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], consumers);
    }
  }
  // Producer: wait until stage i % kStages is free for load i (loads 0..kStages-1 need no wait).
  __device__ bool acquire(int i, volatile int* abort, long long limit) {
    if (i < kStages) return true;
    return mbar_wait(&empty[i % kStages], ((i / kStages) - 1) & 1, abort, limit);
  }
  // Consumer: wait until load i has landed.
  __device__ bool wait_full(int i, volatile int* abort, long long limit) {
    return mbar_wait(&full[i % kStages], (i / kStages) & 1, abort, limit);
  }
  // Consumer warp (one lane): release stage of load i.
  __device__ void release(int i) { mbar_arrive(&empty[i % kStages]); }
  // Producer after an abort: wait (bounded) for the most recent load of every stage, so no
  // transfer is still writing into shared memory when the CTA retires.
  __device__ void drain(int issued, long long limit) {
    int ignore_abort = 0;
    for (int i = max(0, issued - kStages); i < issued; ++i)
      mbar_wait(&full[i % kStages], (i / kStages) & 1, &ignore_abort, limit);
  }
};

}  // namespace hq
