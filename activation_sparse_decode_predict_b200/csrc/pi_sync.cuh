// pi_sync.cuh -- mbarriers, bulk copies, named barriers and a bounded grid
// barrier for the persistent libpi kernels (sm_100a inline PTX).
//
// Every wait here is bounded: it gives up after kTimeoutNs of global time or
// when another CTA has raised the abort flag, records PI_ERR_TIMEOUT in the
// workspace status word and returns false.  Nothing traps.
#pragma once

#include <stdint.h>

#include "pi_common.cuh"

namespace pi {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// 1-D bulk copy global -> shared memory of this CTA, completing on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_sync_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_volatile_s32(const int* p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_volatile_s32(int* p, int v) {
  asm volatile("st.volatile.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Record a timeout and tell every CTA to stop.
__device__ __forceinline__ void raise_abort(Ctrl* ctrl) {
  set_status(&ctrl->status, kStTimeout);
  atomicExch(&ctrl->abort, 1);
}

// Bounded wait for an mbarrier phase.  false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (ld_volatile_s32(&ctrl->abort)) return false;
      if (global_ns() - t0 > kTimeoutNs) {
        raise_abort(ctrl);
        return false;
      }
    }
  }
}

// Grid barrier over the co-resident CTAs of a cooperative launch.  bar_count
// only grows: barrier k (0-based, in launch order) has completed once it
// reaches base + (k + 1) * nctas, where base is the count the previous launch
// left (ctrl->bar_base, read once at kernel start).  One thread per CTA
// arrives after a CTA-wide barrier with a release add; the CTA-wide barrier
// orders the other threads' writes before it.  The waiting thread polls with
// acquire loads, and a CTA-wide barrier after the wait passes the acquired
// view on.  No separate fences: each costs a round trip to L2.
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void grid_arrive(Ctrl* ctrl) { red_release_add(&ctrl->bar_count, 1u); }

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool grid_done(Ctrl* ctrl, unsigned base, unsigned k, unsigned nctas) {
  return (int)(ld_acquire_u32(&ctrl->bar_count) - (base + (k + 1) * nctas)) >= 0;
}

// Polls with acquire loads until the count is reached.
__device__ __forceinline__ bool grid_wait(Ctrl* ctrl, unsigned base, unsigned k, unsigned nctas) {
  if (!grid_done(ctrl, base, k, nctas)) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (grid_done(ctrl, base, k, nctas)) break;
      if ((it & 31u) == 0) {
        if (ld_volatile_s32(&ctrl->abort)) return false;
        if (global_ns() - t0 > kTimeoutNs) {
          raise_abort(ctrl);
          return false;
        }
      }
    }
  }
  return true;
}

}  // namespace pi
