// Pipeline primitives of the persistent decode kernels: shared-memory
// mbarriers, bulk global->shared copies (cp.async.bulk, completion counted in
// bytes on an mbarrier), per-thread cp.async copies and named barriers over
// a subset of the CTA.
//
// Every wait is bounded: after kWaitNs of global time it gives up and the
// caller records an error, so a lost completion can never hang the GPU.
#pragma once

#include <stdint.h>

namespace gdn {

constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s
constexpr int E_TIMEOUT = 16;                // err_flags bit: a pipeline wait gave up

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// Make the initialised barriers visible to the async (bulk copy) proxy.
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Arrive and announce `tx` bytes that bulk copies will complete on the barrier.
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(tx)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait until the barrier's phase of the given parity has completed; false
// when that takes longer than kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try(bar, parity))
    if (global_ns() - t0 > kWaitNs) return false;
  return true;
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to this CTA's shared memory, completed on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// cp.async of 16 bytes from global to shared memory (both addresses 16-byte
// aligned), bypassing L1; `valid` false fills the 16 bytes with zeros. The
// copies of a thread are grouped by commit and awaited by group: wait<N>
// returns once at most N of the thread's groups are still in flight.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Named barrier `id` (1..15) over the first `n` threads (a multiple of 32).
__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// The same, returning the OR of `pred` over the participating threads.
__device__ __forceinline__ bool bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Position (b, hv, vt) of a tile in (sequence, value head, V-tile) order,
// advanced one tile at a time without divisions.
struct TileCursor {
  int b, hv, vt;
  __device__ __forceinline__ void init(int64_t t, int HV, int NVT) {
    const int64_t per_b = (int64_t)HV * NVT;
    b = static_cast<int>(t / per_b);
    const int rem = static_cast<int>(t - (int64_t)b * per_b);
    hv = rem / NVT;
    vt = rem - hv * NVT;
  }
  __device__ __forceinline__ void next(int HV, int NVT) {
    if (++vt == NVT) {
      vt = 0;
      if (++hv == HV) {
        hv = 0;
        ++b;
      }
    }
  }
};

}  // namespace gdn
