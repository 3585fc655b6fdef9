// Pipeline primitives: shared-memory mbarriers (the tensor-core chunk kernel
// waits on them for MMA completion), per-thread cp.async copies global ->
// shared with group waits, and the division-free tile cursor of the
// persistent streaming kernels.
//
// Every mbarrier wait is bounded: after kWaitNs of global time it gives up
// and the caller records an error, so a lost completion can never hang the
// GPU. cp.async group waits complete with the copies themselves.
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
// Make the initialised barriers visible to the async proxy (MMA completions
// arrive on them through it).
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

// Position of a tile: sequence b, value head hv (key head h, hv = h G + gi),
// V-tile vt and the tile's index within the sequence's state (hv NVT + vt),
// advanced one tile at a time without divisions.
struct StreamCursor {
  int b, hv, h, gi, vt, within;
  __device__ __forceinline__ void init(int64_t t, int HV, int NVT, int G) {
    const int64_t per_b = (int64_t)HV * NVT;
    b = static_cast<int>(t / per_b);
    within = static_cast<int>(t - (int64_t)b * per_b);
    hv = within / NVT;
    vt = within - hv * NVT;
    h = hv / G;
    gi = hv - h * G;
  }
  // what the step to the next tile changed: 0 nothing but the V-tile,
  // 1 the value head, 2 the key head, 3 the sequence
  __device__ __forceinline__ int next(int HV, int NVT, int G) {
    ++within;
    if (++vt < NVT) return 0;
    vt = 0;
    if (++hv == HV) {
      hv = h = gi = within = 0;
      ++b;
      return 3;
    }
    if (++gi < G) return 1;
    gi = 0;
    ++h;
    return 2;
  }
};

// cp.async of 4 bytes (both addresses 4-byte aligned), cached in L1.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

}  // namespace gdn
