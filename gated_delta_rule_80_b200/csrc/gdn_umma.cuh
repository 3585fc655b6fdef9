// Fifth-generation tensor core (tcgen05) primitives for sm_100a: tensor
// memory allocation and access, shared-memory matrix descriptors and the
// bf16 x bf16 -> fp32 MMA, issued by one thread of the CTA.
//
// Operand tiles live in shared memory in the canonical K-major layout
// without swizzle: a tile of R rows x C columns (C along the contraction)
// is stored as 8 x 8 "core matrices" of 8 rows x 16 bytes (8 bf16 of one
// row), the core matrix (r / 8, c / 8) at byte (r / 8) * SBO + (c / 8) * LBO
// with LBO = 128 and SBO = (C / 8) * 128. One MMA consumes 16 columns, so
// successive MMAs of a contraction advance the start address by 2 * LBO.
//
// The accumulator of an M = 128 MMA occupies 128 lanes of tensor memory,
// row i in lane i and column j in column j (fp32). Warp w of the CTA may
// access lanes 32 (w % 4) .. 32 (w % 4) + 31 only.
#pragma once

#include <stdint.h>

#include "gdn_pipe.cuh"

namespace gdn {

// byte offset of element (r, c) of a canonical K-major bf16 tile of C columns
__host__ __device__ constexpr uint32_t kmajor_offset(uint32_t r, uint32_t c, uint32_t C) {
  return (r >> 3) * (C * 16u) + (c >> 3) * 128u + (r & 7u) * 16u + (c & 7u) * 2u;
}

// Shared-memory matrix descriptor (canonical K-major, no swizzle):
// start address >> 4 in bits [0,14), LBO >> 4 in [16,30), SBO >> 4 in
// [32,46), descriptor version 1 in [46,48), layout type 0 (no swizzle).
__device__ __forceinline__ uint64_t umma_desc_kmajor(const void* tile, uint32_t C) {
  const uint64_t addr = smem_addr(tile);
  const uint64_t lbo = 128u, sbo = C * 16u;
  return ((addr >> 4) & 0x3FFFull) | (((lbo >> 4) & 0x3FFFull) << 16) | (((sbo >> 4) & 0x3FFFull) << 32) |
         (1ull << 46);
}

// The descriptor of the same tile with its start advanced by `bytes` (a
// multiple of 16): the start address sits in the low 14 bits as address >> 4,
// and shared-memory addresses stay below 2^18, so a plain add cannot carry
// out of the field. This keeps an MMA issue loop at one add per step.
__device__ __forceinline__ uint64_t umma_desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major) and
// an fp32 accumulator: c_format F32 in [4,6), a_format BF16 in [7,10),
// b_format BF16 in [10,13), N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// D (tensor memory) {=, +=} A (shared) x B (shared)^T, one instruction of
// the CTA; `accumulate` false overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  const uint32_t acc = accumulate ? 1u : 0u;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      :
      : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}

// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Tensor memory allocation by one whole warp; the address lands in *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Ordering of tensor-memory traffic and MMAs around thread barriers.
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make this thread's shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of the warp's 32 lanes (thread i: lane i of
// the warp's quarter), and the matching store.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* x) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* x) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(r[i]);
}
// 16x256b shape, two 8-column groups: of the 16 lanes starting at the
// address's lane, thread t of the warp holds lanes (t / 4) and (t / 4 + 8),
// columns 2 (t % 4) and 2 (t % 4) + 1 of each group: r[4 g + 2 h + j] is
// lane (t / 4 + 8 h), column 8 g + 2 (t % 4) + j.
__device__ __forceinline__ void tmem_ld16x256b_x2(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* x) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __uint_as_float(r[i]);
}
// 32 columns of the warp's lanes into registers without waiting: the caller
// waits once (tmem_wait_ld) for several loads in flight before using them.
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 32 columns from registers without waiting (tmem_wait_st before the data is
// used by an MMA or read back)
__device__ __forceinline__ void tmem_st32_issue(uint32_t taddr, const float* x) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(x[0])), "r"(__float_as_uint(x[1])), "r"(__float_as_uint(x[2])), "r"(__float_as_uint(x[3])),
      "r"(__float_as_uint(x[4])), "r"(__float_as_uint(x[5])), "r"(__float_as_uint(x[6])), "r"(__float_as_uint(x[7])),
      "r"(__float_as_uint(x[8])), "r"(__float_as_uint(x[9])), "r"(__float_as_uint(x[10])),
      "r"(__float_as_uint(x[11])), "r"(__float_as_uint(x[12])), "r"(__float_as_uint(x[13])),
      "r"(__float_as_uint(x[14])), "r"(__float_as_uint(x[15])), "r"(__float_as_uint(x[16])),
      "r"(__float_as_uint(x[17])), "r"(__float_as_uint(x[18])), "r"(__float_as_uint(x[19])),
      "r"(__float_as_uint(x[20])), "r"(__float_as_uint(x[21])), "r"(__float_as_uint(x[22])),
      "r"(__float_as_uint(x[23])), "r"(__float_as_uint(x[24])), "r"(__float_as_uint(x[25])),
      "r"(__float_as_uint(x[26])), "r"(__float_as_uint(x[27])), "r"(__float_as_uint(x[28])),
      "r"(__float_as_uint(x[29])), "r"(__float_as_uint(x[30])), "r"(__float_as_uint(x[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* x) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(x[0])), "r"(__float_as_uint(x[1])), "r"(__float_as_uint(x[2])), "r"(__float_as_uint(x[3])),
      "r"(__float_as_uint(x[4])), "r"(__float_as_uint(x[5])), "r"(__float_as_uint(x[6])), "r"(__float_as_uint(x[7])),
      "r"(__float_as_uint(x[8])), "r"(__float_as_uint(x[9])), "r"(__float_as_uint(x[10])),
      "r"(__float_as_uint(x[11])), "r"(__float_as_uint(x[12])), "r"(__float_as_uint(x[13])),
      "r"(__float_as_uint(x[14])), "r"(__float_as_uint(x[15])), "r"(__float_as_uint(x[16])),
      "r"(__float_as_uint(x[17])), "r"(__float_as_uint(x[18])), "r"(__float_as_uint(x[19])),
      "r"(__float_as_uint(x[20])), "r"(__float_as_uint(x[21])), "r"(__float_as_uint(x[22])),
      "r"(__float_as_uint(x[23])), "r"(__float_as_uint(x[24])), "r"(__float_as_uint(x[25])),
      "r"(__float_as_uint(x[26])), "r"(__float_as_uint(x[27])), "r"(__float_as_uint(x[28])),
      "r"(__float_as_uint(x[29])), "r"(__float_as_uint(x[30])), "r"(__float_as_uint(x[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace gdn
