// 5th-generation tensor core (tcgen05) primitives for sm_100a: tensor-memory allocation, the
// shared-memory matrix and instruction descriptors of a kind::f16 MMA, the MMA itself, its
// completion signal on an mbarrier, and tensor-memory loads.
//
// Operand layout (K-major, 128-byte swizzle): a tile of R rows and K 16-bit elements is stored
// as K / 64 blocks of R rows x 128 bytes, element (r, k) at
//     (k / 64) * R * 128 + r * 128 + ((((k / 8) % 8) ^ (r % 8)) * 16) + (k % 8) * 2   bytes
// from a 1024-byte aligned base (the hardware applies the XOR on address bits 4-6 from bits
// 7-9).  Groups of 8 rows are 1024 bytes apart (SBO); the MMA over elements 16 s .. 16 s + 15
// starts at byte (s / 4) * R * 128 + (s % 4) * 32.
#pragma once
#include <cstdint>

namespace iq {

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor of the layout above: start address (16-byte units), leading
// offset 1 (unused by this layout), 8-row stride 1024 bytes, descriptor version 1, layout type
// 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Byte offset of element (r, k) (k a multiple of 8: the start of a 16-byte chunk) in an R-row tile.
__host__ __device__ constexpr int umma_sw128_off(int r, int k, int R) {
  return (k >> 6) * R * 128 + r * 128 + ((((k >> 3) & 7) ^ (r & 7)) << 4);
}

// Instruction descriptor of kind::f16 with fp16 A and B (both K-major) and an fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (tensor memory) = A B^T (+ D when acc != 0); one thread issues it.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}

// The mbarrier receives one arrival once every MMA this thread has issued so far is complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Whole warp: allocate / free `cols` columns (a power of two >= 32) of tensor memory; the base
// address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}

// Whole warp: 16 consecutive 32-bit columns of this thread's lane (the warp's 32 lanes start at
// 32 (warp % 4)); the values are valid after tmem_wait_ld.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace iq
