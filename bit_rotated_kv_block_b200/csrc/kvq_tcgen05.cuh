// Fifth-generation tensor-core (tcgen05) helpers for one CTA (cta_group::1),
// sm_100a only: tensor-memory allocation, shared-memory matrix descriptors,
// the block-scaled MX multiply-accumulate, scale-factor copies into tensor
// memory, completion through an mbarrier and tensor-memory loads.
#pragma once

#include <stdint.h>

#include "kvq_device.cuh"

namespace kvq {

// Shared-memory matrix descriptor of a K-major operand without swizzling:
// the operand is made of "core matrices" of 8 rows x 16 bytes (each row's 16
// bytes contiguous, the 8 rows at a 16-byte pitch); `lbo` is the byte
// distance between core matrices that follow each other along K, `sbo` the
// distance between groups of 8 rows. Bit fields: start address >> 4 in bits
// 0-13, lbo >> 4 in 16-29, sbo >> 4 in 32-45, descriptor version 1 in 46-47,
// base offset 0, layout type 0 (no swizzle) in 61-63.
__device__ __forceinline__ uint64_t umma_desc_kmajor(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::mxf8f6f4 with UE8M0 block scales: A and B
// element formats (0 = E4M3, 5 = E2M1), both K-major, M x N, and the byte
// (0-3) of each scale-factor column that holds this K block's scales.
__host__ __device__ constexpr uint32_t umma_idesc_mx(int a_fmt, int b_fmt, int M, int N, int sf_id) {
  return ((uint32_t)sf_id << 4)            // B scale-factor byte
         | ((uint32_t)a_fmt << 7) | ((uint32_t)b_fmt << 10)
         | ((uint32_t)(N >> 3) << 17)      // N / 8
         | (1u << 23)                      // scale format UE8M0
         | ((uint32_t)(M >> 4) << 24)      // M / 16
         | ((uint32_t)sf_id << 29);        // A scale-factor byte
}

// Instruction descriptor of kind::i8: A unsigned 8-bit, B signed 8-bit, both
// K-major, int32 accumulators, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
  return (2u << 4)                    // D format S32
         | (0u << 7) | (1u << 10)     // A u8, B s8
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Tensor-memory allocation of `ncols` columns (a power of two >= 32) by one
// whole warp; the base address is written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Ordering of tensor-core operations around thread synchronisation.
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Makes this thread's ordinary shared-memory writes (stores, cp.async)
// visible to the tensor core's asynchronous reads.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Copy of 32 rows x 16 bytes from shared memory (a K-major descriptor) into
// tensor-memory lanes 0-31 of 4 columns, replicated into all four lane
// quarters: the scale-factor layout of the block-scaled MMA.
__device__ __forceinline__ void tmem_cp_32x128_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D (+)= (A with its block scales) x (B with its block scales)^T, issued by
// one thread; `sfa`, `sfb`: tensor-memory addresses of the scale factors with
// the byte index in bits 30-31 (the same byte as the descriptor's sf_id).
__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// D (+)= A x B^T with 8-bit integer operands (int32 accumulators), one thread.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One arrival on the mbarrier once every tensor-core operation this thread
// issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Warp-collective load of 16 consecutive 32-bit columns of the warp's 32
// tensor-memory lanes (lane i of the warp gets lane base + i); taddr holds
// the warp's lane base in bits 16-22. Followed by tmem_ld_wait() before use.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// mbarrier arrival count 1 initialisation and a bounded parity wait live in
// kvq_device.cuh (mbar_init, mbar_wait).

}  // namespace kvq
