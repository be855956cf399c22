// tcgen05 helpers shared by the kernels that use the 5th-generation tensor cores: shared-memory
// matrix descriptors, MMAs with A in tensor memory, tensor-memory loads and stores, commits and
// the thread-sync fences.  All PTX is written by hand from the PTX ISA's tcgen05 section.
#pragma once

#include "device_common.cuh"

// Shared-memory matrix descriptor: canonical K-major layout without swizzle; LBO = byte distance
// between adjacent 8x16-byte core matrices along K, SBO = between adjacent 8-row groups.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// A (M x K bytes) from tensor memory: lane = row, four K-bytes per 32-bit column, 8 columns per MMA
__device__ __forceinline__ void umma_i8_ta(uint32_t dtmem, uint32_t atmem, uint64_t db, uint32_t idesc,
                                           uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(dtmem),
      "r"(atmem), "l"(db), "r"(idesc), "r"(accum), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }


// kind::tf32: D (f32, tensor memory) += A (tf32, tensor memory: lane = row, one column per K
// element, 8 columns per MMA) x B (tf32, shared memory descriptor); accum = 0 overwrites D
__device__ __forceinline__ void umma_tf32_ta(uint32_t dtmem, uint32_t atmem, uint64_t db, uint32_t idesc,
                                             uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(dtmem), "r"(atmem), "l"(db),
      "r"(idesc), "r"(accum)
      : "memory");
}

// The tf32 head of an fp32 value by truncation: its bit pattern with the low 13 mantissa bits clear
// (one logic op).  x - head is exact in fp32 and below 2^-10 |x|; a TF32 MMA reads an fp32 operand
// the same way (the low 13 bits ignored), so the two-term split x = head + (x - head) keeps about
// 21 significant bits through the products.
__device__ __forceinline__ uint32_t tf32_head(float x) { return __float_as_uint(x) & 0xFFFFE000u; }

// kind::f16 with both operands in shared memory (descriptors): D (f32, tensor memory) += A x B^T,
// A and B bf16 per the instruction descriptor, K = 16 elements per MMA; accum = 0 overwrites D
__device__ __forceinline__ void umma_f16_ss(uint32_t dtmem, uint64_t da, uint64_t db, uint32_t idesc,
                                            uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(dtmem), "l"(da), "l"(db),
      "r"(idesc), "r"(accum)
      : "memory");
}
