// 5th-generation tensor core (tcgen05) building blocks for sm_100a: tensor-memory
// allocation, MMA issue and completion, tensor-memory loads, and the shared-memory matrix
// and instruction descriptors. Thin inline-PTX shims around the documented instructions.
//
// Conventions used by the kernels here:
//  * one CTA (cta_group::1); a single elected thread issues every tcgen05.mma and the
//    tcgen05.commit that reports their completion on an mbarrier;
//  * operands in shared memory without swizzle, in the "interleaved" canonical layout:
//    8 x 16-byte core matrices (8 rows of 16 bytes, 128 contiguous bytes) placed at a
//    leading-dimension byte offset (LBO) and a stride-dimension byte offset (SBO);
//  * accumulators in tensor memory (fp32). For M = 64 the rows of D sit in lanes 0-15 of
//    each 32-lane sub-partition: row m is lane (m % 16) + 32 (m / 16), column n is column
//    n of the allocation.
#pragma once

#include "wkv_device.cuh"

namespace wkv {

// Allocate ncols tensor-memory columns (a power of two, at least 32) for this CTA. Called
// by one whole warp; the allocation's address is written to *slot in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}

// Let other CTAs on this SM allocate (after this CTA's only allocation).
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Free an allocation; called by one whole warp (the one that allocated).
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Order tensor-core operations around a thread barrier (before / after the bar.sync).
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D (tensor memory, fp32) = A x B (+ D when accumulate != 0); A, B tf32 in shared memory,
// described by smem_desc(); idesc from idesc_tf32().
__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D (tensor memory, fp32) = A x B (+ D when accumulate != 0); A, B bf16 in shared memory
// (kind::f16 with both operands bf16); idesc from idesc_bf16().
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier receives one arrival once every MMA issued so far by this thread is done
// (its operands read and its results in tensor memory).
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 16 consecutive 32-bit columns from the 32 lanes of this warp's sub-partition: thread t
// receives lane (taddr's lane + t), columns taddr's column .. + 15. taddr's lane must be
// 32 x (warp index % 4). Complete with tmem_wait_ld() before using the values.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// x rounded to tf32 (10 explicit mantissa bits), to nearest with ties away from zero; the
// result is an fp32 bit pattern whose low 13 bits are zero.
__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// x = hi + lo as two tf32 values: hi the rounding of x, lo the rounding of the exact
// remainder x - hi; hi.b + hi.b' + lo.b style products then carry about 2^-22 relative
// error instead of tf32's 2^-11.
__device__ __forceinline__ void tf32_split(float x, float& hi, float& lo) {
  hi = tf32_rna(x);
  lo = tf32_rna(__fsub_rn(x, hi));
}

// x = hi + mid + lo as three bf16 values (each the rounding of what the previous ones leave;
// the two subtractions are exact in fp32), together 24 significant bits: products of two
// such splits summed over hi.hi, hi.mid, mid.hi, hi.lo, lo.hi and mid.mid carry about
// 2^-24 relative error, the rounding of an fp32 product.
__device__ __forceinline__ void bf16_split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid,
                                            __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  const float r1 = __fsub_rn(x, __bfloat162float(hi));
  mid = __float2bfloat16_rn(r1);
  lo = __float2bfloat16_rn(__fsub_rn(r1, __bfloat162float(mid)));
}

// Two values split at once with packed conversions and fp32x2 arithmetic (the
// subtractions x - hi as exact fused multiply-adds by -1); same results as bf16_split3.
__device__ __forceinline__ void bf16_split3x2(float2 x, __nv_bfloat162& hi, __nv_bfloat162& mid,
                                              __nv_bfloat162& lo) {
  const float2 neg1 = make_float2(-1.f, -1.f);
  hi = __float22bfloat162_rn(x);
  const float2 r1 = __ffma2_rn(__bfloat1622float2(hi), neg1, x);
  mid = __float22bfloat162_rn(r1);
  lo = __float22bfloat162_rn(__ffma2_rn(__bfloat1622float2(mid), neg1, r1));
}

// Shared-memory matrix descriptor, no swizzle: start address, leading and stride byte
// offsets (all multiples of 16 bytes, addresses below 256 KiB), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of kind::tf32 with an fp32 accumulator: M x N tile, A and B each
// K-major (false) or MN-major (true).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                     // D format: fp32
         | (2u << 7) | (2u << 10)      // A, B format: tf32
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Instruction descriptor of kind::f16 with bf16 A and B and an fp32 accumulator, both
// operands K-major: M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                     // D format: fp32
         | (1u << 7) | (1u << 10)      // A, B format: bf16
         | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

}  // namespace wkv
