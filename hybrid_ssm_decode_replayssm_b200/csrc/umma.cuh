// 5th-generation tensor-core (tcgen05 / UMMA) helpers for sm_100a: operand
// descriptors for shared-memory tiles, the bf16 x bf16 -> fp32 MMA with its
// accumulator in tensor memory (TMEM), completion through an mbarrier, and
// TMEM allocation and loads.  Written from the PTX ISA's tcgen05 instruction
// forms; every instruction here is issued as documented (no multicast).
//
// Operand layout used throughout ("MN-major, no swizzle"): a tile with an M (or
// N) extent and a K extent is stored as core matrices of 8 K-rows x 16 bytes
// (8 bf16 along M/N), each core matrix 128 contiguous bytes (K-row kk at byte
// 16 kk).  Element (mn, k) of the tile lives at byte
//     (mn / 8) * SBO + (k / 8) * LBO + (k % 8) * 16 + (mn % 8) * 2.
// The MMA with K = 16 reads two K-groups of 8; a tile with more K advances the
// descriptor start address by 2 * LBO per K = 16 step.
#pragma once

#include <stdint.h>

namespace rssm {
namespace umma {

// Shared-memory matrix descriptor (sm_100 format): start address, leading-
// and stride-dimension byte offsets (all >> 4), descriptor version 1, no
// swizzle, base offset 0.
__device__ __forceinline__ uint64_t smem_desc_mn(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // version
  return d;                 // layout type 0 = no swizzle (bits 61..63)
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, both MN-major,
// shape M x N (M = 64 or 128, N a multiple of 8 up to 256).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_mn(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | (1u << 15)                   // A MN-major
         | (1u << 16)                   // B MN-major
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A * B, one thread issues.  accumulate = false overwrites D.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
  const uint32_t z = 0u;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate), "r"(z)
      : "memory");
}

// The mbarrier at `bar` (shared) gets one arrival when every MMA this thread
// has issued so far is complete.
__device__ __forceinline__ void commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM allocation: one full warp allocates `ncols` columns (a power of two,
// >= 32) and the base address is written to shared memory at `dst`.
__device__ __forceinline__ void alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Warp-collective load of 32 consecutive fp32 columns of TMEM lane
// (lane base + laneid): v[j] = TMEM[lane][col + j].  The warp may only address
// the 32-lane quarter (warp id % 4) of TMEM; the lane base is in bits 16..31
// of the address.
__device__ __forceinline__ void ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// As ld_32x32b_x32 for 16 consecutive columns.
__device__ __forceinline__ void ld_32x32b_x16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// fp32 -> three bf16 parts whose sum is x to within 2^-24 |x| (each part
// carries the next 8 significant bits: hi = RN(x), mid = RN(x - hi),
// lo = RN(x - hi - mid); both differences are exact in fp32).  Products of a
// part with a bf16 value are exact in fp32, so a bf16 MMA over the three parts
// reproduces an fp32-by-bf16 contraction up to fp32 accumulation rounding.
__device__ __forceinline__ void split3_bf16(float x, uint16_t &hi, uint16_t &mid, uint16_t &lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);
  const __nv_bfloat16 l = __float2bfloat16_rn(r2);
  hi = __bfloat16_as_ushort(h);
  mid = __bfloat16_as_ushort(m);
  lo = __bfloat16_as_ushort(l);
}

// Byte offset of element (mn, k) in an MN-major no-swizzle tile whose K extent
// is kg * 8 (kg K-groups per 8-wide MN chunk): LBO = 128, SBO = kg * 128.
__host__ __device__ constexpr uint32_t mn_offset(int mn, int k, int kg) {
  return (uint32_t)((mn >> 3) * kg * 128 + (k >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

}  // namespace umma
}  // namespace rssm
