// sm100_mx8.cuh -- tcgen05 primitives of the MXFP8 (block-scaled E4M3) GEMM:
// plain bulk copies of the scale bytes, the shared-memory -> TMEM copy of a
// scale block, the block-scaled instruction descriptor and MMA.
#pragma once
#include "sm100.cuh"

namespace vit {

// ---------------------------------------------------------------- MXFP8 (block-scaled E4M3)
// Plain bulk copy global -> shared memory (no tensor map), completing on an
// mbarrier's transaction count.  Both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gmem_src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared memory -> TMEM copy of a 32-row x 16-byte block, replicated into all
// four lane quarters (lanes r, r+32, r+64, r+96 each receive row r as four
// 32-bit columns).  `src_desc` is a no-swizzle K-major matrix descriptor of the
// 512 contiguous bytes (8-row core matrices 128 bytes apart).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t dst_tmem, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(dst_tmem), "l"(src_desc)
               : "memory");
}

// Instruction descriptor of kind::mxf8f6f4 with block scaling: E4M3 x E4M3,
// fp32 accumulation, E8M0 scales, both operands K-major, K = 32 per MMA.
// sf_a / sf_b pick the byte of the 32-bit scale word used by this MMA.
__host__ __device__ constexpr uint32_t idesc_mx8(int M, int N, int sf_a, int sf_b) {
  return (uint32_t(sf_b & 3) << 4)       // B scale-factor byte
         | (0u << 7)                     // A format: E4M3
         | (0u << 10)                    // B format: E4M3
         | (uint32_t(N >> 3) << 17)      // N / 8
         | (1u << 23)                    // scale format: E8M0
         | (uint32_t(M >> 4) << 24)      // M / 16
         | (uint32_t(sf_a & 3) << 29);   // A scale-factor byte
}

// D[tmem] (+)= (A . 2^sfA)[smem desc] * (B . 2^sfB)[smem desc] over K = 32.
// The scale addresses carry the scale byte index in their top two bits.
__device__ __forceinline__ void mma_mx8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

}  // namespace vit
