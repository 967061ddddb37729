// nvfp4.cuh -- what the two NVFP4 fine-stage kernels share (the per-item
// kernel in fp4.cu and the grouped 64-token kernel in attn_fwd_grouped.cu):
// the code and scale tile sizes, the block-scaled S product, the scale copy
// into tensor memory, and the shared-memory descriptors they need.
//
// FastVideo "Optimizations" page, section "FP4 Flash Attention 4 (Blackwell
// only)": Q and K in NVFP4 (E2M1 codes, one E4M3 scale per 16 channels), V in
// its 16-bit format.
//
// Scale layout (the tensor core's): for each (b, h) and each 128-row tile t of
// the tiled sequence, 1024 bytes; byte kh*512 + (r % 32)*16 + (r / 32)*4 + j
// holds the scale of row 128t + r, channels 16(4kh + j) .. 16(4kh + j) + 15.
// One 512-byte half is a 32 x 16-byte matrix that tcgen05.cp.32x128b.warpx4
// moves into tensor memory, where lane r%32 (of every lane quarter), column
// r/32, byte j holds the scale the MMA needs for row r and channel block j of
// a 64-channel product.  A 64-token block is one half (its block id & 1) of
// its scale tile: its rows are columns 2 (kb & 1) and 2 (kb & 1) + 1.
//
// The scales of an S product have no tensor-memory columns of their own: those
// of S0 = Q0 K^T go to [192, 216) and those of S1 to [64, 88), columns of the
// other Q tile's S that hold nothing live between that tile's softmax loading
// its S (P takes only the first 64 columns) and the issue of its next S.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace vsa {
namespace nvfp4 {

constexpr uint32_t kCodeTileBytes = 128 * 64;  // 128 rows x 64 B of E2M1 codes
constexpr uint32_t kSfTileBytes = 1024;        // scales of a 128-row tile

// S: E2M1 x E2M1 with UE4M3 block-16 scales, fp32 accumulate, M = 128, both
// K-major (K = 64 codes per instruction).  Fields: A/B format E2M1 = 1 at bits
// 7 and 10, N>>3 at 17, scale format UE4M3 = 0 at 23, M>>4 at 24.
constexpr uint32_t idesc_s(uint32_t n) { return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24); }

// Shared-memory descriptor, K-major with 64-byte swizzle (layout type 4),
// 8-row atoms of 64 B (SBO 512).
__device__ __forceinline__ uint64_t sdesc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16u >> 4) << 16;
  d |= static_cast<uint64_t>(512u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(4) << 61;
  return d;
}

// Source of tcgen05.cp.32x128b: 32 rows of 16 B, no swizzle, 8-row core
// matrices 128 B apart.
__device__ __forceinline__ uint64_t sdesc_rows16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// D[tmem] (+)= A[smem] * B[smem] with block scales from tensor memory.
__device__ __forceinline__ void mma_fp4_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 rows x 128 bits of shared memory -> 4 columns of tensor memory, copied
// into every lane quarter.
__device__ __forceinline__ void tmem_cp_32x128_w(uint32_t taddr, uint64_t src_desc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(src_desc)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned, a multiple of 16 bytes),
// completion counted on an mbarrier.
__device__ __forceinline__ void bulk_load_w(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// First scale column of the product S_i (inside the other tile's S).
__host__ __device__ constexpr uint32_t sf_col(int i) { return i == 0 ? 192u : 64u; }

}  // namespace nvfp4
}  // namespace vsa
