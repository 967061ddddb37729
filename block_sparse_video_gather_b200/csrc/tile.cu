// tile.cu -- token reorder into spatiotemporal blocks, its inverse, and the
// per-block mean pooling of the coarse stage.
//
// "FastVideo VSA" (vLLM-Omni user guide), introduction and section "Choose
// top-k": the post-patch latent grid is cut into (4, 8, 8) blocks over the
// zero-padded grid; each block is summarised for scoring.
//
// Tiling: one CTA per (b, h, 256 tiled rows), i.e. one 256-token block or
// four 64-token blocks.  A token row of one head is D = 128 bf16 = 256 B,
// moved as 16 lanes x 16 B, so a warp covers two rows per access and the
// tiled side is one contiguous 64 KB run per CTA.  When pooling, the rows
// are also staged in shared memory and thread d sums channel d of a block
// over its slots in slot order in fp32 (the order the coarse stage is
// defined with), then divides once by the real-token count.  Untiling: one
// CTA per (b, h, block).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "items.cuh"
#include "kernels.h"

namespace vsa {

namespace {

using namespace items;


template <int BS, bool POOL, bool F16>
__global__ void __launch_bounds__(kTileThreads) tile_kernel(Geo g, int H, const uint4* __restrict__ x,
                                                            uint4* __restrict__ xt, float* __restrict__ pooled) {
  extern __shared__ __align__(16) uint4 stage[];  // [kItemRows][16] when POOL
  tile_item<BS, POOL, F16>(g, H, blockIdx.x * item_blocks<BS>(), blockIdx.y, x, xt, pooled, stage);
}

template <int BS>
__global__ void __launch_bounds__(kTileThreads) untile_kernel(Geo g, int H, const uint4* __restrict__ xt,
                                                              uint4* __restrict__ x) {
  const int blk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int chunk = threadIdx.x & (kRowChunks - 1);
  const int row0 = threadIdx.x >> 4;
  constexpr int kIters = BS / 16;
  const long long src0 = (static_cast<long long>(bh) * g.Sp + static_cast<long long>(blk) * BS) * kRowChunks;
  uint4 v[kIters];
#pragma unroll
  for (int i = 0; i < kIters; ++i) v[i] = __ldcs(xt + src0 + (row0 + 16 * i) * kRowChunks + chunk);
  const BlockOrigin org = block_origin(g, blk);
#pragma unroll
  for (int i = 0; i < kIters; ++i) {
    const long long s = token_of_slot(g, org, row0 + 16 * i);
    if (s >= 0) x[((static_cast<long long>(b) * g.S + s) * H + h) * kRowChunks + chunk] = v[i];
  }
}

// The two 16-bit values of a packed word as fp32 (exact), for either format.
template <bool F16>
__device__ __forceinline__ float half_lo(uint32_t w) {
  return F16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu))) : bf16_lo(w);
}
template <bool F16>
__device__ __forceinline__ float half_hi(uint32_t w) {
  return F16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16))) : bf16_hi(w);
}

// Untile fused with the gated sum of the compression branch:
// x[token] = x_tiled[slot] + gate[token] * o_compress[block], one fp32 fused
// multiply-add per channel, rounded once to the 16-bit format.  A thread owns
// 8 channels (one 16-byte chunk) of 16 rows; its 8 o_compress values are
// loaded once.
template <int BS, bool F16>
__global__ void __launch_bounds__(kTileThreads) untile_gate_kernel(Geo g, int H, const uint4* __restrict__ xt,
                                                                   const float* __restrict__ o_compress,
                                                                   const uint4* __restrict__ gate,
                                                                   uint4* __restrict__ x) {
  const int blk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int chunk = threadIdx.x & (kRowChunks - 1);
  const int row0 = threadIdx.x >> 4;
  constexpr int kIters = BS / 16;
  const long long src0 = (static_cast<long long>(bh) * g.Sp + static_cast<long long>(blk) * BS) * kRowChunks;
  uint4 v[kIters];
#pragma unroll
  for (int i = 0; i < kIters; ++i) v[i] = __ldcs(xt + src0 + (row0 + 16 * i) * kRowChunks + chunk);
  const float4* cp = reinterpret_cast<const float4*>(o_compress + (static_cast<long long>(bh) * g.NB + blk) * 128) +
                     2 * chunk;
  const float4 c0 = __ldg(cp), c1 = __ldg(cp + 1);
  const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const BlockOrigin org = block_origin(g, blk);
#pragma unroll
  for (int i = 0; i < kIters; ++i) {
    const long long s = token_of_slot(g, org, row0 + 16 * i);
    if (s < 0) continue;
    const long long dst = ((static_cast<long long>(b) * g.S + s) * H + h) * kRowChunks + chunk;
    const uint4 gv = __ldcs(gate + dst);
    const uint32_t ow[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __fmaf_rn(half_lo<F16>(gw[k]), c[2 * k], half_lo<F16>(ow[k]));
      const float hi = __fmaf_rn(half_hi<F16>(gw[k]), c[2 * k + 1], half_hi<F16>(ow[k]));
      r[k] = pack_half2<F16>(lo, hi);
    }
    __stcs(x + dst, make_uint4(r[0], r[1], r[2], r[3]));
  }
}

}  // namespace

template <int BS, bool F16>
cudaError_t launch_tile_t(const Geo& g, int B, int H, const uint4* xi, uint4* xo, float* pooled, cudaStream_t stream) {
  dim3 grid((g.NB + item_blocks<BS>() - 1) / item_blocks<BS>(), B * H);
  if (pooled) {
    const int smem = kItemRows * 256;
    cudaError_t e = cudaFuncSetAttribute(tile_kernel<BS, true, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    tile_kernel<BS, true, F16><<<grid, kTileThreads, smem, stream>>>(g, H, xi, xo, pooled);
  } else {
    tile_kernel<BS, false, false><<<grid, kTileThreads, 0, stream>>>(g, H, xi, xo, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_tile(const Geo& g, int B, int H, const uint16_t* x, uint16_t* xt, float* pooled, bool f16,
                        cudaStream_t stream) {
  const uint4* xi = reinterpret_cast<const uint4*>(x);
  uint4* xo = reinterpret_cast<uint4*>(xt);
  if (g.bs == 256)
    return f16 ? launch_tile_t<256, true>(g, B, H, xi, xo, pooled, stream)
               : launch_tile_t<256, false>(g, B, H, xi, xo, pooled, stream);
  return f16 ? launch_tile_t<64, true>(g, B, H, xi, xo, pooled, stream)
             : launch_tile_t<64, false>(g, B, H, xi, xo, pooled, stream);
}

cudaError_t launch_untile(const Geo& g, int B, int H, const uint16_t* xt, uint16_t* x, cudaStream_t stream) {
  dim3 grid(g.NB, B * H);
  const uint4* xi = reinterpret_cast<const uint4*>(xt);
  uint4* xo = reinterpret_cast<uint4*>(x);
  if (g.bs == 256)
    untile_kernel<256><<<grid, kTileThreads, 0, stream>>>(g, H, xi, xo);
  else
    untile_kernel<64><<<grid, kTileThreads, 0, stream>>>(g, H, xi, xo);
  return cudaGetLastError();
}

cudaError_t launch_untile_gate(const Geo& g, int B, int H, const uint16_t* xt, const float* o_compress,
                               const uint16_t* gate, uint16_t* x, bool f16, cudaStream_t stream) {
  dim3 grid(g.NB, B * H);
  const uint4* xi = reinterpret_cast<const uint4*>(xt);
  const uint4* gi = reinterpret_cast<const uint4*>(gate);
  uint4* xo = reinterpret_cast<uint4*>(x);
  if (g.bs == 256) {
    if (f16) untile_gate_kernel<256, true><<<grid, kTileThreads, 0, stream>>>(g, H, xi, o_compress, gi, xo);
    else untile_gate_kernel<256, false><<<grid, kTileThreads, 0, stream>>>(g, H, xi, o_compress, gi, xo);
  } else {
    if (f16) untile_gate_kernel<64, true><<<grid, kTileThreads, 0, stream>>>(g, H, xi, o_compress, gi, xo);
    else untile_gate_kernel<64, false><<<grid, kTileThreads, 0, stream>>>(g, H, xi, o_compress, gi, xo);
  }
  return cudaGetLastError();
}

}  // namespace vsa
