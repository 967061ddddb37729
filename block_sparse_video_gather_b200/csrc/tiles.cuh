// tiles.cuh -- what the attention kernels share about 128-row tiles:
// validity bits of a tile's slots (real token or padding) and the TMA view
// of a [rows, 128] 16-bit tensor.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace vsa {
namespace tiles {

constexpr int kTileFull = 0, kTilePartial = 1, kTileEmpty = 2;

// Validity bits of the 128 key columns of tile `half` of block kb (bit c of
// word c/32 set = slot half*128 + c holds a real token).  Returns kTileFull
// when every column is real, kTileEmpty when none is, else kTilePartial.
__device__ __forceinline__ int key_tile_mask(const Geo& g, int kb, int half, uint32_t (&w)[4]) {
  if (kb < 0) {
    w[0] = w[1] = w[2] = w[3] = 0u;
    return kTileEmpty;
  }
  const int first = half * 128;
  if (kb < g.n_pre) {
    const int lim = g.n_prefix - kb * g.bs - first;  // real columns of this tile
    if (lim >= 128) return kTileFull;
    if (lim <= 0) return kTileEmpty;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = min(max(lim - 32 * i, 0), 32);
      w[i] = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
    }
    return kTilePartial;
  }
  if (g.vfull) return kTileFull;
  int vt, vh, vw;
  video_block_extent(g, kb - g.n_pre, vt, vh, vw);
  if (vt == g.bt && vh == g.bh && vw == g.bw) return kTileFull;
  const uint32_t rowbits = vw >= 32 ? 0xffffffffu : ((1u << vw) - 1u);
  const int rows_per_word = 32 >> g.lbw;
  uint32_t any = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t word = 0;
    const int row0 = (first + 32 * i) >> g.lbw;
    for (int r = 0; r < rows_per_word; ++r) {
      const int R = row0 + r;
      const int lh = R & (g.bh - 1);
      const int lt = R >> g.lbh;
      if (lt < vt && lh < vh) word |= rowbits << (r << g.lbw);
    }
    w[i] = word;
    any |= word;
  }
  return any ? kTilePartial : kTileEmpty;
}

// Validity bits of the 64 slots of block kb (two words), for 64-token
// blocks.  Returns kTileFull / kTilePartial / kTileEmpty.
__device__ __forceinline__ int block64_mask(const Geo& g, int kb, uint32_t& w0, uint32_t& w1) {
  uint32_t w[4];
  // slots 0..63 of the block are columns 0..63 of "tile 0" of a 128-column view
  w[0] = w[1] = w[2] = w[3] = 0xffffffffu;
  if (kb < 0) {
    w0 = w1 = 0u;
    return kTileEmpty;
  }
  if (kb < g.n_pre) {
    const int lim = g.n_prefix - kb * g.bs;
    if (lim <= 0) {
      w0 = w1 = 0u;
      return kTileEmpty;
    }
    if (lim >= 64) {
      w0 = w1 = 0xffffffffu;
      return kTileFull;
    }
    w0 = lim >= 32 ? 0xffffffffu : ((1u << lim) - 1u);
    w1 = lim <= 32 ? 0u : ((1u << (lim - 32)) - 1u);
    return kTilePartial;
  }
  if (g.vfull) {
    w0 = w1 = 0xffffffffu;
    return kTileFull;
  }
  int vt, vh, vw;
  video_block_extent(g, kb - g.n_pre, vt, vh, vw);
  if (vt == g.bt && vh == g.bh && vw == g.bw) {
    w0 = w1 = 0xffffffffu;
    return kTileFull;
  }
  const uint32_t rowbits = vw >= 32 ? 0xffffffffu : ((1u << vw) - 1u);
  const int rows_per_word = 32 >> g.lbw;
  uint32_t any = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint32_t word = 0;
    const int row0 = (32 * i) >> g.lbw;
    for (int r = 0; r < rows_per_word; ++r) {
      const int R = row0 + r;
      const int lh = R & (g.bh - 1);
      const int lt = R >> g.lbh;
      if (lt < vt && lh < vh) word |= rowbits << (r << g.lbw);
    }
    w[i] = word;
    any |= word;
  }
  w0 = w[0];
  w1 = w[1];
  return any ? kTilePartial : kTileEmpty;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, 128] bf16 row-major viewed as a 2-D tensor; box = 64 columns x box_rows rows, 128-B swizzle.
inline bool make_tmap(CUtensorMap* tm, const void* base, unsigned long long rows, unsigned box_rows, bool f16) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


}  // namespace tiles
}  // namespace vsa
