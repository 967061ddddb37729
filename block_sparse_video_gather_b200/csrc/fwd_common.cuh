// fwd_common.cuh -- what the two 16-bit fine-stage kernels share (the
// per-block kernel in attn_fwd.cu and the grouped 64-token kernel in
// attn_fwd_grouped.cu): the CTA shape, the shared-memory map of Q, the K and
// V rings, the register split, the MMA instruction descriptors, the launch
// parameters, the per-item index helpers and the key-mask application.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tiles.cuh"

namespace vsa {
namespace fwd {

using namespace tiles;

constexpr int kThreads = 384;
// K tiles are needed first (by S) and V tiles a softmax later (by PV): the K
// ring is one stage deeper so its loads start two tile periods ahead.
constexpr int kStagesK = 3, kStagesV = 2;
constexpr uint32_t kHalfBytes = 128 * 128;      // 128 rows x 64 bf16 (one 128-B swizzle column)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;  // 128 rows x 128 bf16
constexpr uint32_t kQBytes = 2 * kTileBytes;     // two Q tiles
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kQBytes;
constexpr uint32_t kSmemV = kSmemK + kStagesK * kTileBytes;
constexpr uint32_t kSmemBar = kSmemV + kStagesV * kTileBytes;
constexpr uint32_t kSmemTotal = kSmemBar + 256 + 1024;  // barriers + 1 KB alignment slack
constexpr uint64_t kTimeoutNs = 2000000000ull;          // 2 s per wait
// Register split: launched at 168 per thread (384 x 168 = 64512); warpgroup 0
// (producer, MMA issuer, two idle warps) gives back down to 104 and the two
// softmax warpgroups take 200 each: 128 x 104 + 256 x 200 = 64512.
constexpr int kRegsLaunch = 168, kRegsLow = 104, kRegsHigh = 200;
static_assert(kThreads * kRegsLaunch == 128 * kRegsLow + 256 * kRegsHigh, "register split must match the launch");

// Q (K-major) x K (K-major); P (TMEM) x V (MN-major); bf16 or fp16 operands.
template <bool F16>
struct Idesc {
  static constexpr uint32_t S = F16 ? idesc_f16_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t PV = F16 ? idesc_f16_f32(128, 128, 0, 1) : idesc_bf16_f32(128, 128, 0, 1);
};

struct Barriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 256, "barrier block too large");

struct Params {
  const int32_t* idx;
  const int32_t* num;
  int max_k;
  int BH;
  uint16_t* o;
  float* lse;
  unsigned int* status;
  float scale_log2;
  Geo g;
  // grouped 64-token kernel: a shared group queue (2 int32 of caller memory,
  // ticket and finished-CTA counters, zero on entry and again on exit), or
  // null for a static assignment of groups to CTAs
  int* queue;
};

// Number of selected blocks of an item (clamped into [0, max_k]).
__device__ __forceinline__ int item_blocks(const Params& p, int item, bool report) {
  int c = __ldg(p.num + item);
  if (c < 0 || c > p.max_k) {
    if (report) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
    c = c < 0 ? 0 : p.max_k;
  }
  return c;
}

// Block id of selection j of an item; -1 if out of range.
__device__ __forceinline__ int item_block_id(const Params& p, int item, int j) {
  const int kb = __ldg(p.idx + static_cast<long long>(item) * p.max_k + j);
  return (kb >= 0 && kb < p.g.NB) ? kb : -1;
}

// Mask of 128-key tile t of an item.  256-token blocks: tile t is half t&1
// of block list[t/2].  64-token blocks: tile t holds blocks list[2t] and
// list[2t+1] (the second may be absent).
template <int BS>
__device__ __forceinline__ int item_tile_mask(const Geo& g, int kb_a, int kb_b, int t, uint32_t (&mw)[4]) {
  if (BS == 256) return key_tile_mask(g, kb_a, t & 1, mw);
  const int sa = block64_mask(g, kb_a, mw[0], mw[1]);
  const int sb = block64_mask(g, kb_b, mw[2], mw[3]);
  if (sa == kTileFull && sb == kTileFull) return kTileFull;
  if (sa == kTileEmpty && sb == kTileEmpty) return kTileEmpty;
  if (sa == kTileFull) mw[0] = mw[1] = 0xffffffffu;
  if (sb == kTileFull) mw[2] = mw[3] = 0xffffffffu;
  return kTilePartial;
}

// 128-key tiles of an item with nb selected blocks.
template <int BS>
__device__ __forceinline__ int item_tiles(int nb) {
  return BS == 256 ? 2 * nb : (nb + 1) / 2;
}

// Set the masked columns of one row of S (32 NW columns, one mask word per
// 32) to -inf.  The mask is the same for every thread, so the branches are
// uniform; columns are handled four at a time whenever each group of four is
// all-real or all-padded.
template <int NW>
__device__ __forceinline__ void apply_key_mask(uint32_t (&sv)[32 * NW], const uint32_t (&mw)[NW]) {
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t m = mw[w];
    if (m == 0xffffffffu) continue;
    // a nibble is mixed if not all four of its bits agree
    const uint32_t x = (m ^ (m >> 1)) | (m ^ (m >> 2)) | (m ^ (m >> 3));
    if ((x & 0x11111111u) == 0u) {
#pragma unroll
      for (int gi = 0; gi < 8; ++gi)
        if (!((m >> (4 * gi)) & 1u)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) sv[32 * w + 4 * gi + c] = 0xff800000u;
        }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (!((m >> c) & 1u)) sv[32 * w + c] = 0xff800000u;
    }
  }
}

// Warp-uniform bounded wait: all lanes wait, then agree.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Barriers* bars, unsigned int* status) {
  bool ok = mbar_wait(bar, parity, &bars->abort, status, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace fwd

// The grouped 64-token kernel (attn_fwd_grouped.cu) serves 64-token plans up
// to this many blocks; launch_attn_fwd uses it for them.
constexpr int kGroupMaxNB = 1024;
cudaError_t launch_attn_fwd_grouped64(const Geo& g, const CUtensorMap& tq, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const fwd::Params& p, int BH, int num_sms, bool f16,
                                      cudaStream_t stream);

}  // namespace vsa
