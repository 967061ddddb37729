// fp4.cu -- NVFP4 Q and K for the fine stage.
//
// FastVideo "Optimizations" page, section "FP4 Flash Attention 4 (Blackwell
// only)": Q and K go to NVFP4 (4-bit E2M1 codes, each block of channels
// sharing one 8-bit E4M3 scale) and V keeps its 16-bit format.  Block length
// 16 (consecutive channels of a token) and scale = E4M3(amax / 6) are NVFP4's
// own definition.
//
// Two kernels:
//
//   quant_nvfp4_kernel  tiled 16-bit rows -> E2M1 codes + E4M3 scales.  One
//                       thread per 16-channel block: amax, scale = E4M3 of
//                       fl32(amax / 6), codes = E2M1 of fl32(x * fl32(1/scale))
//                       (hardware conversions: nearest, ties to even,
//                       saturating), scales scattered into the layout the
//                       tensor core reads (below).  HBM-bound.
//
//   attn_fwd_fp4_kernel the block-sparse attention forward with S = Q K^T as
//                       a block-scaled FP4 product (tcgen05.mma
//                       kind::mxf4nvf4, 16-channel blocks, E4M3 scales read
//                       from tensor memory) and O += P V as a 16-bit product
//                       (P in tensor memory, V in shared memory).
//
// Scale layout (the tensor core's): for each (b, h) and each 128-row tile t of
// the tiled sequence, 1024 bytes; byte kh*512 + (r % 32)*16 + (r / 32)*4 + j
// holds the scale of row 128t + r, channels 16(4kh + j) .. 16(4kh + j) + 15.
// One 512-byte half is a 32 x 16-byte matrix that tcgen05.cp.32x128b.warpx4
// moves into tensor memory, where lane r%32 (of every lane quarter), column
// r/32, byte j holds the scale the MMA needs for row r and channel block j of
// a 64-channel product.
//
// Attention work item: one (b*h, query block) as in the 16-bit kernel (two
// 128-row Q tiles for 256-token blocks, one 64-row tile in the top half of a
// 128-row MMA for 64-token blocks), keys in 128-row tiles (half a 256-token
// block, or two 64-token blocks), the same tensor-memory map (S0, S1, O0, O1:
// all 512 columns) with the scale factors of each S product parked in the
// other Q tile's S columns while those hold nothing live (details below).
//
// Warp roles (384 threads), as in the 16-bit kernel:
//   warp 0      TMA producer: Q codes + scales once per item; per key tile
//               the K codes and the 1 KB scale tiles they belong to (K ring),
//               and V (V ring)
//   warp 1      TMEM owner and MMA issuer (tcgen05.cp of scales, FP4 S MMAs,
//               16-bit PV MMAs)
//   warps 4-11  two softmax warpgroups, one per Q tile, one row per thread
// Per key tile t the MMA thread issues PV0(t), S0(t+1), PV1(t), S1(t+1), so
// one warpgroup's softmax overlaps the other's tensor-core work.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// VSA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "fwd_common.cuh"
#include "kernels.h"
#include "nvfp4.cuh"
#include "tiles.cuh"

namespace vsa {

namespace {

using namespace tiles;
using namespace nvfp4;

// ---------------------------------------------------------------------------
// Conversions
// ---------------------------------------------------------------------------

// Eight fp32 values -> eight E2M1 codes in one word; value 0 in the low nibble
// of byte 0.  Round to nearest, ties to even, saturate at +-6.
__device__ __forceinline__ uint32_t e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5, float x6,
                                           float x7) {
  uint32_t r;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  return r;
}

// fp32 -> E4M3 bits (nearest, ties to even, saturating at 448).
__device__ __forceinline__ uint32_t e4m3_of(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(x), "f"(0.0f));
  return r & 0xffu;
}

// Value of non-negative E4M3 bits (exponent bias 7, 3 mantissa bits; step
// 2^-9 below 2^-6), exact in fp32.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t ex = (b >> 3) & 15u, m = b & 7u;
  return ex == 0 ? static_cast<float>(m) * 0.001953125f : __uint_as_float(((ex + 120u) << 23) | (m << 20));
}

// ---------------------------------------------------------------------------
// Quantisation
// ---------------------------------------------------------------------------

// One thread per 16-channel block: 8 threads per 128-channel row, 32 rows per
// 256-thread block.  rows is a multiple of 128 (whole scale tiles).
template <bool F16>
__global__ void __launch_bounds__(256) quant_nvfp4_kernel(const uint4* __restrict__ x, uint2* __restrict__ codes,
                                                          uint32_t* __restrict__ sf, long long rows) {
  const long long gid = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long row = gid >> 3;
  if (row >= rows) return;  // whole warps: rows is a multiple of 4
  const int b = static_cast<int>(gid & 7);
  const uint4 w0 = __ldg(x + 2 * gid), w1 = __ldg(x + 2 * gid + 1);
  const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (F16) {
      const __half2 h = *reinterpret_cast<const __half2*>(&wd[i]);
      f[2 * i] = __low2float(h);
      f[2 * i + 1] = __high2float(h);
    } else {
      f[2 * i] = bf16_lo(wd[i]);
      f[2 * i + 1] = bf16_hi(wd[i]);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
  const uint32_t sb = e4m3_of(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_value(sb);
  const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(f[i], inv);
  codes[gid] = make_uint2(e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]),
                          e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]));
  // the four scales of a channel half (blocks 4kh .. 4kh+3) form one word
  uint32_t word = sb;
  word |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
  word |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
  word |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
  if ((b & 3) == 0) {
    const long long t = row >> 7;
    const int r = static_cast<int>(row & 127);
    sf[(t * 1024 + (b >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4) >> 2] = word;
  }
}

// ---------------------------------------------------------------------------
// Attention forward with FP4 Q K^T
// ---------------------------------------------------------------------------
//
// The 16-bit kernel's work item, warp roles, pipeline and tensor memory map:
//   [  0,128) S0 (P0 on [0,64))     [128,256) S1 (P1 on [128,192))
//   [256,384) O0                    [384,512) O1
// Keys in 128-row tiles: half a 256-token block, or two selected 64-token
// blocks (the second absent when the count is odd).  The scale factors of a
// block-scaled product have no columns of their own.  Those of S0 = Q0 K^T
// are copied to [192,216) (the Q tile's at +0, the key tile's at +8), those of
// S1 to [64,80): columns of the other tile's S that hold nothing live between
// the moment that tile's softmax has loaded its S (P only takes the first 64
// columns) and the issue of its next S product.  The softmax warpgroups
// signal the load (s_read); the MMA thread waits for it, copies the scales
// (tcgen05.cp, ordered before the MMA that reads them) and issues the product.
// With 64-token blocks there is one Q tile (its 64 rows in the top half of the
// 128-row MMA) and S1 is never written, so no wait is needed; each block of a
// key tile is its own N = 64 product, because its scales are one half of a
// 128-row scale tile (two of the four columns the tensor core reads).

constexpr int kThreads = 384;
constexpr int kStagesK = 4, kStagesV = 3;
constexpr uint32_t kQTileBytes = kCodeTileBytes;  // 128 rows x 64 B of codes
constexpr uint32_t kKTileBytes = kCodeTileBytes;  // 128 keys x 64 B of codes
constexpr uint32_t kKSfBytes = 2 * kSfTileBytes;  // a key tile's scale tiles (two for two 64-token blocks)
constexpr uint32_t kVHalfBytes = 128 * 128;      // 128 keys x 64 channels x 2 B
constexpr uint32_t kVTileBytes = 2 * kVHalfBytes;
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemQsf = kSmemQ + 2 * kQTileBytes;
constexpr uint32_t kSmemK = kSmemQsf + 2 * kSfTileBytes;
constexpr uint32_t kSmemKsf = kSmemK + kStagesK * kKTileBytes;
constexpr uint32_t kSmemV = kSmemKsf + kStagesK * kKSfBytes;
constexpr uint32_t kSmemBar = kSmemV + kStagesV * kVTileBytes;
constexpr uint32_t kSmemTotal = kSmemBar + 256 + 1024;  // barriers + 1 KB alignment slack
static_assert(kSmemK % 1024 == 0 && kSmemV % 1024 == 0 && kSmemBar % 1024 == 0, "1 KB-aligned sections");
constexpr uint32_t kTmO = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kRegsLaunch = 168, kRegsLow = 104, kRegsHigh = 200;
static_assert(kThreads * kRegsLaunch == 128 * kRegsLow + 256 * kRegsHigh, "register split must match the launch");


template <bool F16>
struct IdescPV {
  static constexpr uint32_t v = F16 ? idesc_f16_f32(128, 128, 0, 1) : idesc_bf16_f32(128, 128, 0, 1);
};


struct Barriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], s_read[2], p_full[2], o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 256, "barrier block too large");

struct Params {
  const int32_t* idx;
  const int32_t* num;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  int max_k;
  int BH;
  uint16_t* o;
  float* lse;
  unsigned int* status;
  float scale_log2;
  Geo g;
};

__device__ __forceinline__ int item_blocks(const Params& p, int item, bool report) {
  int c = __ldg(p.num + item);
  if (c < 0 || c > p.max_k) {
    if (report) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
    c = c < 0 ? 0 : p.max_k;
  }
  return c;
}

__device__ __forceinline__ int item_block_id(const Params& p, int item, int j) {
  const int kb = __ldg(p.idx + static_cast<long long>(item) * p.max_k + j);
  return (kb >= 0 && kb < p.g.NB) ? kb : -1;
}


// 128-key tiles of an item with nb selected blocks.
template <int BS>
__device__ __forceinline__ int item_tiles(int nb) {
  return BS == 256 ? 2 * nb : (nb + 1) / 2;
}

// Blocks of key tile t: 256-token blocks, half t&1 of block kb_a (kb_b unused);
// 64-token blocks, blocks kb_a and kb_b (-1 when the count is odd and t is
// the last tile).  Unusable ids come back as -1.
template <int BS>
__device__ __forceinline__ void tile_blocks(const Params& p, int item, int nb, int t, int& kb_a, int& kb_b) {
  if (BS == 256) {
    kb_a = item_block_id(p, item, t >> 1);
    kb_b = -1;
  } else {
    kb_a = item_block_id(p, item, 2 * t);
    kb_b = 2 * t + 1 < nb ? item_block_id(p, item, 2 * t + 1) : -1;
  }
}

// Validity bits of the 128 key columns of tile t; kTileFull / kTilePartial / kTileEmpty.
template <int BS>
__device__ __forceinline__ int tile_mask(const Geo& g, int kb_a, int kb_b, int t, uint32_t (&mw)[4]) {
  if (BS == 256) return key_tile_mask(g, kb_a, t & 1, mw);
  const int sa = block64_mask(g, kb_a, mw[0], mw[1]);
  const int sb = block64_mask(g, kb_b, mw[2], mw[3]);
  if (sa == kTileFull && sb == kTileFull) return kTileFull;
  if (sa == kTileEmpty && sb == kTileEmpty) return kTileEmpty;
  if (sa == kTileFull) mw[0] = mw[1] = 0xffffffffu;
  if (sb == kTileFull) mw[2] = mw[3] = 0xffffffffu;
  return kTilePartial;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Barriers* bars, unsigned int* status) {
  bool ok = mbar_wait(bar, parity, &bars->abort, status, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

// Masked columns of one row of S (128 columns) to -inf; uniform branches.
__device__ __forceinline__ void apply_mask128(uint32_t (&sv)[128], const uint32_t (&mw)[4]) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t m = mw[w];
    if (m == 0xffffffffu) continue;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (!((m >> c) & 1u)) sv[32 * w + c] = 0xff800000u;
  }
}

// Scale-tile halves of the two blocks of 64-token key tile t (bit h for block
// h; an absent or unusable block stands in as block 0).
template <int BS>
__device__ __forceinline__ uint32_t tile_halves(const Params& p, int item, int nb, int t) {
  if (BS == 256) return 0u;
  int kb_a, kb_b;
  tile_blocks<BS>(p, item, nb, t, kb_a, kb_b);
  return (static_cast<uint32_t>(kb_a < 0 ? 0 : kb_a) & 1u) | ((static_cast<uint32_t>(kb_b < 0 ? 0 : kb_b) & 1u) << 1);
}


template <int BS, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sQsf = smem + kSmemQsf;
  uint8_t* sK = smem + kSmemK;
  uint8_t* sKsf = smem + kSmemKsf;
  uint8_t* sV = smem + kSmemV;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + kSmemBar);

  constexpr int kQTiles = BS == 256 ? 2 : 1;  // 128-row query tiles per item
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geo& g = p.g;
  const int total_items = p.BH * g.NB;
  const long long sf_tiles = g.Sp >> 7;  // 128-row scale tiles per head

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_read[i], 128);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 128);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      int kit = 0, vit = 0, qit = 0;
      for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
        const int nb = item_blocks(p, item, false);
        if (nb == 0) continue;
        const int bh = item / g.NB, qb = item - bh * g.NB;
        const long long base = static_cast<long long>(bh) * g.Sp;
        if (!warp_wait(&bars->q_empty, (qit & 1) ^ 1, bars, p.status)) break;
        mbar_arrive_expect_tx_w(&bars->q_full, kQTiles * (kQTileBytes + kSfTileBytes));
        // a 64-token block's rows are the top of a 128-row box, its scales half of a scale tile
        const int q0 = qb * BS;  // first query row inside the head
        for (int i = 0; i < kQTiles; ++i) {
          tma_load_2d_w(sQ + i * kQTileBytes, &tm_q, 0, static_cast<int>(base + q0 + i * 128), &bars->q_full, pol_q);
          const long long tile = bh * sf_tiles + ((q0 >> 7) + i);
          bulk_load_w(sQsf + i * kSfTileBytes, p.q_sf + tile * kSfTileBytes, kSfTileBytes, &bars->q_full);
        }
        ++qit;
        bool stop = false;
        const int n = item_tiles<BS>(nb);
        for (int t = 0; t < n; ++t) {
          // Key rows of this tile: one 128-row box, or two 64-row boxes.
          // Unusable or absent blocks load block 0 -- finite data, masked out
          // by the softmax -- so that no stale shared memory reaches P V.
          int kb_a, kb_b;
          tile_blocks<BS>(p, item, nb, t, kb_a, kb_b);
          const int row_a = BS == 256 ? (kb_a < 0 ? 0 : kb_a) * 256 + (t & 1) * 128 : (kb_a < 0 ? 0 : kb_a) * 64;
          const int row_b = (kb_b < 0 ? 0 : kb_b) * 64;
          const int sk = kit % kStagesK;
          if (!warp_wait(&bars->k_empty[sk], ((kit / kStagesK) & 1) ^ 1, bars, p.status)) {
            stop = true;
            break;
          }
          uint8_t* kdst = sK + sk * kKTileBytes;
          uint8_t* sfdst = sKsf + sk * kKSfBytes;
          mbar_arrive_expect_tx_w(&bars->k_full[sk], kKTileBytes + (BS == 256 ? 1u : 2u) * kSfTileBytes);
          tma_load_2d_w(kdst, &tm_k, 0, static_cast<int>(base + row_a), &bars->k_full[sk], pol_kv);
          bulk_load_w(sfdst, p.k_sf + (bh * sf_tiles + (row_a >> 7)) * kSfTileBytes, kSfTileBytes, &bars->k_full[sk]);
          if (BS == 64) {
            tma_load_2d_w(kdst + kKTileBytes / 2, &tm_k, 0, static_cast<int>(base + row_b), &bars->k_full[sk], pol_kv);
            bulk_load_w(sfdst + kSfTileBytes, p.k_sf + (bh * sf_tiles + (row_b >> 7)) * kSfTileBytes, kSfTileBytes,
                        &bars->k_full[sk]);
          }
          ++kit;
          const int sv = vit % kStagesV;
          if (!warp_wait(&bars->v_empty[sv], ((vit / kStagesV) & 1) ^ 1, bars, p.status)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx_w(&bars->v_full[sv], kVTileBytes);
          for (int hf = 0; hf < 2; ++hf) {
            uint8_t* vdst = sV + sv * kVTileBytes + hf * kVHalfBytes;
            tma_load_2d_w(vdst, &tm_v, hf * 64, static_cast<int>(base + row_a), &bars->v_full[sv], pol_kv);
            if (BS == 64)
              tma_load_2d_w(vdst + kVHalfBytes / 2, &tm_v, hf * 64, static_cast<int>(base + row_b), &bars->v_full[sv],
                            pol_kv);
          }
          ++vit;
        }
        if (stop) break;
      }
      // Drain: every issued copy must land before the CTA's shared memory is released.
      if (qit > 0) mbar_wait_drain(&bars->q_full, (qit - 1) & 1, kTimeoutNs);
      for (int s = 0; s < kStagesK; ++s)
        if (kit > s) {
          const int last = kit - 1 - ((kit - 1 - s) % kStagesK);
          mbar_wait_drain(&bars->k_full[s], (last / kStagesK) & 1, kTimeoutNs);
        }
      for (int s = 0; s < kStagesV; ++s)
        if (vit > s) {
          const int last = vit - 1 - ((vit - 1 - s) % kStagesV);
          mbar_wait_drain(&bars->v_full[s], (last / kStagesV) & 1, kTimeoutNs);
        }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      const uint64_t dq0 = sdesc_sw64(smem_u32(sQ));
      const uint64_t dk0 = sdesc_sw64(smem_u32(sK));
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kVHalfBytes, 1024);
      int kit = 0, vit = 0, qit = 0, tiles = 0, items = 0;
      int sn0 = 0, sn1 = 0;  // S products issued per Q tile
      bool ok = true;
      // S_i = Q_i K^T for key tile t in K stage sk.  Its scales go into the
      // other tile's S columns, free once that tile's softmax has loaded its
      // latest S (with one Q tile that S is never written).
      // khalf: bit h = which half of its scale tile block h of a 64-token key tile is.
      auto issue_s = [&](int i, int sk, uint32_t khalf, uint32_t qshift) -> bool {
        const int j = 1 - i, nj = i == 0 ? sn1 : sn0;
        if (nj > 0 && !warp_wait(&bars->s_read[j], (nj - 1) & 1, bars, p.status)) return false;
        tc_fence_after();
        const uint32_t sf = tmem + sf_col(i);
        const uint8_t* qsf = sQsf + i * kSfTileBytes;
        const uint8_t* ksf = sKsf + sk * kKSfBytes;
        tmem_cp_32x128_w(sf + 0, sdesc_rows16(smem_u32(qsf)));
        tmem_cp_32x128_w(sf + 4, sdesc_rows16(smem_u32(qsf + 512)));
        tmem_cp_32x128_w(sf + 8, sdesc_rows16(smem_u32(ksf)));
        tmem_cp_32x128_w(sf + 12, sdesc_rows16(smem_u32(ksf + 512)));
        const uint32_t d = tmem + 128 * i;
        if (BS == 256) {
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            const uint64_t a = dq0 + ((i * kQTileBytes + kh * 32) >> 4);
            const uint64_t b = dk0 + ((sk * kKTileBytes + kh * 32) >> 4);
            mma_fp4_w(d, a, b, idesc_s(128), sf + 4 * kh, sf + 8 + 4 * kh, kh > 0 ? 1u : 0u);
          }
        } else {
          // one N = 64 product per block; a block's scales are the half
          // (kb & 1) of its scale tile, two columns in
          tmem_cp_32x128_w(sf + 16, sdesc_rows16(smem_u32(ksf + kSfTileBytes)));
          tmem_cp_32x128_w(sf + 20, sdesc_rows16(smem_u32(ksf + kSfTileBytes + 512)));
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
              const uint64_t a = dq0 + ((kh * 32) >> 4);
              const uint64_t b = dk0 + ((sk * kKTileBytes + h * (kKTileBytes / 2) + kh * 32) >> 4);
              mma_fp4_w(d + 64 * h, a, b, idesc_s(64), sf + 4 * kh + qshift, sf + 8 + 8 * h + 4 * kh + 2 * ((khalf >> h) & 1u),
                        kh > 0 ? 1u : 0u);
            }
        }
        if (i == 0) ++sn0; else ++sn1;
        return true;
      };
      auto issue_pv = [&](int i, int sv, bool acc) {
        const uint32_t d = tmem + kTmO + 128 * i, pa = tmem + 128 * i;
        const uint64_t b = dv0 + ((sv * kVTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(d, pa + kk * 8, b + kk * (2048 >> 4), IdescPV<F16>::v, (acc || kk > 0) ? 1u : 0u);
      };
      for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        const int nb = item_blocks(p, item, lane == 0);
        if (nb == 0) continue;
        const int n = item_tiles<BS>(nb);
        // 64-token blocks: the item's rows are one half of their 128-row scale tile
        const uint32_t qshift = BS == 64 ? 2u * static_cast<uint32_t>((item % g.NB) & 1) : 0u;
        if (!(ok = warp_wait(&bars->q_full, qit & 1, bars, p.status))) break;
        ++qit;
        tc_fence_after();
        int sk = kit % kStagesK;
        if (!(ok = warp_wait(&bars->k_full[sk], (kit / kStagesK) & 1, bars, p.status))) break;
        tc_fence_after();
        uint32_t khalf = tile_halves<BS>(p, item, nb, 0);
        if (!(ok = issue_s(0, sk, khalf, qshift))) break;
        mma_commit_w(&bars->s_full[0]);
        if (kQTiles == 2) {
          if (!(ok = issue_s(1, sk, khalf, qshift))) break;
          mma_commit_w(&bars->s_full[1]);
        }
        mma_commit_w(&bars->k_empty[sk]);
        ++kit;
        for (int t = 0; t < n; ++t) {
          const int sv = vit % kStagesV;
          if (!(ok = warp_wait(&bars->v_full[sv], (vit / kStagesV) & 1, bars, p.status))) break;
          if (!(ok = warp_wait(&bars->p_full[0], tiles & 1, bars, p.status))) break;
          if (t == 0 && !(ok = warp_wait(&bars->o_empty[0], (items & 1) ^ 1, bars, p.status))) break;
          tc_fence_after();
          issue_pv(0, sv, t > 0);
          if (t == n - 1) mma_commit_w(&bars->o_full[0]);
          const bool more = t + 1 < n;
          sk = kit % kStagesK;
          if (more) {
            khalf = tile_halves<BS>(p, item, nb, t + 1);
            if (!(ok = warp_wait(&bars->k_full[sk], (kit / kStagesK) & 1, bars, p.status))) break;
            tc_fence_after();
            if (!(ok = issue_s(0, sk, khalf, qshift))) break;
            mma_commit_w(&bars->s_full[0]);
          }
          if (kQTiles == 2) {
            if (!(ok = warp_wait(&bars->p_full[1], tiles & 1, bars, p.status))) break;
            if (t == 0 && !(ok = warp_wait(&bars->o_empty[1], (items & 1) ^ 1, bars, p.status))) break;
            tc_fence_after();
            issue_pv(1, sv, t > 0);
          }
          mma_commit_w(&bars->v_empty[sv]);
          ++vit;
          if (kQTiles == 2 && t == n - 1) mma_commit_w(&bars->o_full[1]);
          if (more) {
            if (kQTiles == 2) {
              if (!(ok = issue_s(1, sk, khalf, qshift))) break;
              mma_commit_w(&bars->s_full[1]);
            }
            mma_commit_w(&bars->k_empty[sk]);
            ++kit;
          }
          ++tiles;
        }
        if (!ok) break;
        mma_commit_w(&bars->q_empty);
        ++items;
      }
      // Drain: wait for every MMA and copy issued by this thread before TMEM and smem go away.
      mma_commit_w(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kTimeoutNs);
    }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) >> 2;  // Q tile
    // 64-token blocks: one query tile per item, held by the first warpgroup
    // in the top 64 rows of its 128-row MMA tile; the second warpgroup idles.
    const bool active = kQTiles == 2 || wg == 0;
    const int quarter = warp & 3;    // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * wg;
    const uint32_t tO = tmem + lane_off + kTmO + 128 * wg;
    const float sl2 = p.scale_log2;
    int tiles = 0, items = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total_items && ok && active; item += gridDim.x) {
      const int nb = item_blocks(p, item, false);
      const int bh = item / g.NB, qb = item - bh * g.NB;
      const long long row = static_cast<long long>(bh) * g.Sp + static_cast<long long>(qb) * BS + wg * 128 + r;
      const bool real_row = BS == 256 || r < 64;
      uint4* orow = reinterpret_cast<uint4*>(p.o + row * 128);
      if (nb == 0) {
        if (!real_row) continue;
#pragma unroll
        for (int c = 0; c < 16; ++c) orow[c] = make_uint4(0, 0, 0, 0);
        p.lse[row] = -INFINITY;
        continue;
      }
      const int n = item_tiles<BS>(nb);
      float m_used = -INFINITY, l = 0.0f;
      for (int t = 0; t < n; ++t) {
        int kb_a, kb_b;
        tile_blocks<BS>(p, item, nb, t, kb_a, kb_b);
        if (wg == 0 && r == 0) {
          const bool bad = BS == 256 ? ((t & 1) == 0 && kb_a < 0) : (kb_a < 0 || (2 * t + 1 < nb && kb_b < 0));
          if (bad) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
        }
        uint32_t mw[4];
        const int mstate = tile_mask<BS>(g, kb_a, kb_b, t, mw);
        if (!(ok = warp_wait(&bars->s_full[wg], tiles & 1, bars, p.status))) break;
        tc_fence_after();
        uint32_t pk[64];
        float lsum = 0.0f, alpha = 1.0f;
        bool rescale = false;
        if (mstate == kTileEmpty) {
          // no real key: the numerators are all zero and the maximum does not move
          tc_fence_before();
          mbar_arrive(&bars->s_read[wg]);
#pragma unroll
          for (int j = 0; j < 64; ++j) pk[j] = 0u;
        } else {
          uint32_t sv[128];
          tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
          tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
          tmem_wait_ld();
          // S is in registers: its last 64 columns may now take the other tile's scales
          tc_fence_before();
          mbar_arrive(&bars->s_read[wg]);
          if (mstate == kTilePartial) apply_mask128(sv, mw);
          float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
            a0 = max3f(a0, __uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1]));
            a1 = max3f(a1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
            a2 = max3f(a2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
            a3 = max3f(a3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
          }
          const float mt = max3f(a0, a1, fmaxf(a2, a3)) * sl2;
          const bool grow = mt > m_used + 8.0f;
          rescale = grow && t > 0 && m_used != -INFINITY;
          alpha = rescale ? ex2_approx(m_used - mt) : 1.0f;
          if (grow) m_used = mt;
          const float msub = (m_used == -INFINITY) ? 0.0f : m_used;
          const uint64_t c2 = f2pack(sl2, sl2), nm2 = f2pack(-msub, -msub);
          uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const uint64_t x = fma2(u2pack(sv[2 * j], sv[2 * j + 1]), c2, nm2);
            float xa, xb;
            f2unpack(x, xa, xb);
            const float pa = ex2_approx(xa), pb = ex2_approx(xb);
            pk[j] = pack_half2<F16>(pa, pb);
            const uint64_t pp = f2pack(pa, pb);
            switch (j & 3) {
              case 0: acc0 = add2(acc0, pp); break;
              case 1: acc1 = add2(acc1, pp); break;
              case 2: acc2 = add2(acc2, pp); break;
              default: acc3 = add2(acc3, pp); break;
            }
          }
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2unpack(acc0, s0, s1);
          f2unpack(acc1, s2, s3);
          f2unpack(acc2, s4, s5);
          f2unpack(acc3, s6, s7);
          lsum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        }
        l = l * alpha + lsum;
        tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        // PV(t-1) has completed: the s_full commit just waited on follows it.
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
            tmem_st32(tO + c * 32, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[wg]);
        ++tiles;
      }
      if (!ok) break;
      // epilogue: O / l -> 16-bit row, lse
      if (!(ok = warp_wait(&bars->o_full[wg], items & 1, bars, p.status))) break;
      tc_fence_after();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + c * 32, ov);
        tmem_wait_ld();
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          wp[j] = pack_half2<F16>(__uint_as_float(ov[2 * j]) * inv, __uint_as_float(ov[2 * j + 1]) * inv);
        if (real_row) {
#pragma unroll
          for (int j = 0; j < 4; ++j) orow[c * 4 + j] = w[j];
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[wg]);
      if (real_row) p.lse[row] = l > 0.0f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      ++items;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// TMA view of [rows, 64] bytes of E2M1 codes, 64-byte swizzle.
bool make_tmap_codes(CUtensorMap* tm, const void* base, unsigned long long rows, unsigned box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {64, rows};
  cuuint64_t strides[1] = {64};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_quant_nvfp4(long long rows, const uint16_t* x, uint8_t* codes, uint8_t* sf, bool f16,
                               cudaStream_t stream) {
  if (rows <= 0 || rows % 128 != 0) return cudaErrorInvalidValue;
  const long long blocks = rows / 32;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = f16 ? quant_nvfp4_kernel<true> : quant_nvfp4_kernel<false>;
  kern<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(reinterpret_cast<const uint4*>(x),
                                                         reinterpret_cast<uint2*>(codes),
                                                         reinterpret_cast<uint32_t*>(sf), rows);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_nvfp4(const Geo& g, const AttnFp4Args& a, cudaStream_t stream) {
  if (g.bs != 256 && g.bs != 64) return cudaErrorNotSupported;
  if (g.Sp % 128 != 0) return cudaErrorNotSupported;
  const unsigned long long rows = static_cast<unsigned long long>(a.BH) * g.Sp;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;
  // key tiles: one 128-row box (256-token blocks) or two 64-row boxes (64-token blocks)
  const unsigned kv_box = g.bs == 256 ? 128 : 64;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_codes(&tq, a.q, rows, 128) || !make_tmap_codes(&tk, a.k, rows, kv_box) ||
      !make_tmap(&tv, a.v, rows, kv_box, a.f16))
    return cudaErrorInvalidValue;
  // 64-token blocks: four query blocks per item (two per 128-row Q tile) over
  // the union of their selections, while the group bitmaps hold the grid
  if (g.bs == 64 && g.NB <= kGroupMaxNB) return launch_attn_fwd_grouped64_fp4(g, tq, tk, tv, a, stream);
  Params p;
  p.idx = a.idx;
  p.num = a.num;
  p.q_sf = a.q_sf;
  p.k_sf = a.k_sf;
  p.max_k = a.max_k;
  p.BH = a.BH;
  p.o = a.o;
  p.lse = a.lse;
  p.status = a.status;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  p.g = g;
  const long long items = static_cast<long long>(a.BH) * g.NB;
  const int grid = static_cast<int>(items < a.num_sms ? items : a.num_sms);
  auto kern = g.bs == 256 ? (a.f16 ? attn_fwd_fp4_kernel<256, true> : attn_fwd_fp4_kernel<256, false>)
                          : (a.f16 ? attn_fwd_fp4_kernel<64, true> : attn_fwd_fp4_kernel<64, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemTotal, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace vsa
