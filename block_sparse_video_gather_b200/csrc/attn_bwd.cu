// attn_bwd.cu -- gradients of the fine stage (dq, dk, dv) with the block
// selection held fixed, on the 5th-generation tensor cores.
//
// The attention step is "FastVideo VSA" (vLLM-Omni user guide, introduction
// and section "Verify routing and fallback"); the FastVideo commit log keeps
// the grad path on separate kernels and prints no formula.  With
// P = softmax(scale q k^T) over each row's selected keys, recomputed from the
// forward's lse:
//   dv = P^T do,  dP = do v^T,  dS = P (dP - delta),  delta_i = do_i . o_i,
//   dq = scale dS k,  dk = scale dS^T q.
// Padded query rows and padded key rows take no part (P = 0 there), so their
// gradients are zero whatever do holds at padded rows.
//
// Four launches:
//   bwd_prep  -delta_i = -do_i . o_i and -lse_i log2(e) per tiled row.
//   k2q       the transposed selection: for each key block, the query blocks
//             that list it (a repeated id is listed again), ascending; rows are
//             placed in order, so the lists do not depend on thread timing.
//   bwd_dkdv  one CTA per (b*h, key block, 128-key half).  K and V stay in
//             shared memory; the 64-row query tiles of every listed query
//             block stream through a 4-stage ring (Q, dO, -lse log2 e, -delta).
//             TMEM: two buffers of S^T (64 columns, P^T written back on the
//             first 32) and dP^T (dS^T on the first 32), dV [256,384),
//             dK [384,512).  Per query tile: S^T = K Q^T, dP^T = V dO^T (N = 64),
//             then dV += P^T dO and dK += dS^T Q; the next tiles' S^T, dP^T
//             run while the elementwise warps work on the current one.
//   bwd_dq    one CTA per (b*h, query block, 128-row half).  Q and dO stay;
//             the K and V tiles of the selected blocks stream.  TMEM: S [0,128),
//             dP [128,256), dQ [256,384), dS (16-bit) [384,448).  Per key tile:
//             S = Q K^T, dP = dO V^T, then dQ += dS K.
// 64-token blocks use the forward's tile-64 arrangement: the resident block
// sits in the top half of a 128-row tile, the streamed 128-wide tiles pair two
// listed blocks (64-row boxes).
// Operands use the two forms of the forward kernel: K-major x K-major for the
// products over the head dimension, TMEM (A) x MN-major shared memory (B) for
// the products over keys or queries.  A tile in shared memory is the TMA image
// of 128 rows x 128 channels (two 64-channel boxes, 128-byte swizzle) and is
// read either way through its descriptor.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 4-11 two warpgroups for the elementwise step and the
// epilogue: a thread owns one TMEM lane (tile row), warpgroup w the columns
// [64w, 64w + 64) of it.  In dkdv, P^T and dS^T are written back over S^T and
// dP^T, so both warpgroups finish reading before either writes (named barrier).  Every mbarrier wait is bounded; on expiry the kernel
// records VSA_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace vsa {

namespace {

using namespace tiles;

constexpr int kThreads = 384;
constexpr uint32_t kHalfBytes = 128 * 128;      // 128 rows x 64 16-bit channels
constexpr uint32_t kTileBytes = 2 * kHalfBytes;  // 128 rows x 128 channels
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
// Register split: launched at 168 per thread (384 x 168 = 64512); warpgroup 0
// (producer, MMA issuer, two idle warps) gives back down to 104 and the two
// elementwise warpgroups take 200 each: 128 x 104 + 256 x 200 = 64512.
constexpr int kRegsLaunch = 168, kRegsLow = 104, kRegsHigh = 200;
static_assert(kThreads * kRegsLaunch == 128 * kRegsLow + 256 * kRegsHigh, "register split must match the launch");

template <bool F16>
struct Idesc {
  static constexpr uint32_t KK = F16 ? idesc_f16_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t TM = F16 ? idesc_f16_f32(128, 128, 0, 1) : idesc_bf16_f32(128, 128, 0, 1);
};

// Word i of four, without dynamic indexing (which would put the array in local memory).
__device__ __forceinline__ uint32_t pick4(const uint32_t (&w)[4], int i) {
  return i == 0 ? w[0] : (i == 1 ? w[1] : (i == 2 ? w[2] : w[3]));
}

// All 128 validity bits of a tile (key_tile_mask sets them only for a
// partial tile; a full or empty one is reported by its return value).
__device__ __forceinline__ int tile_bits(const Geo& g, int blk, int half, uint32_t (&w)[4]) {
  const int st = key_tile_mask(g, blk, half, w);
  if (st != kTilePartial) w[0] = w[1] = w[2] = w[3] = (st == kTileFull) ? 0xffffffffu : 0u;
  return st;
}

__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Barrier among the 256 threads of the two elementwise warpgroups.
__device__ __forceinline__ void wg_pair_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// P and dS for 32 columns of this thread's row: x = s c2 + nl, P = 2^x (0 where
// m has no bit), dS = P (dp + nd).  nl, nd: two columns per 64-bit word.
template <bool F16>
__device__ __forceinline__ void p_ds32(const uint32_t (&sv)[32], const uint32_t (&dv)[32], uint64_t c2,
                                       const uint64_t* nl, const uint64_t* nd, uint32_t m, uint32_t (&pk)[16],
                                       uint32_t (&dk)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint64_t x = fma2(u2pack(sv[2 * j], sv[2 * j + 1]), c2, nl[j]);
    float xa, xb;
    f2unpack(x, xa, xb);
    float pa = ex2_approx(xa), pb = ex2_approx(xb);
    if (m != 0xffffffffu) {
      pa = ((m >> (2 * j)) & 1u) ? pa : 0.0f;
      pb = ((m >> (2 * j + 1)) & 1u) ? pb : 0.0f;
    }
    const uint64_t ds = mul2(f2pack(pa, pb), add2(u2pack(dv[2 * j], dv[2 * j + 1]), nd[j]));
    float da, db;
    f2unpack(ds, da, db);
    pk[j] = pack_half2<F16>(pa, pb);
    dk[j] = pack_half2<F16>(da, db);
  }
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

struct BwdBarriers {
  uint64_t a_full;            // resident tiles (K,V for dkdv; Q,dO for dq)
  uint64_t full[4], empty[4];  // streamed stages (dkdv: Q/dO ring; dq: the V ring)
  uint64_t kfull[3], kempty[3];  // dq: the K ring
  uint32_t mask[3][4];            // validity bits of the streamed tile of each stage (written by the producer)
  uint64_t s_full, s_free, ds_full, ds_free, done, drain;
  uint64_t sbuf[2];               // dkdv: S^T / dP^T buffer b holds a finished tile
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(BwdBarriers) <= 256, "barrier block too large");

__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, BwdBarriers* b, unsigned int* status) {
  bool ok = mbar_wait(bar, parity, &b->abort, status, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void init_barriers(BwdBarriers* b) {
  mbar_init(&b->a_full, 1);
  for (int s = 0; s < 4; ++s) {
    mbar_init(&b->full[s], 1);
    mbar_init(&b->empty[s], 1);
  }
  mbar_init(&b->sbuf[0], 1);
  mbar_init(&b->sbuf[1], 1);
  for (int s = 0; s < 3; ++s) {
    mbar_init(&b->kfull[s], 1);
    mbar_init(&b->kempty[s], 1);
  }
  mbar_init(&b->s_full, 1);
  mbar_init(&b->s_free, 256);
  mbar_init(&b->ds_full, 256);
  mbar_init(&b->ds_free, 1);
  mbar_init(&b->done, 1);
  mbar_init(&b->drain, 1);
  b->abort = 0;
  fence_barrier_init();
  fence_proxy_async_smem();
}

// 128 fp32 TMEM columns of this thread's lane, scaled, to one 16-bit row in
// global memory.  `load` must be the same for the whole warp (the TMEM load
// is a warp-wide instruction); `zero` may differ per thread.
template <bool F16>
__device__ __forceinline__ void store_row(uint32_t taddr, float scale, uint16_t* dst, bool load, bool zero) {
  uint4* out = reinterpret_cast<uint4*>(dst);
  zero = zero || !load;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t v[32];
    if (load) {
      tmem_ld32(taddr + c * 32, v);
      tmem_wait_ld();
    }
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      w[j] = zero ? 0u : pack_half2<F16>(__uint_as_float(v[2 * j]) * scale, __uint_as_float(v[2 * j + 1]) * scale);
#pragma unroll
    for (int j = 0; j < 4; ++j) out[c * 4 + j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

// Columns [c0, c0 + 64) of this thread's lane (fp32, scaled) to 64 16-bit values at dst.
template <bool F16>
__device__ __forceinline__ void store_half_row(uint32_t taddr, float scale, uint16_t* dst, bool load, bool zero) {
  uint4* out = reinterpret_cast<uint4*>(dst);
  zero = zero || !load;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t v[32];
    if (load) {
      tmem_ld32(taddr + c * 32, v);
      tmem_wait_ld();
    }
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      w[j] = zero ? 0u : pack_half2<F16>(__uint_as_float(v[2 * j]) * scale, __uint_as_float(v[2 * j + 1]) * scale);
#pragma unroll
    for (int j = 0; j < 4; ++j) out[c * 4 + j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

struct BwdParams {
  Geo g;
  int BH, max_k;
  const int32_t* idx;
  const int32_t* num;
  const int32_t* k2q_off;  // [BH][NB + 1]
  const int32_t* k2q;      // [BH][NB * max_k]
  const float* nlse2;      // [BH * Sp]  -lse log2(e)
  const float* ndelta;     // [BH * Sp]  -(do . o)
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  unsigned int* status;
  float scale;       // D^-1/2
  float scale_log2;  // D^-1/2 log2(e)
};

// ---------------------------------------------------------------------------
// dk, dv
// ---------------------------------------------------------------------------
// Query tiles of 64 rows: S^T and dP^T take 64 TMEM columns each, so both are
// double-buffered next to dV and dK ([0,64)+64b: S^T of buffer b, P^T written
// back on its first 32 columns; [128,192)+64b: dP^T, dS^T on its first 32;
// [256,384) dV; [384,512) dK).  The MMA warp issues S^T(u+2), dP^T(u+2) right
// after dV(u), dK(u) (which read buffer u&1 first), so the tensor core computes
// the next tiles while the elementwise warps work on the current one.
constexpr uint32_t kQ64Bytes = 64 * 128 * 2;           // 64 rows x 128 channels: two 8 KB halves
constexpr int kKVStages = 4;
constexpr uint32_t kKV_K = 0, kKV_V = kTileBytes, kKV_Stage = 2 * kTileBytes;
constexpr uint32_t kKV_StageBytes = 2 * kQ64Bytes;     // Q + dO
constexpr uint32_t kKV_L = kKV_Stage + kKVStages * kKV_StageBytes;  // -lse log2 e, -delta: 64 + 64 floats a stage
constexpr uint32_t kKV_Bar = kKV_L + kKVStages * 512;
constexpr uint32_t kKV_Smem = kKV_Bar + 256 + 1024;

template <bool F16>
struct Idesc64 {
  static constexpr uint32_t KK = F16 ? idesc_f16_f32(128, 64, 0, 0) : idesc_bf16_f32(128, 64, 0, 0);
};

// 64-token blocks (BS = 64): an item is one key block in the top half of the
// 128-row tile (the 128-row box also brings the next block's rows, finite and
// masked).  A 256-token query block is four 64-row query tiles; a 64-token
// block is one.
template <int BS, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do64,
                         const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + kKV_Bar);
  uint32_t* maskw = &bars->mask[0][0];  // [stage][2]
  const Geo& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kHalves = BS == 256 ? 2 : 1;
  constexpr int kTilesPerBlock = BS / 64;
  const int item = blockIdx.x;
  const int half = BS == 256 ? (item & 1) : 0;
  const int kb = (item / kHalves) % g.NB;
  const int bh = (item / kHalves) / g.NB;
  const int32_t* offs = p.k2q_off + static_cast<long long>(bh) * (g.NB + 1);
  const int lo = __ldg(offs + kb), hi = __ldg(offs + kb + 1);
  const int32_t* list = p.k2q + static_cast<long long>(bh) * g.NB * p.max_k + lo;
  const int nq = kTilesPerBlock * (hi - lo);  // 64-row query tiles
  const long long base = static_cast<long long>(bh) * g.Sp;

  if (threadIdx.x == 0) init_barriers(bars);
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
    const uint64_t pol_last = policy_evict_last();
    int issued = 0;
    bool kv = false;
    if (nq > 0) {
      const int krow = static_cast<int>(base + static_cast<long long>(kb) * BS + half * 128);
      mbar_arrive_expect_tx_w(&bars->a_full, 2 * kTileBytes);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_2d_w(smem + kKV_K + hf * kHalfBytes, &tm_k, hf * 64, krow, &bars->a_full, pol_last);
        tma_load_2d_w(smem + kKV_V + hf * kHalfBytes, &tm_v, hf * 64, krow, &bars->a_full, pol_last);
      }
      kv = true;
      // the next tile's query block id and validity bits are prepared before
      // its stage is free, so that only the copies follow the wait
      int qb_next = __ldg(list);
      for (int u = 0; u < nq; ++u) {
        const int s = u % kKVStages;
        const int qb = qb_next;
        if (u + 1 < nq) qb_next = __ldg(list + (u + 1) / kTilesPerBlock);
        const int qq = u % kTilesPerBlock;  // 64-row part of the query block
        const long long qrow = base + static_cast<long long>(qb) * BS + 64 * qq;
        uint32_t w[4];
        if (BS == 256) {
          tile_bits(g, qb, qq >> 1, w);
        } else {
          block64_mask(g, qb, w[0], w[1]);
        }
        const uint32_t w0 = pick4(w, BS == 256 ? 2 * (qq & 1) : 0), w1 = pick4(w, BS == 256 ? 2 * (qq & 1) + 1 : 1);
        if (!wwait(&bars->empty[s], ((u / kKVStages) & 1) ^ 1, bars, p.status)) break;
        if (lane < 2) maskw[2 * s + lane] = lane ? w1 : w0;  // published by the arrive below
        __syncwarp();
        uint8_t* st = smem + kKV_Stage + s * kKV_StageBytes;
        mbar_arrive_expect_tx_w(&bars->full[s], kKV_StageBytes + 512);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_2d_w(st + hf * (kQ64Bytes / 2), &tm_q64, hf * 64, static_cast<int>(qrow), &bars->full[s], pol_last);
          tma_load_2d_w(st + kQ64Bytes + hf * (kQ64Bytes / 2), &tm_do64, hf * 64, static_cast<int>(qrow),
                        &bars->full[s], pol_last);
        }
        if (lane == 0) {
          bulk_load(smem + kKV_L + s * 512, p.nlse2 + qrow, 256, &bars->full[s]);
          bulk_load(smem + kKV_L + s * 512 + 256, p.ndelta + qrow, 256, &bars->full[s]);
        }
        __syncwarp();
        ++issued;
      }
    }
    // drain every copy in flight before shared memory is released
    if (kv) mbar_wait_drain(&bars->a_full, 0, kTimeoutNs);
    for (int s = 0; s < kKVStages; ++s)
      if (issued > s) {
        const int last = issued - 1 - ((issued - 1 - s) % kKVStages);
        mbar_wait_drain(&bars->full[s], (last / kKVStages) & 1, kTimeoutNs);
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dK = sdesc_sw128(smem_u32(smem + kKV_K), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(smem + kKV_V), 16, 1024);
    const uint64_t dSt = sdesc_sw128(smem_u32(smem + kKV_Stage), 16, 1024);              // K-major view
    const uint64_t mSt = sdesc_sw128(smem_u32(smem + kKV_Stage), kQ64Bytes / 2, 1024);   // MN-major view
    constexpr uint64_t kStage = kKV_StageBytes >> 4, kQ64 = kQ64Bytes >> 4;
    auto issue_sdp = [&](int u) {  // S^T(u), dP^T(u) into buffer u&1
      const int s = u % kKVStages, b = u & 1;
      const uint64_t q_k = dSt + s * kStage, do_k = q_k + kQ64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ok_ = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;        // 128-row K/V tile
        const uint32_t oq = ((kk >> 2) * (kQ64Bytes / 2) + (kk & 3) * 32) >> 4;   // 64-row Q/dO tile
        mma_ss_w(tmem + 64 * b, dK + ok_, q_k + oq, Idesc64<F16>::KK, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ok_ = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
        const uint32_t oq = ((kk >> 2) * (kQ64Bytes / 2) + (kk & 3) * 32) >> 4;
        mma_ss_w(tmem + 128 + 64 * b, dV + ok_, do_k + oq, Idesc64<F16>::KK, kk > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->sbuf[b]);
    };
    bool ok = true;
    if (nq > 0) ok = wwait(&bars->a_full, 0, bars, p.status);
    for (int u = 0; u < 2 && u < nq && ok; ++u) {
      if (!(ok = wwait(&bars->full[u], 0, bars, p.status))) break;
      tc_fence_after();
      issue_sdp(u);
    }
    for (int u = 0; u < nq && ok; ++u) {
      const int s = u % kKVStages, b = u & 1;
      if (!(ok = wwait(&bars->ds_full, u & 1, bars, p.status))) break;
      tc_fence_after();
      const uint64_t q_m = mSt + s * kStage, do_m = q_m + kQ64;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts_w(tmem + 256, tmem + 64 * b + kk * 8, do_m + kk * (2048 >> 4), Idesc<F16>::TM,
                 (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts_w(tmem + 384, tmem + 128 + 64 * b + kk * 8, q_m + kk * (2048 >> 4), Idesc<F16>::TM,
                 (u > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(&bars->empty[s]);
      if (u + 2 < nq) {  // buffer b is free once dV(u), dK(u) have read it (tensor core order)
        if (!(ok = wwait(&bars->full[(u + 2) % kKVStages], ((u + 2) / kKVStages) & 1, bars, p.status))) break;
        tc_fence_after();
        issue_sdp(u + 2);
      }
    }
    mma_commit_w(&bars->done);
    mma_commit_w(&bars->drain);
    mbar_wait_drain(&bars->drain, 0, kTimeoutNs);
  }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ elementwise + epilogue
    const int wg = (warp - 4) >> 2;     // query columns [32 wg, 32 wg + 32) of the 64-row tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tL = tmem + lane_off;
    uint32_t kw[4];
    if (BS == 256) {
      tile_bits(g, kb, half, kw);
    } else {
      block64_mask(g, kb, kw[0], kw[1]);
      kw[2] = kw[3] = 0u;  // rows 64..127 belong to the next block
    }
    const bool kvalid = (pick4(kw, r >> 5) >> (r & 31)) & 1u;
    const uint64_t c2 = f2pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int u = 0; u < nq && ok; ++u) {
      const int s = u % kKVStages, b = u & 1;
      if (!(ok = wwait(&bars->full[s], (u / kKVStages) & 1, bars, p.status))) break;
      const uint32_t m = kvalid ? maskw[2 * s + wg] : 0u;
      if (!(ok = wwait(&bars->sbuf[b], (u >> 1) & 1, bars, p.status))) break;
      tc_fence_after();
      const uint64_t* NL = reinterpret_cast<const uint64_t*>(smem + kKV_L + s * 512);
      const uint64_t* ND = NL + 32;
      uint32_t pk[16], dk16[16];
      {
        uint32_t sv[32], dv[32];
        tmem_ld32(tL + 64 * b + 32 * wg, sv);
        tmem_ld32(tL + 128 + 64 * b + 32 * wg, dv);
        tmem_wait_ld();
        p_ds32<F16>(sv, dv, c2, NL + 16 * wg, ND + 16 * wg, m, pk, dk16);
      }
      wg_pair_sync();  // both halves of S^T and dP^T have been read
      tmem_st16(tL + 64 * b + 16 * wg, pk);
      tmem_st16(tL + 128 + 64 * b + 16 * wg, dk16);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
    }
    if (ok && nq > 0) ok = wwait(&bars->done, 0, bars, p.status);
    tc_fence_after();
    const long long row = base + static_cast<long long>(kb) * BS + half * 128 + r;
    const bool load = ok && nq > 0;  // warp-uniform
    if (BS == 256 || quarter < 2) {  // for 64-token blocks, lanes 64..127 are the next block's rows
      if (wg == 0)
        store_row<F16>(tL + 256, 1.0f, p.dv + row * 128, load, false);
      else
        store_row<F16>(tL + 384, p.scale, p.dk + row * 128, load, false);
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

// ---------------------------------------------------------------------------
// dq
// ---------------------------------------------------------------------------
// K is read by the first MMA of a tile and by its last (dQ += dS K), V only by
// the first: three K stages and two V stages keep the next copies in flight.
constexpr uint32_t kQ_Q = 0, kQ_DO = kTileBytes, kQ_K = 2 * kTileBytes;  // K stages: 3 x 32 KB
constexpr uint32_t kQ_V = kQ_K + 3 * kTileBytes;                          // V stages: 2 x 32 KB
constexpr uint32_t kQ_Bar = kQ_V + 2 * kTileBytes;
constexpr uint32_t kQ_Smem = kQ_Bar + 256 + 1024;

__device__ __forceinline__ int dq_block(const BwdParams& p, long long row_item, int j) {
  const int kb = __ldg(p.idx + row_item * p.max_k + j);
  return (kb >= 0 && kb < p.g.NB) ? kb : -1;
}

// 64-token blocks (BS = 64): an item is one query block in the top half of
// the 128-row tile, and each streamed 128-key tile holds two selected blocks,
// loaded as 64-row boxes (tm_ks, tm_vs).
template <int BS, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ks,
                       const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + kQ_Bar);
  const Geo& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kHalves = BS == 256 ? 2 : 1;
  const int item = blockIdx.x;
  const int half = BS == 256 ? (item & 1) : 0;
  const int qb = (item / kHalves) % g.NB;
  const int bh = (item / kHalves) / g.NB;
  const long long row_item = static_cast<long long>(bh) * g.NB + qb;
  int nb = __ldg(p.num + row_item);
  if (nb < 0 || nb > p.max_k) {
    if (threadIdx.x == 0 && half == 0) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
    nb = nb < 0 ? 0 : p.max_k;
  }
  const int n = BS == 256 ? 2 * nb : (nb + 1) / 2;  // key tiles
  const long long base = static_cast<long long>(bh) * g.Sp;

  if (threadIdx.x == 0) init_barriers(bars);
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
    const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
    int issued = 0, issued_k = 0;  // V and K copies issued
    bool qd = false;
    if (n > 0) {
      const int qrow = static_cast<int>(base + static_cast<long long>(qb) * BS + half * 128);
      mbar_arrive_expect_tx_w(&bars->a_full, 2 * kTileBytes);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_2d_w(smem + kQ_Q + hf * kHalfBytes, &tm_q, hf * 64, qrow, &bars->a_full, pol_first);
        tma_load_2d_w(smem + kQ_DO + hf * kHalfBytes, &tm_do, hf * 64, qrow, &bars->a_full, pol_first);
      }
      qd = true;
      for (int t = 0; t < n; ++t) {
        // rows of the tile's key blocks: one 128-row box, or two 64-row boxes;
        // unusable or absent ids load block 0, which the elementwise step masks out
        int krow0, krow1 = 0;
        uint32_t w[4];
        bool bad;
        if (BS == 256) {
          const int kb0 = dq_block(p, row_item, t >> 1);
          krow0 = static_cast<int>(base + static_cast<long long>(kb0 < 0 ? 0 : kb0) * 256 + (t & 1) * 128);
          tile_bits(g, kb0, t & 1, w);
          bad = kb0 < 0 && half == 0 && (t & 1) == 0;
        } else {
          const int ka = dq_block(p, row_item, 2 * t);
          const int kc = 2 * t + 1 < nb ? dq_block(p, row_item, 2 * t + 1) : -1;
          krow0 = static_cast<int>(base + static_cast<long long>(ka < 0 ? 0 : ka) * 64);
          krow1 = static_cast<int>(base + static_cast<long long>(kc < 0 ? 0 : kc) * 64);
          block64_mask(g, ka, w[0], w[1]);
          block64_mask(g, kc, w[2], w[3]);
          bad = ka < 0 || (2 * t + 1 < nb && kc < 0);
        }
        const int ks = t % 3, vs = t & 1;
        if (!wwait(&bars->kempty[ks], ((t / 3) & 1) ^ 1, bars, p.status)) break;
        if (lane < 4) bars->mask[ks][lane] = pick4(w, lane);  // published by the arrive below
        if (bad && lane == 0) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
        __syncwarp();
        mbar_arrive_expect_tx_w(&bars->kfull[ks], kTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
          uint8_t* dst = smem + kQ_K + ks * kTileBytes + hf * kHalfBytes;
          tma_load_2d_w(dst, &tm_ks, hf * 64, krow0, &bars->kfull[ks], pol_last);
          if (BS == 64) tma_load_2d_w(dst + kHalfBytes / 2, &tm_ks, hf * 64, krow1, &bars->kfull[ks], pol_last);
        }
        if (!wwait(&bars->empty[vs], ((t >> 1) & 1) ^ 1, bars, p.status)) {
          ++issued_k;
          break;
        }
        mbar_arrive_expect_tx_w(&bars->full[vs], kTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
          uint8_t* dst = smem + kQ_V + vs * kTileBytes + hf * kHalfBytes;
          tma_load_2d_w(dst, &tm_vs, hf * 64, krow0, &bars->full[vs], pol_last);
          if (BS == 64) tma_load_2d_w(dst + kHalfBytes / 2, &tm_vs, hf * 64, krow1, &bars->full[vs], pol_last);
        }
        ++issued_k;
        ++issued;
      }
    }
    if (qd) mbar_wait_drain(&bars->a_full, 0, kTimeoutNs);
    for (int s = 0; s < 2; ++s)
      if (issued > s) {
        const int last = issued - 1 - ((issued - 1 - s) & 1);
        mbar_wait_drain(&bars->full[s], (last >> 1) & 1, kTimeoutNs);
      }
    for (int s = 0; s < 3; ++s)
      if (issued_k > s) {
        const int last = issued_k - 1 - ((issued_k - 1 - s) % 3);
        mbar_wait_drain(&bars->kfull[s], (last / 3) & 1, kTimeoutNs);
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dQ = sdesc_sw128(smem_u32(smem + kQ_Q), 16, 1024);
    const uint64_t dDO = sdesc_sw128(smem_u32(smem + kQ_DO), 16, 1024);
    const uint64_t dK = sdesc_sw128(smem_u32(smem + kQ_K), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(smem + kQ_V), 16, 1024);
    const uint64_t mK = sdesc_sw128(smem_u32(smem + kQ_K), kHalfBytes, 1024);
    constexpr uint64_t kTile = kTileBytes >> 4;
    // S(t+1) and dP(t+1) are issued as soon as the elementwise warps have read
    // S(t) and dP(t) (s_free), so the tensor core works while they form dS(t).
    auto issue_sdp = [&](int t) {  // S(t), dP(t); V(t) is released when they complete
      const int ks = t % 3, vs = t & 1;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
        mma_ss_w(tmem + 0, dQ + off, dK + ks * kTile + off, Idesc<F16>::KK, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
        mma_ss_w(tmem + 128, dDO + off, dV + vs * kTile + off, Idesc<F16>::KK, kk > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->s_full);
      mma_commit_w(&bars->empty[vs]);
    };
    auto wait_kv = [&](int t) {
      return wwait(&bars->kfull[t % 3], (t / 3) & 1, bars, p.status) &&
             wwait(&bars->full[t & 1], (t >> 1) & 1, bars, p.status);
    };
    bool ok = true;
    if (n > 0) ok = wwait(&bars->a_full, 0, bars, p.status) && wait_kv(0);
    if (ok && n > 0) {
      tc_fence_after();
      issue_sdp(0);
    }
    for (int t = 0; t < n && ok; ++t) {
      if (!(ok = wwait(&bars->s_free, t & 1, bars, p.status))) break;
      if (t + 1 < n) {
        if (!(ok = wait_kv(t + 1))) break;
        tc_fence_after();
        issue_sdp(t + 1);
      }
      if (!(ok = wwait(&bars->ds_full, t & 1, bars, p.status))) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(tmem + 256, tmem + 384 + kk * 8, mK + (t % 3) * kTile + kk * (2048 >> 4), Idesc<F16>::TM,
                 (t > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(&bars->kempty[t % 3]);
      mma_commit_w(&bars->ds_free);
    }
    mma_commit_w(&bars->done);
    mma_commit_w(&bars->drain);
    mbar_wait_drain(&bars->drain, 0, kTimeoutNs);
  }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ elementwise + epilogue
    const int wg = (warp - 4) >> 2;     // key columns [64 wg, 64 wg + 64)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off, tP = tS + 128, tDS = tS + 384;
    uint32_t rw[4];
    if (BS == 256) {
      tile_bits(g, qb, half, rw);
    } else {
      block64_mask(g, qb, rw[0], rw[1]);
      rw[2] = rw[3] = 0u;  // rows 64..127 belong to the next block
    }
    const bool rvalid = (pick4(rw, r >> 5) >> (r & 31)) & 1u;
    const long long row = base + static_cast<long long>(qb) * BS + half * 128 + r;
    const float nl = rvalid ? __ldg(p.nlse2 + row) : 0.0f;
    const float nd = rvalid ? __ldg(p.ndelta + row) : 0.0f;
    uint64_t nl2[16], nd2[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      nl2[j] = f2pack(nl, nl);
      nd2[j] = f2pack(nd, nd);
    }
    const uint64_t c2 = f2pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int t = 0; t < n && ok; ++t) {
      if (!(ok = wwait(&bars->s_full, t & 1, bars, p.status))) break;
      // the key tile's validity bits: written before its copy was announced on kfull
      if (!(ok = wwait(&bars->kfull[t % 3], (t / 3) & 1, bars, p.status))) break;
      uint32_t kw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) kw[i] = bars->mask[t % 3][i];
      tc_fence_after();
      uint32_t sv[2][32], dv[2][32], pk[16], dk16[2][16];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        tmem_ld32(tS + (2 * wg + cc) * 32, sv[cc]);
        tmem_ld32(tP + (2 * wg + cc) * 32, dv[cc]);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);  // S and dP may be overwritten by the next tile
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
        p_ds32<F16>(sv[cc], dv[cc], c2, nl2, nd2, rvalid ? pick4(kw, 2 * wg + cc) : 0u, pk, dk16[cc]);
      if (t > 0 && !(ok = wwait(&bars->ds_free, (t - 1) & 1, bars, p.status))) break;  // dQ(t-1) read dS
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) tmem_st16(tDS + (2 * wg + cc) * 16, dk16[cc]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
    }
    if (ok && n > 0) ok = wwait(&bars->done, 0, bars, p.status);
    tc_fence_after();
    if (BS == 256 || quarter < 2)  // for 64-token blocks, lanes 64..127 are the next block's rows
      store_half_row<F16>(tS + 256 + 64 * wg, p.scale, p.dq + row * 128 + 64 * wg, ok && n > 0, !rvalid);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// preparation: delta and lse2 per tiled row; transposed selection per head
// ---------------------------------------------------------------------------
template <bool F16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dO,
                                                       const float* __restrict__ lse, float* __restrict__ nlse2,
                                                       float* __restrict__ ndelta, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 16 + (threadIdx.x >> 4);
  const int chunk = threadIdx.x & 15;
  float acc = 0.0f;
  if (row < rows) {
    const uint4 a = __ldg(o + row * 16 + chunk), b = __ldg(dO + row * 16 + chunk);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float alo, ahi, blo, bhi;
      if (F16) {
        alo = __half2float(__ushort_as_half(static_cast<unsigned short>(aw[k] & 0xFFFFu)));
        ahi = __half2float(__ushort_as_half(static_cast<unsigned short>(aw[k] >> 16)));
        blo = __half2float(__ushort_as_half(static_cast<unsigned short>(bw[k] & 0xFFFFu)));
        bhi = __half2float(__ushort_as_half(static_cast<unsigned short>(bw[k] >> 16)));
      } else {
        alo = bf16_lo(aw[k]);
        ahi = bf16_hi(aw[k]);
        blo = bf16_lo(bw[k]);
        bhi = bf16_hi(bw[k]);
      }
      acc = __fmaf_rn(alo, blo, acc);
      acc = __fmaf_rn(ahi, bhi, acc);
    }
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && chunk == 0) {
    ndelta[row] = -acc;
    nlse2[row] = -__ldg(lse + row) * kLog2e;
  }
}

// One CTA per (b*h).  Counts per key block, offsets, then rows in order.
// Grids up to this many blocks build the transposed selection from a bitmap
// (NB x NB bits of shared memory: 128 KB at 1024 blocks).
constexpr int kK2qBitmapMaxNB = 1024;

__host__ __device__ constexpr size_t k2q_smem_bytes(int NB) {
  return NB <= kK2qBitmapMaxNB
             ? (static_cast<size_t>(NB) * ((NB + 31) / 32) + 2 * static_cast<size_t>(NB)) * sizeof(int)
             : 2 * static_cast<size_t>(NB) * sizeof(int);
}

// The transposed selection of one head: for each key block, the query blocks
// that list it, ascending.  Grids of at most kK2qBitmapMaxNB blocks set one
// bit per (key block, query block) and read each key block's list off its
// bitmap (every step parallel); a head whose lists repeat an id (the repeat is
// listed again) and larger grids place the rows one query block at a time.
__global__ void __launch_bounds__(256) k2q_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ num,
                                                  int NB, int max_k, int32_t* __restrict__ k2q_off,
                                                  int32_t* __restrict__ k2q, unsigned int* status) {
  extern __shared__ int kq_sm[];
  const int bh = blockIdx.x;
  const int32_t* ih = idx + static_cast<long long>(bh) * NB * max_k;
  const int32_t* nh = num + static_cast<long long>(bh) * NB;
  int32_t* list = k2q + static_cast<long long>(bh) * NB * max_k;
  int32_t* off = k2q_off + static_cast<long long>(bh) * (NB + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  bool bad = false;
  if (NB <= kK2qBitmapMaxNB) {
    const int W = (NB + 31) >> 5;
    uint32_t* bits = reinterpret_cast<uint32_t*>(kq_sm);  // [NB key blocks][W words of query blocks]
    int* cnt = kq_sm + NB * W;                            // [NB]
    for (int i = tid; i < NB * W; i += blockDim.x) bits[i] = 0u;
    __syncthreads();
    bool dup = false;
    for (long long e = tid; e < static_cast<long long>(NB) * max_k; e += blockDim.x) {
      const int r = static_cast<int>(e / max_k), t = static_cast<int>(e - static_cast<long long>(r) * max_k);
      int c = nh[r];
      if (c < 0 || c > max_k) {
        bad = true;
        c = c < 0 ? 0 : max_k;
      }
      if (t >= c) continue;
      const int kb = ih[e];
      if (kb < 0 || kb >= NB) {
        bad = true;
        continue;
      }
      const uint32_t bit = 1u << (r & 31);
      if (atomicOr(&bits[kb * W + (r >> 5)], bit) & bit) dup = true;
    }
    if (bad) atomicCAS(status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
    if (!__syncthreads_or(dup)) {
      for (int kb = tid; kb < NB; kb += blockDim.x) {
        int n = 0;
        for (int w = 0; w < W; ++w) n += __popc(bits[kb * W + w]);
        cnt[kb] = n;
      }
      __syncthreads();
      if (warp == 0) {  // exclusive scan of the counts: lane l sums a contiguous run
        const int per = (NB + 31) / 32, lo = lane * per, hi = min(NB, lo + per);
        int sum = 0;
        for (int c = lo; c < hi; ++c) sum += cnt[c];
        int incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += y;
        }
        int run = incl - sum;
        for (int c = lo; c < hi; ++c) {
          const int x = cnt[c];
          cnt[c] = run;
          off[c] = run;
          run += x;
        }
        if (lane == 31) off[NB] = incl;
      }
      __syncthreads();
      for (int kb = tid; kb < NB; kb += blockDim.x) {
        int pos = cnt[kb];
        for (int w = 0; w < W; ++w) {
          uint32_t b = bits[kb * W + w];
          while (b) {
            list[pos++] = w * 32 + __ffs(b) - 1;
            b &= b - 1u;
          }
        }
      }
      return;
    }
    __syncthreads();  // the bitmap is given up; the shared memory is reused below
  }

  // one query block at a time (repeated ids, or grids beyond the bitmap)
  int* cnt = kq_sm;        // [NB]
  int* cur = kq_sm + NB;   // [NB]
  for (int c = tid; c < NB; c += blockDim.x) {
    cnt[c] = 0;
    cur[c] = 0;
  }
  __syncthreads();
  for (long long e = tid; e < static_cast<long long>(NB) * max_k; e += blockDim.x) {
    const int r = static_cast<int>(e / max_k), t = static_cast<int>(e - static_cast<long long>(r) * max_k);
    int c = nh[r];
    if (c < 0 || c > max_k) {
      bad = true;
      c = c < 0 ? 0 : max_k;
    }
    if (t >= c) continue;
    const int kb = ih[e];
    if (kb < 0 || kb >= NB) {
      bad = true;
      continue;
    }
    atomicAdd(&cnt[kb], 1);
  }
  if (bad) atomicCAS(status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int c = 0; c < NB; ++c) {
      const int x = cnt[c];
      cnt[c] = run;
      off[c] = run;
      run += x;
    }
    off[NB] = run;
  }
  __syncthreads();
  for (int r = 0; r < NB; ++r) {
    int c = nh[r];
    c = c < 0 ? 0 : (c > max_k ? max_k : c);
    for (int t = tid; t < c; t += blockDim.x) {
      const int kb = ih[static_cast<long long>(r) * max_k + t];
      if (kb < 0 || kb >= NB) continue;
      list[cnt[kb] + atomicAdd(&cur[kb], 1)] = r;
    }
    __syncthreads();
  }
}

}  // namespace

size_t attn_bwd_workspace_bytes(const Geo& g, int BH, int max_k) {
  const size_t rows = static_cast<size_t>(BH) * g.Sp;
  size_t b = 2 * rows * sizeof(float);                                   // lse2, delta
  b += static_cast<size_t>(BH) * (g.NB + 1) * sizeof(int32_t);           // k2q offsets
  b = (b + 15) & ~size_t(15);
  b += static_cast<size_t>(BH) * g.NB * max_k * sizeof(int32_t);        // k2q lists
  return b;
}

template <int BS, bool F16>
cudaError_t launch_bwd_kernels(const Geo& g, const AttnBwdArgs& a, const BwdParams& p, cudaStream_t stream) {
  const unsigned long long rows = static_cast<unsigned long long>(a.BH) * g.Sp;
  CUtensorMap tq, tk, tv, tdo, tks, tvs, tq64, tdo64;
  if (!make_tmap(&tq, a.q, rows, 128, F16) || !make_tmap(&tk, a.k, rows, 128, F16) ||
      !make_tmap(&tv, a.v, rows, 128, F16) || !make_tmap(&tdo, a.dO, rows, 128, F16))
    return cudaErrorInvalidValue;
  if (!make_tmap(&tq64, a.q, rows, 64, F16) || !make_tmap(&tdo64, a.dO, rows, 64, F16))
    return cudaErrorInvalidValue;
  if (BS == 256) {
    tks = tk;
    tvs = tv;
  } else if (!make_tmap(&tks, a.k, rows, 64, F16) || !make_tmap(&tvs, a.v, rows, 64, F16)) {
    return cudaErrorInvalidValue;
  }
  const unsigned items = static_cast<unsigned>((BS == 256 ? 2ull : 1ull) * a.BH * g.NB);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<BS, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kKV_Smem)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_bwd_dq_kernel<BS, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kQ_Smem)) != cudaSuccess)
    return e;
  attn_bwd_dkdv_kernel<BS, F16><<<items, kThreads, kKV_Smem, stream>>>(tq64, tk, tv, tdo64, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  attn_bwd_dq_kernel<BS, F16><<<items, kThreads, kQ_Smem, stream>>>(tq, tks, tvs, tdo, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const Geo& g, const AttnBwdArgs& a, cudaStream_t stream) {
  if (g.bs != 256 && g.bs != 64) return cudaErrorNotSupported;
  const unsigned long long rows = static_cast<unsigned long long>(a.BH) * g.Sp;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* lse2 = reinterpret_cast<float*>(ws);
  float* delta = lse2 + rows;
  int32_t* k2q_off = reinterpret_cast<int32_t*>(delta + rows);
  size_t off_bytes = 2 * rows * sizeof(float) + static_cast<size_t>(a.BH) * (g.NB + 1) * sizeof(int32_t);
  off_bytes = (off_bytes + 15) & ~size_t(15);
  int32_t* k2q = reinterpret_cast<int32_t*>(ws + off_bytes);

  const unsigned prep_blocks = static_cast<unsigned>((rows + 15) / 16);
  if (a.f16)
    bwd_prep_kernel<true><<<prep_blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(a.o),
                                                           reinterpret_cast<const uint4*>(a.dO), a.lse, lse2, delta,
                                                           static_cast<long long>(rows));
  else
    bwd_prep_kernel<false><<<prep_blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(a.o),
                                                            reinterpret_cast<const uint4*>(a.dO), a.lse, lse2, delta,
                                                            static_cast<long long>(rows));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the bitmap and counts (or, beyond the bitmap, two int32 per key block:
  // counts, then write positions); above the default 48 KB the kernel opts in
  // (the API caps NB at kBwdMaxBlocks)
  const size_t k2q_smem = k2q_smem_bytes(g.NB);
  if (k2q_smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(k2q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(k2q_smem))) != cudaSuccess)
    return e;
  k2q_kernel<<<a.BH, 256, k2q_smem, stream>>>(a.idx, a.num, g.NB, a.max_k, k2q_off, k2q, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  BwdParams p;
  p.g = g;
  p.BH = a.BH;
  p.max_k = a.max_k;
  p.idx = a.idx;
  p.num = a.num;
  p.k2q_off = k2q_off;
  p.k2q = k2q;
  p.nlse2 = lse2;
  p.ndelta = delta;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.status = a.status;
  p.scale = static_cast<float>(1.0 / 11.313708498984761);            // 128^-1/2
  p.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);
  if (g.bs == 256)
    return a.f16 ? launch_bwd_kernels<256, true>(g, a, p, stream) : launch_bwd_kernels<256, false>(g, a, p, stream);
  return a.f16 ? launch_bwd_kernels<64, true>(g, a, p, stream) : launch_bwd_kernels<64, false>(g, a, p, stream);
}

}  // namespace vsa
