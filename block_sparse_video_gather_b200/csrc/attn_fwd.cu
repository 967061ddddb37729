// attn_fwd.cu -- fine stage of VSA: block-sparse flash attention forward on
// the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA loads).
//
// "FastVideo VSA" (vLLM-Omni user guide), introduction and section "Verify
// routing and fallback": each query block attends only to the tokens of its
// selected key/value blocks; non-causal; scale head_size^-1/2.  FastVideo
// commit log (examples/inference/basic/README.md): rows carry different
// counts, including zero.
//
// Work item: one (b*h, query block) of 256 tokens = two 128-row Q tiles.
// Each selected key block is two 128-key tiles.  Persistent CTAs, one per SM,
// take items in head-major order so the K/V of a head stay hot in L2.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q (64 KB per item), K and V tiles (32 KB each)
//               into a 3-stage K ring and a 2-stage V ring (224 KB of shared
//               memory in all), completion counted on mbarriers.
//   warp 1      TMEM owner (512 columns) and single-thread MMA issuer.
//   warps 4-7   softmax + epilogue of Q tile 0 (one thread per query row)
//   warps 8-11  softmax + epilogue of Q tile 1
//
// Tensor memory (128 lanes x 512 fp32 columns):
//   [  0,128) S0 = Q0 K^T   (P0 = bf16 softmax numerators, aliased on [0,64))
//   [128,256) S1 = Q1 K^T   (P1 on [128,192))
//   [256,384) O0            [384,512) O1
// Per KV tile the MMA thread issues, in order:
//   PV0(t)  S0(t+1)  PV1(t)  S1(t+1)
// so softmax of tile 0 overlaps the tensor-core work of tile 1 and back.
// S MMAs: A = Q (K-major, smem), B = K tile (K-major, smem).
// PV MMAs: A = P (TMEM), B = V tile (MN-major, smem); O accumulates in TMEM.
//
// Online softmax in the log2 domain with a lazy maximum: the running max used
// for the exponentials only moves when a row's new tile max exceeds it by more
// than 8 (a factor 256), and only then is that row of O rescaled in TMEM.
// Numerators stay <= 256, safe in bf16 and fp32; o = O / l and
// lse = (m + log2 l) ln 2 use the same maximum, so the result is exact.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// VSA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "fwd_common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace vsa {

namespace {

using namespace tiles;
using namespace fwd;

template <int BS, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sK = smem + kSmemK;
  uint8_t* sV = smem + kSmemV;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + kSmemBar);

  constexpr int kQTiles = BS == 256 ? 2 : 1;  // 128-row query tiles per item
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geo& g = p.g;
  const int total_items = p.BH * g.NB;

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
    {
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
        mbar_arrive_expect_tx_w(&bars->q_full, kQTiles * kTileBytes);
        const int qrow = static_cast<int>(base + static_cast<long long>(qb) * BS);
        for (int i = 0; i < kQTiles; ++i)
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d_w(sQ + i * kTileBytes + hf * kHalfBytes, &tm_q, hf * 64, qrow + i * 128, &bars->q_full, pol_q);
        ++qit;
        bool stop = false;
        const int n = item_tiles<BS>(nb);
        for (int t = 0; t < n && !stop; ++t) {
          // Key rows of this tile: one 128-row box (256-token blocks) or two
          // 64-row boxes (64-token blocks).  Unusable or absent blocks load
          // block 0 -- finite data, masked out by the softmax -- so that no
          // stale shared memory can reach the PV product.
          int krow0, krow1 = 0;
          if (BS == 256) {
            const int kb0 = item_block_id(p, item, t >> 1);
            const int kb = kb0 < 0 ? 0 : kb0;
            krow0 = static_cast<int>(base + static_cast<long long>(kb) * 256 + (t & 1) * 128);
          } else {
            const int ka = item_block_id(p, item, 2 * t);
            const int kb = 2 * t + 1 < nb ? item_block_id(p, item, 2 * t + 1) : -1;
            krow0 = static_cast<int>(base + static_cast<long long>(ka < 0 ? 0 : ka) * 64);
            krow1 = static_cast<int>(base + static_cast<long long>(kb < 0 ? 0 : kb) * 64);
          }
          const int sk = kit % kStagesK;
          if (!warp_wait(&bars->k_empty[sk], ((kit / kStagesK) & 1) ^ 1, bars, p.status)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx_w(&bars->k_full[sk], kTileBytes);
          for (int hf = 0; hf < 2; ++hf) {
            uint8_t* dst = sK + sk * kTileBytes + hf * kHalfBytes;
            tma_load_2d_w(dst, &tm_k, hf * 64, krow0, &bars->k_full[sk], pol_kv);
            if (BS == 64) tma_load_2d_w(dst + kHalfBytes / 2, &tm_k, hf * 64, krow1, &bars->k_full[sk], pol_kv);
          }
          ++kit;
          const int sv = vit % kStagesV;
          if (!warp_wait(&bars->v_empty[sv], ((vit / kStagesV) & 1) ^ 1, bars, p.status)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx_w(&bars->v_full[sv], kTileBytes);
          for (int hf = 0; hf < 2; ++hf) {
            uint8_t* dst = sV + sv * kTileBytes + hf * kHalfBytes;
            tma_load_2d_w(dst, &tm_v, hf * 64, krow0, &bars->v_full[sv], pol_kv);
            if (BS == 64) tma_load_2d_w(dst + kHalfBytes / 2, &tm_v, hf * 64, krow1, &bars->v_full[sv], pol_kv);
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
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    {
      // Descriptors are built once; each MMA only adds a constant to the
      // start-address field (smem addresses stay below 2^18, so the 14-bit
      // field never carries).  A lean issue loop keeps the tensor core fed:
      // rebuilding descriptors per instruction made this thread the bottleneck.
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kHalfBytes, 1024);
      constexpr uint64_t kTileDesc = kTileBytes >> 4;
      int kit = 0, vit = 0, qit = 0, tiles = 0, items = 0;
      bool ok = true;
      auto issue_s = [&](int i, int sk) {
        const uint32_t d = tmem + i * 128;
        const uint64_t a = dq0 + i * kTileDesc, b = dk0 + sk * kTileDesc;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss_w(d, a + off, b + off, Idesc<F16>::S, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int sv, bool acc) {
        const uint32_t d = tmem + 256 + i * 128, pa = tmem + i * 128;
        const uint64_t b = dv0 + sv * kTileDesc;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ts_w(d, pa + kk * 8, b + kk * (2048 >> 4), Idesc<F16>::PV, (acc || kk > 0) ? 1u : 0u);
      };
      for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        const int nb = item_blocks(p, item, lane == 0);
        if (nb == 0) continue;
        const int n = item_tiles<BS>(nb);
        if (!(ok = warp_wait(&bars->q_full, qit & 1, bars, p.status))) break;
        ++qit;
        tc_fence_after();
        int sk = kit % kStagesK;
        if (!(ok = warp_wait(&bars->k_full[sk], (kit / kStagesK) & 1, bars, p.status))) break;
        tc_fence_after();
        issue_s(0, sk);
        mma_commit_w(&bars->s_full[0]);
        if (kQTiles == 2) {
          issue_s(1, sk);
          mma_commit_w(&bars->s_full[1]);
        }
        mma_commit_w(&bars->k_empty[sk]);
        ++kit;
        for (int t = 0; t < n; ++t) {
          const int sv = vit % kStagesV;
          if (!(ok = warp_wait(&bars->v_full[sv], (vit / kStagesV) & 1, bars, p.status))) break;
          if (!(ok = warp_wait(&bars->p_full[0], tiles & 1, bars, p.status))) break;
          if (t == 0 && !(ok = warp_wait(&bars->o_empty[0], (items & 1) ^ 1, bars, p.status)))
            break;
          tc_fence_after();
          issue_pv(0, sv, t > 0);
          if (t == n - 1) mma_commit_w(&bars->o_full[0]);
          const bool more = t + 1 < n;
          sk = kit % kStagesK;
          if (more) {
            if (!(ok = warp_wait(&bars->k_full[sk], (kit / kStagesK) & 1, bars, p.status))) break;
            tc_fence_after();
            issue_s(0, sk);
            mma_commit_w(&bars->s_full[0]);
          }
          if (kQTiles == 2) {
            if (!(ok = warp_wait(&bars->p_full[1], tiles & 1, bars, p.status))) break;
            if (t == 0 && !(ok = warp_wait(&bars->o_empty[1], (items & 1) ^ 1, bars, p.status)))
              break;
            tc_fence_after();
            issue_pv(1, sv, t > 0);
          }
          mma_commit_w(&bars->v_empty[sv]);
          ++vit;
          if (kQTiles == 2 && t == n - 1) mma_commit_w(&bars->o_full[1]);
          if (more) {
            if (kQTiles == 2) {
              issue_s(1, sk);
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
      // Drain: wait for every MMA issued by this thread before TMEM and smem go away.
      mma_commit_w(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kTimeoutNs);
    }
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
    const uint32_t tS = tmem + lane_off + wg * 128;
    const uint32_t tO = tmem + lane_off + 256 + wg * 128;
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
        int kb_a, kb_b = -1;
        if (BS == 256) {
          kb_a = item_block_id(p, item, t >> 1);
        } else {
          kb_a = item_block_id(p, item, 2 * t);
          if (2 * t + 1 < nb) {
            kb_b = item_block_id(p, item, 2 * t + 1);
            if (kb_b < 0 && r == 0) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
          }
        }
        if (kb_a < 0 && wg == 0 && r == 0) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
        uint32_t mw[4];
        const int mstate = item_tile_mask<BS>(g, kb_a, kb_b, t, mw);
        if (!(ok = warp_wait(&bars->s_full[wg], tiles & 1, bars, p.status))) break;
        tc_fence_after();
        uint32_t pk[64];
        float lsum = 0.0f, alpha = 1.0f;
        bool rescale = false;
        if (mstate == kTileEmpty) {
          // no real key: the numerators are all zero and the maximum does not move
#pragma unroll
          for (int j = 0; j < 64; ++j) pk[j] = 0u;
        } else {
          uint32_t sv[128];
          tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
          tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
          tmem_wait_ld();
          if (mstate == kTilePartial) apply_key_mask(sv, mw);
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
            uint64_t pp;
            {
              float xa, xb;
              f2unpack(x, xa, xb);
              pp = f2pack(ex2_approx(xa), ex2_approx(xb));
            }
            {
              float p0, p1;
              f2unpack(pp, p0, p1);
              pk[j] = pack_half2<F16>(p0, p1);
            }
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
        // Rescale this row of O when its maximum moved (warp-uniform branch;
        // rows that did not move use alpha = 1).  PV(t-1) is complete: the
        // s_full commit just waited on follows it in issue order.
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
      // epilogue: O / l -> bf16 row, lse
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

}  // namespace

cudaError_t launch_attn_fwd(const Geo& g, const AttnArgs& a, cudaStream_t stream) {
  if (g.bs != 256 && g.bs != 64) return cudaErrorNotSupported;
  const unsigned long long rows = static_cast<unsigned long long>(a.BH) * g.Sp;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;
  const unsigned kv_box = g.bs == 256 ? 128 : 64;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, a.q, rows, 128, a.f16) || !make_tmap(&tk, a.k, rows, kv_box, a.f16) ||
      !make_tmap(&tv, a.v, rows, kv_box, a.f16))
    return cudaErrorInvalidValue;
  Params p;
  p.idx = a.idx;
  p.num = a.num;
  p.max_k = a.max_k;
  p.BH = a.BH;
  p.o = a.o;
  p.lse = a.lse;
  p.status = a.status;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  p.g = g;
  p.queue = a.queue;
  if (g.bs == 64 && g.NB <= kGroupMaxNB)  // groups of four query blocks over their union
    return launch_attn_fwd_grouped64(g, tq, tk, tv, p, a.BH, a.num_sms, a.f16, stream);
  const long long items = static_cast<long long>(a.BH) * g.NB;
  const int grid = static_cast<int>(items < a.num_sms ? items : a.num_sms);
  auto kern = g.bs == 256 ? (a.f16 ? attn_fwd_kernel<256, true> : attn_fwd_kernel<256, false>)
                          : (a.f16 ? attn_fwd_kernel<64, true> : attn_fwd_kernel<64, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemTotal, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace vsa
