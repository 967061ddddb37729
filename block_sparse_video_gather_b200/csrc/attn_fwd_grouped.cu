// attn_fwd_grouped.cu -- fine stage of VSA for 64-token blocks (the tile-64
// layout of the FastVideo commit log, examples/inference/basic/README.md:
// rows of any length, zero included), with four query blocks per work item,
// two per 128-row Q tile, each Q tile over the union of its two selections;
// Q and K 16-bit, or NVFP4 (FastVideo "Optimizations" page, section "FP4
// Flash Attention 4": E2M1 codes with E4M3 scales, V and P 16-bit).
// "FastVideo VSA" (vLLM-Omni user guide), introduction: each query block
// attends only to the tokens of its selected blocks; non-causal; scale
// head_size^-1/2.
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
using namespace fwd;

// ===========================================================================
// 64-token blocks, grouped.
//
// A 64-row query block fills only half of an M = 128 product, and one block
// per item leaves the second softmax warpgroup idle.  Here a work item is a
// group of four consecutive query blocks of one head -- two 128-row Q tiles
// (query blocks 0-1 and 2-3), one per softmax warpgroup, the 256-token
// kernel's schedule.  Each Q tile walks its own key stream, two 64-key blocks
// per 128-key tile: first the blocks both Q tiles selected (ascending), then
// the blocks only it selected (ascending).  Step t of the group carries tile
// t of each Q tile that still has one; for t < ns (the shared blocks paired
// among themselves) the two tiles are the same and are loaded once, later
// steps load one tile per Q tile.  Each softmax warp serves one query block
// (warps 0-1 of a warpgroup the first, 2-3 the second) and looks up, per key
// tile, whether its block selected each half: unselected halves are masked,
// and a warp whose block selected neither half skips the exponentials (P =
// 0).  Against one stream over the union of all four selections this cuts
// the products of a group by the blocks only the other Q tile selected.
//
// A fourth role builds the groups: warp 2 reads the four index rows, sets one
// bit per (query block, selected block) in shared-memory bitmaps (double
// buffered, two groups ahead), forms the bitmap of the blocks both Q tiles
// selected, counts each Q tile's tiles and hands the group over on grp_full;
// the eleven consuming warps (the K and V producers, MMA, eight softmax
// warps) release it on grp_free.  Block ids outside [0, NB) are skipped and
// counts outside [0, max_k] clamped (both reported); a list that names a
// block twice puts the whole group in list order instead ("concat": each
// query block's list, two ids per tile, only that block's rows unmasked, the
// same stream for both Q tiles), so a repeated id counts twice as in the
// ungrouped kernel.
//
// Groups go to CTAs statically (every gridDim.x-th group) or, with a caller
// workspace, through a shared queue: the builder takes tickets with an atomic
// add, the groups holding prefix query tiles first (dense under the tile-64
// rule, the longest), and publishes an end marker past the last group; the
// last CTA to finish resets the counters.  Either way the consumers stop on
// the end marker.
//
// The bitmaps hold kGroupMaxNB blocks: the host uses this kernel for
// 64-token blocks when NB <= kGroupMaxNB.
// ===========================================================================
constexpr int kGroupBlocks = 4;
constexpr int kGroupMaxWords = 32;
static_assert(kGroupMaxNB == 32 * kGroupMaxWords, "bitmap capacity");

// Shared-memory map of the two variants.  16-bit Q and K: the five 32 KB tile
// stages after Q; a step that loads one tile per Q tile takes two K and two V
// stages, and a V stage is held a softmax longer than a K stage (S issues
// right after its load, P V only after the softmax), so the V ring gets the
// deeper share.  NVFP4 Q and K: a Q tile is 8 KB of codes + a 1 KB scale
// tile, a key tile 8 KB of codes + a 1 KB scale tile assembled from its two
// blocks' halves, so both rings get four stages.
template <bool FP4>
struct GMap;
template <>
struct GMap<false> {
  static constexpr int kKS = 2, kVS = 3;
  static constexpr uint32_t kQ = 0, kQsf = 0, kK = kQ + 2 * kTileBytes, kKsf = 0;
  static constexpr uint32_t kKStage = kTileBytes, kKsfStage = 0;
  static constexpr uint32_t kV = kK + kKS * kKStage;
  static constexpr uint32_t kBar = kV + kVS * kTileBytes;
};
template <>
struct GMap<true> {
  static constexpr int kKS = 4, kVS = 4;
  static constexpr uint32_t kQTile = nvfp4::kCodeTileBytes;
  static constexpr uint32_t kQ = 0, kQsf = kQ + 2 * kQTile, kK = kQsf + 2 * nvfp4::kSfTileBytes;
  static constexpr uint32_t kKStage = nvfp4::kCodeTileBytes, kKsfStage = nvfp4::kSfTileBytes;
  static constexpr uint32_t kKsf = kK + kKS * kKStage;
  static constexpr uint32_t kV = kKsf + kKS * kKsfStage;
  static constexpr uint32_t kBar = kV + kVS * kTileBytes;
};
static_assert(GMap<false>::kBar == kSmemBar, "16-bit map: the per-block kernel's");
static_assert(GMap<true>::kK % 1024 == 0 && GMap<true>::kV % 1024 == 0, "1 KB-aligned rings");
constexpr int kMaxStages = 4;

constexpr int kShared = kGroupBlocks;  // bitmap of the blocks both Q tiles use

struct GroupInfo {
  int concat;  // 1: walk each list as given (a list repeats an id)
  int ns;      // leading steps whose tile is the same for both Q tiles
  int len[2];  // 128-key tiles of each Q tile's key stream (0 for an absent Q tile)
  int nq;      // 128-row query tiles (1 for a group of two query blocks)
  int cnt[kGroupBlocks];
  int gi;      // the group (b*h * groups per head + query block / 4), -1: no more groups
  // selection bitmaps of the four query blocks; [kShared]: blocks selected
  // by a query block of each Q tile
  uint32_t bm[kGroupBlocks + 1][kGroupMaxWords];
};

struct GroupBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t s_read[2];  // NVFP4: S_i loaded by its softmax (its last 64 columns free for scales)
  uint64_t grp_full[2], grp_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t kBarBytes = 512;
static_assert(sizeof(GroupBarriers) <= kBarBytes, "barrier block too large");

template <bool FP4>
struct GSmem {
  static constexpr uint32_t kGroups = GMap<FP4>::kBar + kBarBytes;
  static constexpr uint32_t kTotal = kGroups + 2 * sizeof(GroupInfo) + 1024;
  static_assert(kTotal <= 232448, "grouped kernel exceeds the shared memory of one CTA");
};

// Launch parameters: the 16-bit kernel's, plus the NVFP4 scale tiles.
struct GroupParams : Params {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
};
constexpr uint32_t kGroupConsumers = 11;  // two producers, MMA, 8 softmax warps: one arrival each

__device__ __forceinline__ bool gwarp_wait(uint64_t* bar, uint32_t parity, GroupBarriers* bars,
                                           unsigned int* status) {
  bool ok = mbar_wait(bar, parity, &bars->abort, status, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

// Group of ticket d of a shared queue: the groups holding prefix query tiles
// (dense under the tile-64 rule, the longest) of every head first, then the
// others head by head -- the longest work is handed out first.
__device__ __forceinline__ int queue_group(const Geo& g, int BH, int ngq, int d) {
  const int npq = min(ngq, (g.n_pre + kGroupBlocks - 1) / kGroupBlocks);
  if (d < BH * npq) return (d / npq) * ngq + d % npq;
  const int e = d - BH * npq, nv = ngq - npq;
  return (e / nv) * ngq + npq + e % nv;
}

// Block id at position t of index row `row`, or -1 when outside [0, NB).
__device__ __forceinline__ int row_block_id(const Params& p, int row, int t) {
  const int kb = __ldg(p.idx + static_cast<long long>(row) * p.max_k + t);
  return (kb >= 0 && kb < p.g.NB) ? kb : -1;
}

// The key stream of Q tile qt of a group: 128-key tile after 128-key tile,
// the two block ids (-1: absent or unusable) and the query blocks that use
// each.  Union: the shared blocks ascending, then the blocks only Q tile qt
// selected ascending.  Concat: the four lists as given, the same stream for
// both Q tiles.
struct GroupWalk {
  int a;       // union: word a of the shared bitmap, then (a >= W) word a - W of Q tile qt's own
  uint32_t b;  // union: bits of that word still to visit; concat: next pair of list a
  __device__ __forceinline__ void init(const GroupInfo& gb) {
    a = 0;
    b = gb.concat ? 0u : gb.bm[kShared][0];
  }
  __device__ __forceinline__ int pop_union(const GroupInfo& gb, int W, int qt) {
    while (b == 0u) {
      if (++a >= 2 * W) return -1;
      const int w = a - W;
      b = w < 0 ? gb.bm[kShared][a] : (gb.bm[2 * qt][w] | gb.bm[2 * qt + 1][w]) & ~gb.bm[kShared][w];
    }
    const int bit = __ffs(b) - 1;
    b &= b - 1u;
    return (a < W ? a : a - W) * 32 + bit;
  }
  // Next tile: ids ka, kb, and the one query block that uses them in list
  // order (owner), or -1 for the union, where each query block's bitmap says.
  __device__ __forceinline__ void next(const GroupInfo& gb, const Params& p, int row0, int W, int qt, int& ka,
                                       int& kb, int& owner) {
    if (!gb.concat) {
      ka = pop_union(gb, W, qt);
      kb = pop_union(gb, W, qt);
      owner = -1;
      return;
    }
    while (a < kGroupBlocks && 2 * static_cast<int>(b) >= gb.cnt[a]) {
      ++a;
      b = 0u;
    }
    if (a >= kGroupBlocks) {  // past the last list (not reached: len counts the pairs)
      ka = kb = owner = -1;
      return;
    }
    const int t = 2 * static_cast<int>(b);
    ka = row_block_id(p, row0 + a, t);
    kb = t + 1 < gb.cnt[a] ? row_block_id(p, row0 + a, t + 1) : -1;
    owner = a;
    ++b;
  }
};

// Whether query block j of the group uses block kb of a tile (kb < 0: no).
__device__ __forceinline__ bool group_uses(const GroupInfo& gb, int owner, int j, int kb) {
  if (kb < 0) return false;
  if (owner >= 0) return owner == j;
  return (gb.bm[j][kb >> 5] >> (kb & 31)) & 1u;
}

// Softmax of one 128-column S row whose halves (two 64-key blocks) may be
// unselected (ha / hb false: those columns are ignored); log2 domain with the
// lazy maximum of the kernel above.  Writes the 16-bit numerators into pk
// (zero for an unselected half, whose maximum and exponentials are skipped)
// and returns their sum.  One body for every case keeps the loop's code small.
template <bool F16>
__device__ __forceinline__ float softmax_halves(uint32_t (&sv)[128], bool ha, bool hb, float sl2, int t,
                                                float& m_used, float& alpha, bool& rescale, uint32_t (&pk)[64]) {
  float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 0 ? ha : hb) {
#pragma unroll
      for (int c = 64 * h; c < 64 * h + 64; c += 8) {
        a0 = max3f(a0, __uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1]));
        a1 = max3f(a1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
        a2 = max3f(a2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
        a3 = max3f(a3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
      }
    }
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
  for (int h = 0; h < 2; ++h) {
    if (h == 0 ? ha : hb) {
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int j = 32 * h + jj;
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
        switch (jj & 3) {
          case 0: acc0 = add2(acc0, pp); break;
          case 1: acc1 = add2(acc1, pp); break;
          case 2: acc2 = add2(acc2, pp); break;
          default: acc3 = add2(acc3, pp); break;
        }
      }
    } else {
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) pk[32 * h + jj] = 0u;
    }
  }
  float s0, s1, s2, s3, s4, s5, s6, s7;
  f2unpack(acc0, s0, s1);
  f2unpack(acc1, s2, s3);
  f2unpack(acc2, s4, s5);
  f2unpack(acc3, s6, s7);
  return ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
}

// FP4: Q and K as NVFP4 codes with E4M3 scale tiles (tm_q: 128-row boxes of
// 64-byte code rows; tm_k: 64-row boxes), S = Q K^T a block-scaled FP4
// product per 64-token block of the key tile (N = 64), its scales copied into
// the other Q tile's free S columns once that tile's softmax has loaded its
// latest S (s_read); V, P and O as in the 16-bit variant.
template <bool F16, bool FP4>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_grouped64_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ GroupParams p) {
  using M = GMap<FP4>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + M::kQ;
  uint8_t* sQsf = smem + M::kQsf;
  uint8_t* sK = smem + M::kK;
  uint8_t* sKsf = smem + M::kKsf;
  uint8_t* sV = smem + M::kV;
  GroupBarriers* bars = reinterpret_cast<GroupBarriers*>(smem + M::kBar);
  GroupInfo* grp = reinterpret_cast<GroupInfo*>(smem + GSmem<FP4>::kGroups);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geo& g = p.g;
  const int ngq = (g.NB + kGroupBlocks - 1) / kGroupBlocks;  // groups per head
  const int total_groups = p.BH * ngq;
  const int W = (g.NB + 31) >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < M::kKS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < M::kVS; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_read[i], 128);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 128);
      mbar_init(&bars->grp_full[i], 1);
      mbar_init(&bars->grp_free[i], kGroupConsumers);
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
  if (warp == 2) {
    // ------------------------------------------------------------ group builder
    for (int gl = 0;; ++gl) {
      // the next group: a ticket of the shared queue, or every gridDim.x-th group
      int gi;
      if (p.queue) {
        int tk = 0;
        if (lane == 0) tk = atomicAdd(p.queue, 1);
        tk = __shfl_sync(0xffffffffu, tk, 0);
        gi = tk < total_groups ? queue_group(g, p.BH, ngq, tk) : -1;
      } else {
        gi = blockIdx.x + gl * static_cast<int>(gridDim.x);
        if (gi >= total_groups) gi = -1;
      }
      const int buf = gl & 1;
      if (gl >= 2 && !gwarp_wait(&bars->grp_free[buf], ((gl >> 1) - 1) & 1, bars, p.status)) break;
      GroupInfo& gb = grp[buf];
      if (gi < 0) {  // past the last group: an end marker for the consumers
        if (lane == 0) gb.gi = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->grp_full[buf]);
        break;
      }
      for (int i = lane; i < (kGroupBlocks + 1) * kGroupMaxWords; i += 32) (&gb.bm[0][0])[i] = 0u;
      __syncwarp();
      const int bh = gi / ngq, qb0 = (gi - bh * ngq) * kGroupBlocks;
      const int nqb = min(kGroupBlocks, g.NB - qb0);
      bool repeat = false, bad = false;
      int cnts[kGroupBlocks];
#pragma unroll
      for (int j = 0; j < kGroupBlocks; ++j) {
        int c = 0;
        if (j < nqb) {
          const long long row = static_cast<long long>(bh) * g.NB + qb0 + j;
          c = __ldg(p.num + row);
          if (c < 0 || c > p.max_k) {
            bad = true;
            c = c < 0 ? 0 : p.max_k;
          }
          for (int t = lane; t < c; t += 32) {
            const int kb = __ldg(p.idx + row * p.max_k + t);
            if (kb < 0 || kb >= g.NB) {
              bad = true;
              continue;
            }
            const uint32_t bit = 1u << (kb & 31);
            if (atomicOr(&gb.bm[j][kb >> 5], bit) & bit) repeat = true;
          }
        }
        cnts[j] = c;
      }
      __syncwarp();
      repeat = __any_sync(0xffffffffu, repeat);
      bad = __any_sync(0xffffffffu, bad);
      if (bad && lane == 0) atomicCAS(p.status, 0u, (unsigned)VSA_ERR_BAD_INDEX);
      // blocks of both Q tiles, of Q tile 0 only, of Q tile 1 only (a group
      // of two query blocks has no Q tile 1: all its blocks are Q tile 0's)
      int cs = 0, c0 = 0, c1 = 0;
      for (int w = lane; w < W; w += 32) {
        const uint32_t u0 = gb.bm[0][w] | gb.bm[1][w], u1 = gb.bm[2][w] | gb.bm[3][w], sh = u0 & u1;
        gb.bm[kShared][w] = sh;
        cs += __popc(sh);
        c0 += __popc(u0 & ~sh);
        c1 += __popc(u1 & ~sh);
      }
      cs = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cs)));
      c0 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c0)));
      c1 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c1)));
      if (lane == 0) {
        const int nq = (nqb + 1) / 2;
        if (repeat) {  // one stream, the lists as given, for every Q tile
          int n = 0;
#pragma unroll
          for (int j = 0; j < kGroupBlocks; ++j) n += (cnts[j] + 1) / 2;
          gb.ns = nq == 2 ? n : 0;
          gb.len[0] = n;
          gb.len[1] = nq == 2 ? n : 0;
        } else {
          gb.ns = cs / 2;
          gb.len[0] = (cs + c0 + 1) / 2;
          gb.len[1] = (cs + c1 + 1) / 2;
        }
        gb.gi = gi;
        gb.concat = repeat ? 1 : 0;
        gb.nq = nq;
#pragma unroll
        for (int j = 0; j < kGroupBlocks; ++j) gb.cnt[j] = cnts[j];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->grp_full[buf]);
    }
  } else if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    // Warp 0 loads Q and the K tiles, warp 3 the V tiles: each waits only on
    // its own ring, so a K load never queues behind a V stage that is still
    // read (a step may take two stages of each).
    const bool vside = warp == 3;
    tma_prefetch_desc(vside ? &tm_v : &tm_k);
    if (!vside) tma_prefetch_desc(&tm_q);
    const uint64_t pol_kv = policy_evict_last();
    const uint64_t pol_q = policy_evict_first();
    const int stages = vside ? M::kVS : M::kKS;
    const long long sf_tiles = g.Sp >> 7;  // NVFP4: 128-row scale tiles per head
    uint8_t* const ring = vside ? sV : sK;
    uint64_t* const full = vside ? bars->v_full : bars->k_full;
    uint64_t* const empty = vside ? bars->v_empty : bars->k_empty;
    const CUtensorMap* const tm = vside ? &tm_v : &tm_k;
    int it = 0, qit = 0;
    bool stop = false;
    for (int gl = 0; !stop; ++gl) {
      const int buf = gl & 1;
      if (!gwarp_wait(&bars->grp_full[buf], (gl >> 1) & 1, bars, p.status)) break;
      const GroupInfo& gb = grp[buf];
      const int gi = gb.gi;
      if (gi < 0) break;
      const int ns = gb.ns, len0 = gb.len[0], len1 = gb.len[1], nq = gb.nq;
      const int n = max(len0, len1);
      const int bh = gi / ngq, qb0 = (gi - bh * ngq) * kGroupBlocks;
      const long long base = static_cast<long long>(bh) * g.Sp;
      const int row0 = bh * g.NB + qb0;
      if (n > 0) {
        if (!vside) {
          if (!gwarp_wait(&bars->q_empty, (qit & 1) ^ 1, bars, p.status)) break;
          const int qrow = static_cast<int>(base + static_cast<long long>(qb0) * 64);
          if constexpr (FP4) {  // codes + the Q tile's scale tile (qb0 * 64 is 256-row aligned)
            mbar_arrive_expect_tx_w(&bars->q_full, nq * (M::kQTile + nvfp4::kSfTileBytes));
            for (int i = 0; i < nq; ++i) {
              tma_load_2d_w(sQ + i * M::kQTile, &tm_q, 0, qrow + i * 128, &bars->q_full, pol_q);
              const long long tile = bh * sf_tiles + ((qb0 * 64 + i * 128) >> 7);
              nvfp4::bulk_load_w(sQsf + i * nvfp4::kSfTileBytes, p.q_sf + tile * nvfp4::kSfTileBytes,
                                 nvfp4::kSfTileBytes, &bars->q_full);
            }
          } else {
            mbar_arrive_expect_tx_w(&bars->q_full, nq * kTileBytes);
            for (int i = 0; i < nq; ++i)
              for (int hf = 0; hf < 2; ++hf)
                tma_load_2d_w(sQ + i * kTileBytes + hf * kHalfBytes, &tm_q, hf * 64, qrow + i * 128, &bars->q_full,
                              pol_q);
          }
          ++qit;
        }
        // one stage per distinct tile of a step, Q tile 0's first
        auto load = [&](int krow0, int krow1) -> bool {
          const int st = it % stages;
          if (!gwarp_wait(&empty[st], ((it / stages) & 1) ^ 1, bars, p.status)) return false;
          if (FP4 && !vside) {
            // K codes: a 64-row box per block, stacked into one 128-row tile.
            // Scales: a 64-token block is one half of its scale tile, so the
            // two blocks' halves are assembled into one 128-row scale tile (block
            // a's rows 0-63, block b's 64-127): in each 16-byte row r%32 of each
            // channel half, block a's 8 bytes of columns 2 (kb & 1) .. +1, then
            // block b's.  Generic stores, made visible to the tensor core's copy
            // by a proxy fence before the stage is announced on k_full.
            const long long r0h = krow0 - base, r1h = krow1 - base;
            const uint8_t* ta = p.k_sf + (bh * sf_tiles + (r0h >> 7)) * nvfp4::kSfTileBytes + 8 * ((r0h >> 6) & 1);
            const uint8_t* tb = p.k_sf + (bh * sf_tiles + (r1h >> 7)) * nvfp4::kSfTileBytes + 8 * ((r1h >> 6) & 1);
            uint8_t* sfd = sKsf + st * M::kKsfStage;
#pragma unroll
            for (int e = lane; e < 128; e += 32) {  // 2 channel halves x 32 rows x 2 blocks of 8 bytes
              const int kh = e >> 6, rr = (e >> 1) & 31, blk = e & 1;
              const uint32_t off = kh * 512 + rr * 16;
              const uint2 v = __ldg(reinterpret_cast<const uint2*>((blk ? tb : ta) + off));
              *reinterpret_cast<uint2*>(sfd + off + 8 * blk) = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive_expect_tx_w(&full[st], M::kKStage);
            uint8_t* kdst = sK + st * M::kKStage;
            tma_load_2d_w(kdst, &tm_k, 0, krow0, &full[st], pol_kv);
            tma_load_2d_w(kdst + M::kKStage / 2, &tm_k, 0, krow1, &full[st], pol_kv);
          } else {
            mbar_arrive_expect_tx_w(&full[st], kTileBytes);
            for (int hf = 0; hf < 2; ++hf) {
              uint8_t* dst = ring + st * kTileBytes + hf * kHalfBytes;
              tma_load_2d_w(dst, tm, hf * 64, krow0, &full[st], pol_kv);
              tma_load_2d_w(dst + kHalfBytes / 2, tm, hf * 64, krow1, &full[st], pol_kv);
            }
          }
          ++it;
          return true;
        };
        GroupWalk walk[2];
        walk[0].init(gb);
        walk[1].init(gb);
        for (int t = 0; t < n && !stop; ++t) {
          // the rows of each Q tile's tile (absent or unusable blocks load block 0:
          // finite data, masked by every warp)
          int r0[2] = {0, 0}, r1[2] = {0, 0};
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (t >= gb.len[j]) continue;
            int ka, kb, owner;
            walk[j].next(gb, p, row0, W, j, ka, kb, owner);
            r0[j] = static_cast<int>(base + static_cast<long long>(ka < 0 ? 0 : ka) * 64);
            r1[j] = static_cast<int>(base + static_cast<long long>(kb < 0 ? 0 : kb) * 64);
          }
          const bool shared = t < ns;  // both Q tiles' tile t is the same: one stage
          const bool a0 = t < len0, a1 = t < len1 && !shared;
          if ((a0 && !load(r0[0], r1[0])) || (a1 && !load(r0[1], r1[1]))) stop = true;
        }
        if (stop) break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->grp_free[buf]);
    }
    // Drain: every issued copy must land before the CTA's shared memory is released.
    if (qit > 0) mbar_wait_drain(&bars->q_full, (qit - 1) & 1, kTimeoutNs);
    for (int st = 0; st < stages; ++st)
      if (it > st) {
        const int last = it - 1 - ((it - 1 - st) % stages);
        mbar_wait_drain(&full[st], (last / stages) & 1, kTimeoutNs);
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dq0 = FP4 ? nvfp4::sdesc_sw64(smem_u32(sQ)) : sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dk0 = FP4 ? nvfp4::sdesc_sw64(smem_u32(sK)) : sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kHalfBytes, 1024);
    constexpr uint64_t kTileDesc = kTileBytes >> 4;
    int kit = 0, vit = 0, qit = 0;
    int tiles0 = 0, tiles1 = 0, items0 = 0, items1 = 0;  // per Q tile: P V products, groups
    int sn0 = 0, sn1 = 0;                                // NVFP4: S products issued per Q tile
    bool ok = true;
    // S_i = Q_i K^T for the key tile in K stage sk
    auto issue_s = [&](int i, int sk) -> bool {
      const uint32_t d = tmem + i * 128;
      if constexpr (FP4) {
        // the scales go into the other Q tile's S columns: free once its softmax
        // has loaded its latest S
        const int j = 1 - i, nj = j == 0 ? sn0 : sn1;
        if (nj > 0 && !gwarp_wait(&bars->s_read[j], (nj - 1) & 1, bars, p.status)) return false;
        tc_fence_after();
        const uint32_t sf = tmem + nvfp4::sf_col(i);
        const uint8_t* qsf = sQsf + i * nvfp4::kSfTileBytes;
        const uint8_t* ksf = sKsf + sk * M::kKsfStage;
        nvfp4::tmem_cp_32x128_w(sf + 0, nvfp4::sdesc_rows16(smem_u32(qsf)));
        nvfp4::tmem_cp_32x128_w(sf + 4, nvfp4::sdesc_rows16(smem_u32(qsf + 512)));
        nvfp4::tmem_cp_32x128_w(sf + 8, nvfp4::sdesc_rows16(smem_u32(ksf)));
        nvfp4::tmem_cp_32x128_w(sf + 12, nvfp4::sdesc_rows16(smem_u32(ksf + 512)));
        // the Q tile and the key tile are each one whole scale tile: two N = 128
        // products (64 channels each)
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          const uint64_t a = dq0 + ((i * M::kQTile + kh * 32) >> 4);
          const uint64_t b = dk0 + ((sk * M::kKStage + kh * 32) >> 4);
          nvfp4::mma_fp4_w(d, a, b, nvfp4::idesc_s(128), sf + 4 * kh, sf + 8 + 4 * kh, kh > 0 ? 1u : 0u);
        }
        if (i == 0) ++sn0; else ++sn1;
      } else {
        const uint64_t a = dq0 + i * kTileDesc, b = dk0 + sk * kTileDesc;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss_w(d, a + off, b + off, Idesc<F16>::S, kk > 0 ? 1u : 0u);
        }
      }
      return true;
    };
    auto issue_pv = [&](int i, int sv, bool acc) {
      const uint32_t d = tmem + 256 + i * 128, pa = tmem + i * 128;
      const uint64_t b = dv0 + sv * kTileDesc;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, pa + kk * 8, b + kk * (2048 >> 4), Idesc<F16>::PV, (acc || kk > 0) ? 1u : 0u);
    };
    for (int gl = 0; ok; ++gl) {
      const int buf = gl & 1;
      if (!(ok = gwarp_wait(&bars->grp_full[buf], (gl >> 1) & 1, bars, p.status))) break;
      if (grp[buf].gi < 0) break;
      const int ns = grp[buf].ns, len0 = grp[buf].len[0], len1 = grp[buf].len[1];
      const int n = max(len0, len1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->grp_free[buf]);
      if (n == 0) continue;
      if (!(ok = gwarp_wait(&bars->q_full, qit & 1, bars, p.status))) break;
      ++qit;
      tc_fence_after();
      // Per step t: PV0(t), S0(t+1), PV1(t), S1(t+1); t = -1 issues the first S
      // products.  A shared step's tile is one K and one V stage, released by
      // Q tile 1's product; other steps take one stage per Q tile.  One loop
      // over the Q tiles (not unrolled), so every product is issued from one
      // place in the code: the issuing thread stays lean.
      int sk = 0, sv = 0;
      for (int t = -1; t < n && ok; ++t) {
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          const int lj = j ? len1 : len0;
          if (t >= 0 && t < lj) {  // P V product of Q tile j at step t
            const bool shared = t < ns;
            if (j == 0 || !shared) {
              sv = vit % M::kVS;
              if (!(ok = gwarp_wait(&bars->v_full[sv], (vit / M::kVS) & 1, bars, p.status))) break;
            }
            const int tj = j ? tiles1 : tiles0;
            if (!(ok = gwarp_wait(&bars->p_full[j], tj & 1, bars, p.status))) break;
            if (t == 0) {
              const int ij = j ? items1 : items0;
              if (!(ok = gwarp_wait(&bars->o_empty[j], (ij & 1) ^ 1, bars, p.status))) break;
            }
            tc_fence_after();
            issue_pv(j, sv, t > 0);
            if (j) ++tiles1; else ++tiles0;
            if (t == lj - 1) mma_commit_w(&bars->o_full[j]);
            if (j == 1 || !shared) {  // the V stage's last reader is issued
              mma_commit_w(&bars->v_empty[sv]);
              ++vit;
            }
          }
          const int u = t + 1;
          if (u < lj) {  // S product of Q tile j at step t + 1
            const bool shared = u < ns;
            if (j == 0 || !shared) {
              sk = kit % M::kKS;
              if (!(ok = gwarp_wait(&bars->k_full[sk], (kit / M::kKS) & 1, bars, p.status))) break;
              tc_fence_after();
            }
            if (!(ok = issue_s(j, sk))) break;
            mma_commit_w(&bars->s_full[j]);
            if (j == 1 || !shared) {  // the K stage's last reader is issued
              mma_commit_w(&bars->k_empty[sk]);
              ++kit;
            }
          }
        }
        // Q is read by the S products only: once the group's last S is issued,
        // the next group's Q may load while the last P V products run
        if (ok && t + 2 == n) mma_commit_w(&bars->q_empty);
      }
      if (!ok) break;
      if (len0 > 0) ++items0;
      if (len1 > 0) ++items1;
    }
    // Drain: wait for every MMA issued by this thread before TMEM and smem go away.
    mma_commit_w(&bars->drain);
    mbar_wait_drain(&bars->drain, 0, kTimeoutNs);
  }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) >> 2;  // Q tile
    const int quarter = warp & 3;    // TMEM lane quarter of this warp
    const int jq = 2 * wg + (quarter >> 1);  // query block of the group this warp serves
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + wg * 128;
    const uint32_t tO = tmem + lane_off + 256 + wg * 128;
    const float sl2 = p.scale_log2;
    int tiles = 0, items = 0;
    bool ok = true;
    for (int gl = 0; ok; ++gl) {
      const int buf = gl & 1;
      if (!(ok = gwarp_wait(&bars->grp_full[buf], (gl >> 1) & 1, bars, p.status))) break;
      const GroupInfo& gb = grp[buf];
      const int gi = gb.gi;
      if (gi < 0) break;
      const int nq = gb.nq;
      const int n = wg < nq ? gb.len[wg] : 0;  // this Q tile's key tiles
      const int bh = gi / ngq, qb0 = (gi - bh * ngq) * kGroupBlocks;
      const int row0 = bh * g.NB + qb0;  // index row of the group's first query block (NB <= kGroupMaxNB)
      if (n == 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->grp_free[buf]);
        if (wg < nq) {  // nothing selected by either query block of this Q tile
          const long long row = static_cast<long long>(bh) * g.Sp + static_cast<long long>(qb0) * 64 + wg * 128 + r;
          uint4* orow = reinterpret_cast<uint4*>(p.o + row * 128);
#pragma unroll
          for (int c = 0; c < 16; ++c) orow[c] = make_uint4(0, 0, 0, 0);
          p.lse[row] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY, l = 0.0f;
      GroupWalk walk;
      walk.init(gb);
      for (int t = 0; t < n; ++t) {
        int ka, kb, owner;
        walk.next(gb, p, row0, W, wg, ka, kb, owner);
        // this warp's query block: which halves of the tile it selected
        const int sa = group_uses(gb, owner, jq, ka) ? ka : -1;
        const int sb = group_uses(gb, owner, jq, kb) ? kb : -1;
        uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;
        const int st_a = block64_mask(g, sa, w0, w1);
        const int st_b = block64_mask(g, sb, w2, w3);
        if (!(ok = gwarp_wait(&bars->s_full[wg], tiles & 1, bars, p.status))) break;
        tc_fence_after();
        uint32_t pk[64];
        float lsum = 0.0f, alpha = 1.0f;
        bool rescale = false;
        const bool ha = st_a != kTileEmpty, hb = st_b != kTileEmpty;
        if (ha || hb) {
          uint32_t sv[128];  // an unselected half holds finite S values; the mask below overwrites them
          tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
          tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
          tmem_wait_ld();
          if constexpr (FP4) {  // S is in registers: its last 64 columns may take the other tile's scales
            tc_fence_before();
            mbar_arrive(&bars->s_read[wg]);
          }
          if (st_a == kTilePartial || st_b == kTilePartial) {
            // padded slots of a selected block (an unselected half is skipped below)
            const uint32_t mw[4] = {st_a == kTilePartial ? w0 : 0xffffffffu, st_a == kTilePartial ? w1 : 0xffffffffu,
                                    st_b == kTilePartial ? w2 : 0xffffffffu, st_b == kTilePartial ? w3 : 0xffffffffu};
            apply_key_mask(sv, mw);
          }
          lsum = softmax_halves<F16>(sv, ha, hb, sl2, t, m_used, alpha, rescale, pk);
        } else {
          // nothing selected in this tile by this warp's query block
          if constexpr (FP4) {  // S is not needed: its columns are free now
            tc_fence_before();
            mbar_arrive(&bars->s_read[wg]);
          }
#pragma unroll
          for (int j = 0; j < 64; ++j) pk[j] = 0u;
        }
        l = l * alpha + lsum;
        tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        // Rescale this row of O when its maximum moved (warp-uniform branch).
        // PV(t-1) is complete: the s_full commit just waited on follows it.
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->grp_free[buf]);
      // epilogue: O / l -> 16-bit row, lse
      if (!(ok = gwarp_wait(&bars->o_full[wg], items & 1, bars, p.status))) break;
      tc_fence_after();
      const long long row = static_cast<long long>(bh) * g.Sp + static_cast<long long>(qb0) * 64 + wg * 128 + r;
      uint4* orow = reinterpret_cast<uint4*>(p.o + row * 128);
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
#pragma unroll
        for (int j = 0; j < 4; ++j) orow[c * 4 + j] = w[j];
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[wg]);
      p.lse[row] = l > 0.0f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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
  // the last CTA to finish leaves the queue's counters at zero for the next call
  // (every CTA has taken its last ticket by now)
  if (p.queue && threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.queue + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      p.queue[0] = 0;
      p.queue[1] = 0;
    }
  }
}

template <bool FP4>
cudaError_t launch_grouped(const Geo& g, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const GroupParams& p, int BH, int num_sms, bool f16, cudaStream_t stream) {
  const long long groups = static_cast<long long>(BH) * ((g.NB + kGroupBlocks - 1) / kGroupBlocks);
  const int grid = static_cast<int>(groups < num_sms ? groups : num_sms);
  auto kern = f16 ? attn_fwd_grouped64_kernel<true, FP4> : attn_fwd_grouped64_kernel<false, FP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GSmem<FP4>::kTotal);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, GSmem<FP4>::kTotal, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_grouped64(const Geo& g, const CUtensorMap& tq, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const fwd::Params& p, int BH, int num_sms, bool f16,
                                      cudaStream_t stream) {
  GroupParams gp;
  static_cast<fwd::Params&>(gp) = p;
  gp.q_sf = gp.k_sf = nullptr;
  return launch_grouped<false>(g, tq, tk, tv, gp, BH, num_sms, f16, stream);
}

cudaError_t launch_attn_fwd_grouped64_fp4(const Geo& g, const CUtensorMap& tq, const CUtensorMap& tk,
                                          const CUtensorMap& tv, const AttnFp4Args& a, cudaStream_t stream) {
  GroupParams gp;
  gp.idx = a.idx;
  gp.num = a.num;
  gp.max_k = a.max_k;
  gp.BH = a.BH;
  gp.o = a.o;
  gp.lse = a.lse;
  gp.status = a.status;
  gp.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  gp.g = g;
  gp.queue = a.queue;  // null: groups go to CTAs statically
  gp.q_sf = a.q_sf;
  gp.k_sf = a.k_sf;
  return launch_grouped<true>(g, tq, tk, tv, gp, a.BH, a.num_sms, a.f16, stream);
}

}  // namespace vsa
