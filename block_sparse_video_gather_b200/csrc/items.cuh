// items.cuh -- the per-CTA work items of the front end, shared by the
// standalone tile / coarse kernels and the fused front-end kernel: tiling
// (with block means) of one (b*h, block), and scoring + selection (+ the
// compression branch) of 8 query blocks of one head.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace vsa {
namespace items {

constexpr int kTileThreads = 256;
constexpr int kRowChunks = 16;  // 16 B chunks per 256 B row (D = 128)

// Where the tokens of one block live in the untiled sequence.  Computed
// once per CTA (three divisions); each slot then costs shifts and two
// multiply-adds.  Slot (lt, lh, lw) of a video block sits at grid point
// (t0 + lt, y0 + lh, x0 + lw); slot s of a prefix tile is token p0 + s.
struct BlockOrigin {
  bool prefix;
  long long p0;   // first token of a prefix tile
  int plim;       // real tokens of a prefix tile
  int t0, y0, x0; // grid origin of a video block
};

__device__ __forceinline__ BlockOrigin block_origin(const Geo& g, int blk) {
  BlockOrigin o;
  o.prefix = blk < g.n_pre;
  o.p0 = static_cast<long long>(blk) * g.bs;
  o.plim = g.n_prefix - blk * g.bs;
  const int vb = blk - g.n_pre;
  const int bW = vb % g.nW, bH = (vb / g.nW) % g.nH, bT = vb / (g.nW * g.nH);
  o.t0 = bT * g.bt;
  o.y0 = bH * g.bh;
  o.x0 = bW * g.bw;
  return o;
}

// Token index of slot `slot` of the block, or -1 for a padded slot.
__device__ __forceinline__ long long token_of_slot(const Geo& g, const BlockOrigin& o, int slot) {
  if (o.prefix) return slot < o.plim ? o.p0 + slot : -1;
  const int x = o.x0 + (slot & (g.bw - 1));
  const int y = o.y0 + ((slot >> g.lbw) & (g.bh - 1));
  const int t = o.t0 + (slot >> (g.lbw + g.lbh));
  if (t >= g.T || y >= g.Hg || x >= g.Wg) return -1;
  return g.n_prefix + (static_cast<long long>(t) * g.Hg + y) * g.Wg + x;
}

__device__ __forceinline__ int block_real_count(const Geo& g, int blk) {
  if (blk < g.n_pre) return min(g.bs, g.n_prefix - blk * g.bs);
  int vt, vh, vw;
  video_block_extent(g, blk - g.n_pre, vt, vh, vw);
  return vt * vh * vw;
}

// Token rows one tile item covers: one 256-token block or four 64-token
// blocks, so every item moves 64 KB whatever the block size.
constexpr int kItemRows = 256;
template <int BS>
__host__ __device__ constexpr int item_blocks() {
  return kItemRows / BS;
}

// Tile blocks blk0 .. blk0 + item_blocks<BS>() - 1 (those below NB) of head
// bh: copy their token rows into the tiled layout (padding zero-filled) and,
// with POOL, write each block's fp32 channel means (channel d of a block is
// summed over its slots in slot order, then divided once by its real-token
// count).  `stage` is kItemRows * 256 bytes of shared memory (used only with
// POOL).
template <int BS, bool POOL, bool F16>
__device__ __forceinline__ void tile_item(const Geo& g, int H, int blk0, int bh, const uint4* __restrict__ x,
                                          uint4* __restrict__ xt, float* __restrict__ pooled, uint4* stage) {
  constexpr int kBlocks = item_blocks<BS>();
  constexpr int kPer = BS / 16;  // row groups of one block per thread
  const int b = bh / H, h = bh - b * H;
  const int chunk = threadIdx.x & (kRowChunks - 1);
  const int row0 = threadIdx.x >> 4;  // 0..15

  uint4 v[kBlocks * kPer];
#pragma unroll
  for (int j = 0; j < kBlocks; ++j) {
    const int blk = blk0 + j;
    const bool live = blk < g.NB;
    const BlockOrigin org = block_origin(g, live ? blk : blk0);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const long long s = live ? token_of_slot(g, org, row0 + 16 * i) : -1;
      if (s >= 0) {
        const long long src = ((static_cast<long long>(b) * g.S + s) * H + h) * kRowChunks + chunk;
        v[j * kPer + i] = __ldcs(x + src);
      } else {
        v[j * kPer + i] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  const long long dst0 = (static_cast<long long>(bh) * g.Sp + static_cast<long long>(blk0) * BS) * kRowChunks;
#pragma unroll
  for (int j = 0; j < kBlocks; ++j) {
    if (blk0 + j >= g.NB) break;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int row = j * BS + row0 + 16 * i;
      xt[dst0 + row * kRowChunks + chunk] = v[j * kPer + i];
      if (POOL) stage[row * kRowChunks + chunk] = v[j * kPer + i];
    }
  }
  if (POOL) {
    __syncthreads();
    const int d = threadIdx.x & 127;
    const uint16_t* st = reinterpret_cast<const uint16_t*>(stage);
    for (int j = threadIdx.x >> 7; j < kBlocks && blk0 + j < g.NB; j += kTileThreads / 128) {
      float s = 0.0f;
#pragma unroll 8
      for (int slot = 0; slot < BS; ++slot) {
        const uint16_t hv = st[(j * BS + slot) * 128 + d];
        const float f = F16 ? __half2float(__ushort_as_half(hv)) : __uint_as_float(static_cast<uint32_t>(hv) << 16);
        s = __fadd_rn(s, f);
      }
      const float mean = __fdiv_rn(s, static_cast<float>(block_real_count(g, blk0 + j)));
      pooled[(static_cast<long long>(bh) * g.NB + blk0 + j) * 128 + d] = mean;
    }
  }
}


constexpr int kRows = 8;     // query blocks per score item (one per warp in the selection)
constexpr int kThreads = 256;
constexpr int kChunk = kThreads;  // key blocks per pass: one per thread
// One buffer of the key-mean ring: kChunk keys x 16 channels at a row stride
// of 20 floats (or fewer keys x more channels); two buffers.
constexpr int kSlabFloats = kChunk * 20;

// fp32 loads: read-only path for inputs of the launch, L2-only for data
// that other CTAs of the same launch wrote.
template <bool COHERENT>
__device__ __forceinline__ float ldf(const float* p) {
  return COHERENT ? __ldcg(p) : __ldg(p);
}

// 16-byte global -> shared copy through L2 (cp.async.cg); a source size of
// 0 writes zeros.  All copies of a thread stay in flight until cp_async_wait.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most one committed group of this thread is still in flight.
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__host__ __device__ constexpr size_t score_smem_bytes_c(int NB) {
  return sizeof(float) * (kRows * 128 + 2 * kSlabFloats) + sizeof(uint32_t) * kRows * static_cast<size_t>(NB) +
         sizeof(float) * kRows;
}
inline size_t score_smem_bytes(int NB) { return score_smem_bytes_c(NB); }

// Monotone map fp32 -> uint32 (larger score -> larger key); -0 counts as +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key (the score back from its key; -0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The k-th largest of the order keys key[lo .. NB-1] as the selection's
// threshold: the largest v with #{key >= v} >= topk, found bit by bit.  Once
// exactly topk keys are >= v the selection is decided (no tie straddles v,
// and the selection pass takes every key >= v), so the search stops there.
// KR > 0: each lane holds its candidates lo + lane + 32 i (i < KR) in
// registers for the passes (NB - lo <= 32 KR); KR = 0 reads them from
// shared memory every pass.  Absent candidates count as 0, below every
// candidate threshold (>= 1).
template <int KR>
__device__ __forceinline__ uint32_t select_threshold(const uint32_t* key, int lo, int NB, int topk, int lane) {
  uint32_t kr[KR > 0 ? KR : 1];
#pragma unroll
  for (int i = 0; i < KR; ++i) {
    const int j = lo + lane + 32 * i;
    kr[i] = j < NB ? key[j] : 0u;
  }
  uint32_t tau = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    unsigned cnt = 0;
    if (KR > 0) {
#pragma unroll
      for (int i = 0; i < KR; ++i) cnt += kr[i] >= cand;
    } else {
      for (int j = lo + lane; j < NB; j += 32) cnt += key[j] >= cand;
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= static_cast<unsigned>(topk)) {
      tau = cand;
      if (cnt == static_cast<unsigned>(topk)) break;
    }
  }
  return tau;
}

// Scores, selection and compression branch of query blocks r0 .. r0+7 of
// head bh.  `sm` is score_smem_bytes(NB) of shared memory.  COHERENT: the
// block means were written by other CTAs of the same launch, so they are
// read through L2 only (never the read-only path).
//
// A thread owns one key block of the current pass (up to kChunk blocks) and
// all eight query blocks: eight fused-multiply-add chains over the channels in
// order (four channels per step: one 16-byte load of the key row, one
// broadcast 16-byte load per query row), so each key row is read from shared
// memory once.  Key means reach shared memory by cp.async through L2 in
// slabs of channels (16 for a full pass, more when the pass has fewer keys),
// two buffers: the next slab loads while the current one is scored.
//
// The selection follows `rule` (common.cuh): a forced-empty row writes count
// 0; a prefix query row under the tile-64 rule lists every block; any other
// row lists the rule's n_pre prefix blocks, then its top-k among the blocks
// n_pre .. NB-1 (every block under the plain rule), then -1 up to the stride.
template <bool SELECT, bool COMPRESS, bool COHERENT>
__device__ __forceinline__ void score_item(int NB, int topk, const SelectRule& rule, int r0, int bh,
                                           const float* qbar, const float* kbar, int32_t* __restrict__ idx,
                                           int32_t* __restrict__ num, const float* vbar,
                                           float* __restrict__ o_compress, float scale, float* sm) {
  float* q_s = sm;                                                          // [kRows][128]
  float* k_s = q_s + kRows * 128;                                           // [2][kSlabFloats]
  uint32_t* keys = reinterpret_cast<uint32_t*>(k_s + 2 * kSlabFloats);     // [kRows][NB]
  float* wsum = reinterpret_cast<float*>(keys + kRows * NB);                // [kRows]

  const int tid = threadIdx.x;
  const float* qh = qbar + static_cast<long long>(bh) * NB * 128;
  const float* kh = kbar + static_cast<long long>(bh) * NB * 128;

  static_assert(kRows * 128 == 4 * kThreads, "one 16-byte copy of query means per thread");
  {
    const int i = 4 * tid;
    const bool ok = r0 + (i >> 7) < NB;
    cp_async16(q_s + i, ok ? qh + static_cast<long long>(r0) * 128 + i : qh, ok);  // rows past NB read as 0
  }

  for (int c0 = 0; c0 < NB; c0 += kChunk) {
    const int nk = min(kChunk, NB - c0);
    int C = 16;  // channels per slab: as many as one buffer holds for this pass
    while (C < 128 && nk * (2 * C + 4) <= kSlabFloats) C *= 2;
    const int stride = C + 4;  // 16-byte rows, conflict-free float4 reads
    const int nslab = 128 / C, units = nk * (C / 4);
    auto issue = [&](int sl) {  // slab sl into buffer sl & 1, one commit group
      float* dst = k_s + (sl & 1) * kSlabFloats;
      const int cpr = C / 4;
      for (int u = tid; u < units; u += kThreads) {
        const int key = u / cpr, part = u - key * cpr;
        cp_async16(dst + key * stride + 4 * part, kh + static_cast<long long>(c0 + key) * 128 + sl * C + 4 * part,
                   true);
      }
      cp_async_commit();
    };
    __syncthreads();  // the previous pass no longer reads the buffers
    issue(0);
    float acc[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r] = 0.0f;
    for (int sl = 0; sl < nslab; ++sl) {
      if (sl + 1 < nslab) {
        issue(sl + 1);
        cp_async_wait_1();
      } else {
        cp_async_wait_0();
      }
      __syncthreads();  // slab sl (and the query rows) visible to every thread
      if (tid < nk) {
        const float* kr = k_s + (sl & 1) * kSlabFloats + tid * stride;
        const float* qc = q_s + sl * C;
#pragma unroll 4
        for (int d = 0; d < C; d += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(kr + d);
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const float4 qv = *reinterpret_cast<const float4*>(qc + r * 128 + d);
            acc[r] = __fmaf_rn(qv.x, kv.x, acc[r]);
            acc[r] = __fmaf_rn(qv.y, kv.y, acc[r]);
            acc[r] = __fmaf_rn(qv.z, kv.z, acc[r]);
            acc[r] = __fmaf_rn(qv.w, kv.w, acc[r]);
          }
        }
      }
      __syncthreads();  // buffer sl & 1 is free for slab sl + 2
    }
    if (tid < nk) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) keys[r * NB + c0 + tid] = order_key(acc[r]);
    }
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; SELECT && r < kRows; r += kThreads / 32) {
    const int row = r0 + r;
    if (row >= NB) break;
    const long long rid = static_cast<long long>(bh) * NB + row;
    int32_t* out = idx + rid * rule.stride;
    if (rule.keep && __ldg(rule.keep + rid) == 0) {  // forced empty
      for (int j = lane; j < rule.stride; j += 32) out[j] = -1;
      if (lane == 0) num[rid] = 0;
      continue;
    }
    if (row < rule.n_pre) {  // prefix query tile: every block
      for (int j = lane; j < rule.stride; j += 32) out[j] = j < NB ? j : -1;
      if (lane == 0) num[rid] = NB;
      continue;
    }
    const int lo = rule.n_pre;  // candidates lo .. NB-1; blocks 0 .. lo-1 always listed
    for (int j = lane; j < lo; j += 32) out[j] = j;
    const uint32_t* key = keys + r * NB;
    const int nc = NB - lo;  // candidates
    const uint32_t tau = nc <= 32 * 8    ? select_threshold<8>(key, lo, NB, topk, lane)
                         : nc <= 32 * 20 ? select_threshold<20>(key, lo, NB, topk, lane)
                                         : select_threshold<0>(key, lo, NB, topk, lane);
    unsigned gt = 0;
    for (int j = lo + lane; j < NB; j += 32) gt += key[j] > tau;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int need = topk - static_cast<int>(gt);  // ties at tau to take, lowest ids first
    int pos = lo, ties = 0;
    for (int base = lo; base < NB; base += 32) {
      const int j = base + lane;
      const uint32_t u = (j < NB) ? key[j] : 0u;
      const bool is_gt = (j < NB) && u > tau;
      const bool is_eq = (j < NB) && u == tau;
      const uint32_t eq = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = is_gt || (is_eq && ties + __popc(eq & lt_mask) < need);
      const uint32_t sm_ = __ballot_sync(0xffffffffu, sel);
      if (sel) out[pos + __popc(sm_ & lt_mask)] = j;
      pos += __popc(sm_);
      ties += __popc(eq);
    }
    for (int j = lo + topk + lane; j < rule.stride; j += 32) out[j] = -1;
    if (lane == 0) num[rid] = lo + topk;
  }
  if (!COMPRESS) return;

  __syncthreads();  // the selection is done reading the keys
  float* w = reinterpret_cast<float*>(keys);
  for (int r = warp; r < kRows; r += kThreads / 32) {
    uint32_t* key = keys + r * NB;
    uint32_t kmax = 0;
    for (int j = lane; j < NB; j += 32) kmax = max(kmax, key[j]);
    const float m = key_value(__reduce_max_sync(0xffffffffu, kmax));
    float l = 0.0f;
    for (int j = lane; j < NB; j += 32) {
      const float e = expf((key_value(key[j]) - m) * scale);
      w[r * NB + j] = e;  // same word, same thread: the key is read before it is overwritten
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) wsum[r] = l;
  }
  __syncthreads();
  const int d = tid & 127;
  const int rbase = (tid >> 7) * (kRows / 2);  // rows rbase .. rbase + kRows/2 - 1
  const float* vh = vbar + static_cast<long long>(bh) * NB * 128 + d;
  const float* wr = w + rbase * NB;
  float acc[kRows / 2];
#pragma unroll
  for (int i = 0; i < kRows / 2; ++i) acc[i] = 0.0f;
  for (int c = 0; c < NB; ++c) {
    const float vv = ldf<COHERENT>(vh + static_cast<long long>(c) * 128);
#pragma unroll
    for (int i = 0; i < kRows / 2; ++i) acc[i] = __fmaf_rn(wr[i * NB + c], vv, acc[i]);
  }
#pragma unroll
  for (int i = 0; i < kRows / 2; ++i) {
    const int row = r0 + rbase + i;
    if (row < NB) o_compress[(static_cast<long long>(bh) * NB + row) * 128 + d] = __fdiv_rn(acc[i], wsum[rbase + i]);
  }
}


}  // namespace items
}  // namespace vsa
