// front.cu -- the whole front end of VSA in one launch: tile q, k, v (with
// the block means the coarse stage scores), then scores + per-row top-k
// (+ the compression branch).
//
// "FastVideo VSA" (vLLM-Omni user guide), introduction and section "Choose
// top-k" (tile, pool, score, keep top-k); section "Checkpoint behavior" and
// the FastVideo commit log for the gate-compress branch.
//
// One CTA per work item, two kinds:
//   tile item   (tensor, b*h, 256 tiled rows: one 256-token block or four
//               64-token blocks): tile_item of items.cuh; an item that pools
//               announces its block means on the head's arrival counter
//               (writes, fence, barrier, atomic add);
//   score item  (b*h, 8 query blocks): waits until every pooled item of its
//               head has arrived, then score_item of items.cuh with loads
//               through L2.
// Grid order (linear blockIdx.x): tile items of head 0; then for h >= 1 the
// tile items of head h followed by the score items of head h-1; then the
// score items of the last head; then, when no compression branch needs the
// block means of v, the v tiles of every head.  A score item therefore only
// waits on items with a lower index, dispatched before it, a head's scoring
// overlaps the tiling of the next head, and the last head's scoring overlaps
// the v tiles instead of trailing the whole tiling pass.  The wait is bounded (2 s); on expiry the item records
// VSA_ERR_TIMEOUT and returns.
//
// The arrival counters live in a caller workspace of 2 int32 per (b, h)
// (arrivals, finished score items), zero before the launch; the last score
// item of a head sets both back to zero, so the workspace is zero again after
// every launch that did not time out.
#include "common.cuh"
#include "items.cuh"
#include "kernels.h"

namespace vsa {

namespace {

using namespace items;

constexpr unsigned long long kWaitNs = 2000000000ull;

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int BS, bool F16, bool SELECT, bool COMPRESS>
__global__ void __launch_bounds__(kTileThreads, 3) front_kernel(FrontArgs a) {
  extern __shared__ __align__(16) uint4 smem[];
  const Geo& g = a.g;
  const int NB = g.NB;
  constexpr bool kScore = SELECT || COMPRESS;
  constexpr int kBlocks = item_blocks<BS>();
  const int nT = (NB + kBlocks - 1) / kBlocks;  // tile items per tensor and head
  // tile items per head segment: q, k (and v when the scoring needs its means)
  const int nA = (COMPRESS || !kScore) ? 3 * nT : 2 * nT;
  const int nB = kScore ? (NB + kRows - 1) / kRows : 0;
  const int per = nA + nB;

  // decode the work item
  const int L = blockIdx.x;
  int head, item;
  bool is_tile;
  if (!kScore) {
    head = L / nA;
    item = L - head * nA;
    is_tile = true;
  } else if (L < nA) {
    head = 0;
    item = L;
    is_tile = true;
  } else if (L < a.BH * per) {
    const int s = (L - nA) / per + 1;
    const int off = (L - nA) - (s - 1) * per;
    if (s < a.BH && off < nA) {
      head = s;
      item = off;
      is_tile = true;
    } else if (s < a.BH) {
      head = s - 1;
      item = off - nA;
      is_tile = false;
    } else {
      head = a.BH - 1;
      item = off;
      is_tile = false;
    }
  } else {  // v tiles that no score item waits for, after every score item
    const int vi = L - a.BH * per;
    head = vi / nT;
    item = 2 * nT + (vi - head * nT);
    is_tile = true;
  }

  if (is_tile) {
    const int tensor = item / nT;  // 0 q, 1 k, 2 v
    const int blk = (item - tensor * nT) * kBlocks;
    if (tensor == 0) {
      tile_item<BS, true, F16>(g, a.H, blk, head, a.q, a.qt, a.qbar, smem);
    } else if (tensor == 1) {
      tile_item<BS, true, F16>(g, a.H, blk, head, a.k, a.kt, a.kbar, smem);
    } else if (COMPRESS) {
      tile_item<BS, true, F16>(g, a.H, blk, head, a.v, a.vt, a.vbar, smem);
    } else {
      tile_item<BS, false, F16>(g, a.H, blk, head, a.v, a.vt, nullptr, smem);
    }
    if (kScore && (tensor < 2 || COMPRESS)) {
      __threadfence();  // each writer of the block means orders its writes
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(a.arrive + head, 1);
      }
    }
    return;
  }

  // score item: wait for the head's block means
  __shared__ int s_ready;
  if (threadIdx.x == 0) {
    const int target = (COMPRESS ? 3 : 2) * nT;
    const unsigned long long t0 = globaltimer_ns();
    int ready = 1;
    while (ld_acquire_gpu(a.arrive + head) < target) {
      if (globaltimer_ns() - t0 > kWaitNs) {
        atomicCAS(a.status, 0u, static_cast<unsigned>(VSA_ERR_TIMEOUT));
        ready = 0;
        break;
      }
      __nanosleep(256);
    }
    s_ready = ready;
  }
  __syncthreads();
  if (!s_ready) return;
  score_item<SELECT, COMPRESS, true>(NB, a.topk, a.rule, item * kRows, head, a.qbar, a.kbar, a.idx, a.num, a.vbar,
                                     a.o_compress, a.scale, reinterpret_cast<float*>(smem));
  if (threadIdx.x == 0) {
    // every score item of the head has passed its wait once the last one gets here
    if (atomicAdd(a.done + head, 1) == nB - 1) {
      a.arrive[head] = 0;
      a.done[head] = 0;
    }
  }
}

template <int BS, bool F16, bool SELECT, bool COMPRESS>
cudaError_t launch_front_t(const FrontArgs& a, cudaStream_t stream) {
  constexpr bool kScore = SELECT || COMPRESS;
  const int NB = a.g.NB;
  size_t smem = static_cast<size_t>(kItemRows) * 256;
  if (kScore) smem = smem > score_smem_bytes(NB) ? smem : score_smem_bytes(NB);
  cudaError_t e = cudaFuncSetAttribute(front_kernel<BS, F16, SELECT, COMPRESS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long nB = kScore ? (NB + kRows - 1) / kRows : 0;
  const long long nT = (NB + item_blocks<BS>() - 1) / item_blocks<BS>();
  const long long grid = static_cast<long long>(a.BH) * (3LL * nT + nB);
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  front_kernel<BS, F16, SELECT, COMPRESS><<<static_cast<unsigned>(grid), kTileThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int BS, bool F16>
cudaError_t launch_front_bs(const FrontArgs& a, cudaStream_t stream) {
  const bool sel = a.topk > 0, cmp = a.vbar != nullptr;
  if (sel && cmp) return launch_front_t<BS, F16, true, true>(a, stream);
  if (sel) return launch_front_t<BS, F16, true, false>(a, stream);
  if (cmp) return launch_front_t<BS, F16, false, true>(a, stream);
  return launch_front_t<BS, F16, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_front(const FrontArgs& a, cudaStream_t stream) {
  if (a.g.bs == 256) return a.f16 ? launch_front_bs<256, true>(a, stream) : launch_front_bs<256, false>(a, stream);
  return a.f16 ? launch_front_bs<64, true>(a, stream) : launch_front_bs<64, false>(a, stream);
}

}  // namespace vsa
