// coarse.cu -- coarse stage of VSA: block scores, per-row top-k, and the
// bool-map compaction.
//
// "FastVideo VSA" (vLLM-Omni user guide), introduction and section "Choose
// top-k": every query block scores all key/value blocks and keeps its top-k
// (top-k counts blocks, 0 < topk <= num_blocks).  FastVideo commit log
// (examples/inference/basic/README.md): a bool block map is compacted into
// q2k_idx / q2k_num with rows of any length, zero included.
//
// score_topk: one CTA per (b*h, group of 8 query blocks); the work item is
// score_item of items.cuh.  The selection rule is either the VSA top-k over
// every block or the tile-64 rule of the commit log (prefix query tiles
// dense, video query tiles the prefix plus a top-k of the video tiles; rows
// may be forced empty) -- see SelectRule in common.cuh.  The pooled K of the head streams through shared
// memory in chunks of 64 blocks (copied with cp.async; 16-byte rows of 132
// floats, read four channels at a time); a thread owns one key block and two query blocks and
// runs two independent fused-multiply-add chains in channel order -- the
// exact fp32 order the selection is defined with.  Scores never reach HBM:
// they stay in shared memory as order-keys.
// One warp per query block then finds the k-th largest key by a bitwise
// search of at most 32 steps (each step: count keys >= candidate, warp
// reduction; it stops once exactly k keys pass), and writes the selected ids
// in ascending order with ballots; ties at the threshold go to the lower
// block index.
//
// Compression branch ("FastVideo VSA", section "Checkpoint behavior": the
// learned gate_compress projection; FastVideo commit log: the gate-compress
// branch pools per tile).  The same CTA turns its 8 score rows into softmax
// weights over all blocks, exp(scale (s - max)), kept in shared memory in
// place of the keys, and every thread accumulates one channel of four rows
// against the pooled V of the head streamed in block order:
// o_compress[r] = sum_c w_rc vbar[c] / sum_c w_rc.  The weights come from the
// very fp32 scores the selection ranks.
#include "common.cuh"
#include "items.cuh"
#include "kernels.h"

namespace vsa {

namespace {

using namespace items;

template <bool SELECT, bool COMPRESS>
__global__ void __launch_bounds__(kThreads) score_topk_kernel(int NB, int topk, SelectRule rule,
                                                              const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              int32_t* __restrict__ idx, int32_t* __restrict__ num,
                                                              const float* __restrict__ vbar,
                                                              float* __restrict__ o_compress, float scale) {
  extern __shared__ __align__(16) float sm[];
  score_item<SELECT, COMPRESS, false>(NB, topk, rule, blockIdx.x * kRows, blockIdx.y, qbar, kbar, idx, num, vbar,
                                      o_compress, scale, sm);
}

__global__ void __launch_bounds__(256) map_to_index_kernel(const uint8_t* __restrict__ map, long long rows, int NK,
                                                           int32_t* __restrict__ idx, int32_t* __restrict__ num) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const uint8_t* m = map + row * NK;
  int32_t* out = idx + row * NK;
  int pos = 0;
  for (int base = 0; base < NK; base += 32) {
    const int j = base + lane;
    const bool sel = (j < NK) && m[j] != 0;
    const uint32_t b = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(b & lt_mask)] = j;
    pos += __popc(b);
  }
  for (int j = pos + lane; j < NK; j += 32) out[j] = -1;
  if (lane == 0) num[row] = pos;
}

}  // namespace


template <bool SELECT, bool COMPRESS>
cudaError_t launch_coarse_t(int BH, int NB, int topk, const SelectRule& rule, const float* qbar, const float* kbar,
                            int32_t* idx, int32_t* num, const float* vbar, float* o_compress, float scale,
                            cudaStream_t stream) {
  const size_t smem = score_smem_bytes(NB);
  cudaError_t e = cudaFuncSetAttribute(score_topk_kernel<SELECT, COMPRESS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((NB + kRows - 1) / kRows, BH);
  score_topk_kernel<SELECT, COMPRESS><<<grid, kThreads, smem, stream>>>(NB, topk, rule, qbar, kbar, idx, num, vbar,
                                                                          o_compress, scale);
  return cudaGetLastError();
}

cudaError_t launch_score_topk(int BH, int NB, int topk, const SelectRule& rule, const float* qbar,
                              const float* kbar, int32_t* idx, int32_t* num, cudaStream_t stream) {
  return launch_coarse_t<true, false>(BH, NB, topk, rule, qbar, kbar, idx, num, nullptr, nullptr, 0.0f, stream);
}

cudaError_t launch_coarse_compress(int BH, int NB, int topk, const float* qbar, const float* kbar,
                                   const float* vbar, int32_t* idx, int32_t* num, float* o_compress, float scale,
                                   cudaStream_t stream) {
  const SelectRule plain{topk, 0, nullptr};
  if (topk > 0)
    return launch_coarse_t<true, true>(BH, NB, topk, plain, qbar, kbar, idx, num, vbar, o_compress, scale, stream);
  return launch_coarse_t<false, true>(BH, NB, 0, plain, qbar, kbar, nullptr, nullptr, vbar, o_compress, scale,
                                      stream);
}

cudaError_t launch_map_to_index(const uint8_t* map, long long rows, int NK, int32_t* idx, int32_t* num,
                                cudaStream_t stream) {
  const long long blocks = (rows + 7) / 8;
  map_to_index_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(map, rows, NK, idx, num);
  return cudaGetLastError();
}

}  // namespace vsa
