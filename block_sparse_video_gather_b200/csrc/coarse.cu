// coarse.cu -- coarse stage of VSA: block scores, per-row top-k, and the
// bool-map compaction.
//
// "FastVideo VSA" (vLLM-Omni user guide), introduction and section "Choose
// top-k": every query block scores all key/value blocks and keeps its top-k
// (top-k counts blocks, 0 < topk <= num_blocks).  FastVideo commit log
// (examples/inference/basic/README.md): a bool block map is compacted into
// q2k_idx / q2k_num with rows of any length, zero included.
//
// score_topk: one CTA per (b*h, group of 16 query blocks).  The pooled K of
// the head streams through shared memory in chunks of 64 blocks (row stride
// 129 floats, so the 32 threads of a warp hit 32 banks); a thread owns one key
// block and four query blocks and runs four independent fused-multiply-add
// chains in channel order -- the exact fp32 order the selection is defined
// with.  Scores never reach HBM: they stay in shared memory as order-keys.
// One warp per query block then finds the k-th largest key by a 32-step
// bitwise search (each step: count keys >= candidate, warp reduction), and
// writes the selected ids in ascending order with ballots; ties at the
// threshold go to the lower block index.
//
// Compression branch ("FastVideo VSA", section "Checkpoint behavior": the
// learned gate_compress projection; FastVideo commit log: the gate-compress
// branch pools per tile).  The same CTA turns its 16 score rows into softmax
// weights over all blocks, exp(scale (s - max)), kept in shared memory in
// place of the keys, and every thread accumulates one channel of eight rows
// against the pooled V of the head streamed in block order:
// o_compress[r] = sum_c w_rc vbar[c] / sum_c w_rc.  The weights come from the
// very fp32 scores the selection ranks.
#include "common.cuh"
#include "kernels.h"

namespace vsa {

namespace {

constexpr int kRows = 16;      // query blocks per CTA
constexpr int kChunk = 64;     // key blocks per shared-memory chunk
constexpr int kKStride = 129;  // padded row stride (floats)
constexpr int kThreads = 256;

// Monotone map fp32 -> uint32 (larger score -> larger key); -0 counts as +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key (the score back from its key; -0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <bool SELECT, bool COMPRESS>
__global__ void __launch_bounds__(kThreads) score_topk_kernel(int NB, int topk, const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              int32_t* __restrict__ idx, int32_t* __restrict__ num,
                                                              const float* __restrict__ vbar,
                                                              float* __restrict__ o_compress, float scale) {
  extern __shared__ __align__(16) float sm[];
  float* q_s = sm;                               // [kRows][128]
  float* k_s = q_s + kRows * 128;                // [kChunk][129]
  uint32_t* keys = reinterpret_cast<uint32_t*>(k_s + kChunk * kKStride);  // [kRows][NB]
  float* wsum = reinterpret_cast<float*>(keys + kRows * NB);              // [kRows]

  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  const float* qh = qbar + static_cast<long long>(bh) * NB * 128;
  const float* kh = kbar + static_cast<long long>(bh) * NB * 128;

  for (int i = tid; i < kRows * 128; i += kThreads) {
    const int r = i >> 7;
    q_s[i] = (r0 + r < NB) ? qh[static_cast<long long>(r0) * 128 + i] : 0.0f;
  }

  const int j_loc = tid % kChunk;
  const int rg = tid / kChunk;  // 0..3, owns query rows rg*4 .. rg*4+3
  for (int c0 = 0; c0 < NB; c0 += kChunk) {
    __syncthreads();
    const int nrow = min(kChunk, NB - c0);
    for (int i = tid; i < kChunk * 128; i += kThreads) {
      const int jr = i >> 7, d = i & 127;
      k_s[jr * kKStride + d] = (jr < nrow) ? kh[static_cast<long long>(c0) * 128 + i] : 0.0f;
    }
    __syncthreads();
    if (j_loc < nrow) {
      float acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
      const float* kr = k_s + j_loc * kKStride;
      const float* q0 = q_s + (rg * 4) * 128;
#pragma unroll 8
      for (int d = 0; d < 128; ++d) {
        const float kv = kr[d];
        acc0 = __fmaf_rn(q0[d], kv, acc0);
        acc1 = __fmaf_rn(q0[128 + d], kv, acc1);
        acc2 = __fmaf_rn(q0[256 + d], kv, acc2);
        acc3 = __fmaf_rn(q0[384 + d], kv, acc3);
      }
      const int j = c0 + j_loc;
      keys[(rg * 4 + 0) * NB + j] = order_key(acc0);
      keys[(rg * 4 + 1) * NB + j] = order_key(acc1);
      keys[(rg * 4 + 2) * NB + j] = order_key(acc2);
      keys[(rg * 4 + 3) * NB + j] = order_key(acc3);
    }
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; SELECT && r < kRows; r += kThreads / 32) {
    const int row = r0 + r;
    if (row >= NB) break;
    const uint32_t* key = keys + r * NB;
    // k-th largest key: the largest v with #{key >= v} >= topk
    uint32_t tau = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      unsigned cnt = 0;
      for (int j = lane; j < NB; j += 32) cnt += key[j] >= cand;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= static_cast<unsigned>(topk)) tau = cand;
    }
    unsigned gt = 0;
    for (int j = lane; j < NB; j += 32) gt += key[j] > tau;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int need = topk - static_cast<int>(gt);  // ties at tau to take, lowest ids first
    int32_t* out = idx + (static_cast<long long>(bh) * NB + row) * topk;
    int pos = 0, ties = 0;
    for (int base = 0; base < NB; base += 32) {
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
    if (lane == 0) num[static_cast<long long>(bh) * NB + row] = topk;
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
  const int rbase = (tid >> 7) * (kRows / 2);  // rows rbase .. rbase + 7
  const float* vh = vbar + static_cast<long long>(bh) * NB * 128 + d;
  const float* wr = w + rbase * NB;
  float acc[kRows / 2];
#pragma unroll
  for (int i = 0; i < kRows / 2; ++i) acc[i] = 0.0f;
  for (int c = 0; c < NB; ++c) {
    const float vv = __ldg(vh + static_cast<long long>(c) * 128);
#pragma unroll
    for (int i = 0; i < kRows / 2; ++i) acc[i] = __fmaf_rn(wr[i * NB + c], vv, acc[i]);
  }
#pragma unroll
  for (int i = 0; i < kRows / 2; ++i) {
    const int row = r0 + rbase + i;
    if (row < NB) o_compress[(static_cast<long long>(bh) * NB + row) * 128 + d] = __fdiv_rn(acc[i], wsum[rbase + i]);
  }
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

size_t score_topk_smem_bytes(int NB) {
  return sizeof(float) * (kRows * 128 + kChunk * kKStride) + sizeof(uint32_t) * kRows * static_cast<size_t>(NB) +
         sizeof(float) * kRows;
}

template <bool SELECT, bool COMPRESS>
cudaError_t launch_coarse_t(int BH, int NB, int topk, const float* qbar, const float* kbar, int32_t* idx,
                            int32_t* num, const float* vbar, float* o_compress, float scale, cudaStream_t stream) {
  const size_t smem = score_topk_smem_bytes(NB);
  cudaError_t e = cudaFuncSetAttribute(score_topk_kernel<SELECT, COMPRESS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((NB + kRows - 1) / kRows, BH);
  score_topk_kernel<SELECT, COMPRESS><<<grid, kThreads, smem, stream>>>(NB, topk, qbar, kbar, idx, num, vbar,
                                                                          o_compress, scale);
  return cudaGetLastError();
}

cudaError_t launch_score_topk(int BH, int NB, int topk, const float* qbar, const float* kbar, int32_t* idx,
                              int32_t* num, cudaStream_t stream) {
  return launch_coarse_t<true, false>(BH, NB, topk, qbar, kbar, idx, num, nullptr, nullptr, 0.0f, stream);
}

cudaError_t launch_coarse_compress(int BH, int NB, int topk, const float* qbar, const float* kbar,
                                   const float* vbar, int32_t* idx, int32_t* num, float* o_compress, float scale,
                                   cudaStream_t stream) {
  if (topk > 0)
    return launch_coarse_t<true, true>(BH, NB, topk, qbar, kbar, idx, num, vbar, o_compress, scale, stream);
  return launch_coarse_t<false, true>(BH, NB, 0, qbar, kbar, nullptr, nullptr, vbar, o_compress, scale, stream);
}

cudaError_t launch_map_to_index(const uint8_t* map, long long rows, int NK, int32_t* idx, int32_t* num,
                                cudaStream_t stream) {
  const long long blocks = (rows + 7) / 8;
  map_to_index_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(map, rows, NK, idx, num);
  return cudaGetLastError();
}

}  // namespace vsa
