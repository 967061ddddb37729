// kernels.h -- internal launch entry points of the VSA kernels (not public ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace vsa {

// tile.cu
cudaError_t launch_tile(const Geo& g, int B, int H, const uint16_t* x, uint16_t* xt, float* pooled,
                        bool f16, cudaStream_t stream);
cudaError_t launch_untile(const Geo& g, int B, int H, const uint16_t* xt, uint16_t* x, cudaStream_t stream);
// x = x_tiled + gate * o_compress[block], untiled; gate in the untiled layout.
cudaError_t launch_untile_gate(const Geo& g, int B, int H, const uint16_t* xt, const float* o_compress,
                               const uint16_t* gate, uint16_t* x, bool f16, cudaStream_t stream);

// coarse.cu
cudaError_t launch_score_topk(int BH, int NB, int topk, const SelectRule& rule, const float* qbar,
                              const float* kbar, int32_t* idx, int32_t* num, cudaStream_t stream);
// topk == 0: the compression branch alone (idx, num unused).
cudaError_t launch_coarse_compress(int BH, int NB, int topk, const float* qbar, const float* kbar,
                                   const float* vbar, int32_t* idx, int32_t* num, float* o_compress, float scale,
                                   cudaStream_t stream);
cudaError_t launch_map_to_index(const uint8_t* map, long long rows, int NK, int32_t* idx, int32_t* num,
                                cudaStream_t stream);

// front.cu: tile q, k, v (+ block means) and the coarse stage in one launch.
struct FrontArgs {
  Geo g;
  int H, BH;
  int topk;                        // 0: no selection
  SelectRule rule;                 // with topk > 0: stride, prefix rule, forced-empty rows
  const uint4 *q, *k, *v;          // [B,S,H,D] 16-bit
  uint4 *qt, *kt, *vt;             // [B,H,Sp,D]
  float *qbar, *kbar, *vbar;       // [B,H,NB,D]; vbar null: no compression branch
  int32_t *idx, *num;              // selection (topk > 0)
  float* o_compress;               // [B,H,NB,D] (with vbar)
  float scale;                     // D^-1/2
  int *arrive, *done;              // [B*H] each, zero on entry, zero again on exit
  unsigned int* status;
  bool f16;
};
cudaError_t launch_front(const FrontArgs& a, cudaStream_t stream);

// attn_fwd.cu
struct AttnArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const int32_t* num;
  int max_k;
  int BH;
  uint16_t* o;
  float* lse;
  unsigned int* status;
  int num_sms;
  bool f16;    // fp16 tensors (else bf16)
  int* queue;  // 2 int32 of caller memory for the grouped kernel's shared queue, or null
};
cudaError_t launch_attn_fwd(const Geo& g, const AttnArgs& a, cudaStream_t stream);

// fp4.cu: NVFP4 codes + scales of tiled 16-bit rows (rows a multiple of 128),
// and the fine stage with FP4 Q K^T.
cudaError_t launch_quant_nvfp4(long long rows, const uint16_t* x, uint8_t* codes, uint8_t* sf, bool f16,
                               cudaStream_t stream);
struct AttnFp4Args {
  const uint8_t *q, *q_sf;  // codes [B,H,Sp,64] bytes, scales (tensor-core layout)
  const uint8_t *k, *k_sf;
  const uint16_t* v;        // [B,H,Sp,D] 16-bit
  const int32_t* idx;
  const int32_t* num;
  int max_k;
  int BH;
  uint16_t* o;
  float* lse;
  unsigned int* status;
  int num_sms;
  bool f16;  // v and o are fp16 (else bf16)
  int* queue = nullptr;  // 64-token plans: the grouped kernel's shared group queue (2 int32), or null
};
cudaError_t launch_attn_fwd_nvfp4(const Geo& g, const AttnFp4Args& a, cudaStream_t stream);
// attn_fwd_grouped.cu: the grouped 64-token kernel with NVFP4 Q and K (four
// query blocks per item); launch_attn_fwd_nvfp4 uses it for 64-token plans of
// up to kGroupMaxNB blocks.  tq: 128-row boxes of codes, tk / tv: 64-row boxes.
cudaError_t launch_attn_fwd_grouped64_fp4(const Geo& g, const CUtensorMap& tq, const CUtensorMap& tk,
                                          const CUtensorMap& tv, const AttnFp4Args& a, cudaStream_t stream);

// attn_bwd.cu
struct AttnBwdArgs {
  const uint16_t *q, *k, *v, *o, *dO;  // tiled [B,H,Sp,D]
  const float* lse;                    // [B,H,Sp]
  const int32_t* idx;
  const int32_t* num;
  int max_k;
  int BH;
  uint16_t *dq, *dk, *dv;  // tiled [B,H,Sp,D]
  void* workspace;         // attn_bwd_workspace_bytes
  unsigned int* status;
  bool f16;
};
size_t attn_bwd_workspace_bytes(const Geo& g, int BH, int max_k);
// The transposed selection of one head is built in shared memory (8 bytes per
// key block): at most this many blocks per head.
constexpr int kBwdMaxBlocks = 28672;
cudaError_t launch_attn_bwd(const Geo& g, const AttnBwdArgs& a, cudaStream_t stream);

}  // namespace vsa
