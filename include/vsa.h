/*
 * vsa.h -- C ABI of the Video Sparse Attention (VSA) forward path on B200.
 *
 * The method ("FastVideo VSA", vLLM-Omni user guide, introduction): the
 * post-patch latent grid of a video DiT is cut into spatiotemporal blocks;
 * every query block scores all key/value blocks on block-pooled Q and K,
 * keeps its top-k, and runs attention against the tokens of those blocks
 * only.  The forward path, in stream order:
 *
 *   vsa_tile(q), vsa_tile(k) (with pooled means), vsa_tile(v)
 *   vsa_coarse_topk(qbar, kbar)          -> q2k_idx, q2k_num
 *      (or vsa_coarse_topk_prefix for the tile-64 layout's rule,
 *       or vsa_map_to_index(bool map)    -> q2k_idx, q2k_num)
 *   vsa_sparse_attn_fwd(q, k, v, index)  -> o, lse      (tiled layout)
 *   vsa_untile(o)
 *
 * or, with the front end in one launch,
 *
 *   vsa_tile_coarse(q, k, v)             -> tiled q, k, v, means, q2k_idx, q2k_num
 *   vsa_sparse_attn_fwd_ex(...)          -> o, lse
 *   vsa_untile(o)
 *
 * The gate-compress branch adds pooled v to the front end,
 * vsa_coarse_compress (or the compression outputs of vsa_tile_coarse) and
 * vsa_untile_gate in place of vsa_untile.  vsa_sparse_attn_bwd gives the
 * fine stage's gradients for a fixed selection.  The _ex calls and
 * vsa_tile_coarse take bf16 or fp16.  For FP4 Q and K, vsa_quantize_nvfp4
 * (tiled q, tiled k) and vsa_sparse_attn_fwd_nvfp4 replace the fine stage.
 * vsa_tile_coarse_prefix is the one-launch front end with the tile-64
 * selection.  The _ws fine-stage calls take a caller workspace with which
 * the 64-token kernel hands out its work items from a shared queue.
 *
 * Conventions shared by every call
 *  - bf16 / fp16 tensors are passed as pointers to their raw 16-bit patterns.
 *  - Untiled layout: [B, S, H, D] (token-major, heads inside), S = n_prefix +
 *    T*Hg*Wg tokens, video tokens in (t, y, x) raster order after the prefix.
 *  - Tiled layout: [B, H, Sp, D], Sp = NB * block_tokens.  Block b holds rows
 *    [b*bs, (b+1)*bs).  Prefix tiles come first and hold the prefix tokens in
 *    order.  Video blocks follow in raster order over (bT, bH, bW); inside a
 *    block, token (lt, lh, lw) sits at slot (lt*bh + lh)*bw + lw.  Slots whose
 *    grid coordinates fall outside (T, Hg, Wg) are padding and hold zeros.
 *  - D must be 128 (the only head size the B200 kernels are built for).
 *  - Every device pointer must be 16-byte aligned and every buffer is owned
 *    by the caller; the library allocates no device memory in any call.
 *  - Every call is asynchronous on `stream` and returns an int status.  A
 *    rejected argument returns before any device work is queued.  Errors found on the device
 *    (bad block ids, counts above max_k, a pipeline wait that ran out) are
 *    recorded in a per-device status word read by vsa_get_status().
 *  - Nothing falls back: unsupported input is an error, never rerouted.
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VSA_API __attribute__((visibility("default")))
#else
#define VSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *vsa_stream_t;

/* Opaque, host-only description of one video geometry. */
typedef struct vsa_plan *vsa_plan_t;

/* 16-bit floating-point formats of Q, K, V and o ("FastVideo VSA", section
 * "Verify routing and fallback": the kernel takes FP16 or BF16 tensors).
 * The calls without an _ex suffix are bf16. */
typedef enum vsa_dtype { VSA_BF16 = 0, VSA_F16 = 1 } vsa_dtype_t;

enum vsa_status {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, non-positive size */
    VSA_ERR_UNSUPPORTED = 2,   /* D != 128, block tokens not 64 or 256, odd tile count, not sm_100 */
    VSA_ERR_TOPK = 3,          /* topk <= 0 or topk > num_blocks */
    VSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    VSA_ERR_BAD_INDEX = 5,     /* device: a block id outside [0, NB) or a count outside [0, max_k] */
    VSA_ERR_TIMEOUT = 6,       /* device: a pipeline wait ran out; the kernel stopped early */
    VSA_ERR_NO_DEVICE = 7      /* no usable CUDA device */
};

/*
 * Geometry ("FastVideo VSA", section "Choose top-k": blocks of (4, 8, 8)
 * tokens over the zero-padded latent grid; num_blocks = ceil(T/bt) *
 * ceil(Hg/bh) * ceil(Wg/bw), e.g. (31, 22, 40) -> 120).
 *
 * vsa_plan_create_prefix adds n_prefix tokens ahead of the grid, tiled in
 * order into ceil(n_prefix / bs) contiguous tiles (the tile-64 layout of
 * the FastVideo commit log, examples/inference/basic/README.md).
 * Block sizes: bt*bh*bw must be 64 or 256 and each of bt, bh, bw a power of
 * two.  Returns VSA_ERR_INVALID_ARG / VSA_ERR_UNSUPPORTED on bad sizes.
 * The plan is host memory owned by the caller; free it with vsa_plan_destroy.
 */
VSA_API int vsa_plan_create(int T, int Hg, int Wg, int bt, int bh, int bw, vsa_plan_t *out);
VSA_API int vsa_plan_create_prefix(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                           vsa_plan_t *out);
VSA_API void vsa_plan_destroy(vsa_plan_t plan);

/* Sizes of a plan: block count NB, real tokens S, padded tokens Sp, tokens per block. */
VSA_API int vsa_plan_sizes(vsa_plan_t plan, int *num_blocks, int64_t *seq_len, int64_t *padded_len,
                   int *block_tokens);

/*
 * The routing fields the page logs ("FastVideo VSA", section "Choose
 * top-k"): seq_len, dit_seq_shape, block_size, num_blocks, topk and
 * keep_ratio, written as one NUL-terminated line into buf (at most n bytes).
 */
VSA_API int vsa_plan_describe(vsa_plan_t plan, int topk, char *buf, size_t n);

/*
 * Tile: x [B,S,H,D] bf16 -> x_tiled [B,H,Sp,D] bf16 (padding zero-filled).
 * If pooled is not NULL it also receives the per-block mean of the real
 * tokens, [B,H,NB,D] fp32, summed in slot order in fp32 and divided once by
 * the real-token count (the block summary the coarse stage scores; "FastVideo
 * VSA", introduction).  x and x_tiled must not overlap.
 */
VSA_API int vsa_tile(vsa_plan_t plan, const uint16_t *x, uint16_t *x_tiled, float *pooled,
             int B, int H, int D, vsa_stream_t stream);

/* vsa_tile for either 16-bit format (the pooled means are fp32 either way). */
VSA_API int vsa_tile_ex(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *x, uint16_t *x_tiled,
                        float *pooled, int B, int H, int D, vsa_stream_t stream);

/* Untile ("FastVideo VSA", introduction: the inverse of the regrouping into
 * contiguous blocks, back to the model's token order): x_tiled [B,H,Sp,D] ->
 * x [B,S,H,D]; padded rows are dropped.  A pure 16-bit copy: the same call
 * serves bf16 and fp16. */
VSA_API int vsa_untile(vsa_plan_t plan, const uint16_t *x_tiled, uint16_t *x, int B, int H, int D,
               vsa_stream_t stream);

/*
 * Coarse stage ("FastVideo VSA", introduction and section "Choose top-k"):
 * score[i][j] = qbar[i] . kbar[j] (fp32, one fused multiply-add per channel
 * in channel order) for every (b, h); every query block i keeps the topk
 * largest scores, ties to the lower block index, written to
 * q2k_idx [B,H,NB,topk] in ascending block order; q2k_num [B,H,NB] = topk.
 * qbar, kbar: [B,H,NB,D] fp32 as produced by vsa_tile.  0 < topk <= NB,
 * else VSA_ERR_TOPK; VSA_ERR_UNSUPPORTED for NB > 2048 (the scores of eight
 * query blocks are staged in shared memory) or D != 128.
 */
VSA_API int vsa_coarse_topk(vsa_plan_t plan, const float *qbar, const float *kbar, int B, int H, int D,
                    int topk, int32_t *q2k_idx, int32_t *q2k_num, vsa_stream_t stream);

/*
 * Coarse stage with its compression branch ("FastVideo VSA", section
 * "Checkpoint behavior": checkpoints carry a learned gate_compress
 * projection; FastVideo commit log: the gate-compress branch pools per tile).
 * The pages print no formula; this call computes the plainest reading:
 *   o_compress[r] = sum_c softmax_c(D^-1/2 qbar[r] . kbar[c]) vbar[c]
 * over all NB blocks of each (b, h), from the fp32 scores vsa_coarse_topk
 * ranks (fp32 weights and accumulation).
 *   qbar, kbar, vbar : [B,H,NB,D] fp32 block means (vsa_tile / vsa_tile_ex
 *                      with pooled output, for q, k and v)
 *   o_compress       : [B,H,NB,D] fp32, caller-owned
 *   topk > 0         : also the selection of vsa_coarse_topk into q2k_idx
 *                      [B,H,NB,topk] / q2k_num [B,H,NB], same results bit for bit;
 *   topk == 0        : the branch alone (selection from a block map);
 *                      q2k_idx and q2k_num must then be NULL.
 * Errors: VSA_ERR_TOPK for topk < 0 or topk > NB; VSA_ERR_INVALID_ARG for a
 * null or misaligned pointer, or index outputs given with topk == 0;
 * VSA_ERR_UNSUPPORTED for NB > 2048 or D != 128.
 */
VSA_API int vsa_coarse_compress(vsa_plan_t plan, const float *qbar, const float *kbar, const float *vbar,
                                int B, int H, int D, int topk, int32_t *q2k_idx, int32_t *q2k_num,
                                float *o_compress, vsa_stream_t stream);

/*
 * Untile fused with the gated sum of the two branches (same reading as
 * vsa_coarse_compress): for every real token s of block r,
 *   o[b,s,h,:] = o_tiled[b,h,slot(s),:] + gate[b,s,h,:] * o_compress[b,h,r,:]
 * one fp32 fused multiply-add per channel, rounded once to dtype.
 *   o_tiled    : tiled [B,H,Sp,D] (the fine stage's o), dtype
 *   o_compress : [B,H,NB,D] fp32 (vsa_coarse_compress)
 *   gate       : [B,S,H,D] dtype, untiled (the caller's gate_compress projection)
 *   o          : [B,S,H,D] dtype, caller-owned; must not overlap the inputs
 */
VSA_API int vsa_untile_gate(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *o_tiled, const float *o_compress,
                            const uint16_t *gate, uint16_t *o, int B, int H, int D, vsa_stream_t stream);

/*
 * The front end in one launch: vsa_tile_ex of q, k and v (block means of q
 * and k always, of v when vbar is not NULL) followed, per head, by the coarse
 * stage of vsa_coarse_topk (topk > 0) and/or the compression branch of
 * vsa_coarse_compress (vbar and o_compress not NULL).  Every output is bit
 * for bit the one the separate calls write.  topk == 0 with vbar == NULL
 * tiles only (selection from a block map).
 *   q, k, v                : [B,S,H,D] dtype
 *   q_tiled, k_tiled, v_tiled : [B,H,Sp,D] dtype, caller-owned
 *   qbar, kbar (, vbar)    : [B,H,NB,D] fp32, caller-owned
 *   q2k_idx, q2k_num       : as vsa_coarse_topk (NULL when topk == 0)
 *   o_compress             : [B,H,NB,D] fp32 (NULL exactly when vbar is NULL)
 *   workspace              : 2*B*H int32 of device memory, zero before the
 *                            first call; each call leaves it zero unless it
 *                            reports VSA_ERR_TIMEOUT, after which the caller
 *                            zeroes it again.  Calls that share a workspace
 *                            must not run concurrently.
 * The scoring of a head waits (at most 2 s) for the tiling of that head
 * inside the same launch; on expiry the status word holds VSA_ERR_TIMEOUT.
 * Errors: as vsa_tile_ex and vsa_coarse_compress; VSA_ERR_INVALID_ARG for a
 * null or misaligned workspace.
 */
VSA_API int vsa_tile_coarse(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                            const uint16_t *v, int B, int H, int D, int topk, uint16_t *q_tiled,
                            uint16_t *k_tiled, uint16_t *v_tiled, float *qbar, float *kbar, float *vbar,
                            int32_t *q2k_idx, int32_t *q2k_num, float *o_compress, int32_t *workspace,
                            vsa_stream_t stream);

/*
 * vsa_tile_coarse without a caller workspace: the arrival counters live in
 * a static device array of the library (2 int32 per (b, h), B*H <= 4096,
 * 32 KB per device), cleared by an asynchronous memset on `stream` before
 * each launch.  The call allocates no memory.  The pages have no
 * counterpart: it is an API convenience of this library.
 *   Same arguments, outputs and errors as vsa_tile_coarse, minus workspace;
 *   VSA_ERR_UNSUPPORTED when B*H > 4096.
 *   Calls on one device share the one array: calls that may overlap (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.
 *   The first call on a device looks up the array's address (host-side
 *   set-up); make that first call before any stream capture.
 */
VSA_API int vsa_tile_coarse_static(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                                   const uint16_t *v, int B, int H, int D, int topk, uint16_t *q_tiled,
                                   uint16_t *k_tiled, uint16_t *v_tiled, float *qbar, float *kbar, float *vbar,
                                   int32_t *q2k_idx, int32_t *q2k_num, float *o_compress, vsa_stream_t stream);

/*
 * Coarse stage of the tile-64 layout (FastVideo commit log,
 * examples/inference/basic/README.md: prefix query tiles attend every tile,
 * video query tiles attend the prefix plus a top-k of the video tiles, and
 * some rows select nothing).  With the plan's n_pre prefix tiles (blocks
 * 0 .. n_pre-1) and the block scores of vsa_coarse_topk:
 *   - a row whose row_keep byte is 0 selects nothing: count 0;
 *   - a prefix query tile (row < n_pre) selects every block: count NB;
 *   - a video query tile selects blocks 0 .. n_pre-1 and the topk video
 *     blocks of highest score among n_pre .. NB-1 (ties to the lower block
 *     index): count n_pre + topk.
 * Ids are written ascending; entries past a row's count are -1.
 *   qbar, kbar : [B,H,NB,D] fp32 block means (vsa_tile)
 *   row_keep   : [B,H,NB] bytes (0 = forced empty) or NULL (every row kept)
 *   max_k      : row stride of q2k_idx; at least NB when the plan has prefix
 *                tiles, else at least topk
 *   q2k_idx    : [B,H,NB,max_k] int32, q2k_num: [B,H,NB] int32, caller-owned
 * Without prefix tiles and with every row kept this is vsa_coarse_topk with
 * a row stride of max_k.
 * Errors: VSA_ERR_TOPK unless 0 < topk <= NB - n_pre; VSA_ERR_INVALID_ARG for
 * a max_k below the longest row or a null / misaligned pointer;
 * VSA_ERR_UNSUPPORTED for NB > 2048 or D != 128.
 */
VSA_API int vsa_coarse_topk_prefix(vsa_plan_t plan, const float *qbar, const float *kbar, const uint8_t *row_keep,
                                   int B, int H, int D, int topk, int max_k, int32_t *q2k_idx, int32_t *q2k_num,
                                   vsa_stream_t stream);

/*
 * The front end in one launch with the selection of vsa_coarse_topk_prefix:
 * vsa_tile_ex of q, k and v with the block means of q and k, then, per head,
 * the tile-64 selection -- bit for bit the outputs of vsa_tile_ex and
 * vsa_coarse_topk_prefix.
 *   q, k, v                   : [B,S,H,D] dtype
 *   row_keep, topk, max_k     : as vsa_coarse_topk_prefix
 *   q_tiled, k_tiled, v_tiled : [B,H,Sp,D] dtype; qbar, kbar: [B,H,NB,D] fp32
 *   q2k_idx, q2k_num          : [B,H,NB,max_k] / [B,H,NB] int32
 *   workspace                 : as vsa_tile_coarse (2*B*H int32, zero before
 *                               the first call, zero again after each call
 *                               that did not report VSA_ERR_TIMEOUT)
 * Errors: as vsa_tile_ex and vsa_coarse_topk_prefix.
 */
VSA_API int vsa_tile_coarse_prefix(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                                   const uint16_t *v, const uint8_t *row_keep, int B, int H, int D, int topk,
                                   int max_k, uint16_t *q_tiled, uint16_t *k_tiled, uint16_t *v_tiled, float *qbar,
                                   float *kbar, int32_t *q2k_idx, int32_t *q2k_num, int32_t *workspace,
                                   vsa_stream_t stream);

/*
 * Bool block map -> index (FastVideo commit log: map_to_index):
 * map [B,H,NQ,NK] (one byte per entry, non-zero = selected) ->
 * q2k_idx [B,H,NQ,NK] (selected ids ascending, then -1), q2k_num [B,H,NQ]
 * (0 allowed).
 */
VSA_API int vsa_map_to_index(const uint8_t *map, int B, int H, int NQ, int NK, int32_t *q2k_idx,
                     int32_t *q2k_num, vsa_stream_t stream);

/*
 * Fine stage ("FastVideo VSA", introduction and section "Verify routing and
 * fallback"; FastVideo commit log for non-uniform and zero-count rows):
 * for every query token i of block r, attention over the real tokens of
 * blocks q2k_idx[r, 0 .. q2k_num[r]-1] with scale D^-1/2, non-causal.
 *   q, k, v  : tiled [B,H,Sp,D] bf16
 *   q2k_idx  : [B,H,NB,max_k] int32;  q2k_num: [B,H,NB] int32
 *   o        : tiled [B,H,Sp,D] bf16; lse: [B,H,Sp] fp32, natural log of
 *              sum_j exp(scale q.k_j).  A row of count 0 gives o = 0 and
 *              lse = -inf.  Padded query rows are computed like any other.
 * bf16 products, fp32 accumulation and fp32 online softmax.
 * Block ids outside [0, NB) are skipped and counts outside [0, max_k] are
 * clamped; both set VSA_ERR_BAD_INDEX in the device status word.
 * For 64-token blocks the block count must be even.
 */
VSA_API int vsa_sparse_attn_fwd(vsa_plan_t plan, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *q2k_idx, const int32_t *q2k_num, int max_k,
                        int B, int H, int D, uint16_t *o, float *lse, vsa_stream_t stream);

/* vsa_sparse_attn_fwd for either 16-bit format: q, k, v and o share dtype
 * (fp16: the softmax numerators are rounded to fp16 for the PV product). */
VSA_API int vsa_sparse_attn_fwd_ex(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                                   const uint16_t *v, const int32_t *q2k_idx, const int32_t *q2k_num,
                                   int max_k, int B, int H, int D, uint16_t *o, float *lse,
                                   vsa_stream_t stream);

/*
 * vsa_sparse_attn_fwd_ex with a caller workspace that lets the 64-token
 * fine stage (four query blocks per work item, two per 128-row query tile,
 * each query tile over the union of its two selections) hand out its work
 * items from a shared queue -- the items whose
 * query blocks are prefix tiles (dense under the tile-64 rule) first -- instead
 * of a fixed item-to-CTA assignment.  Same results bit for bit; the schedule
 * is this library's, the pages have no counterpart.
 *   workspace : 2 int32 of device memory, 16-byte aligned, caller-owned, zero
 *               before the first call; each call leaves it zero unless it
 *               reports VSA_ERR_TIMEOUT, after which the caller zeroes it
 *               again.  Calls that share a workspace must not run
 *               concurrently.  Unused by 256-token plans.
 * Errors: as vsa_sparse_attn_fwd_ex; VSA_ERR_INVALID_ARG for a null or
 * misaligned workspace.
 */
VSA_API int vsa_sparse_attn_fwd_ws(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                                   const uint16_t *v, const int32_t *q2k_idx, const int32_t *q2k_num, int max_k,
                                   int B, int H, int D, uint16_t *o, float *lse, int32_t *workspace,
                                   vsa_stream_t stream);

/*
 * NVFP4 quantisation of tiled Q or K (FastVideo "Optimizations" page, section
 * "FP4 Flash Attention 4 (Blackwell only)": Q and K as NVFP4: 4-bit E2M1 codes, one
 * E4M3 scale per block of channels; block length and scale rule are NVFP4's own).
 * For every 16-channel block of a row: s = E4M3(fl32(amax / 6)) and each
 * value's code = E2M1(fl32(x * fl32(1 / s))) (1/s := 0 when s is 0); both
 * roundings to nearest, ties to even, saturating (448, 6); E2M1 keeps the
 * sign, zero included.
 *   x_tiled : tiled [B,H,Sp,D] dtype
 *   codes   : [B,H,Sp,D/2] bytes, caller-owned; channel 2j in the low nibble
 *             of byte j, 2j+1 in the high nibble
 *   scales  : B*H*Sp*D/16 bytes, caller-owned, in the tensor core's layout:
 *             for each (b, h) and each 128-row tile t of the head's Sp rows,
 *             1024 bytes; byte kh*512 + (r%32)*16 + (r/32)*4 + j holds the
 *             scale of row 128t + r, channels 16(4kh + j) .. 16(4kh + j) + 15
 * Sp must be a multiple of 128 (always for 256-token blocks; an even block
 * count for 64-token blocks), else VSA_ERR_UNSUPPORTED.
 */
VSA_API int vsa_quantize_nvfp4(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *x_tiled, int B, int H, int D,
                               uint8_t *codes, uint8_t *scales, vsa_stream_t stream);

/*
 * Fine stage with NVFP4 Q and K (same page and section): the attention of
 * vsa_sparse_attn_fwd_ex computed on the values the codes stand for,
 * q_i = s_q * e2m1(code), k_j likewise; S = Q K^T runs as a block-scaled FP4
 * product with fp32 accumulation, P and V stay 16-bit (dtype).
 *   q_codes, q_scales, k_codes, k_scales : from vsa_quantize_nvfp4
 *   v, o : tiled [B,H,Sp,D] dtype;  lse: [B,H,Sp] fp32
 *   q2k_idx, q2k_num, max_k : as in vsa_sparse_attn_fwd
 * Same error behaviour as vsa_sparse_attn_fwd; Sp must be a multiple of 128.
 */
VSA_API int vsa_sparse_attn_fwd_nvfp4(vsa_plan_t plan, vsa_dtype_t dtype, const uint8_t *q_codes,
                                      const uint8_t *q_scales, const uint8_t *k_codes, const uint8_t *k_scales,
                                      const uint16_t *v, const int32_t *q2k_idx, const int32_t *q2k_num, int max_k,
                                      int B, int H, int D, uint16_t *o, float *lse, vsa_stream_t stream);

/*
 * vsa_sparse_attn_fwd_nvfp4 with a caller workspace: for 64-token plans of at
 * most 1024 blocks (four query blocks per work item) the items are handed out
 * from a shared queue, prefix groups first, as in vsa_sparse_attn_fwd_ws.
 * Same results bit for bit.
 *   workspace : 2 int32 of device memory, 16-byte aligned, caller-owned, zero
 *               before the first call; each call leaves it zero unless it
 *               reports VSA_ERR_TIMEOUT.  Calls that share a workspace must not
 *               run concurrently.  Unused by 256-token plans.
 * Errors: as vsa_sparse_attn_fwd_nvfp4; VSA_ERR_INVALID_ARG for a null or
 * misaligned workspace.
 */
VSA_API int vsa_sparse_attn_fwd_nvfp4_ws(vsa_plan_t plan, vsa_dtype_t dtype, const uint8_t *q_codes,
                                         const uint8_t *q_scales, const uint8_t *k_codes, const uint8_t *k_scales,
                                         const uint16_t *v, const int32_t *q2k_idx, const int32_t *q2k_num,
                                         int max_k, int B, int H, int D, uint16_t *o, float *lse,
                                         int32_t *workspace, vsa_stream_t stream);

/*
 * Backward of the fine stage with the selection held fixed (the FastVideo
 * commit log keeps the grad path on separate kernels; the pages print no
 * formula, so this is the derivative of the fine stage): with
 * P = softmax(D^-1/2 q k^T) over each row's selected real keys,
 *   dv = P^T do,  dS = P (do v^T - rowsum(do * o)),
 *   dq = D^-1/2 dS k,  dk = D^-1/2 dS^T q.
 *   q, k, v, o, dO : tiled [B,H,Sp,D] dtype (o and lse from the forward call
 *                    with the same q2k_idx / q2k_num)
 *   lse            : [B,H,Sp] fp32 from the forward call
 *   dq, dk, dv     : tiled [B,H,Sp,D] dtype, caller-owned; padded rows get 0
 *                    and the dO of padded rows is ignored
 *   workspace      : device memory of vsa_sparse_attn_bwd_workspace bytes,
 *                    caller-owned, contents need not be initialised
 * 16-bit operands (P, dS rounded to dtype for the tensor cores), fp32
 * accumulation.  Both block sizes (256 tokens, and the 64-token tiles of the
 * FastVideo commit log's layout).
 * Block ids outside [0, NB) and counts outside [0, max_k] are skipped /
 * clamped and set VSA_ERR_BAD_INDEX in the device status word.
 * VSA_ERR_UNSUPPORTED for NB > 28672 (the transposed selection of a head is
 * built in shared memory, 8 bytes per block) or D != 128.
 */
VSA_API int vsa_sparse_attn_bwd_workspace(vsa_plan_t plan, int B, int H, int max_k, size_t *bytes);
VSA_API int vsa_sparse_attn_bwd(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t *q, const uint16_t *k,
                                const uint16_t *v, const uint16_t *o, const float *lse, const uint16_t *dO,
                                const int32_t *q2k_idx, const int32_t *q2k_num, int max_k, int B, int H, int D,
                                uint16_t *dq, uint16_t *dk, uint16_t *dv, void *workspace, vsa_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the status word of the current
 * device: *device_status receives VSA_OK or the first device-detected error
 * (VSA_ERR_BAD_INDEX, VSA_ERR_TIMEOUT) since the last read.
 */
VSA_API int vsa_get_status(vsa_stream_t stream, int *device_status);

/* Static text for a status code. */
VSA_API const char *vsa_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */
