/*
 * vsa_oracle.c -- plain CPU oracle of the Video Sparse Attention forward path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header, table or helper with the CUDA library, and neither calls the other.
 *
 * What it computes, step by step, and where each step is stated:
 *
 *  geometry  "FastVideo VSA" (vLLM-Omni user guide), section "Choose top-k":
 *            the post-patch latent grid (T, H, W) is cut into blocks of
 *            (4, 8, 8) tokens; num_blocks counts the zero-padded grid, e.g.
 *            (31, 22, 40) -> 8 * 3 * 5 = 120.  A prefix of n_prefix tokens
 *            (the tile-64 layout of the FastVideo commit log,
 *            examples/inference/basic/README.md) is cut into contiguous tiles
 *            placed before the video blocks.
 *  tile      same page, introduction: tokens are regrouped so that every
 *            spatiotemporal block is contiguous.  Blocks are in raster order
 *            over (bT, bH, bW); tokens inside a block in raster order over
 *            (lt, lh, lw); padding sits at its grid coordinates and is zero.
 *  pool      same page, introduction ("for every query block, VSA scores the
 *            key/value blocks"): a block is summarised by the mean of its
 *            valid tokens.  Sum in slot order in fp32, then one fp32 division.
 *  score     block score = pooled q . pooled k, one fused multiply-add per
 *            channel in channel order, fp32 (no scale: ranking ignores it).
 *  top-k     same page, sections "Enable the backend" and "Choose top-k":
 *            each query block keeps its topk highest-scoring key blocks,
 *            0 < topk <= num_blocks; ties go to the lower block index; the
 *            kept indices are written in ascending order.
 *  map       FastVideo commit log: a bool block map [B,H,NQ,NK] is compacted
 *            into q2k_idx (ascending, -1 padded) and q2k_num (may be 0).
 *  prefix    FastVideo commit log, the tile-64 layout: prefix query tiles
 *  top-k     attend every tile; a video query tile attends the prefix tiles
 *            plus the top-k video tiles by the same block score (same tie
 *            rule); rows the caller marks are forced empty (count 0).
 *  attention "FastVideo VSA", sections introduction and "Verify routing and
 *            fallback": non-causal attention of every query token of a block
 *            against the valid tokens of its selected blocks only, scale
 *            head_size^-1/2, equal Q/KV lengths and head counts, no mask.
 *            Computed in double from the bf16 inputs.  A row with count 0
 *            gives o = 0 and lse = -inf (commit log: zero-count rows).
 *  untile    inverse of tile; padded rows are dropped.
 *  backward  the gradients of the attention step with the selection held
 *            fixed (the commit log keeps the grad path on its own kernels; the
 *            pages print no formula, so this is the definition): with
 *            P_ij = softmax_j(scale q_i.k_j) over row i's keys,
 *            dv_j = sum_i P_ij do_i, dP_ij = do_i.v_j,
 *            dS_ij = P_ij (dP_ij - sum_l P_il dP_il),
 *            dq_i = scale sum_j dS_ij k_j, dk_j = scale sum_i dS_ij q_i,
 *            summed over the real query rows only (padded rows are not
 *            outputs of the method), in double.
 *  compress  "FastVideo VSA", section "Checkpoint behavior", and the FastVideo
 *            commit log (the gate-compress branch pools per tile): the pages
 *            name a learned gate_compress projection and a branch that pools
 *            per block but print no formula.  Reading taken: the branch is
 *            dense attention among the pooled blocks of a head,
 *            o_c[r] = sum_c softmax_c(scale qbar_r . kbar_c) vbar_c, in double
 *            from the fp32 block means; every token of block r receives
 *            o_c[r], scaled channel-wise by the caller's gate and added to the
 *            sparse branch: o_i = o_fine_i + gate_i * o_c[block(i)].
 *
 * bf16 / fp16 tensors are passed as their raw 16-bit patterns (the page
 * names "FP16 or BF16" inputs; pool and attention take a dtype flag).  Build with
 * -ffp-contract=off so that every fp32 operation rounds as written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_INDEX 2
#define ORACLE_ERR_NOMEM 3

typedef struct {
    int n_prefix, T, Hg, Wg, bt, bh, bw;
    int bs;           /* tokens per block */
    int nT, nH, nW;   /* blocks along each grid axis */
    int n_pre;        /* prefix tiles */
    int NB;           /* total blocks */
    long S;           /* real tokens */
    long Sp;          /* padded tokens = NB * bs */
} geom_t;

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

static int geom_init(geom_t *g, int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw) {
    if (n_prefix < 0 || T < 1 || Hg < 1 || Wg < 1 || bt < 1 || bh < 1 || bw < 1) return ORACLE_ERR_ARG;
    g->n_prefix = n_prefix; g->T = T; g->Hg = Hg; g->Wg = Wg;
    g->bt = bt; g->bh = bh; g->bw = bw;
    g->bs = bt * bh * bw;
    g->nT = ceil_div(T, bt); g->nH = ceil_div(Hg, bh); g->nW = ceil_div(Wg, bw);
    g->n_pre = ceil_div(n_prefix, g->bs);
    g->NB = g->n_pre + g->nT * g->nH * g->nW;
    g->S = (long)n_prefix + (long)T * Hg * Wg;
    g->Sp = (long)g->NB * g->bs;
    return ORACLE_OK;
}

/* out[0..7] = bs, nT, nH, nW, n_pre, NB, S, Sp */
int oracle_geometry(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw, long *out) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    out[0] = g.bs; out[1] = g.nT; out[2] = g.nH; out[3] = g.nW; out[4] = g.n_pre;
    out[5] = g.NB; out[6] = g.S; out[7] = g.Sp;
    return ORACLE_OK;
}

/* Position in the tiled sequence of untiled token s. */
static long tiled_pos_of_token(const geom_t *g, long s) {
    if (s < g->n_prefix) return s; /* prefix tiles are contiguous and come first */
    long v = s - g->n_prefix;
    int x = (int)(v % g->Wg);
    int y = (int)((v / g->Wg) % g->Hg);
    int t = (int)(v / ((long)g->Wg * g->Hg));
    int bT = t / g->bt, lt = t % g->bt;
    int bH = y / g->bh, lh = y % g->bh;
    int bW = x / g->bw, lw = x % g->bw;
    long blk = (long)g->n_pre + ((long)bT * g->nH + bH) * g->nW + bW;
    long slot = ((long)lt * g->bh + lh) * g->bw + lw;
    return blk * g->bs + slot;
}

/* Whether slot `slot` of block `blk` holds a real token (else it is padding). */
static int slot_is_valid(const geom_t *g, int blk, int slot) {
    if (blk < g->n_pre) return (long)blk * g->bs + slot < g->n_prefix;
    int vb = blk - g->n_pre;
    int bW = vb % g->nW, bH = (vb / g->nW) % g->nH, bT = vb / (g->nW * g->nH);
    int lw = slot % g->bw, lh = (slot / g->bw) % g->bh, lt = slot / (g->bw * g->bh);
    return bT * g->bt + lt < g->T && bH * g->bh + lh < g->Hg && bW * g->bw + lw < g->Wg;
}

static int block_valid_count(const geom_t *g, int blk) {
    int c = 0;
    for (int s = 0; s < g->bs; ++s) c += slot_is_valid(g, blk, s);
    return c;
}

int oracle_block_valid_counts(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw, int *counts) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    for (int b = 0; b < g.NB; ++b) counts[b] = block_valid_count(&g, b);
    return ORACLE_OK;
}

static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE binary16 -> float: sign, 5-bit exponent (bias 15), 10-bit fraction;
 * exponent 0 is subnormal (fraction * 2^-24), exponent 31 is inf/nan. */
static float f16_to_f32(uint16_t h) {
    const int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, e - 15);
    return (float)(sign ? -v : v);
}

/* dtype 0: bf16, 1: fp16 (the kernel takes "FP16 or BF16" inputs). */
static float half_to_f32(uint16_t h, int dtype) { return dtype ? f16_to_f32(h) : bf16_to_f32(h); }

int oracle_half_to_f32(const uint16_t *x, float *y, long n, int dtype) {
    for (long i = 0; i < n; ++i) y[i] = half_to_f32(x[i], dtype);
    return ORACLE_OK;
}

/* tile: x [B,S,H,D] -> xt [B,H,Sp,D]; padded rows are zero. */
int oracle_tile(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                const uint16_t *x, uint16_t *xt, int B, int H, int D) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    memset(xt, 0, sizeof(uint16_t) * (size_t)B * H * g.Sp * D);
    for (int b = 0; b < B; ++b)
        for (long s = 0; s < g.S; ++s) {
            long p = tiled_pos_of_token(&g, s);
            for (int h = 0; h < H; ++h)
                memcpy(xt + (((size_t)b * H + h) * g.Sp + p) * D,
                       x + (((size_t)b * g.S + s) * H + h) * D, sizeof(uint16_t) * D);
        }
    return ORACLE_OK;
}

/* untile: xt [B,H,Sp,D] -> x [B,S,H,D]; padded rows are dropped. */
int oracle_untile(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                  const uint16_t *xt, uint16_t *x, int B, int H, int D) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    for (int b = 0; b < B; ++b)
        for (long s = 0; s < g.S; ++s) {
            long p = tiled_pos_of_token(&g, s);
            for (int h = 0; h < H; ++h)
                memcpy(x + (((size_t)b * g.S + s) * H + h) * D,
                       xt + (((size_t)b * H + h) * g.Sp + p) * D, sizeof(uint16_t) * D);
        }
    return ORACLE_OK;
}

/* pool: xt [B,H,Sp,D] -> pooled [B,H,NB,D] fp32 mean over the valid slots,
 * summed in slot order with one fp32 rounding per addition. */
int oracle_pool(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                const uint16_t *xt, float *pooled, int B, int H, int D, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
#pragma omp parallel for schedule(static)
    for (int bhh = 0; bhh < B * H; ++bhh)
        for (int blk = 0; blk < g.NB; ++blk) {
            int count = block_valid_count(&g, blk);
            for (int d = 0; d < D; ++d) {
                float s = 0.0f;
                for (int slot = 0; slot < g.bs; ++slot)
                    if (slot_is_valid(&g, blk, slot))
                        s = s + half_to_f32(xt[((size_t)bhh * g.Sp + (size_t)blk * g.bs + slot) * D + d], dtype);
                pooled[((size_t)bhh * g.NB + blk) * D + d] = s / (float)count;
            }
        }
    return ORACLE_OK;
}

/* score: s[b,h,i,j] = sum_d qbar[i,d] * kbar[j,d], fused multiply-add in d order. */
int oracle_score(const float *qbar, const float *kbar, float *s, int B, int H, int NB, int D) {
#pragma omp parallel for schedule(static)
    for (int bhh = 0; bhh < B * H; ++bhh)
        for (int i = 0; i < NB; ++i)
            for (int j = 0; j < NB; ++j) {
                const float *qi = qbar + ((size_t)bhh * NB + i) * D;
                const float *kj = kbar + ((size_t)bhh * NB + j) * D;
                float acc = 0.0f;
                for (int d = 0; d < D; ++d) acc = fmaf(qi[d], kj[d], acc);
                s[((size_t)bhh * NB + i) * NB + j] = acc;
            }
    return ORACLE_OK;
}

typedef struct { float v; int j; } scored_t;

/* Descending score; equal scores keep the lower block index first. */
static int by_score_then_index(const void *a, const void *b) {
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int by_index(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* top-k: s [B,H,NB,NB] -> idx [B,H,NB,topk] ascending, num [B,H,NB] = topk. */
int oracle_topk(const float *s, int B, int H, int NB, int topk, int32_t *idx, int32_t *num) {
    if (topk < 1 || topk > NB) return ORACLE_ERR_ARG;
    scored_t *row = (scored_t *)malloc(sizeof(scored_t) * NB);
    int *keep = (int *)malloc(sizeof(int) * topk);
    if (!row || !keep) { free(row); free(keep); return ORACLE_ERR_NOMEM; }
    for (long r = 0; r < (long)B * H * NB; ++r) {
        for (int j = 0; j < NB; ++j) { row[j].v = s[r * NB + j]; row[j].j = j; }
        qsort(row, NB, sizeof(scored_t), by_score_then_index);
        for (int t = 0; t < topk; ++t) keep[t] = row[t].j;
        qsort(keep, topk, sizeof(int), by_index);
        for (int t = 0; t < topk; ++t) idx[r * topk + t] = keep[t];
        num[r] = topk;
    }
    free(row);
    free(keep);
    return ORACLE_OK;
}

/*
 * top-k with dense prefix tiles (FastVideo commit log: in the tile-64 layout
 * the prefix query tiles attend every tile and a video query tile attends the
 * prefix plus the top-k of the video tiles; some rows are forced empty).
 *   s        : [B,H,NB,NB] block scores (oracle_score)
 *   n_pre    : prefix tiles, blocks 0 .. n_pre-1
 *   topk     : video tiles kept per video query tile, 0 < topk <= NB - n_pre
 *   row_keep : [B,H,NB] bytes or NULL; a row whose byte is 0 selects nothing
 *   max_k    : row stride of idx, at least the longest row (NB when n_pre > 0)
 * A prefix query tile lists every tile (count NB).  A video query tile lists
 * the prefix tiles, then the topk video tiles of highest score, ties to the
 * lower index: count n_pre + topk, all ids ascending.  Unused entries are -1.
 */
int oracle_topk_prefix(const float *s, int B, int H, int NB, int n_pre, int topk, const uint8_t *row_keep,
                       int max_k, int32_t *idx, int32_t *num) {
    int nvid = NB - n_pre;
    if (n_pre < 0 || nvid < 1 || topk < 1 || topk > nvid) return ORACLE_ERR_ARG;
    if (max_k < (n_pre > 0 ? NB : topk)) return ORACLE_ERR_ARG;
    scored_t *row = (scored_t *)malloc(sizeof(scored_t) * nvid);
    int *keep = (int *)malloc(sizeof(int) * topk);
    if (!row || !keep) { free(row); free(keep); return ORACLE_ERR_NOMEM; }
    for (long r = 0; r < (long)B * H * NB; ++r) {
        int32_t *out = idx + r * max_k;
        int blk = (int)(r % NB), c = 0;
        if (row_keep && !row_keep[r]) {
            c = 0;
        } else if (blk < n_pre) {
            for (int j = 0; j < NB; ++j) out[c++] = j;
        } else {
            for (int j = 0; j < n_pre; ++j) out[c++] = j;
            for (int j = 0; j < nvid; ++j) { row[j].v = s[r * NB + n_pre + j]; row[j].j = n_pre + j; }
            qsort(row, nvid, sizeof(scored_t), by_score_then_index);
            for (int t = 0; t < topk; ++t) keep[t] = row[t].j;
            qsort(keep, topk, sizeof(int), by_index);
            for (int t = 0; t < topk; ++t) out[c++] = keep[t];
        }
        for (int j = c; j < max_k; ++j) out[j] = -1;
        num[r] = c;
    }
    free(row);
    free(keep);
    return ORACLE_OK;
}

/* map_to_index: map [B,H,NQ,NK] bool -> idx [B,H,NQ,NK] (ascending, -1 padded), num. */
int oracle_map_to_index(const uint8_t *map, int B, int H, int NQ, int NK, int32_t *idx, int32_t *num) {
    for (long r = 0; r < (long)B * H * NQ; ++r) {
        int c = 0;
        for (int j = 0; j < NK; ++j)
            if (map[r * NK + j]) idx[r * NK + c++] = j;
        for (int j = c; j < NK; ++j) idx[r * NK + j] = -1;
        num[r] = c;
    }
    return ORACLE_OK;
}

/*
 * attention on selected blocks, for an explicit list of query rows.
 *   q, k, v : tiled [B,H,Sp,D] bf16 bits
 *   idx     : [B,H,NB,max_k] block ids; num: [B,H,NB] counts
 *   rows    : flat indices into [B,H,Sp]; o_rows [n_rows, D], lse_rows [n_rows]
 * For query token i of block r: keys are the valid slots of blocks
 * idx[r, 0..num[r]-1]; o_i = sum_j softmax_j(scale q_i.k_j) v_j,
 * lse_i = log sum_j exp(scale q_i.k_j), scale = 1/sqrt(D).
 */
/* Where the q or k operand of the attention lives: 16-bit patterns, or NVFP4
 * codes and scales (nvfp4_value below). */
typedef struct {
    const uint16_t *bits;
    const uint8_t *codes, *sf;
    int dtype;
} operand_t;

static double nvfp4_value(const uint8_t *codes, const uint8_t *sf, size_t row, int D, int d);

/* Element d of tiled row `row` (flat over [B,H,Sp]) of an operand. */
static double operand_value(const operand_t *op, size_t row, int D, int d) {
    if (op->bits) return half_to_f32(op->bits[row * D + d], op->dtype);
    return nvfp4_value(op->codes, op->sf, row, D, d);
}

static int attn_rows_core(const geom_t *gp, const operand_t *qop, const operand_t *kop, const uint16_t *v,
                          const int32_t *idx, const int32_t *num, int max_k, int D, const int64_t *rows,
                          long n_rows, double *o_rows, double *lse_rows, int dtype);

int oracle_attn_rows(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                     const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *idx, const int32_t *num, int max_k,
                     int B, int H, int D, const int64_t *rows, long n_rows,
                     double *o_rows, double *lse_rows, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    (void)B; (void)H; /* rows are flat indices into [B,H,Sp] */
    const operand_t qop = {q, NULL, NULL, dtype}, kop = {k, NULL, NULL, dtype};
    return attn_rows_core(&g, &qop, &kop, v, idx, num, max_k, D, rows, n_rows, o_rows, lse_rows, dtype);
}

static int attn_rows_core(const geom_t *gp, const operand_t *qop, const operand_t *kop, const uint16_t *v,
                          const int32_t *idx, const int32_t *num, int max_k, int D, const int64_t *rows,
                          long n_rows, double *o_rows, double *lse_rows, int dtype) {
    const geom_t g = *gp;
    if (D < 1 || D > 512 || max_k < 1) return ORACLE_ERR_ARG;
    const double scale = 1.0 / sqrt((double)D);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
    for (long n = 0; n < n_rows; ++n) {
        long flat = rows[n];
        long i = flat % g.Sp;
        long bhh = flat / g.Sp;
        int rblk = (int)(i / g.bs);
        int cnt = num[bhh * g.NB + rblk];
        double *o = o_rows + (size_t)n * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (cnt <= 0 || cnt > max_k) {
            lse_rows[n] = -INFINITY;
            if (cnt != 0) bad = 1;
            continue;
        }
        double qi[512];
        for (int d = 0; d < D; ++d) qi[d] = operand_value(qop, (size_t)bhh * g.Sp + i, D, d);
        double *logit = (double *)malloc(sizeof(double) * (size_t)cnt * g.bs);
        long *key = (long *)malloc(sizeof(long) * (size_t)cnt * g.bs);
        long nk = 0;
        for (int t = 0; t < cnt; ++t) {
            int kb = idx[(bhh * g.NB + rblk) * (long)max_k + t];
            if (kb < 0 || kb >= g.NB) { bad = 1; continue; }
            for (int slot = 0; slot < g.bs; ++slot) {
                if (!slot_is_valid(&g, kb, slot)) continue;
                long j = (long)kb * g.bs + slot;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += qi[d] * operand_value(kop, (size_t)bhh * g.Sp + j, D, d);
                logit[nk] = scale * dot;
                key[nk] = j;
                ++nk;
            }
        }
        if (nk == 0) {
            lse_rows[n] = -INFINITY;
        } else {
            double m = -INFINITY;
            for (long t = 0; t < nk; ++t) if (logit[t] > m) m = logit[t];
            double l = 0.0;
            for (long t = 0; t < nk; ++t) {
                double p = exp(logit[t] - m);
                l += p;
                const uint16_t *vj = v + ((size_t)bhh * g.Sp + key[t]) * D;
                for (int d = 0; d < D; ++d) o[d] += p * (double)half_to_f32(vj[d], dtype);
            }
            for (int d = 0; d < D; ++d) o[d] /= l;
            lse_rows[n] = m + log(l);
        }
        free(logit);
        free(key);
    }
    return bad ? ORACLE_ERR_INDEX : ORACLE_OK;
}

/* Softmax of one query row over its selected keys, in double.  Fills the key
 * rows (tiled indices) and P; returns the key count, -1 on a bad block id. */
static long row_softmax(const geom_t *g, const uint16_t *q, const uint16_t *k, const int32_t *idx,
                        const int32_t *num, int max_k, int D, long bhh, long i, int dtype,
                        long *key, double *p) {
    int rblk = (int)(i / g->bs);
    int cnt = num[bhh * g->NB + rblk];
    if (cnt < 0 || cnt > max_k) return -1;
    const double scale = 1.0 / sqrt((double)D);
    const uint16_t *qi = q + ((size_t)bhh * g->Sp + i) * D;
    long nk = 0;
    for (int t = 0; t < cnt; ++t) {
        int kb = idx[(bhh * g->NB + rblk) * (long)max_k + t];
        if (kb < 0 || kb >= g->NB) return -1;
        for (int slot = 0; slot < g->bs; ++slot) {
            if (!slot_is_valid(g, kb, slot)) continue;
            long j = (long)kb * g->bs + slot;
            const uint16_t *kj = k + ((size_t)bhh * g->Sp + j) * D;
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += (double)half_to_f32(qi[d], dtype) * (double)half_to_f32(kj[d], dtype);
            p[nk] = scale * dot;
            key[nk] = j;
            ++nk;
        }
    }
    double m = -INFINITY;
    for (long t = 0; t < nk; ++t) if (p[t] > m) m = p[t];
    double l = 0.0;
    for (long t = 0; t < nk; ++t) { p[t] = exp(p[t] - m); l += p[t]; }
    for (long t = 0; t < nk; ++t) p[t] /= l;
    return nk;
}

/* dP_ij = do_i . v_j for the row's keys, and delta_i = sum_j P_ij dP_ij. */
static double row_dp(const uint16_t *v, const uint16_t *dO, long bhh, long i, long Sp, int D, int dtype,
                     const long *key, const double *p, long nk, double *dp) {
    const uint16_t *doi = dO + ((size_t)bhh * Sp + i) * D;
    double delta = 0.0;
    for (long t = 0; t < nk; ++t) {
        const uint16_t *vj = v + ((size_t)bhh * Sp + key[t]) * D;
        double x = 0.0;
        for (int d = 0; d < D; ++d) x += (double)half_to_f32(doi[d], dtype) * (double)half_to_f32(vj[d], dtype);
        dp[t] = x;
        delta += p[t] * x;
    }
    return delta;
}

static long max_keys(const geom_t *g, int max_k) { return (long)max_k * g->bs; }

/*
 * backward, query side: dq for an explicit list of query rows (flat indices
 * into [B,H,Sp]); padded rows give dq = 0.  dq_rows [n_rows, D] double.
 */
int oracle_attn_bwd_q_rows(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                           const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dO,
                           const int32_t *idx, const int32_t *num, int max_k, int B, int H, int D,
                           const int64_t *rows, long n_rows, double *dq_rows, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    (void)B; (void)H;
    if (D < 1 || max_k < 1) return ORACLE_ERR_ARG;
    const double scale = 1.0 / sqrt((double)D);
    int bad = 0;
#pragma omp parallel reduction(| : bad)
    {
        long *key = (long *)malloc(sizeof(long) * (size_t)max_keys(&g, max_k));
        double *p = (double *)malloc(sizeof(double) * (size_t)max_keys(&g, max_k));
        double *dp = (double *)malloc(sizeof(double) * (size_t)max_keys(&g, max_k));
        if (!key || !p || !dp) bad = 1;
#pragma omp for schedule(dynamic, 4)
        for (long n = 0; n < n_rows; ++n) {
            double *out = dq_rows + (size_t)n * D;
            for (int d = 0; d < D; ++d) out[d] = 0.0;
            if (bad) continue;
            long i = rows[n] % g.Sp, bhh = rows[n] / g.Sp;
            if (!slot_is_valid(&g, (int)(i / g.bs), (int)(i % g.bs))) continue;
            long nk = row_softmax(&g, q, k, idx, num, max_k, D, bhh, i, dtype, key, p);
            if (nk < 0) { bad = 1; continue; }
            double delta = row_dp(v, dO, bhh, i, g.Sp, D, dtype, key, p, nk, dp);
            for (long t = 0; t < nk; ++t) {
                double ds = p[t] * (dp[t] - delta) * scale;
                const uint16_t *kj = k + ((size_t)bhh * g.Sp + key[t]) * D;
                for (int d = 0; d < D; ++d) out[d] += ds * (double)half_to_f32(kj[d], dtype);
            }
        }
        free(key); free(p); free(dp);
    }
    return bad ? ORACLE_ERR_INDEX : ORACLE_OK;
}

/*
 * backward, key side: dk and dv [B,H,Sp,D] double for every key row, summed
 * over every real query row of the head (small problems only: the cost is
 * the whole attention, twice).  Padded key rows get 0.
 */
int oracle_attn_bwd_kv(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                       const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dO,
                       const int32_t *idx, const int32_t *num, int max_k, int B, int H, int D,
                       double *dk, double *dv, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    if (D < 1 || max_k < 1) return ORACLE_ERR_ARG;
    const double scale = 1.0 / sqrt((double)D);
    memset(dk, 0, sizeof(double) * (size_t)B * H * g.Sp * D);
    memset(dv, 0, sizeof(double) * (size_t)B * H * g.Sp * D);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long bhh = 0; bhh < (long)B * H; ++bhh) {
        long *key = (long *)malloc(sizeof(long) * (size_t)max_keys(&g, max_k));
        double *p = (double *)malloc(sizeof(double) * (size_t)max_keys(&g, max_k));
        double *dp = (double *)malloc(sizeof(double) * (size_t)max_keys(&g, max_k));
        if (!key || !p || !dp) { bad = 1; free(key); free(p); free(dp); continue; }
        for (long i = 0; i < g.Sp; ++i) {
            if (!slot_is_valid(&g, (int)(i / g.bs), (int)(i % g.bs))) continue;
            long nk = row_softmax(&g, q, k, idx, num, max_k, D, bhh, i, dtype, key, p);
            if (nk < 0) { bad = 1; continue; }
            double delta = row_dp(v, dO, bhh, i, g.Sp, D, dtype, key, p, nk, dp);
            const uint16_t *doi = dO + ((size_t)bhh * g.Sp + i) * D;
            const uint16_t *qi = q + ((size_t)bhh * g.Sp + i) * D;
            for (long t = 0; t < nk; ++t) {
                double *dvj = dv + ((size_t)bhh * g.Sp + key[t]) * D;
                double *dkj = dk + ((size_t)bhh * g.Sp + key[t]) * D;
                double ds = p[t] * (dp[t] - delta) * scale;
                for (int d = 0; d < D; ++d) {
                    dvj[d] += p[t] * (double)half_to_f32(doi[d], dtype);
                    dkj[d] += ds * (double)half_to_f32(qi[d], dtype);
                }
            }
        }
        free(key); free(p); free(dp);
    }
    return bad ? ORACLE_ERR_INDEX : ORACLE_OK;
}

/*
 * compression branch: dense attention among the block means of each head.
 *   qbar, kbar, vbar : [B,H,NB,D] fp32 block means
 *   out              : [B,H,NB,D] double
 * out[r] = sum_c a_rc vbar[c], a_rc = exp(z_rc - max_c z) / sum_c exp(z_rc - max_c z),
 * z_rc = scale * sum_d qbar[r,d] kbar[c,d] (double), scale = 1/sqrt(D).
 */
int oracle_compress(const float *qbar, const float *kbar, const float *vbar, int B, int H, int NB, int D,
                    double *out) {
    if (B < 1 || H < 1 || NB < 1 || D < 1) return ORACLE_ERR_ARG;
    const double scale = 1.0 / sqrt((double)D);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long row = 0; row < (long)B * H * NB; ++row) {
        long bhh = row / NB;
        const float *qr = qbar + (size_t)row * D;
        const float *kh = kbar + (size_t)bhh * NB * D;
        const float *vh = vbar + (size_t)bhh * NB * D;
        double *o = out + (size_t)row * D;
        double *z = (double *)malloc(sizeof(double) * (size_t)NB);
        if (!z) { bad = 1; continue; }
        double m = -INFINITY;
        for (int c = 0; c < NB; ++c) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += (double)qr[d] * (double)kh[(size_t)c * D + d];
            z[c] = scale * dot;
            if (z[c] > m) m = z[c];
        }
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        double l = 0.0;
        for (int c = 0; c < NB; ++c) {
            double p = exp(z[c] - m);
            l += p;
            for (int d = 0; d < D; ++d) o[d] += p * (double)vh[(size_t)c * D + d];
        }
        for (int d = 0; d < D; ++d) o[d] /= l;
        free(z);
    }
    return bad ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * gated sum of the two branches for an explicit list of real tokens.
 *   rows       : flat indices into the tiled [B,H,Sp]; the token of each must be real
 *   o_fine     : [n_rows, D] double, the sparse branch of those rows
 *   gate       : untiled [B,S,H,D] 16-bit patterns (bf16 or fp16)
 *   o_compress : [B,H,NB,D] double (oracle_compress)
 *   out        : [n_rows, D] double = o_fine + gate * o_compress[block of the row]
 */
int oracle_gate_rows(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                     const int64_t *rows, long n_rows, const double *o_fine, const uint16_t *gate,
                     const double *o_compress, int B, int H, int D, double *out, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    if (D < 1) return ORACLE_ERR_ARG;
    /* tiled slot -> real token index (or -1), built by walking the tokens */
    long *token_of_slot = (long *)malloc(sizeof(long) * (size_t)g.Sp);
    if (!token_of_slot) return ORACLE_ERR_NOMEM;
    for (long i = 0; i < g.Sp; ++i) token_of_slot[i] = -1;
    for (long s = 0; s < g.S; ++s) token_of_slot[tiled_pos_of_token(&g, s)] = s;
    int bad = 0;
    for (long n = 0; n < n_rows; ++n) {
        long flat = rows[n];
        long i = flat % g.Sp;
        long bhh = flat / g.Sp;
        long b = bhh / H, h = bhh % H;
        long s = token_of_slot[i];
        if (s < 0 || b >= B) { bad = 1; continue; }
        const uint16_t *gi = gate + (((size_t)b * g.S + s) * H + h) * D;
        const double *oc = o_compress + ((size_t)bhh * g.NB + i / g.bs) * D;
        for (int d = 0; d < D; ++d)
            out[(size_t)n * D + d] = o_fine[(size_t)n * D + d] + (double)half_to_f32(gi[d], dtype) * oc[d];
    }
    free(token_of_slot);
    return bad ? ORACLE_ERR_INDEX : ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * NVFP4 Q and K.  FastVideo "Optimizations" page, section "FP4 Flash
 * Attention 4 (Blackwell only)": Q and K go to NVFP4 -- 4-bit E2M1
 * codes, each block of channels sharing one 8-bit E4M3 scale -- and V keeps
 * its 16-bit format.  The page
 * fixes neither the block length nor how a scale is chosen; the readings
 * taken are NVFP4's own definition:
 *   - a block is 16 consecutive channels of one token;
 *   - its scale is amax / 6 (6 = the largest E2M1 magnitude), one fp32
 *     division, rounded to E4M3;
 *   - each value becomes x * (1 / scale), one fp32 reciprocal and one fp32
 *     multiply, rounded to E2M1; a scale that rounds to 0 gives 1/scale := 0.
 * Both roundings take the nearest representable value, ties to the one whose
 * last mantissa bit is 0, and stop at the largest finite value (448, 6); E2M1
 * keeps the sign of its input, zero included.
 * Formats: E4M3 = sign, 4 exponent bits (bias 7), 3 mantissa bits, step 2^-9
 * below 2^-6; E2M1 = sign, 2 exponent bits (bias 1), 1 mantissa bit, step 0.5
 * below 1: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * Storage: codes [rows, D/2] bytes, channel 2j in the low nibble of byte j and
 * 2j+1 in the high nibble; scales [rows, D/16] bytes, block order.
 * --------------------------------------------------------------------------- */

/* v >= 0 rounded to the binary grid with `mbits` mantissa bits whose smallest
 * normal binade is 2^emin (below it the step stays 2^(emin - mbits)); ties to
 * the even multiple of the step. */
static double round_to_grid(double v, int mbits, int emin) {
    if (v == 0.0) return 0.0;
    int e;
    frexp(v, &e);         /* v = f 2^e with f in [1/2, 1): leading bit 2^(e-1) */
    int lead = e - 1;
    if (lead < emin) lead = emin;
    const double step = ldexp(1.0, lead - mbits);
    return nearbyint(v / step) * step; /* v / step is exact; default mode: half to even */
}

/* Bits of an E4M3 magnitude already on the grid (0 <= v <= 448). */
static uint8_t e4m3_bits(double v) {
    if (v < ldexp(1.0, -6)) return (uint8_t)(v / ldexp(1.0, -9));
    int e;
    frexp(v, &e);
    const int lead = e - 1;
    const int mant = (int)(v / ldexp(1.0, lead - 3)) - 8;
    return (uint8_t)(((lead + 7) << 3) | mant);
}

static double e4m3_value(uint8_t b) {
    const int ex = (b >> 3) & 15, mant = b & 7;
    const double mag = ex == 0 ? ldexp((double)mant, -9) : ldexp(8.0 + mant, ex - 10);
    return (b & 0x80) ? -mag : mag;
}

/* Bits of an E2M1 magnitude already on the grid (0 <= m <= 6). */
static int e2m1_bits(double m) {
    if (m < 1.0) return (int)(m / 0.5);
    int e;
    frexp(m, &e);
    const int lead = e - 1;
    const int mant = (int)(m / ldexp(1.0, lead - 1)) - 2;
    return ((lead + 1) << 1) | mant;
}

static double e2m1_value(int c) {
    const int ex = (c >> 1) & 3, mant = c & 1;
    const double mag = ex == 0 ? 0.5 * mant : ldexp(2.0 + mant, ex - 2);
    return (c & 8) ? -mag : mag;
}

static double nvfp4_value(const uint8_t *codes, const uint8_t *sf, size_t row, int D, int d) {
    const uint8_t byte = codes[row * (size_t)(D / 2) + d / 2];
    const int c = (d & 1) ? (byte >> 4) : (byte & 15);
    return e2m1_value(c) * e4m3_value(sf[row * (size_t)(D / 16) + d / 16]);
}

int oracle_quant_nvfp4(const uint16_t *x, long rows, int D, uint8_t *codes, uint8_t *sf, int dtype) {
    if (rows < 0 || D < 16 || D % 16) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (int b = 0; b < D / 16; ++b) {
            float xs[16], amax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                xs[j] = half_to_f32(x[(size_t)r * D + 16 * b + j], dtype);
                if (fabsf(xs[j]) > amax) amax = fabsf(xs[j]);
            }
            const float s32 = amax / 6.0f;
            double s = round_to_grid((double)s32, 3, -6);
            if (s > 448.0) s = 448.0;
            const uint8_t sb = e4m3_bits(s);
            sf[(size_t)r * (D / 16) + b] = sb;
            const float sdec = (float)e4m3_value(sb);
            const float inv = sdec == 0.0f ? 0.0f : 1.0f / sdec;
            uint8_t *out = codes + (size_t)r * (D / 2) + 8 * b;
            for (int j = 0; j < 16; ++j) {
                const float y = xs[j] * inv;
                double m = round_to_grid(fabs((double)y), 1, 0);
                if (m > 6.0) m = 6.0;
                const int c = e2m1_bits(m) | (signbit(y) ? 8 : 0);
                if (j % 2 == 0)
                    out[j / 2] = (uint8_t)c;
                else
                    out[j / 2] = (uint8_t)(out[j / 2] | (c << 4));
            }
        }
    }
    return ORACLE_OK;
}

/* The values NVFP4 codes and scales stand for: y [rows, D] doubles. */
int oracle_dequant_nvfp4(const uint8_t *codes, const uint8_t *sf, long rows, int D, double *y) {
    if (rows < 0 || D < 16 || D % 16) return ORACLE_ERR_ARG;
    for (long r = 0; r < rows; ++r)
        for (int d = 0; d < D; ++d) y[(size_t)r * D + d] = nvfp4_value(codes, sf, (size_t)r, D, d);
    return ORACLE_OK;
}

/* E4M3 bits of fp32 values (the scale rounding above, exposed for its pins). */
int oracle_e4m3_round(const float *x, long n, uint8_t *bits) {
    for (long i = 0; i < n; ++i) {
        if (!(x[i] >= 0.0f)) return ORACLE_ERR_ARG;
        double s = round_to_grid((double)x[i], 3, -6);
        if (s > 448.0) s = 448.0;
        bits[i] = e4m3_bits(s);
    }
    return ORACLE_OK;
}

/* Attention of explicit query rows with NVFP4 q and k (codes + scales in the
 * storage above, tiled row order) and 16-bit v: the same definition as
 * oracle_attn_rows, on the values the codes stand for. */
int oracle_attn_rows_nvfp4(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw,
                           const uint8_t *qc, const uint8_t *qs, const uint8_t *kc, const uint8_t *ks,
                           const uint16_t *v, const int32_t *idx, const int32_t *num, int max_k,
                           int D, const int64_t *rows, long n_rows, double *o_rows, double *lse_rows, int dtype) {
    geom_t g;
    int rc = geom_init(&g, n_prefix, T, Hg, Wg, bt, bh, bw);
    if (rc) return rc;
    if (D < 16 || D % 16) return ORACLE_ERR_ARG;
    const operand_t qop = {NULL, qc, qs, dtype}, kop = {NULL, kc, ks, dtype};
    return attn_rows_core(&g, &qop, &kop, v, idx, num, max_k, D, rows, n_rows, o_rows, lse_rows, dtype);
}

/* Highest thread count OpenMP will use here (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
