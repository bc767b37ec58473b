/*
 * csa2_oracle.h -- CPU oracle for the CSA2 decode step over an FP4 global KV
 * cache.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product path (libcsa2.so and its
 * Python binding) never does, and the two share no code, header or table.
 *
 * Plain, slow, single-threaded C in fp64 on exactly decoded values.  Every
 * selection is an explicit full sort.  No blocking, fusion or reordering.
 *
 * Sources (web pages on DeepSeek-V4.1-Flash; cited by tag below):
 *   [REL] "DeepSeek-V4.1-Flash 发布：100 万上下文 + FP4 KV Cache + 跨层注意力复用"
 *         (feinterview.poetries.top)
 *   [CNB] "DeepSeek V4.1 Flash 发布，百万上下文开始算缓存这笔账" (cnblogs, OpenCSG)
 *   [YOM] yomxxx.com post on the V4.1-Flash CED/CSA2 paper (2026-09-14)
 *   [TUC] "V4.1 Flash 内测，梁文锋又当回了梁圣" (tucaod.com; paper walk-through)
 *
 * Readings where the pages are silent are stated at each function.
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer modes [YOM §二 mode table; REL §CSA2]. */
enum { CSA2O_FULL = 0, CSA2O_REINDEX = 1, CSA2O_REUSE = 2 };

/* Return codes. */
enum { CSA2O_OK = 0, CSA2O_EARG = 1 };

/* ---------------------------------------------------------------- formats */

/* bf16 bit pattern -> value (the upper half of an IEEE binary32). */
double csa2o_bf16_value(uint16_t bits);
/* fp64 -> bf16, round to nearest, ties to even (finite inputs). */
uint16_t csa2o_bf16_round(double v);

/* OCP FP4 E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 * [REL §FP4 KV; YOM §三] name the format; its values follow from the layout. */
double csa2o_e2m1_value(uint8_t code);
/* OCP FP8 E4M3 ("fn"): sign bit 7, exponent bits 6..3 (bias 7), mantissa
 * bits 2..0; S.1111.111 is NaN, no infinities, max finite 448. */
double csa2o_e4m3_value(uint8_t bits);

/* Nearest E2M1 code to q by search over the 8 magnitudes; equal distance
 * picks the even code; beyond 6 saturates to 6; the sign bit is kept
 * (negative q that rounds to zero gives 0x8).  q must be finite. */
uint8_t csa2o_e2m1_encode(float q);
/* Nearest finite E4M3 to t by search over all finite codes; equal distance
 * picks the even code; beyond 448 saturates to 448 (sign kept).  NaN -> 0x7F. */
uint8_t csa2o_e4m3_encode(float t);

/* ------------------------------------------------------- A1/A2 FP4 codec */

/* Quantise bf16 rows x[rows][ch] (ch % 16 == 0) to FP4:
 *   codes[rows][ch/2]  two E2M1 codes per byte, even channel in the low nibble
 *   scales[rows][ch/16] one E4M3 scale per 16 channels, no global scale
 * Per group: amax = max|x|; t = fp32(amax)/6 (fp32 division); s = E4M3(t);
 * s == 0 -> all codes 0x0, else code_i = E2M1(fp32(x_i)/s) (fp32 division).
 * [REL §FP4 KV; YOM §三 FP4; TUC §缓存精度与持久化分层]. */
int csa2o_quantize_fp4(const uint16_t *x, int64_t rows, int32_t ch,
                       uint8_t *codes, uint8_t *scales);

/* v = e2m1(code) * e4m3(scale), exact; y[rows][ch] in fp64. */
int csa2o_dequantize_fp4(const uint8_t *codes, const uint8_t *scales,
                         int64_t rows, int32_t ch, double *y);

/* -------------------------------------------------------- KV cache view */

/* Rows of sequence b live in a row pool.  Position p of sequence b is row
 *   page_table == NULL : b * seq_stride + p
 *   page_table != NULL : page_table[b * max_pages + p / page_rows] * page_rows
 *                        + p % page_rows
 * codes/scales: FP4 main KV rows (d/2 and d/16 bytes); idxk: bf16 indexer K
 * rows (di values). */
typedef struct {
  const uint8_t  *codes;
  const uint8_t  *scales;
  const uint16_t *idxk;
  const int32_t  *page_table;
  int32_t page_rows;
  int32_t max_pages;
  int64_t seq_stride;
  int64_t pool_rows;   /* rows in the pool; every mapped row must be below */
} csa2o_kv;

typedef struct {
  int32_t d;        /* main-KV channels (512) */
  int32_t h;        /* query heads (16) */
  int32_t hi;       /* indexer heads (8) */
  int32_t di;       /* indexer head dim (64) */
  int32_t blk;      /* HSI block size in positions (8) */
  int32_t w;        /* SWA window rows (128) */
} csa2o_dims;

/* Row index of position p in sequence b, or -1 when it falls outside the pool. */
int64_t csa2o_row_of(const csa2o_kv *kv, int32_t b, int64_t p);

/* ---------------------------------------------------- A3..A7 the indexer */

/* Indexer score of every position p < C of one sequence:
 *   s[p] = sum_h w_h * max(0, q_h . idxk[p])        (fp64 on bf16 values)
 * The score form is this build's reading (the pages only say "score"). */
int csa2o_scores(const csa2o_kv *kv, const csa2o_dims *dm, int32_t b, int64_t C,
                 const uint16_t *q_idx /*[hi][di]*/, const float *w /*[hi]*/,
                 double *s /*[C]*/);

/* Block maxima bm[j] = max over positions [blk*j, min(blk*j+blk, C)). */
int csa2o_block_max(const double *s, int64_t C, int32_t blk, double *bm);

/* The n_sel = min(k, n) best of n candidates by (value desc, id asc), where
 * candidate i has value v[i] and id ids ? ids[i] : i; written ascending by id
 * into out.  Returns n_sel.  A full sort, nothing cleverer. */
int64_t csa2o_select_topk(const double *v, const int64_t *ids, int64_t n,
                          int64_t k, int32_t *out);

/* Decoder Hierarchical Sparse Indexer pool: the min(pool_blocks, ceil(C/blk))
 * blocks with the largest block max, ids ascending.  Returns the count.
 * [REL §CSA2 last paragraph; YOM §二 HSI paragraph; TUC HSI figure text]. */
int64_t csa2o_pool(const double *bm, int64_t nblk, int32_t pool_blocks,
                   int32_t *pool);

/* One decode step of a CSA2 layer group for a batch of sequences.
 *   modes[L]              FULL / REINDEX / REUSE per layer
 *   n_rows[B]             visible global entries C_b
 *   q_idx[L][B][hi][di]   bf16 indexer queries (ignored for REUSE)
 *   w[L][B][hi]           fp32 indexer head weights (ignored for REUSE)
 *   q[L][B][h][d]         bf16 main queries
 *   swa[L][B][w][d]       E4M3 sliding-window KV, per layer
 *   swa_len[B]            valid window rows (<= w), rows 0..swa_len-1
 *   top_k (512), pool_blocks (2048; 0 = no HSI pool)
 * Outputs:
 *   idx[L][B][top_k], idx_count[L][B]     selected positions, ascending
 *   pool[B][pool_blocks], pool_count[B]   HSI pool of the last FULL layer
 *   out[L][B][h][d]                       attention output, fp64
 * FULL: score all C positions, build the pool from block maxima, pick the
 * exact Top-k over all positions.  REINDEX: rescore with its own q_idx only
 * positions inside the pool (all positions when pool_blocks == 0), Top-k.
 * REUSE: copy the latest indices.  [REL §CSA2; YOM §二; TUC §CSA2注意力]. */
int csa2o_layer_group(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B,
                      const int64_t *n_rows, int32_t L, const int32_t *modes,
                      const uint16_t *q_idx, const float *w, const uint16_t *q,
                      const uint8_t *swa, const int32_t *swa_len, int32_t top_k,
                      int32_t pool_blocks, double sm_scale, int32_t *idx,
                      int32_t *idx_count, int32_t *pool, int32_t *pool_count,
                      double *out);

/* ------------------------------------------------------ A8 the attention */

/* Decode attention of one sequence for one layer: keys = values = the rows
 *   [ dequant(main KV at idx[0..n_idx-1]) ; e4m3 SWA rows 0..swa_len-1 ]
 * logits l_hj = sm_scale * q_h . R_j, one softmax over all n_idx + swa_len
 * keys, out_h = sum_j softmax_j R_j.  fp64 throughout.  No keys -> zeros.
 * [TUC core-attention figure text: selection, Top-K, concatenation]. */
int csa2o_attention(const csa2o_kv *kv, const csa2o_dims *dm, int32_t b,
                    const uint16_t *q /*[h][d]*/, const int32_t *idx,
                    int32_t n_idx, const uint8_t *swa /*[w][d]*/,
                    int32_t swa_len, double sm_scale, double *out /*[h][d]*/);

/* ------------------------------ multi-query decode (next row of work) */

/* Verification of Q draft positions in one step (the drafts' entries are
 * already in the caches): query t < Q of sequence b is one decode step that
 * sees the first C_t = n_rows[b] - (Q - 1 - t) global entries (fewer than 0
 * means none) and the window rows [max(0, e_t - w), e_t) of its layer, with
 * e_t = swa_len[b] - (Q - 1 - t).  Per-query inputs and outputs carry a query
 * axis after the batch axis: q_idx [L][B][Q][hi][di], w [L][B][Q][hi],
 * q [L][B][Q][h][d], idx [L][B][Q][top_k], idx_count [L][B][Q],
 * pool [B][Q][pool_blocks], pool_count [B][Q], out [L][B][Q][h][d]; the
 * window is swa [L][B][w + Q - 1][d] with swa_len[B] <= w + Q - 1 valid rows.
 * Each (b, t) is computed by csa2o_layer_group on its own truncated view.
 * [CNB / REL: DSpark drafts several positions and the main model verifies
 * them in one pass]; causal visibility among drafts is this build's reading. */
int csa2o_layer_group_multi(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B, int32_t Q,
                            const int64_t *n_rows, int32_t L, const int32_t *modes,
                            const uint16_t *q_idx, const float *w, const uint16_t *q,
                            const uint8_t *swa, const int32_t *swa_len, int32_t top_k,
                            int32_t pool_blocks, double sm_scale, int32_t *idx,
                            int32_t *idx_count, int32_t *pool, int32_t *pool_count,
                            double *out);

/* --------------------------------------- cache append (next row of work) */

/* Indexer-K projection of one main-KV entry:
 *   out[j] = bf16_RNE( sum_c x[c] * w_idx[c * di + j] ),  c < d, j < di
 * with x and w_idx bf16, every product exact and the sum in fp64.  The
 * pages say the indexer K is projected from the main KV entry instead of a
 * separate compression of the hidden state [YOM §二 last paragraph; TUC
 * §CSA2]; this build projects the entry as produced (bf16, before its FP4
 * storage rounding) with a d x di bf16 matrix. */
int csa2o_project_idxk(const uint16_t *x /*[d]*/, const uint16_t *w_idx /*[d][di]*/,
                       int32_t d, int32_t di, uint16_t *out /*[di]*/);

/* Append one decode step's new entries (one global entry per sequence, one
 * sliding-window entry per layer and sequence):
 *   for each b: p = n_rows[b]; row = csa2o_row_of(kv, b, p); the position must
 *     also be below the sequence's capacity (seq_stride when contiguous,
 *     max_pages * page_rows when paged);
 *     codes/scales[row] = csa2o_quantize_fp4(x[b]) ; idxk[row] =
 *     csa2o_project_idxk(x[b]) ; n_rows[b] = p + 1.
 *     A sequence whose row is not mapped is left as it is (its counters too)
 *     and the call returns CSA2O_EARG after processing the others.
 *   for each layer l and b: slot = swa_pos[b] % w ;
 *     swa[l][b][slot][c] = E4M3_RNE_satfinite(x_swa[l][b][c]) ;
 *   then swa_pos[b] += 1, swa_len[b] = min(swa_pos[b], w).
 * The main KV is FP4 with E4M3 scales and the window KV stays FP8 [YOM §三];
 * each layer keeps its own window [REL §CSA2].  Storing the window entry
 * without a scale, and as a ring of w slots, is this build's reading. */
int csa2o_cache_append(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B,
                       uint8_t *codes, uint8_t *scales, uint16_t *idxk,
                       int64_t *n_rows, const uint16_t *x /*[B][d]*/,
                       const uint16_t *w_idx /*[d][di]*/, int32_t L,
                       const uint16_t *x_swa /*[L][B][d]*/, uint8_t *swa /*[L][B][w][d]*/,
                       int64_t *swa_pos /*[B]*/, int32_t *swa_len /*[B]*/);

#ifdef __cplusplus
}
#endif
#endif
