/*
 * csa2.h -- C ABI of libcsa2.so: the CSA2 (Compressed Sparse Attention 2)
 * decode step over an FP4 global KV cache, on one NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on DeepSeek-V4.1-Flash), cited by tag:
 *   [REL] "DeepSeek-V4.1-Flash 发布：100 万上下文 + FP4 KV Cache + 跨层注意力复用"
 *         (feinterview.poetries.top)
 *   [CNB] "DeepSeek V4.1 Flash 发布，百万上下文开始算缓存这笔账" (cnblogs, OpenCSG)
 *   [YOM] yomxxx.com post on the V4.1-Flash CED/CSA2 paper (2026-09-14)
 *   [TUC] "V4.1 Flash 内测，梁文锋又当回了梁圣" (tucaod.com; paper walk-through)
 *
 * Conventions shared by every entry point
 *  - Every pointer argument named as device memory must be a device pointer
 *    of the current CUDA device; the caller allocates and owns every buffer.
 *    The library allocates nothing, frees nothing and never synchronises,
 *    except csa2_sync_status(), which exists to synchronise.
 *  - All work is enqueued on the given stream and is asynchronous.
 *  - Argument, shape and alignment errors are detected on the host and
 *    returned before anything is launched.  Launch failures return
 *    CSA2_ERR_CUDA.  Problems only the device can see (a page-table entry
 *    outside the row pool, an expired bounded wait) never fault: the kernel
 *    clamps, records a bit in the status word at the start of the workspace,
 *    and csa2_sync_status() reports it as CSA2_ERR_DEVICE_CHECK or
 *    CSA2_ERR_TIMEOUT.
 *  - csa2_last_error() returns a thread-local message for the last failure.
 *  - Device pointers must be 16-byte aligned (CSA2_ERR_ALIGNMENT otherwise).
 *  - Shapes are fixed to the decode configuration of the pages and of the
 *    synthetic workloads: main-KV rows of CSA2_D = 512 channels, CSA2_H = 16
 *    query heads, an indexer of CSA2_HI = 8 heads x CSA2_DI = 64, blocks of
 *    CSA2_BLK = 8 positions, a sliding window of CSA2_W = 128 rows.
 */
#ifndef CSA2_API_H_
#define CSA2_API_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa2_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum {
  CSA2_D = 512,          /* main-KV channels per entry                         */
  CSA2_H = 16,           /* query heads sharing one main-KV row (K = V)        */
  CSA2_HI = 8,           /* indexer heads                                      */
  CSA2_DI = 64,          /* indexer head dimension                             */
  CSA2_BLK = 8,          /* positions per HSI block [YOM §二 HSI]              */
  CSA2_W = 128,          /* sliding-window rows [REL §CED; YOM §一]            */
  CSA2_MAX_TOPK = 512,   /* Top-512 [REL §CSA2; YOM §二 table]                 */
  CSA2_MAX_POOL = 2048,  /* 2,048 blocks = 16,384 positions [YOM §二 HSI]      */
  CSA2_MAX_ROWS = 1 << 20, /* visible entries per sequence (1M context)       */
  CSA2_MAX_QUERY = 1024    /* queries per sequence per step (drafts, prefill)  */
};

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,  /* NULL pointer, bad enum, bad count              */
  CSA2_ERR_SHAPE = 2,        /* a size outside what the kernels support        */
  CSA2_ERR_ALIGNMENT = 3,    /* a pointer not 16-byte aligned                  */
  CSA2_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than required        */
  CSA2_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed           */
  CSA2_ERR_TIMEOUT = 6,      /* a device-side bounded wait expired             */
  CSA2_ERR_DEVICE_CHECK = 7  /* a device-side bounds check clamped an index    */
} csa2_status;

typedef enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 } csa2_mode;

/*
 * FP4 main-KV cache, E2M1 values with one E4M3 scale per 16 channels and no
 * global scale ("NVFP4 without its global scale") [REL §FP4 KV; YOM §三;
 * TUC §缓存精度与持久化分层], stored as two planes over a pool of rows:
 *   codes  [pool_rows][CSA2_D/2]  two E2M1 codes per byte, even channel in
 *                                 the low nibble
 *   scales [pool_rows][CSA2_D/16] E4M3 bit patterns
 *   idx_k  [pool_rows][CSA2_DI]   bf16 indexer K of each row, projected from
 *                                 the main-KV entry [YOM §二 last paragraph]
 * Position p (0 <= p < n_rows[b]) of sequence b is pool row
 *   page_table == NULL: b * seq_stride + p
 *   otherwise:          page_table[b * max_pages + p / page_rows] * page_rows
 *                       + p % page_rows      (page_rows must be 64)
 * A row outside [0, pool_rows) is never dereferenced: it reads as zeros and
 * sets CSA2_ERR_DEVICE_CHECK.  All pointers are device pointers.
 */
typedef struct {
  const uint8_t *codes;
  const uint8_t *scales;
  const uint16_t *idx_k;
  const int32_t *page_table; /* [batch][max_pages] or NULL                     */
  int32_t page_rows;         /* 64 when paged, ignored otherwise               */
  int32_t max_pages;
  const int32_t *n_rows;     /* [batch] visible entries C_b (device)           */
  int32_t batch;
  int32_t max_rows;          /* host upper bound of every n_rows[b]            */
  int64_t seq_stride;        /* contiguous layout only                         */
  int64_t pool_rows;
} csa2_kv_view;

/* ---------------------------------------------------------------- status */

const char *csa2_status_string(csa2_status s);
/* Thread-local text of the last error returned on this thread ("" if none). */
const char *csa2_last_error(void);

/* Bytes at the start of every workspace: the device status word (word 0)
 * and the Full scan's tile counter (word 16), which every scan launch
 * returns to zero before it completes.  A workspace serves one call at a
 * time (calls enqueued on one stream, or otherwise ordered). */
#define CSA2_WS_HEADER 256
/* Zero the header of a workspace (status word and scan counter; enqueued on
 * stream).  Call once before the first use of a workspace, and again after
 * a call whose csa2_sync_status reported CSA2_ERR_TIMEOUT (a scan that gave
 * up may leave its counter non-zero). */
csa2_status csa2_workspace_init(void *ws, size_t ws_bytes, csa2_stream_t stream);
/* Synchronise the stream, read and clear the status word: CSA2_OK, or the
 * first device-side problem recorded since the last call. */
csa2_status csa2_sync_status(void *ws, csa2_stream_t stream);

/* --------------------------------------------------------- cache append */

/*
 * Append one decode step's new entries to the caches (the step that runs
 * before csa2_layer_group; yomxxx.com CSA2 paper notes, section 二, last
 * paragraph, and section 三; release note, section "Compressed Sparse
 * Attention 2 (CSA2)"):
 *   for each sequence b, at position p = kv->n_rows[b]:
 *     codes/scales row of p  <- FP4 of x[b] (as csa2_quantize_fp4),
 *     idx_k row of p         <- bf16_rne(x[b] @ w_idx)  (fp32 accumulation),
 *     kv->n_rows[b]          <- p + 1;
 *   for each layer l < n_layers and sequence b, at slot s = swa_pos[b] % 128:
 *     swa[l][b][s][:]        <- E4M3 (round to nearest even, saturating to
 *                               +-448, no scale) of x_swa[l][b][:],
 *   then swa_pos[b] += 1 and swa_len[b] = min(swa_pos[b], 128).
 * Arguments (device memory, caller-owned, 16-byte aligned):
 *   kv      the cache; its codes, scales, idx_k and n_rows arrays are
 *           WRITTEN by this call (the view's const qualifiers notwithstanding).
 *           The new position must lie below the sequence's capacity
 *           (seq_stride rows when contiguous, max_pages * 64 when paged) on a
 *           mapped page; kv->max_rows is not checked against it (raise it
 *           before the next decode step reads the longer sequence).
 *   x       bf16 [batch][512]; w_idx bf16 [512][64];
 *   n_layers >= 0 window layers; when 0, x_swa, swa, swa_pos and swa_len
 *           may be NULL;  x_swa bf16 [n_layers][batch][512];
 *           swa E4M3 [n_layers][batch][128][512];  swa_pos, swa_len int32
 *           [batch], swa_pos >= 0.
 *   ws      a workspace of at least CSA2_WS_HEADER bytes (status word).
 * Errors: argument problems return before any launch.  A position with no
 * row (full sequence, unmapped page) or a negative swa_pos leaves that
 * sequence's cache and counters unchanged and records CSA2_ERR_DEVICE_CHECK
 * for csa2_sync_status.  Two launches; asynchronous on stream.
 */
csa2_status csa2_cache_append(const csa2_kv_view *kv, const uint16_t *x, const uint16_t *w_idx,
                              int32_t n_layers, const uint16_t *x_swa, uint8_t *swa,
                              int32_t *swa_pos, int32_t *swa_len, void *ws, size_t ws_bytes,
                              csa2_stream_t stream);

/* Self-test of the device-side failure path: launches one warp that waits on
 * a barrier nothing completes, through the same bounded wait every pipeline
 * wait in this library uses; after `cycles` SM clock cycles (1,000 to
 * 2,000,000,000) the wait gives up, records the timeout bit in the status
 * word of ws, and the kernel returns.  The next csa2_sync_status then returns
 * CSA2_ERR_TIMEOUT and the context stays usable.  Nothing faults or hangs. */
csa2_status csa2_selftest_bounded_wait(void *ws, size_t ws_bytes, int64_t cycles,
                                       csa2_stream_t stream);

/* ---------------------------------------------------------------- tracing */

/*
 * Optional per-launch timing.  While a trace is set on the calling thread,
 * every entry point records trace->events[trace->count] (a cudaEvent_t the
 * caller created with timing enabled) on its stream just before each kernel
 * launch, with the kernel's stage name in trace->names[], and one event named
 * "end" after its last launch; count advances by one per event and recording
 * stops silently at capacity (at most 64).  Stage i lasts from event i to
 * event i+1.  NULL turns tracing off.  Tracing adds event records only.
 */
typedef struct {
  void *events[64];
  const char *names[64];
  int32_t capacity;
  int32_t count;
} csa2_trace;
void csa2_trace_set(csa2_trace *trace);

/* ------------------------------------------------------------- FP4 codec */

/*
 * Quantise rows of bf16 values x[rows][ch] (ch a multiple of 16) to the FP4
 * planes codes[rows][ch/2] and scales[rows][ch/16] [REL §FP4 KV; YOM §三].
 * Per group of 16: amax = max|x|; t = amax / 6 in fp32 (correctly rounded);
 * scale = E4M3(t) round-to-nearest-even, saturating at 448; a zero scale
 * gives all codes 0x0; otherwise code_i = E2M1(x_i / scale), nearest-even,
 * saturating at 6, sign kept (a negative value that rounds to zero is 0x8).
 * Inputs must be finite.  rows may be 0.  Device pointers.
 */
csa2_status csa2_quantize_fp4(const uint16_t *x_bf16, int64_t rows, int32_t ch,
                              uint8_t *codes, uint8_t *scales, csa2_stream_t stream);

/* y[rows][ch] = bf16(e2m1(code) * e4m3(scale)); exact (every product is a
 * bf16 value).  Device pointers. */
csa2_status csa2_dequantize_fp4(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                                int32_t ch, uint16_t *y_bf16, csa2_stream_t stream);

/* ------------------------------------------------------------ the indexer */

/*
 * Workspace bytes csa2_index_full / csa2_index_reindex need for this view.
 */
size_t csa2_index_workspace_size(const csa2_kv_view *kv, int32_t top_k, int32_t pool_blocks);

/*
 * Full-mode indexer [REL §CSA2 "Full"; YOM §二 mode table and HSI paragraph;
 * TUC §CSA2注意力].  For every sequence b, over all visible positions p < C_b:
 *   s[p] = sum_h w[b][h] * max(0, q_idx[b][h] . idx_k[row(b,p)])
 * (the score form is this library's reading; the pages only say "score"),
 * block maxima over blocks of CSA2_BLK positions, and
 *   pool[b][0..pool_count[b])  the min(pool_blocks, ceil(C_b/8)) blocks with
 *                              the largest block maxima, ascending block ids
 *                              (the decoder Hierarchical Sparse Indexer pool)
 *   idx[b][0..idx_count[b])    the min(top_k, C_b) positions with the largest
 *                              s, ascending, ties to the lower position
 * Entries past the counts are -1.  pool_blocks = 0 builds no pool (pool and
 * pool_count may be NULL).  top_k in [1, 512]; pool_blocks in {0} or
 * [top_k ... 2048].  q_idx: bf16 [batch][8][64]; w: fp32 [batch][8];
 * idx: int32 [batch][top_k]; pool: int32 [batch][pool_blocks].  Device.
 */
csa2_status csa2_index_full(const csa2_kv_view *kv, const uint16_t *q_idx, const float *w,
                            int32_t top_k, int32_t pool_blocks, int32_t *idx,
                            int32_t *idx_count, int32_t *pool, int32_t *pool_count,
                            void *ws, size_t ws_bytes, csa2_stream_t stream);

/*
 * Reindex-mode indexer [REL §CSA2 "Reindex"; YOM §二 table: reuses the Full
 * layer's main KV and indexer K, rescores with its own indexer query].
 * With a pool (pool != NULL) only the positions of the pool blocks are
 * rescored [YOM §二 HSI: later indexers search only inside the pool]; with
 * pool == NULL every visible position is.  Output as csa2_index_full.
 * pool: int32 [batch][pool_stride] ascending block ids, pool_count [batch].
 */
csa2_status csa2_index_reindex(const csa2_kv_view *kv, const uint16_t *q_idx, const float *w,
                               const int32_t *pool, const int32_t *pool_count,
                               int32_t pool_stride, int32_t top_k, int32_t *idx,
                               int32_t *idx_count, void *ws, size_t ws_bytes,
                               csa2_stream_t stream);

/*
 * csa2_index_full without any device allocation by the caller.  The pages
 * have no counterpart: this is an integration convenience.  It is for callers
 * that cannot allocate device memory while they run -- plugins or custom ops
 * inside a host framework that owns all device memory through its own
 * allocator, serving loops that must not pay cudaMalloc's implicit device
 * synchronisation, processes already at their memory limit.
 *
 * Same arguments, checks and outputs as csa2_index_full, minus the
 * workspace.  Its scratch is one static device array of
 * CSA2_NOALLOC_SCRATCH_BYTES (2 MiB) inside libcsa2.so, which every GPU that
 * loads the library holds until the process exits.  A batch and context
 * needing more scratch than that (csa2_index_workspace_size() larger than
 * CSA2_NOALLOC_SCRATCH_BYTES; e.g. batch x ceil(context / 8) x 4 bytes above
 * about 2 MB) is rejected with CSA2_ERR_WORKSPACE before any launch.
 * The first call on each device looks up the array's device address (with
 * that device current), and again whenever the device's current context is
 * a different one (after cudaDeviceReset the module loads at a new
 * address); make that first call before any stream capture.
 * Every call shares the one array: calls whose work overlaps on the GPU
 * (two streams, two threads) race and must be serialised by the caller.
 * Device-side range checks still clamp, but their status bit stays in the
 * shared scratch (cleared at the start of each call) and is not reported;
 * use csa2_index_full with csa2_sync_status to diagnose such inputs.
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (2u << 20)
csa2_status csa2_index_full_noalloc(const csa2_kv_view *kv, const uint16_t *q_idx,
                                    const float *w, int32_t top_k, int32_t pool_blocks,
                                    int32_t *idx, int32_t *idx_count, int32_t *pool,
                                    int32_t *pool_count, csa2_stream_t stream);

/* ---------------------------------------------------------- the attention */

size_t csa2_attn_workspace_size(int32_t batch, int32_t n_layers);

/*
 * Sparse + sliding-window decode attention of one layer [TUC core-attention
 * figure text: Selection / Top-K / Concatenation; REL §CED: 128-token SWA at
 * every layer with FP8 KV].  For each sequence b and head h:
 *   keys = values = [ dequant(main KV at idx[b][0..idx_count[b]) ) ;
 *                     E4M3 window swa[b][0..swa_len[b]) ]
 *   out[b][h] = softmax_j(sm_scale * q[b][h] . key_j) . values
 * one softmax over both branches (MQA: the 16 heads share each row as K and
 * V).  No keys gives zeros.  q: bf16 [batch][16][512], any finite values
 * (each head is scaled by a power of two into fp16's range for the MMAs and
 * the logits are scaled back exactly);
 * idx: int32 [batch][idx_stride]; swa: uint8 E4M3 [batch][128][512];
 * swa_len: int32 [batch] (<= 128); out: bf16 [batch][16][512].  Device.
 */
csa2_status csa2_sparse_attn_decode(const uint16_t *q, const csa2_kv_view *kv,
                                    const int32_t *idx, const int32_t *idx_count,
                                    int32_t idx_stride, const uint8_t *swa,
                                    const int32_t *swa_len, float sm_scale, uint16_t *out,
                                    void *ws, size_t ws_bytes, csa2_stream_t stream);

/* ---------------------------------------------------------- a layer group */

/*
 * One decode step of a group of CSA2 layers sharing one main-KV cache
 * [REL §CSA2; YOM §二: layers statically Full, Reindex or Reuse; every layer
 * keeps its own query and SWA KV; decoder = Full+3 Reuse, then 4 x
 * (Reindex+3 Reuse)].  Layer 0 must be FULL.  A REINDEX layer rescores the
 * pool of the latest FULL layer (all positions when pool_blocks == 0).  A
 * REUSE layer takes the latest FULL/REINDEX indices unchanged.
 * Per-layer inputs are stacked on a leading layer axis:
 *   q_idx bf16 [L][batch][8][64], w fp32 [L][batch][8] (read for FULL and
 *   REINDEX layers only), q bf16 [L][batch][16][512],
 *   swa E4M3 [L][batch][128][512], swa_len int32 [batch].
 * Outputs: idx int32 [L][batch][top_k] and idx_count [L][batch] (REUSE layers
 * receive a copy of the indices they used), pool int32 [batch][pool_blocks]
 * and pool_count [batch] of the last FULL layer (may be NULL when
 * pool_blocks == 0), out bf16 [L][batch][16][512].
 * modes points to HOST memory; everything else is device memory.
 *
 * Multi-query step (n_query = Q in [2, CSA2_MAX_QUERY]): Q new positions per
 * sequence whose entries are already in the caches, each attending causally:
 * verification of draft positions (the release note and the cnblogs article
 * describe DSpark drafting several positions that the main model verifies in
 * one pass; Q <= 8) and chunked prefill (Q new tokens of a prompt).  Query t of sequence
 * b sees the first kv.n_rows[b] - (Q-1-t) global entries and the window rows
 * [max(0, e_t - 128), e_t) with e_t = swa_len[b] - (Q-1-t).  Every per-query
 * array gains a query axis after the batch axis, so "batch" above reads
 * batch x Q: q_idx [L][batch][Q][8][64], w [L][batch][Q][8],
 * q [L][batch][Q][16][512], idx [L][batch][Q][top_k], idx_count
 * [L][batch][Q], pool [batch][Q][pool_blocks], pool_count [batch][Q],
 * out [L][batch][Q][16][512]; the window is swa [L][batch][128 + Q - 1][512]
 * with swa_len [batch] <= 128 + Q - 1.  The scan reads every indexer-K row
 * once per pass of up to 8 queries (one MMA of N = 8 x queries, padded to
 * 16/32/64), i.e. ceil(Q / 8) times.
 * batch x Q must not exceed 65535.
 */
typedef struct {
  csa2_kv_view kv;
  int32_t n_layers;
  const int32_t *modes; /* host [n_layers] */
  const uint16_t *q_idx;
  const float *w;
  const uint16_t *q;
  const uint8_t *swa;
  const int32_t *swa_len;
  int32_t top_k;
  int32_t pool_blocks;
  float sm_scale;
  int32_t *idx;
  int32_t *idx_count;
  int32_t *pool;
  int32_t *pool_count;
  uint16_t *out;
  int32_t n_query; /* queries (draft positions) per sequence; 0 or 1 = one */
} csa2_group_desc;

size_t csa2_group_workspace_size(const csa2_group_desc *desc);
csa2_status csa2_layer_group(const csa2_group_desc *desc, void *ws, size_t ws_bytes,
                             csa2_stream_t stream);

/* ------------------------------------------------ context-parallel decode */

/*
 * One decode step of a layer group with every sequence's positions cut into
 * `world` contiguous shards of shard_rows (S) rows: rank r holds positions
 * [r*S, (r+1)*S) of every sequence in its own cache, a csa2_kv_view whose
 * n_rows are the shard's visible rows (csa2_cp_local_rows) and whose
 * max_rows <= S.  Scores, block maxima and attention rows are per position,
 * and every selection of the step is a Top-k under one total order (the key,
 * then the lower position or block) [REL §CSA2; YOM §二 mode table and HSI
 * paragraph], so the step is local work on each shard plus three exchanges.
 * The caller runs each exchange as an all-gather over the ranks in rank
 * order (NCCL over NVLink, or any transport): the library moves no data
 * between ranks and never waits on another rank.
 *   1. FULL layer (and REINDEX without a pool): csa2_cp_block_max ->
 *      all-gather -> csa2_cp_pool: the pool (P = pool_blocks, or top_k
 *      blocks without a pool), the same on every rank.
 *   2. Selection: csa2_cp_filter (unit 8: the pool blocks this shard owns) ->
 *      csa2_cp_select_local -> all-gather -> csa2_cp_select_merge: the
 *      layer's Top-k positions, the same on every rank and equal to the
 *      one-GPU csa2_layer_group result (the keys exchanged are bit-identical
 *      to those the one-GPU rescore ranks).
 *   3. Attention: csa2_cp_filter (unit 1: the selected rows this shard owns)
 *      -> csa2_cp_attn_partial -> all-gather -> csa2_cp_attn_combine.
 * The sliding window lives on one rank: pass the window lengths there and
 * zeros on the others.  Every call is asynchronous on its stream and records
 * device checks in the status word of ws, like the rest of this ABI.
 * Count arrays (n_rows, counts, index lists) need 4-byte alignment only.
 */
enum { CSA2_CP_MAX_WORLD = 16 };

typedef struct {
  int32_t rank;       /* this shard, 0 <= rank < world                          */
  int32_t world;      /* shards, 1 <= world <= CSA2_CP_MAX_WORLD                 */
  int32_t shard_rows; /* S: a multiple of 128; world * S <= CSA2_MAX_ROWS        */
} csa2_cp_shard;

/* Bytes of workspace that every csa2_cp_* call of one rank needs for a group
 * of n_layers layers (status word, local selection scratch, attention split
 * partials, regrouped block maxima).  0 on a bad argument. */
size_t csa2_cp_workspace_size(const csa2_cp_shard *sh, int32_t batch, int32_t n_layers,
                              int32_t top_k);

/* Floats in one rank's attention partial: n_layers * batch * 16 * (512 + 2). */
size_t csa2_cp_partial_floats(int32_t batch, int32_t n_layers);

/* local_rows[b] = clamp(n_rows[b] - rank * S, 0, S): the shard's visible rows.
 * n_rows, local_rows: device int32 [batch].  A negative n_rows[b] is a device
 * check. */
csa2_status csa2_cp_local_rows(const csa2_cp_shard *sh, const int32_t *n_rows, int32_t batch,
                               int32_t *local_rows, void *ws, size_t ws_bytes,
                               csa2_stream_t stream);

/* Block maxima over the shard: bm[b][j] = max of the score
 * s = sum_h w_h * relu(q_idx_h . k) over the shard's visible rows 8j..8j+7
 * [YOM §二 HSI], by the same scan as csa2_index_full.  q_idx bf16
 * [batch][8][64], w fp32 [batch][8], bm fp32 [batch][S / 8] (entries at or
 * past the visible blocks are left as they are).  kv: this shard's view. */
csa2_status csa2_cp_block_max(const csa2_cp_shard *sh, const csa2_kv_view *kv,
                              const uint16_t *q_idx, const float *w, float *bm, void *ws,
                              size_t ws_bytes, csa2_stream_t stream);

/* The pool from the all-gathered block maxima bm_all fp32 [world][batch][S/8]
 * (rank-major, as an all-gather of every rank's bm lays them out): the top P
 * blocks by block maximum over the blocks of the global visible rows n_rows
 * (int32 [batch]), ties to the lower block.  pool int32 [batch][P] ascending
 * global block ids, -1 padded; pool_count int32 [batch].  P in
 * [1, CSA2_MAX_POOL]. */
csa2_status csa2_cp_pool(const csa2_cp_shard *sh, const float *bm_all, const int32_t *n_rows,
                         int32_t batch, int32_t P, int32_t *pool, int32_t *pool_count,
                         void *ws, size_t ws_bytes, csa2_stream_t stream);

/* The ids in list that this shard owns, made local.  unit = 8 for block ids
 * (shard range [rank*S/8, (rank+1)*S/8)), 1 for positions ([rank*S,
 * (rank+1)*S)).  out[b] = the ids x of list[b][0 .. count[b]) in the range,
 * as x - range start, in list order, -1 padded to out_stride; out_count[b]
 * their number (at most out_stride).  copy and copy_count (both or neither)
 * receive list [batch][stride] and count verbatim.  stride and out_stride in
 * [1, CSA2_MAX_POOL]; a count outside [0, stride] is a device check. */
csa2_status csa2_cp_filter(const csa2_cp_shard *sh, int32_t unit, const int32_t *list,
                           const int32_t *count, int32_t stride, int32_t batch, int32_t *out,
                           int32_t *out_count, int32_t out_stride, int32_t *copy,
                           int32_t *copy_count, void *ws, size_t ws_bytes,
                           csa2_stream_t stream);

/* The shard's Top-k among its candidate blocks cand int32 [batch][cand_stride]
 * (local block ids, ascending; cand_count [batch]), scored with q_idx / w as
 * in csa2_index_reindex, exported for the merge: send uint32
 * [batch][top_k][2] = (key, global position) in ascending position, then
 * (0, 0xFFFFFFFF).  The key is the fp32 score mapped to an unsigned integer
 * of the same order (0 is never a key).  send: 8-byte aligned. */
csa2_status csa2_cp_select_local(const csa2_cp_shard *sh, const csa2_kv_view *kv,
                                 const uint16_t *q_idx, const float *w, const int32_t *cand,
                                 const int32_t *cand_count, int32_t cand_stride, int32_t top_k,
                                 uint32_t *send, void *ws, size_t ws_bytes,
                                 csa2_stream_t stream);

/* The global Top-k of job `job` (ties to the lower position) from the
 * all-gathered exports gathered uint32 [world][n_jobs][batch][top_k][2]
 * (several layers' exports may share one all-gather).  idx int32
 * [batch][top_k] ascending global positions, -1 padded; idx_count [batch].
 * world * top_k <= 8192. */
csa2_status csa2_cp_select_merge(const csa2_cp_shard *sh, const uint32_t *gathered,
                                 int32_t n_jobs, int32_t job, int32_t batch, int32_t top_k,
                                 int32_t *idx, int32_t *idx_count, void *ws, size_t ws_bytes,
                                 csa2_stream_t stream);

/* Batched forms (one launch, or one pair of launches, instead of one per job
 * or per layer; results identical to the per-job calls).  Jobs that share a
 * candidate list (a FULL layer and the REINDEX layers of its pool) are
 * layers of the group's arrays, named by host arrays of layer numbers. */
enum { CSA2_CP_MAX_JOBS = 8 };

/* csa2_cp_select_local for n_jobs jobs (1 <= n_jobs <= CSA2_CP_MAX_JOBS):
 * job j scores with layer layer[j] of q_idx bf16 [n_layers][batch][8][64] and
 * w fp32 [n_layers][batch][8] (layer: host int32 [n_jobs], each in
 * [0, n_layers)) and exports to send + j * batch * top_k * 2 (send uint32
 * [n_jobs][batch][top_k][2], as n_jobs consecutive single-job exports).  ws
 * as for csa2_cp_workspace_size(sh, batch, n_layers >= n_jobs, top_k). */
csa2_status csa2_cp_select_local_jobs(const csa2_cp_shard *sh, const csa2_kv_view *kv,
                                      int32_t n_jobs, const int32_t *layer, int32_t n_layers,
                                      const uint16_t *q_idx, const float *w,
                                      const int32_t *cand, const int32_t *cand_count,
                                      int32_t cand_stride, int32_t top_k, uint32_t *send,
                                      void *ws, size_t ws_bytes, csa2_stream_t stream);

/* csa2_cp_select_merge for jobs 0 .. n_jobs - 1 of gathered: job j's global
 * Top-k goes to layer layer[j] of idx int32 [n_layers][batch][top_k] and
 * idx_count int32 [n_layers][batch] (layer: host int32 [n_jobs], each in
 * [0, n_layers); 1 <= n_jobs <= CSA2_CP_MAX_JOBS). */
csa2_status csa2_cp_select_merge_jobs(const csa2_cp_shard *sh, const uint32_t *gathered,
                                      int32_t n_jobs, const int32_t *layer, int32_t n_layers,
                                      int32_t batch, int32_t top_k, int32_t *idx,
                                      int32_t *idx_count, void *ws, size_t ws_bytes,
                                      csa2_stream_t stream);

/* csa2_cp_filter (unit 1) for every layer: layer l keeps the positions of
 * idx[src[l]] (idx int32 [n_layers][batch][stride], counts idx_count
 * [n_layers][batch]) that this shard owns, as local positions, into
 * idx_local[l] / idx_local_count[l] (same shapes); a layer with src[l] != l
 * (a REUSE layer) also receives idx[src[l]] and its count verbatim in idx[l]
 * / idx_count[l].  src: host int32 [n_layers] with src[l] <= l and
 * src[src[l]] == src[l]; 1 <= n_layers <= 32; stride in [1, CSA2_MAX_POOL]. */
csa2_status csa2_cp_filter_layers(const csa2_cp_shard *sh, int32_t n_layers, const int32_t *src,
                                  int32_t *idx, int32_t *idx_count, int32_t stride,
                                  int32_t batch, int32_t *idx_local, int32_t *idx_local_count,
                                  void *ws, size_t ws_bytes, csa2_stream_t stream);

/* The shard's attention partial for every layer: over its selected rows
 * idx_local int32 [L][batch][idx_stride] (local positions from csa2_cp_filter,
 * counts idx_count [L][batch]) and the window rows swa_len[b] (zeros on ranks
 * without the window), the unnormalised softmax numerator and its (max, sum)
 * per head, as csa2_sparse_attn_decode computes them before normalising.
 * q bf16 [L][batch][16][512], swa E4M3 [L][batch][128][512].  partial fp32
 * [csa2_cp_partial_floats]: O [L][batch][16][512], then (max in log2 units of
 * sm_scale * q.k, sum) [L][batch][16][2].  n_layers <= 32. */
csa2_status csa2_cp_attn_partial(const csa2_cp_shard *sh, const csa2_kv_view *kv,
                                 int32_t n_layers, const uint16_t *q, const uint8_t *swa,
                                 const int32_t *swa_len, const int32_t *idx_local,
                                 const int32_t *idx_count, int32_t idx_stride, float sm_scale,
                                 float *partial, void *ws, size_t ws_bytes,
                                 csa2_stream_t stream);

/* out bf16 [L][batch][16][512] from the all-gathered partials gathered fp32
 * [world][csa2_cp_partial_floats]: the log-sum-exp merge over the ranks,
 * zeros where no rank had a key. */
csa2_status csa2_cp_attn_combine(const csa2_cp_shard *sh, const float *gathered,
                                 int32_t n_layers, int32_t batch, uint16_t *out, void *ws,
                                 size_t ws_bytes, csa2_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_API_H_ */
