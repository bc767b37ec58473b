// capi_index.cu -- C ABI of the indexer, the attention and the layer group:
// host-side checks, workspace layout, TMA tensor maps, and the launch DAG.
//
// Layer group schedule (release note section "Compressed Sparse Attention 2
// (CSA2)"; yomxxx.com CSA2 notes, section 二, mode table and HSI paragraph):
//   for each FULL layer f:
//     scan(q_f) -> block maxima -> block Top-P (P = pool_blocks, or top_k
//     blocks when there is no pool) -> rescore + Top-k of f and of every
//     REINDEX layer up to the next FULL layer (one launch; they depend only
//     on the pool) ;
//   REINDEX without a pool: its own scan -> block Top-k -> rescore + Top-k ;
//   one attention launch for every layer (REUSE layers read the indices of
//   the latest FULL/REINDEX layer) ; one merge launch when split-KV is used.
// Exact Top-k of a FULL layer over all positions is taken over the positions
// of its Top-P blocks: every one of the k best positions lies in a block whose
// maximum is among the k best block maxima (ties to the lower position and
// block), so P >= k blocks hold them all.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "capi_common.h"
#include "csa2_internal.cuh"
#include "kernels.h"

namespace csa2 {

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over rows of 64 values (128 B), 128B swizzle, zero OOB fill.
static csa2_status map_rows64(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t gdim[2] = {64, rows < 1 ? 1 : rows};
  cuuint64_t gstride[1] = {128};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CSA2_OK;
}

// ------------------------------------------------------------ validation
static csa2_status check_kv(const csa2_kv_view* kv) {
  CSA2_REQUIRE(kv != nullptr, CSA2_ERR_INVALID_ARG, "kv is NULL");
  CSA2_REQUIRE_PTR(kv->codes);
  CSA2_REQUIRE_PTR(kv->scales);
  CSA2_REQUIRE_PTR(kv->idx_k);
  CSA2_REQUIRE(kv->n_rows != nullptr, CSA2_ERR_INVALID_ARG, "kv->n_rows is NULL");
  CSA2_REQUIRE(kv->batch >= 1 && kv->batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", kv->batch);
  CSA2_REQUIRE(kv->max_rows >= 0 && kv->max_rows <= CSA2_MAX_ROWS, CSA2_ERR_SHAPE,
               "max_rows = %d outside [0, %d]", kv->max_rows, (int)CSA2_MAX_ROWS);
  CSA2_REQUIRE(kv->pool_rows >= 0 && kv->pool_rows <= (int64_t)0x7FFF0000, CSA2_ERR_SHAPE,
               "pool_rows = %lld", (long long)kv->pool_rows);
  if (kv->page_table) {
    CSA2_REQUIRE(kv->page_rows == 64, CSA2_ERR_SHAPE, "page_rows = %d (must be 64)", kv->page_rows);
    CSA2_REQUIRE((int64_t)kv->max_pages * 64 >= kv->max_rows, CSA2_ERR_SHAPE,
                 "max_pages = %d cannot hold max_rows = %d", kv->max_pages, kv->max_rows);
  } else {
    CSA2_REQUIRE(kv->seq_stride >= kv->max_rows, CSA2_ERR_SHAPE,
                 "seq_stride = %lld < max_rows = %d", (long long)kv->seq_stride, kv->max_rows);
    CSA2_REQUIRE(kv->seq_stride % 64 == 0, CSA2_ERR_ALIGNMENT,
                 "seq_stride = %lld is not a multiple of 64 rows", (long long)kv->seq_stride);
    CSA2_REQUIRE((int64_t)(kv->batch - 1) * kv->seq_stride + kv->max_rows <= kv->pool_rows,
                 CSA2_ERR_SHAPE, "the row pool of %lld rows is too small for the layout",
                 (long long)kv->pool_rows);
  }
  return CSA2_OK;
}

static csa2_status check_topk(int top_k, int pool_blocks) {
  CSA2_REQUIRE(top_k >= 1 && top_k <= CSA2_MAX_TOPK, CSA2_ERR_SHAPE, "top_k = %d outside [1, %d]",
               top_k, (int)CSA2_MAX_TOPK);
  CSA2_REQUIRE(pool_blocks == 0 || (pool_blocks >= top_k && pool_blocks <= CSA2_MAX_POOL),
               CSA2_ERR_SHAPE, "pool_blocks = %d must be 0 or in [top_k, %d]", pool_blocks,
               (int)CSA2_MAX_POOL);
  return CSA2_OK;
}

csa2_status check_index_args(const csa2_kv_view* kv, int top_k, int pool_blocks) {
  csa2_status r = check_kv(kv);
  if (r) return r;
  return check_topk(top_k, pool_blocks);
}

// ------------------------------------------------------------ workspace
struct IndexWs {
  uint32_t* status;
  float* bm;
  int32_t bm_stride;
  int32_t* sel;
  int32_t* sel_count;
  int32_t sel_stride;
  size_t bytes;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// nq queries per sequence: block maxima and candidates per (sequence, query).
static IndexWs index_ws_layout(const csa2_kv_view* kv, int top_k, uint8_t* base, int nq = 1) {
  IndexWs w{};
  const size_t vb = (size_t)kv->batch * nq;
  const int nblk = (kv->max_rows + CSA2_BLK - 1) / CSA2_BLK;
  w.bm_stride = ((nblk + 15) / 16) * 16;
  if (w.bm_stride == 0) w.bm_stride = 16;
  w.sel_stride = top_k;
  size_t off = CSA2_WS_HEADER;
  w.status = reinterpret_cast<uint32_t*>(base);
  w.bm = reinterpret_cast<float*>(base + off);
  off = align256(off + vb * w.bm_stride * sizeof(float));
  w.sel = reinterpret_cast<int32_t*>(base + off);
  off = align256(off + vb * w.sel_stride * sizeof(int32_t));
  w.sel_count = reinterpret_cast<int32_t*>(base + off);
  off = align256(off + vb * sizeof(int32_t));
  w.bytes = off;
  return w;
}

static ScanParams scan_params(const csa2_kv_view* kv, const float* w, const IndexWs& ws,
                              int nq) {
  ScanParams p{};
  p.n_rows = kv->n_rows;
  p.page_table = kv->page_table;
  p.max_pages = kv->max_pages;
  p.max_rows = kv->max_rows;
  p.seq_stride = kv->seq_stride;
  p.pool_rows = kv->pool_rows;
  p.w = w;
  p.bm = ws.bm;
  p.bm_stride = ws.bm_stride;
  p.batch = kv->batch;
  p.tiles_per_seq = (kv->max_rows + SC_TILE - 1) / SC_TILE;
  p.nq = nq;
  p.q_first = 0;
  p.nq_pass = nq;
  p.tail = 0;
  p.status = ws.status;
  p.sched = ws.status + CSA2_WS_SCHED_WORD;  // the scan's tile counters in the header
  return p;
}

static RescoreParams rescore_params(const csa2_kv_view* kv, const int32_t* cand,
                                    const int32_t* cand_count, int cand_stride, int top_k,
                                    uint32_t* status, int nq = 1) {
  RescoreParams p{};
  p.nq = nq;
  p.idx_k = kv->idx_k;
  p.page_table = kv->page_table;
  p.max_pages = kv->max_pages;
  p.max_rows = kv->max_rows;
  p.seq_stride = kv->seq_stride;
  p.pool_rows = kv->pool_rows;
  p.n_rows = kv->n_rows;
  p.cand = cand;
  p.cand_count = cand_count;
  p.cand_stride = cand_stride;
  p.top_k = top_k;
  p.status = status;
  return p;
}

// scan + block select: candidates (top P blocks by block max) into sel
static csa2_status run_scan_select(const csa2_kv_view* kv, const uint16_t* q_idx, const float* w,
                                   int P, int32_t* sel, int32_t* sel_count, int sel_stride,
                                   const IndexWs& ws, cudaStream_t st, int nq = 1) {
  CUtensorMap map_k, map_q;
  csa2_status r = map_rows64(&map_k, kv->idx_k, (uint64_t)kv->pool_rows, 64);
  if (r) return r;
  // one scan launch per pass of up to CSA2_SCAN_QUERIES queries: each reads
  // the indexer K once and scores that many queries per row
  ScanParams sp = scan_params(kv, w, ws, nq);
  int box_rows = 0;
  for (int q0 = 0; q0 < nq; q0 += CSA2_SCAN_QUERIES) {
    sp.q_first = q0;
    sp.nq_pass = nq - q0 < CSA2_SCAN_QUERIES ? nq - q0 : CSA2_SCAN_QUERIES;
    sp.tail = nq - (q0 + sp.nq_pass);
    if (scan_query_rows(sp.nq_pass) != box_rows) {
      box_rows = scan_query_rows(sp.nq_pass);
      r = map_rows64(&map_q, q_idx, (uint64_t)kv->batch * nq * CSA2_HI, box_rows);
      if (r) return r;
    }
    trace_mark("scan", st);
    CSA2_CUDA(launch_scan(map_k, map_q, sp, num_sms(), st));
  }
  trace_mark("block_select", st);
  CSA2_CUDA(launch_block_select(ws.bm, ws.bm_stride, kv->n_rows, kv->max_rows, kv->batch * nq, nq,
                                P, sel, sel_stride, sel_count, ws.status, st));
  return CSA2_OK;
}

static int cand_blocks_max(const csa2_kv_view* kv, int P) {
  const int nblk = (kv->max_rows + CSA2_BLK - 1) / CSA2_BLK;
  return P < nblk ? P : nblk;
}

// ------------------------------------------------------------ group plan
struct GroupWs {
  IndexWs ix;
  float* part_o;
  float* part_ml;
  int nsplit;
  size_t bytes;
};

static int group_nq(const csa2_group_desc* d) { return d->n_query < 1 ? 1 : d->n_query; }

static GroupWs group_ws_layout(const csa2_group_desc* d, uint8_t* base) {
  GroupWs g{};
  const int nq = group_nq(d), vb = d->kv.batch * nq;
  g.ix = index_ws_layout(&d->kv, d->top_k, base, nq);
  g.nsplit = attn_nsplit(vb * d->n_layers, num_sms());
  const size_t slots = (size_t)vb * d->n_layers * g.nsplit;
  g.part_o = reinterpret_cast<float*>(base + g.ix.bytes);
  g.part_ml = reinterpret_cast<float*>(base + g.ix.bytes + slots * CSA2_H * CSA2_D * sizeof(float));
  g.bytes = g.ix.bytes + align256(attn_partial_bytes(vb, d->n_layers, g.nsplit));
  return g;
}

// ------------------------------------------------- context-parallel decode
#define CSA2_REQUIRE_I32(p)                                                         \
  do {                                                                             \
    if ((p) == nullptr) return ::csa2::fail(CSA2_ERR_INVALID_ARG, "%s is NULL", #p); \
    if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)                                  \
      return ::csa2::fail(CSA2_ERR_ALIGNMENT, "%s is not 4-byte aligned", #p);       \
  } while (0)

static csa2_status check_shard(const csa2_cp_shard* sh) {
  CSA2_REQUIRE(sh != nullptr, CSA2_ERR_INVALID_ARG, "shard is NULL");
  CSA2_REQUIRE(sh->world >= 1 && sh->world <= CSA2_CP_MAX_WORLD, CSA2_ERR_SHAPE,
               "world = %d outside [1, %d]", sh->world, (int)CSA2_CP_MAX_WORLD);
  CSA2_REQUIRE(sh->rank >= 0 && sh->rank < sh->world, CSA2_ERR_INVALID_ARG,
               "rank = %d outside [0, %d)", sh->rank, sh->world);
  CSA2_REQUIRE(sh->shard_rows > 0 && sh->shard_rows % 128 == 0, CSA2_ERR_SHAPE,
               "shard_rows = %d is not a positive multiple of 128", sh->shard_rows);
  CSA2_REQUIRE((int64_t)sh->world * sh->shard_rows <= CSA2_MAX_ROWS, CSA2_ERR_SHAPE,
               "world x shard_rows = %lld > %d", (long long)sh->world * sh->shard_rows,
               (int)CSA2_MAX_ROWS);
  return CSA2_OK;
}

static csa2_status check_shard_kv(const csa2_cp_shard* sh, const csa2_kv_view* kv) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  if ((r = check_kv(kv))) return r;
  CSA2_REQUIRE(kv->max_rows <= sh->shard_rows, CSA2_ERR_SHAPE,
               "kv->max_rows = %d > shard_rows = %d", kv->max_rows, sh->shard_rows);
  return CSA2_OK;
}

static int cp_nsplit(int batch, int n_layers) {
  const int ns = attn_nsplit(batch * n_layers, num_sms());
  return ns < 2 ? 2 : ns;  // the partials must stay unmerged for the exchange
}

struct CpWs {
  uint32_t* status;
  int32_t* sel;        // [jobs][batch][top_k] local Top-k
  int32_t* sel_count;  // [jobs][batch]
  float* part_o;       // attention split partials
  float* part_ml;
  float* bm;           // [batch][world * S / 8] regrouped block maxima
  int nsplit;
  size_t bytes;
};

static CpWs cp_ws_layout(const csa2_cp_shard* sh, int batch, int n_layers, int top_k,
                         uint8_t* base) {
  CpWs w{};
  w.nsplit = cp_nsplit(batch, n_layers);
  // local selections of up to RS_MAX_JOBS jobs (no more than the layers)
  const size_t n_sel = n_layers < RS_MAX_JOBS ? (size_t)n_layers : (size_t)RS_MAX_JOBS;
  size_t off = CSA2_WS_HEADER;
  w.status = reinterpret_cast<uint32_t*>(base);
  w.sel = reinterpret_cast<int32_t*>(base + off);
  off = align256(off + n_sel * batch * top_k * sizeof(int32_t));
  w.sel_count = reinterpret_cast<int32_t*>(base + off);
  off = align256(off + n_sel * batch * sizeof(int32_t));
  const size_t slots = (size_t)batch * n_layers * w.nsplit;
  w.part_o = reinterpret_cast<float*>(base + off);
  w.part_ml = reinterpret_cast<float*>(base + off + slots * CSA2_H * CSA2_D * sizeof(float));
  off = align256(off + attn_partial_bytes(batch, n_layers, w.nsplit));
  w.bm = reinterpret_cast<float*>(base + off);
  off = align256(off + (size_t)batch * sh->world * (sh->shard_rows / CSA2_BLK) * sizeof(float));
  w.bytes = off;
  return w;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

size_t csa2_index_workspace_size(const csa2_kv_view* kv, int32_t top_k, int32_t pool_blocks) {
  (void)pool_blocks;
  if (!kv || top_k < 1) return 0;
  return index_ws_layout(kv, top_k, nullptr).bytes;
}

csa2_status csa2_index_full(const csa2_kv_view* kv, const uint16_t* q_idx, const float* w,
                            int32_t top_k, int32_t pool_blocks, int32_t* idx, int32_t* idx_count,
                            int32_t* pool, int32_t* pool_count, void* ws, size_t ws_bytes,
                            csa2_stream_t stream) {
  csa2_status r = check_kv(kv);
  if (r) return r;
  if ((r = check_topk(top_k, pool_blocks))) return r;
  CSA2_REQUIRE_PTR(q_idx);
  CSA2_REQUIRE_PTR(w);
  CSA2_REQUIRE_PTR(idx);
  CSA2_REQUIRE_PTR(idx_count);
  CSA2_REQUIRE_PTR(ws);
  if (pool_blocks > 0) {
    CSA2_REQUIRE_PTR(pool);
    CSA2_REQUIRE_PTR(pool_count);
  }
  const IndexWs lay = index_ws_layout(kv, top_k, static_cast<uint8_t*>(ws));
  CSA2_REQUIRE(ws_bytes >= lay.bytes, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes,
               lay.bytes);
  cudaStream_t st = (cudaStream_t)stream;
  const int P = pool_blocks > 0 ? pool_blocks : top_k;
  int32_t* sel = pool_blocks > 0 ? pool : lay.sel;
  int32_t* sel_count = pool_blocks > 0 ? pool_count : lay.sel_count;
  const int sel_stride = pool_blocks > 0 ? pool_blocks : lay.sel_stride;
  if ((r = run_scan_select(kv, q_idx, w, P, sel, sel_count, sel_stride, lay, st))) return r;
  RescoreParams rp = rescore_params(kv, sel, sel_count, sel_stride, top_k, lay.status);
  rp.job[0] = RescoreJob{q_idx, w, idx, idx_count, top_k};
  trace_mark("rescore", st);
  CSA2_CUDA(launch_rescore(rp, 1, kv->batch, cand_blocks_max(kv, P), st));
  trace_mark("end", st);
  return CSA2_OK;
}

csa2_status csa2_index_reindex(const csa2_kv_view* kv, const uint16_t* q_idx, const float* w,
                               const int32_t* pool, const int32_t* pool_count,
                               int32_t pool_stride, int32_t top_k, int32_t* idx,
                               int32_t* idx_count, void* ws, size_t ws_bytes,
                               csa2_stream_t stream) {
  csa2_status r = check_kv(kv);
  if (r) return r;
  if ((r = check_topk(top_k, 0))) return r;
  CSA2_REQUIRE_PTR(q_idx);
  CSA2_REQUIRE_PTR(w);
  CSA2_REQUIRE_PTR(idx);
  CSA2_REQUIRE_PTR(idx_count);
  CSA2_REQUIRE_PTR(ws);
  const IndexWs lay = index_ws_layout(kv, top_k, static_cast<uint8_t*>(ws));
  CSA2_REQUIRE(ws_bytes >= lay.bytes, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes,
               lay.bytes);
  cudaStream_t st = (cudaStream_t)stream;
  if (pool) {
    CSA2_REQUIRE_PTR(pool_count);
    CSA2_REQUIRE(pool_stride >= 1 && pool_stride <= CSA2_MAX_POOL, CSA2_ERR_SHAPE,
                 "pool_stride = %d outside [1, %d]", pool_stride, (int)CSA2_MAX_POOL);
    RescoreParams rp = rescore_params(kv, pool, pool_count, pool_stride, top_k, lay.status);
    rp.job[0] = RescoreJob{q_idx, w, idx, idx_count, top_k};
    trace_mark("rescore", st);
  CSA2_CUDA(launch_rescore(rp, 1, kv->batch, cand_blocks_max(kv, pool_stride), st));
    trace_mark("end", st);
    return CSA2_OK;
  }
  if ((r = run_scan_select(kv, q_idx, w, top_k, lay.sel, lay.sel_count, lay.sel_stride, lay, st)))
    return r;
  RescoreParams rp = rescore_params(kv, lay.sel, lay.sel_count, lay.sel_stride, top_k, lay.status);
  rp.job[0] = RescoreJob{q_idx, w, idx, idx_count, top_k};
  trace_mark("rescore", st);
  CSA2_CUDA(launch_rescore(rp, 1, kv->batch, cand_blocks_max(kv, top_k), st));
  trace_mark("end", st);
  return CSA2_OK;
}

size_t csa2_attn_workspace_size(int32_t batch, int32_t n_layers) {
  if (batch < 1 || n_layers < 1) return 0;
  const int ns = attn_nsplit(batch * n_layers, num_sms());
  return CSA2_WS_HEADER + align256(attn_partial_bytes(batch, n_layers, ns));
}

static csa2_status fill_attn_common(AttnParams& ap, const csa2_kv_view* kv, const int32_t* swa_len,
                                    float sm_scale, int idx_stride, int nq = 1) {
  ap.batch = kv->batch * nq;
  ap.nq = nq;
  ap.swa_rows = CSA2_W + nq - 1;
  ap.idx_stride = idx_stride;
  ap.codes = kv->codes;
  ap.scales = kv->scales;
  ap.page_table = kv->page_table;
  ap.max_pages = kv->max_pages;
  ap.max_rows = kv->max_rows;
  ap.seq_stride = kv->seq_stride;
  ap.pool_rows = kv->pool_rows;
  ap.n_rows = kv->n_rows;
  ap.swa_len = swa_len;
  ap.scale_log2 = sm_scale * 1.4426950408889634f;
  return CSA2_OK;
}

// Attention for every (layer, sequence) unit of a launch.  The tensor-core
// kernel runs one 5-CTA cluster per unit at one CTA per SM: the shape for a
// decode step whose units fit in about two waves of it.  Larger batches (many
// sequences, or many queries per sequence) run the split-KV kernel instead,
// several small CTAs per SM with their partials merged through L2, which
// keeps more units in flight.
static cudaError_t launch_attention(const AttnParams& ap, cudaStream_t st) {
  const int64_t ctas = (int64_t)ap.batch * ap.n_layers * ATTN_TC_CTAS_PER_UNIT;
  if (ctas > 2LL * num_sms()) return launch_attn(ap, st, /*merge=*/true);
  return launch_attn_tc(ap, st);
}

csa2_status csa2_sparse_attn_decode(const uint16_t* q, const csa2_kv_view* kv, const int32_t* idx,
                                    const int32_t* idx_count, int32_t idx_stride,
                                    const uint8_t* swa, const int32_t* swa_len, float sm_scale,
                                    uint16_t* out, void* ws, size_t ws_bytes,
                                    csa2_stream_t stream) {
  csa2_status r = check_kv(kv);
  if (r) return r;
  CSA2_REQUIRE_PTR(q);
  CSA2_REQUIRE_PTR(idx);
  CSA2_REQUIRE_PTR(idx_count);
  CSA2_REQUIRE_PTR(swa);
  CSA2_REQUIRE_PTR(swa_len);
  CSA2_REQUIRE_PTR(out);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(idx_stride >= 1 && idx_stride <= CSA2_MAX_TOPK, CSA2_ERR_SHAPE,
               "idx_stride = %d outside [1, %d]", idx_stride, (int)CSA2_MAX_TOPK);
  CSA2_REQUIRE(sm_scale == sm_scale, CSA2_ERR_INVALID_ARG, "sm_scale is NaN");
  const size_t need = csa2_attn_workspace_size(kv->batch, 1);
  CSA2_REQUIRE(ws_bytes >= need, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  AttnParams ap{};
  fill_attn_common(ap, kv, swa_len, sm_scale, idx_stride);
  ap.n_layers = 1;
  ap.nsplit = attn_nsplit(kv->batch, num_sms());
  ap.layer[0] = AttnLayer{q, swa, idx, idx_count, nullptr, nullptr, out};
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t slots = (size_t)kv->batch * ap.nsplit;
  ap.part_o = reinterpret_cast<float*>(base + CSA2_WS_HEADER);
  ap.part_ml = reinterpret_cast<float*>(base + CSA2_WS_HEADER + slots * CSA2_H * CSA2_D * 4);
  ap.status = static_cast<uint32_t*>(ws);
  CSA2_CUDA(launch_attention(ap, (cudaStream_t)stream));
  trace_mark("end", (cudaStream_t)stream);
  return CSA2_OK;
}

size_t csa2_group_workspace_size(const csa2_group_desc* d) {
  if (!d || d->n_layers < 1 || d->top_k < 1 || d->kv.batch < 1) return 0;
  return group_ws_layout(d, nullptr).bytes;
}

csa2_status csa2_layer_group(const csa2_group_desc* d, void* ws, size_t ws_bytes,
                             csa2_stream_t stream) {
  CSA2_REQUIRE(d != nullptr, CSA2_ERR_INVALID_ARG, "desc is NULL");
  const csa2_kv_view* kv = &d->kv;
  csa2_status r = check_kv(kv);
  if (r) return r;
  if ((r = check_topk(d->top_k, d->pool_blocks))) return r;
  const int L = d->n_layers, B = kv->batch, nq = group_nq(d), VB = B * nq;
  CSA2_REQUIRE(d->n_query >= 0 && d->n_query <= CSA2_MAX_QUERY, CSA2_ERR_SHAPE,
               "n_query = %d outside [0, %d]", d->n_query, (int)CSA2_MAX_QUERY);
  CSA2_REQUIRE(VB <= 65535, CSA2_ERR_SHAPE, "batch x n_query = %d > 65535", VB);
  CSA2_REQUIRE(L >= 1 && L <= AT_MAX_LAYERS, CSA2_ERR_SHAPE, "n_layers = %d outside [1, %d]", L,
               AT_MAX_LAYERS);
  CSA2_REQUIRE(d->modes != nullptr, CSA2_ERR_INVALID_ARG, "modes is NULL");
  for (int l = 0; l < L; l++)
    CSA2_REQUIRE(d->modes[l] >= CSA2_FULL && d->modes[l] <= CSA2_REUSE, CSA2_ERR_INVALID_ARG,
                 "modes[%d] = %d", l, d->modes[l]);
  CSA2_REQUIRE(d->modes[0] == CSA2_FULL, CSA2_ERR_INVALID_ARG,
               "layer 0 must be FULL (REINDEX and REUSE reuse an earlier FULL layer's cache)");
  CSA2_REQUIRE_PTR(d->q_idx);
  CSA2_REQUIRE_PTR(d->w);
  CSA2_REQUIRE_PTR(d->q);
  CSA2_REQUIRE_PTR(d->swa);
  CSA2_REQUIRE_PTR(d->swa_len);
  CSA2_REQUIRE_PTR(d->idx);
  CSA2_REQUIRE_PTR(d->idx_count);
  CSA2_REQUIRE_PTR(d->out);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(d->sm_scale == d->sm_scale, CSA2_ERR_INVALID_ARG, "sm_scale is NaN");
  if (d->pool_blocks > 0) {
    CSA2_REQUIRE_PTR(d->pool);
    CSA2_REQUIRE_PTR(d->pool_count);
  }
  const GroupWs g = group_ws_layout(d, static_cast<uint8_t*>(ws));
  CSA2_REQUIRE(ws_bytes >= g.bytes, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes,
               g.bytes);
  cudaStream_t st = (cudaStream_t)stream;
  const int K = d->top_k;
  const size_t qi_stride = (size_t)VB * CSA2_HI * CSA2_DI, w_stride = (size_t)VB * CSA2_HI;
  auto layer_idx = [&](int l) { return d->idx + (size_t)l * VB * K; };
  auto layer_cnt = [&](int l) { return d->idx_count + (size_t)l * VB; };

  // Indexer: per FULL layer, one scan + block select and one rescore launch
  // for the FULL layer and the REINDEX layers that share its pool.
  const bool hsi = d->pool_blocks > 0;
  for (int l = 0; l < L; l++) {
    if (d->modes[l] == CSA2_REUSE) continue;
    if (d->modes[l] == CSA2_REINDEX && hsi) continue;  // batched with its FULL layer
    const uint16_t* qi = d->q_idx + l * qi_stride;
    const float* wl = d->w + l * w_stride;
    const int P = hsi ? d->pool_blocks : K;
    int32_t* sel = hsi ? d->pool : g.ix.sel;
    int32_t* sel_count = hsi ? d->pool_count : g.ix.sel_count;
    const int sel_stride = hsi ? d->pool_blocks : g.ix.sel_stride;
    if ((r = run_scan_select(kv, qi, wl, P, sel, sel_count, sel_stride, g.ix, st, nq))) return r;
    RescoreParams rp = rescore_params(kv, sel, sel_count, sel_stride, K, g.ix.status, nq);
    int nj = 0;
    rp.job[nj++] = RescoreJob{qi, wl, layer_idx(l), layer_cnt(l), K};
    if (hsi && d->modes[l] == CSA2_FULL) {
      for (int x = l + 1; x < L && d->modes[x] != CSA2_FULL; x++) {
        if (d->modes[x] != CSA2_REINDEX) continue;
        if (nj == RS_MAX_JOBS) {
          trace_mark("rescore", st);
          CSA2_CUDA(launch_rescore(rp, nj, VB, cand_blocks_max(kv, P), st));
          nj = 0;
        }
        rp.job[nj++] =
            RescoreJob{d->q_idx + x * qi_stride, d->w + x * w_stride, layer_idx(x), layer_cnt(x), K};
      }
    }
    trace_mark("rescore", st);
    CSA2_CUDA(launch_rescore(rp, nj, VB, cand_blocks_max(kv, P), st));
  }

  // Attention for every layer in one launch.
  AttnParams ap{};
  fill_attn_common(ap, kv, d->swa_len, d->sm_scale, K, nq);
  ap.n_layers = L;
  ap.nsplit = g.nsplit;
  ap.part_o = g.part_o;
  ap.part_ml = g.part_ml;
  ap.status = g.ix.status;
  int src = 0;
  for (int l = 0; l < L; l++) {
    if (d->modes[l] != CSA2_REUSE) src = l;
    const bool reuse = d->modes[l] == CSA2_REUSE;
    ap.layer[l] = AttnLayer{d->q + (size_t)l * VB * CSA2_H * CSA2_D,
                            d->swa + (size_t)l * B * ap.swa_rows * CSA2_D,
                            layer_idx(src),
                            layer_cnt(src),
                            reuse ? layer_idx(l) : nullptr,
                            reuse ? layer_cnt(l) : nullptr,
                            d->out + (size_t)l * VB * CSA2_H * CSA2_D};
  }
  CSA2_CUDA(launch_attention(ap, st));
  trace_mark("end", st);
  return CSA2_OK;
}

// ------------------------------------------------------------ cache append
csa2_status csa2_cache_append(const csa2_kv_view* kv, const uint16_t* x, const uint16_t* w_idx,
                              int32_t n_layers, const uint16_t* x_swa, uint8_t* swa,
                              int32_t* swa_pos, int32_t* swa_len, void* ws, size_t ws_bytes,
                              csa2_stream_t stream) {
  csa2_status r = check_kv(kv);
  if (r) return r;
  CSA2_REQUIRE_PTR(x);
  CSA2_REQUIRE_PTR(w_idx);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(n_layers >= 0 && n_layers <= 65535 * 4, CSA2_ERR_SHAPE, "n_layers = %d", n_layers);
  if (n_layers > 0) {
    CSA2_REQUIRE_PTR(x_swa);
    CSA2_REQUIRE_PTR(swa);
    CSA2_REQUIRE(swa_pos != nullptr && swa_len != nullptr, CSA2_ERR_INVALID_ARG,
                 "swa_pos and swa_len are required when n_layers > 0");
  }
  AppendParams p{};
  p.codes = const_cast<uint8_t*>(kv->codes);
  p.scales = const_cast<uint8_t*>(kv->scales);
  p.idx_k = const_cast<uint16_t*>(kv->idx_k);
  p.page_table = kv->page_table;
  p.max_pages = kv->max_pages;
  p.seq_stride = kv->seq_stride;
  p.pool_rows = kv->pool_rows;
  p.n_rows = const_cast<int32_t*>(kv->n_rows);
  p.batch = kv->batch;
  p.x = x;
  p.w_idx = w_idx;
  p.n_layers = n_layers;
  p.x_swa = x_swa;
  p.swa = swa;
  p.swa_pos = swa_pos;
  p.swa_len = swa_len;
  p.status = static_cast<uint32_t*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  CSA2_CUDA(launch_append(p, st));
  trace_mark("end", st);
  return CSA2_OK;
}

// ------------------------------------------------- context-parallel decode
size_t csa2_cp_workspace_size(const csa2_cp_shard* sh, int32_t batch, int32_t n_layers,
                              int32_t top_k) {
  if (check_shard(sh) != CSA2_OK || batch < 1 || n_layers < 1 || top_k < 1) return 0;
  return cp_ws_layout(sh, batch, n_layers, top_k, nullptr).bytes;
}

size_t csa2_cp_partial_floats(int32_t batch, int32_t n_layers) {
  if (batch < 1 || n_layers < 1) return 0;
  return (size_t)n_layers * batch * CSA2_H * (CSA2_D + 2);
}

csa2_status csa2_cp_local_rows(const csa2_cp_shard* sh, const int32_t* n_rows, int32_t batch,
                               int32_t* local_rows, void* ws, size_t ws_bytes,
                               csa2_stream_t stream) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  CSA2_REQUIRE_I32(n_rows);
  CSA2_REQUIRE_I32(local_rows);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_CUDA(launch_cp_local_rows(n_rows, batch, (int64_t)sh->rank * sh->shard_rows,
                                 sh->shard_rows, local_rows, static_cast<uint32_t*>(ws),
                                 (cudaStream_t)stream));
  return CSA2_OK;
}

csa2_status csa2_cp_block_max(const csa2_cp_shard* sh, const csa2_kv_view* kv,
                              const uint16_t* q_idx, const float* w, float* bm, void* ws,
                              size_t ws_bytes, csa2_stream_t stream) {
  csa2_status r = check_shard_kv(sh, kv);
  if (r) return r;
  CSA2_REQUIRE_PTR(q_idx);
  CSA2_REQUIRE_PTR(w);
  CSA2_REQUIRE_PTR(bm);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  cudaStream_t st = (cudaStream_t)stream;
  IndexWs iw{};
  iw.status = static_cast<uint32_t*>(ws);
  iw.bm = bm;
  iw.bm_stride = sh->shard_rows / CSA2_BLK;
  CUtensorMap map_k, map_q;
  if ((r = map_rows64(&map_k, kv->idx_k, (uint64_t)kv->pool_rows, 64))) return r;
  if ((r = map_rows64(&map_q, q_idx, (uint64_t)kv->batch * CSA2_HI, scan_query_rows(1)))) return r;
  ScanParams sp = scan_params(kv, w, iw, 1);
  trace_mark("scan", st);
  CSA2_CUDA(launch_scan(map_k, map_q, sp, num_sms(), st));
  return CSA2_OK;
}

csa2_status csa2_cp_pool(const csa2_cp_shard* sh, const float* bm_all, const int32_t* n_rows,
                         int32_t batch, int32_t P, int32_t* pool, int32_t* pool_count, void* ws,
                         size_t ws_bytes, csa2_stream_t stream) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  CSA2_REQUIRE_PTR(bm_all);
  CSA2_REQUIRE_I32(n_rows);
  CSA2_REQUIRE_I32(pool);
  CSA2_REQUIRE_I32(pool_count);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_REQUIRE(P >= 1 && P <= CSA2_MAX_POOL, CSA2_ERR_SHAPE, "P = %d outside [1, %d]", P,
               (int)CSA2_MAX_POOL);
  const CpWs lay = cp_ws_layout(sh, batch, 1, 1, static_cast<uint8_t*>(ws));
  const int nb = sh->shard_rows / CSA2_BLK;
  const bool regroup = sh->world > 1 && batch > 1;
  CSA2_REQUIRE(ws_bytes >= (regroup ? lay.bytes : (size_t)CSA2_WS_HEADER), CSA2_ERR_WORKSPACE,
               "workspace %zu < %zu bytes", ws_bytes, regroup ? lay.bytes : (size_t)CSA2_WS_HEADER);
  cudaStream_t st = (cudaStream_t)stream;
  const float* bm = bm_all;
  if (regroup) {
    CSA2_CUDA(launch_cp_bm_regroup(bm_all, sh->world, batch, nb, lay.bm, st));
    bm = lay.bm;
  }
  trace_mark("block_select", st);
  CSA2_CUDA(launch_block_select(bm, sh->world * nb, n_rows, sh->world * sh->shard_rows, batch, 1,
                                P, pool, P, pool_count, lay.status, st));
  return CSA2_OK;
}

csa2_status csa2_cp_filter(const csa2_cp_shard* sh, int32_t unit, const int32_t* list,
                           const int32_t* count, int32_t stride, int32_t batch, int32_t* out,
                           int32_t* out_count, int32_t out_stride, int32_t* copy,
                           int32_t* copy_count, void* ws, size_t ws_bytes,
                           csa2_stream_t stream) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  CSA2_REQUIRE(unit == 1 || unit == CSA2_BLK, CSA2_ERR_INVALID_ARG, "unit = %d (1 or %d)", unit,
               (int)CSA2_BLK);
  CSA2_REQUIRE_I32(list);
  CSA2_REQUIRE_I32(count);
  CSA2_REQUIRE_I32(out);
  CSA2_REQUIRE_I32(out_count);
  CSA2_REQUIRE((copy == nullptr) == (copy_count == nullptr), CSA2_ERR_INVALID_ARG,
               "copy and copy_count must both be given or both be NULL");
  if (copy) {
    CSA2_REQUIRE_I32(copy);
    CSA2_REQUIRE_I32(copy_count);
  }
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_REQUIRE(stride >= 1 && stride <= CSA2_MAX_POOL, CSA2_ERR_SHAPE,
               "stride = %d outside [1, %d]", stride, (int)CSA2_MAX_POOL);
  CSA2_REQUIRE(out_stride >= 1 && out_stride <= CSA2_MAX_POOL, CSA2_ERR_SHAPE,
               "out_stride = %d outside [1, %d]", out_stride, (int)CSA2_MAX_POOL);
  CpFilterParams p{};
  p.n_lists = 1;
  p.list[0] = list;
  p.count[0] = count;
  p.out[0] = out;
  p.out_count[0] = out_count;
  p.copy[0] = copy;
  p.copy_count[0] = copy_count;
  p.stride = stride;
  p.lo = sh->rank * (sh->shard_rows / unit);
  p.hi = p.lo + sh->shard_rows / unit;
  p.out_stride = out_stride;
  p.status = static_cast<uint32_t*>(ws);
  CSA2_CUDA(launch_cp_filter(p, batch, (cudaStream_t)stream));
  return CSA2_OK;
}

csa2_status csa2_cp_filter_layers(const csa2_cp_shard* sh, int32_t n_layers, const int32_t* src,
                                  int32_t* idx, int32_t* idx_count, int32_t stride,
                                  int32_t batch, int32_t* idx_local, int32_t* idx_local_count,
                                  void* ws, size_t ws_bytes, csa2_stream_t stream) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  CSA2_REQUIRE(n_layers >= 1 && n_layers <= CP_MAX_LISTS, CSA2_ERR_SHAPE,
               "n_layers = %d outside [1, %d]", n_layers, (int)CP_MAX_LISTS);
  CSA2_REQUIRE(src != nullptr, CSA2_ERR_INVALID_ARG, "src is NULL");
  for (int l = 0; l < n_layers; l++) {
    CSA2_REQUIRE(src[l] >= 0 && src[l] <= l && src[src[l]] == src[l], CSA2_ERR_INVALID_ARG,
                 "src[%d] = %d: each layer reads itself or an earlier layer that reads itself",
                 l, src[l]);
  }
  CSA2_REQUIRE_I32(idx);
  CSA2_REQUIRE_I32(idx_count);
  CSA2_REQUIRE_I32(idx_local);
  CSA2_REQUIRE_I32(idx_local_count);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_REQUIRE(stride >= 1 && stride <= CSA2_MAX_POOL, CSA2_ERR_SHAPE,
               "stride = %d outside [1, %d]", stride, (int)CSA2_MAX_POOL);
  CpFilterParams p{};
  p.n_lists = n_layers;
  const int64_t ls = (int64_t)batch * stride;  // one layer's index list
  for (int l = 0; l < n_layers; l++) {
    p.list[l] = idx + src[l] * ls;
    p.count[l] = idx_count + (int64_t)src[l] * batch;
    p.out[l] = idx_local + l * ls;
    p.out_count[l] = idx_local_count + (int64_t)l * batch;
    p.copy[l] = src[l] != l ? idx + l * ls : nullptr;
    p.copy_count[l] = src[l] != l ? idx_count + (int64_t)l * batch : nullptr;
  }
  p.stride = stride;
  p.lo = sh->rank * sh->shard_rows;
  p.hi = p.lo + sh->shard_rows;
  p.out_stride = stride;
  p.status = static_cast<uint32_t*>(ws);
  CSA2_CUDA(launch_cp_filter(p, batch, (cudaStream_t)stream));
  return CSA2_OK;
}

}  // extern "C"

namespace csa2 {
// The shard's Top-k of n_jobs jobs over one candidate list: one rescore
// launch (a cluster per (job, sequence)) and one export launch.
static csa2_status cp_select_local_impl(const csa2_cp_shard* sh, const csa2_kv_view* kv,
                                        int n_jobs, const uint16_t* const* q_idx,
                                        const float* const* w, const int32_t* cand,
                                        const int32_t* cand_count, int32_t cand_stride,
                                        int32_t top_k, uint2* const* send, void* ws,
                                        size_t ws_bytes, cudaStream_t st) {
  csa2_status r = check_shard_kv(sh, kv);
  if (r) return r;
  if ((r = check_topk(top_k, 0))) return r;
  for (int j = 0; j < n_jobs; j++) {
    CSA2_REQUIRE(q_idx[j] != nullptr && aligned16(q_idx[j]), CSA2_ERR_ALIGNMENT,
                 "job %d: q_idx is NULL or not 16-byte aligned", j);
    CSA2_REQUIRE(w[j] != nullptr && aligned16(w[j]), CSA2_ERR_ALIGNMENT,
                 "job %d: w is NULL or not 16-byte aligned", j);
    CSA2_REQUIRE(send[j] != nullptr && (reinterpret_cast<uintptr_t>(send[j]) & 7u) == 0,
                 CSA2_ERR_ALIGNMENT, "send is NULL or not 8-byte aligned");
  }
  CSA2_REQUIRE_I32(cand);
  CSA2_REQUIRE_I32(cand_count);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(cand_stride >= 1 && cand_stride <= CSA2_MAX_POOL, CSA2_ERR_SHAPE,
               "cand_stride = %d outside [1, %d]", cand_stride, (int)CSA2_MAX_POOL);
  const CpWs lay = cp_ws_layout(sh, kv->batch, n_jobs, top_k, static_cast<uint8_t*>(ws));
  const size_t need = reinterpret_cast<uint8_t*>(lay.part_o) - static_cast<uint8_t*>(ws);
  CSA2_REQUIRE(ws_bytes >= need, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  const int B = kv->batch;
  RescoreParams rp = rescore_params(kv, cand, cand_count, cand_stride, top_k, lay.status);
  CpExportParams xp{};
  for (int j = 0; j < n_jobs; j++) {
    int32_t* sel = lay.sel + (int64_t)j * B * top_k;
    int32_t* sel_count = lay.sel_count + (int64_t)j * B;
    rp.job[j] = RescoreJob{q_idx[j], w[j], sel, sel_count, top_k};
    xp.q_idx[j] = q_idx[j];
    xp.w[j] = w[j];
    xp.idx[j] = sel;
    xp.idx_count[j] = sel_count;
    xp.send[j] = send[j];
  }
  trace_mark("rescore", st);
  CSA2_CUDA(launch_rescore(rp, n_jobs, B, cand_blocks_max(kv, cand_stride), st));
  xp.n_jobs = n_jobs;
  xp.idx_k = kv->idx_k;
  xp.page_table = kv->page_table;
  xp.max_pages = kv->max_pages;
  xp.max_rows = kv->max_rows;
  xp.seq_stride = kv->seq_stride;
  xp.pool_rows = kv->pool_rows;
  xp.n_rows = kv->n_rows;
  xp.top_k = top_k;
  xp.pos_base = sh->rank * sh->shard_rows;
  xp.status = lay.status;
  CSA2_CUDA(launch_cp_export(xp, B, st));
  return CSA2_OK;
}

// The global Top-k of gathered jobs job0 .. job0 + n_sel - 1 in one launch
// (a CTA per (sequence, job)).
static csa2_status cp_select_merge_impl(const csa2_cp_shard* sh, const uint32_t* gathered,
                                        int n_jobs, int job0, int n_sel, int batch, int top_k,
                                        int32_t* const* idx, int32_t* const* idx_count,
                                        void* ws, size_t ws_bytes, cudaStream_t st) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  if ((r = check_topk(top_k, 0))) return r;
  CSA2_REQUIRE(gathered != nullptr && (reinterpret_cast<uintptr_t>(gathered) & 7u) == 0,
               CSA2_ERR_ALIGNMENT, "gathered is NULL or not 8-byte aligned");
  for (int j = 0; j < n_sel; j++) {
    CSA2_REQUIRE_I32(idx[j]);
    CSA2_REQUIRE_I32(idx_count[j]);
  }
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_REQUIRE(sh->world * top_k <= cp_merge_capacity(), CSA2_ERR_SHAPE,
               "world x top_k = %d > %d", sh->world * top_k, cp_merge_capacity());
  CpMergeParams p{};
  p.gathered = reinterpret_cast<const uint2*>(gathered);
  p.world = sh->world;
  p.n_jobs = n_jobs;
  p.job0 = job0;
  p.n_sel = n_sel;
  p.batch = batch;
  p.top_k = top_k;
  for (int j = 0; j < n_sel; j++) {
    p.idx[j] = idx[j];
    p.idx_count[j] = idx_count[j];
  }
  CSA2_CUDA(launch_cp_merge_select(p, st));
  return CSA2_OK;
}
}  // namespace csa2

extern "C" {

csa2_status csa2_cp_select_local(const csa2_cp_shard* sh, const csa2_kv_view* kv,
                                 const uint16_t* q_idx, const float* w, const int32_t* cand,
                                 const int32_t* cand_count, int32_t cand_stride, int32_t top_k,
                                 uint32_t* send, void* ws, size_t ws_bytes,
                                 csa2_stream_t stream) {
  uint2* s0 = reinterpret_cast<uint2*>(send);
  return cp_select_local_impl(sh, kv, 1, &q_idx, &w, cand, cand_count, cand_stride, top_k, &s0,
                              ws, ws_bytes, (cudaStream_t)stream);
}

csa2_status csa2_cp_select_local_jobs(const csa2_cp_shard* sh, const csa2_kv_view* kv,
                                      int32_t n_jobs, const int32_t* layer, int32_t n_layers,
                                      const uint16_t* q_idx, const float* w,
                                      const int32_t* cand, const int32_t* cand_count,
                                      int32_t cand_stride, int32_t top_k, uint32_t* send,
                                      void* ws, size_t ws_bytes, csa2_stream_t stream) {
  if (!kv) return fail(CSA2_ERR_INVALID_ARG, "kv is NULL");
  CSA2_REQUIRE(n_jobs >= 1 && n_jobs <= RS_MAX_JOBS, CSA2_ERR_SHAPE,
               "n_jobs = %d outside [1, %d]", n_jobs, (int)RS_MAX_JOBS);
  CSA2_REQUIRE(layer != nullptr, CSA2_ERR_INVALID_ARG, "layer is NULL");
  CSA2_REQUIRE_PTR(q_idx);
  CSA2_REQUIRE_PTR(w);
  CSA2_REQUIRE(send != nullptr, CSA2_ERR_INVALID_ARG, "send is NULL");
  const uint16_t* qs[RS_MAX_JOBS];
  const float* ws_[RS_MAX_JOBS];
  uint2* sends[RS_MAX_JOBS];
  const int64_t B = kv->batch;
  for (int j = 0; j < n_jobs; j++) {
    CSA2_REQUIRE(layer[j] >= 0 && layer[j] < n_layers, CSA2_ERR_INVALID_ARG,
                 "layer[%d] = %d outside [0, %d)", j, layer[j], n_layers);
    qs[j] = q_idx + layer[j] * B * CSA2_HI * CSA2_DI;
    ws_[j] = w + layer[j] * B * CSA2_HI;
    sends[j] = reinterpret_cast<uint2*>(send) + j * B * top_k;
  }
  return cp_select_local_impl(sh, kv, n_jobs, qs, ws_, cand, cand_count, cand_stride, top_k,
                              sends, ws, ws_bytes, (cudaStream_t)stream);
}

csa2_status csa2_cp_select_merge(const csa2_cp_shard* sh, const uint32_t* gathered,
                                 int32_t n_jobs, int32_t job, int32_t batch, int32_t top_k,
                                 int32_t* idx, int32_t* idx_count, void* ws, size_t ws_bytes,
                                 csa2_stream_t stream) {
  CSA2_REQUIRE(n_jobs >= 1 && job >= 0 && job < n_jobs, CSA2_ERR_INVALID_ARG,
               "job = %d, n_jobs = %d", job, n_jobs);
  return cp_select_merge_impl(sh, gathered, n_jobs, job, 1, batch, top_k, &idx, &idx_count, ws,
                              ws_bytes, (cudaStream_t)stream);
}

csa2_status csa2_cp_select_merge_jobs(const csa2_cp_shard* sh, const uint32_t* gathered,
                                      int32_t n_jobs, const int32_t* layer, int32_t n_layers,
                                      int32_t batch, int32_t top_k, int32_t* idx,
                                      int32_t* idx_count, void* ws, size_t ws_bytes,
                                      csa2_stream_t stream) {
  CSA2_REQUIRE(n_jobs >= 1 && n_jobs <= RS_MAX_JOBS, CSA2_ERR_SHAPE,
               "n_jobs = %d outside [1, %d]", n_jobs, (int)RS_MAX_JOBS);
  CSA2_REQUIRE(layer != nullptr, CSA2_ERR_INVALID_ARG, "layer is NULL");
  CSA2_REQUIRE(idx != nullptr && idx_count != nullptr, CSA2_ERR_INVALID_ARG,
               "idx or idx_count is NULL");
  int32_t* outs[RS_MAX_JOBS];
  int32_t* counts[RS_MAX_JOBS];
  for (int j = 0; j < n_jobs; j++) {
    CSA2_REQUIRE(layer[j] >= 0 && layer[j] < n_layers, CSA2_ERR_INVALID_ARG,
                 "layer[%d] = %d outside [0, %d)", j, layer[j], n_layers);
    outs[j] = idx + (int64_t)layer[j] * batch * top_k;
    counts[j] = idx_count + (int64_t)layer[j] * batch;
  }
  return cp_select_merge_impl(sh, gathered, n_jobs, 0, n_jobs, batch, top_k, outs, counts, ws,
                              ws_bytes, (cudaStream_t)stream);
}

csa2_status csa2_cp_attn_partial(const csa2_cp_shard* sh, const csa2_kv_view* kv,
                                 int32_t n_layers, const uint16_t* q, const uint8_t* swa,
                                 const int32_t* swa_len, const int32_t* idx_local,
                                 const int32_t* idx_count, int32_t idx_stride, float sm_scale,
                                 float* partial, void* ws, size_t ws_bytes,
                                 csa2_stream_t stream) {
  csa2_status r = check_shard_kv(sh, kv);
  if (r) return r;
  CSA2_REQUIRE(n_layers >= 1 && n_layers <= AT_MAX_LAYERS, CSA2_ERR_SHAPE,
               "n_layers = %d outside [1, %d]", n_layers, AT_MAX_LAYERS);
  CSA2_REQUIRE_PTR(q);
  CSA2_REQUIRE_PTR(swa);
  CSA2_REQUIRE_I32(swa_len);
  CSA2_REQUIRE_I32(idx_local);
  CSA2_REQUIRE_I32(idx_count);
  CSA2_REQUIRE_PTR(partial);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(idx_stride >= 1 && idx_stride <= CSA2_MAX_TOPK, CSA2_ERR_SHAPE,
               "idx_stride = %d outside [1, %d]", idx_stride, (int)CSA2_MAX_TOPK);
  CSA2_REQUIRE(sm_scale == sm_scale, CSA2_ERR_INVALID_ARG, "sm_scale is NaN");
  const int B = kv->batch;
  const CpWs lay = cp_ws_layout(sh, B, n_layers, 1, static_cast<uint8_t*>(ws));
  const size_t need = reinterpret_cast<uint8_t*>(lay.bm) - static_cast<uint8_t*>(ws);
  CSA2_REQUIRE(ws_bytes >= need, CSA2_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  AttnParams ap{};
  fill_attn_common(ap, kv, swa_len, sm_scale, idx_stride);
  ap.n_layers = n_layers;
  ap.nsplit = lay.nsplit;
  ap.part_o = lay.part_o;
  ap.part_ml = lay.part_ml;
  ap.status = lay.status;
  for (int l = 0; l < n_layers; l++)
    ap.layer[l] = AttnLayer{q + (size_t)l * B * CSA2_H * CSA2_D,
                            swa + (size_t)l * B * CSA2_W * CSA2_D,
                            idx_local + (size_t)l * B * idx_stride,
                            idx_count + (size_t)l * B,
                            nullptr,
                            nullptr,
                            nullptr};  // nsplit >= 2: the output is never written here
  CSA2_CUDA(launch_attn(ap, st, /*merge=*/false));
  const size_t o_floats = (size_t)n_layers * B * CSA2_H * CSA2_D;
  CpAttnMergeParams mp{};
  mp.part_o = lay.part_o;
  mp.part_ml = lay.part_ml;
  mp.o_pstride = CSA2_H * CSA2_D;
  mp.o_sstride = (int64_t)lay.nsplit * CSA2_H * CSA2_D;
  mp.ml_pstride = CSA2_H * 2;
  mp.ml_sstride = (int64_t)lay.nsplit * CSA2_H * 2;
  mp.nparts = lay.nsplit;
  mp.batch = B;
  mp.out_o = partial;
  mp.out_ml = partial + o_floats;
  CSA2_CUDA(launch_cp_attn_merge(mp, n_layers, false, st));
  return CSA2_OK;
}

csa2_status csa2_cp_attn_combine(const csa2_cp_shard* sh, const float* gathered,
                                 int32_t n_layers, int32_t batch, uint16_t* out, void* ws,
                                 size_t ws_bytes, csa2_stream_t stream) {
  csa2_status r = check_shard(sh);
  if (r) return r;
  CSA2_REQUIRE_PTR(gathered);
  CSA2_REQUIRE_PTR(out);
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE, "workspace %zu < %d bytes",
               ws_bytes, CSA2_WS_HEADER);
  CSA2_REQUIRE(batch >= 1 && batch <= 65535, CSA2_ERR_SHAPE, "batch = %d", batch);
  CSA2_REQUIRE(n_layers >= 1 && n_layers <= 65535, CSA2_ERR_SHAPE, "n_layers = %d", n_layers);
  CSA2_REQUIRE(sh->world <= CP_MAX_PARTS, CSA2_ERR_SHAPE, "world = %d > %d", sh->world,
               CP_MAX_PARTS);
  const size_t per_rank = csa2_cp_partial_floats(batch, n_layers);
  const size_t o_floats = (size_t)n_layers * batch * CSA2_H * CSA2_D;
  CpAttnMergeParams mp{};
  mp.part_o = gathered;
  mp.part_ml = gathered + o_floats;
  mp.o_pstride = (int64_t)per_rank;
  mp.o_sstride = CSA2_H * CSA2_D;
  mp.ml_pstride = (int64_t)per_rank;
  mp.ml_sstride = CSA2_H * 2;
  mp.nparts = sh->world;
  mp.batch = batch;
  mp.out = out;
  CSA2_CUDA(launch_cp_attn_merge(mp, n_layers, true, (cudaStream_t)stream));
  return CSA2_OK;
}

}  // extern "C"
