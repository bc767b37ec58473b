// kernels.h -- launch interfaces between the C ABI (capi*.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

#include <mutex>

namespace csa2 {

// Host-side set-up that a launcher does once per device (kernel attributes,
// resident-CTA counts), thread-safe; devices beyond the table run it every time.
struct PerDeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::once_flag flag[kMaxDevices];
  cudaError_t err[kMaxDevices] = {};
  int value[kMaxDevices] = {};
  template <class F>  // F: cudaError_t (int& value)
  cudaError_t run(F f, int* out = nullptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) {
      int v = 0;
      e = f(v);
      if (out) *out = v;
      return e;
    }
    std::call_once(flag[dev], [&] { err[dev] = f(value[dev]); });
    if (out) *out = value[dev];
    return err[dev];
  }
};


void trace_mark(const char* stage, cudaStream_t st);  // capi.cu

// score.cu -------------------------------------------------------------
struct ScanParams {
  const int32_t* n_rows;
  const int32_t* page_table;
  int32_t max_pages;
  int32_t max_rows;
  int64_t seq_stride;
  int64_t pool_rows;
  const float* w;
  float* bm;
  int32_t bm_stride;
  int32_t batch;
  int32_t tiles_per_seq;
  int32_t nq;        // queries per sequence; w and bm are [batch * nq][...]
  int32_t q_first;   // this launch scores queries [q_first, q_first + nq_pass)
  int32_t nq_pass;   // 1..8
  int32_t tail;      // nq - (q_first + nq_pass): later queries not in this launch
  uint32_t* status;
  uint32_t* sched;   // tile counter, zero at launch and again at exit (workspace header)
};
constexpr int SC_TILE = 128;
// Word of the workspace header where the scan's tile counter lives (the
// status word is word 0); it is zero between launches.
constexpr int CSA2_WS_SCHED_WORD = 16;
constexpr int CSA2_SCAN_QUERIES = 8;  // queries one scan launch scores (MMA N <= 64)

constexpr int RS_MAX_JOBS = 8;
static_assert(RS_MAX_JOBS == CSA2_CP_MAX_JOBS, "jobs of one rescore launch");
struct RescoreJob {
  const uint16_t* q_idx;
  const float* w;
  int32_t* idx;
  int32_t* idx_count;
  int32_t idx_stride;
};
struct RescoreParams {
  RescoreJob job[RS_MAX_JOBS];
  const uint16_t* idx_k;
  const int32_t* page_table;
  int32_t max_pages;
  int32_t max_rows;
  int64_t seq_stride;
  int64_t pool_rows;
  const int32_t* n_rows;
  const int32_t* cand;
  const int32_t* cand_count;
  int32_t cand_stride;
  int32_t top_k;
  int32_t nq;        // queries per sequence: blockIdx.y runs over batch * nq
  uint32_t* status;
};

int num_sms();  // SMs of the current device (capi.cu)
cudaError_t launch_scan(const CUtensorMap& map_k, const CUtensorMap& map_q, const ScanParams& p,
                        int num_sms, cudaStream_t st);
cudaError_t launch_rescore(const RescoreParams& p, int n_jobs, int batch, int n_cand_blocks,
                           cudaStream_t st);
// batch counts sequences x queries (nq per sequence).
cudaError_t launch_block_select(const float* bm, int bm_stride, const int32_t* n_rows,
                                int max_rows, int batch, int nq, int k_req, int32_t* sel,
                                int sel_stride, int32_t* sel_count, uint32_t* status,
                                cudaStream_t st);
int scan_query_rows(int nq);

// attn.cu --------------------------------------------------------------
constexpr int AT_MAX_LAYERS = 32;
struct AttnLayer {
  const uint16_t* q;
  const uint8_t* swa;
  const int32_t* idx;
  const int32_t* idx_count;
  int32_t* idx_copy;
  int32_t* idx_copy_count;
  uint16_t* out;
};
struct AttnParams {
  AttnLayer layer[AT_MAX_LAYERS];
  int32_t n_layers, batch, idx_stride, nsplit;
  const uint8_t* codes;
  const uint8_t* scales;
  const int32_t* page_table;
  int32_t max_pages;
  int32_t max_rows;
  int64_t seq_stride;
  int64_t pool_rows;
  const int32_t* n_rows;
  const int32_t* swa_len;
  float scale_log2;
  int32_t nq;        // queries per sequence: blockIdx.y runs over batch * nq
  int32_t swa_rows;  // window rows per (layer, sequence): 128 + nq - 1
  float* part_o;   // [n_layers][batch][nsplit][16][512] split partials (nsplit > 1)
  float* part_ml;  // [n_layers][batch][nsplit][16][2] their max and sum
  uint32_t* status;
};
int attn_nsplit(int pairs, int num_sms);
size_t attn_partial_bytes(int batch, int n_layers, int nsplit);
// merge = false leaves the split partials in part_o / part_ml (nsplit > 1).
cudaError_t launch_attn(const AttnParams& p, cudaStream_t st, bool merge = true);
// The tensor-core attention: one 5-CTA cluster per (layer, sequence), merged
// in the cluster, bf16 output (part_o / part_ml unused).
constexpr int ATTN_TC_CTAS_PER_UNIT = 5;  // attn_tc_kernel: CTAs (one cluster) per (layer, sequence)
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t st);

// ------------------------------------------------------------ cache append
struct AppendParams {
  uint8_t* codes;
  uint8_t* scales;
  uint16_t* idx_k;
  const int32_t* page_table;
  int32_t max_pages;
  int64_t seq_stride;
  int64_t pool_rows;
  int32_t* n_rows;
  int32_t batch;
  const uint16_t* x;       // [batch][512] new main-KV entries, bf16
  const uint16_t* w_idx;   // [512][64] indexer-K projection, bf16
  int32_t n_layers;
  const uint16_t* x_swa;   // [n_layers][batch][512] new window entries, bf16
  uint8_t* swa;            // [n_layers][batch][128][512] E4M3 window rings
  int32_t* swa_pos;        // [batch] window entries written so far
  int32_t* swa_len;        // [batch] valid window rows
  uint32_t* status;
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t st);

// ------------------------------------------------- context-parallel decode
constexpr int CP_MAX_PARTS = 16;  // shards (and attention splits) one merge combines
constexpr int CP_MAX_LISTS = AT_MAX_LAYERS;  // lists one filter launch handles
struct CpFilterParams {
  // list u (blockIdx.y, u < n_lists):
  const int32_t* list[CP_MAX_LISTS];   // [batch][stride] ascending ids
  const int32_t* count[CP_MAX_LISTS];  // [batch]
  int32_t* out[CP_MAX_LISTS];          // [batch][out_stride]
  int32_t* out_count[CP_MAX_LISTS];    // [batch]
  int32_t* copy[CP_MAX_LISTS];         // optional verbatim copy of list / count
  int32_t* copy_count[CP_MAX_LISTS];
  int32_t n_lists;
  int32_t stride;        // <= CSA2_MAX_POOL
  int32_t lo, hi;        // kept: lo <= id < hi, written as id - lo
  int32_t out_stride;
  uint32_t* status;
};
struct CpExportParams {
  const uint16_t* idx_k;
  const int32_t* page_table;
  int32_t max_pages;
  int32_t max_rows;
  int64_t seq_stride;
  int64_t pool_rows;
  const int32_t* n_rows;     // this shard's visible rows per sequence
  // job j (blockIdx.z, j < n_jobs):
  const uint16_t* q_idx[RS_MAX_JOBS];     // [batch][8][64]
  const float* w[RS_MAX_JOBS];            // [batch][8]
  const int32_t* idx[RS_MAX_JOBS];        // [batch][top_k] local positions, ascending
  const int32_t* idx_count[RS_MAX_JOBS];  // [batch]
  uint2* send[RS_MAX_JOBS];               // [batch][top_k] (key, global position)
  int32_t n_jobs;
  int32_t top_k;
  int32_t pos_base;          // global position of local position 0
  uint32_t* status;
};
struct CpMergeParams {
  const uint2* gathered;  // [world][n_jobs][batch][top_k]
  int32_t world, n_jobs, batch, top_k;
  // launch job j (blockIdx.y, j < n_sel) merges gathered job job0 + j into:
  int32_t job0, n_sel;
  int32_t* idx[RS_MAX_JOBS];        // [batch][top_k]
  int32_t* idx_count[RS_MAX_JOBS];  // [batch]
};
struct CpAttnMergeParams {
  const float* part_o;
  const float* part_ml;
  int64_t o_pstride, o_sstride, ml_pstride, ml_sstride;  // floats
  int32_t nparts, batch;
  float* out_o;      // merged partials [slot][16][512] (local merge)
  float* out_ml;     // [slot][16][2]
  uint16_t* out;     // bf16 [slot][16][512] (final merge)
};
cudaError_t launch_cp_local_rows(const int32_t* n_rows, int batch, int64_t lo, int shard_rows,
                                 int32_t* local_rows, uint32_t* status, cudaStream_t st);
cudaError_t launch_cp_bm_regroup(const float* src, int world, int batch, int nb, float* dst,
                                 cudaStream_t st);
cudaError_t launch_cp_filter(const CpFilterParams& p, int batch, cudaStream_t st);
cudaError_t launch_cp_export(const CpExportParams& p, int batch, cudaStream_t st);
cudaError_t launch_cp_merge_select(const CpMergeParams& p, cudaStream_t st);
cudaError_t launch_cp_attn_merge(const CpAttnMergeParams& p, int n_layers, bool final_out,
                                 cudaStream_t st);
int cp_merge_capacity();

}  // namespace csa2
