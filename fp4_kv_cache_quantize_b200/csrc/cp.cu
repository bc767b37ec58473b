// cp.cu -- context-parallel decode: every sequence's positions are cut into
// contiguous shards of S rows, shard r = positions [r*S, (r+1)*S) on rank r,
// and one decode step becomes local work on each shard plus small exchanges
// (the sharding follows from the method: scores, block maxima and attention
// rows are per position, and the release note's section "Compressed Sparse
// Attention 2 (CSA2)" and the yomxxx.com notes' section 二 define every
// selection as a Top-k over positions or blocks, which decomposes over
// shards).
//
// What runs where (kernels of this file marked *):
//   scan over the shard's rows            -> its block maxima [B][S/8]
//   exchange (all-gather)                  -> [world][B][S/8]
//   * cp_bm_regroup_kernel                 -> [B][world*S/8] (global block order)
//   block select over the global maxima    -> the pool, the same on every rank
//   * cp_filter_kernel                     -> the pool blocks this shard owns
//   rescore + Top-k over owned candidates  -> local Top-k (local positions)
//   * cp_export_kernel                     -> (key, global position) pairs
//   exchange (all-gather)                  -> [world][jobs][B][k] pairs
//   * cp_merge_select_kernel               -> the global Top-k, every rank
//   * cp_filter_kernel                     -> the selected rows this shard owns
//   attention over them (+ the window on the rank that holds it), split-KV
//   * cp_attn_merge_kernel<false>          -> one (O, max, sum) per head
//   exchange (all-gather)                  -> [world] partials
//   * cp_attn_merge_kernel<true>           -> the bf16 output
//
// Exactness: a shard's Top-k under the same total order (key, then lower
// position) contains every element of the global Top-k that lies in the
// shard, so the Top-k of the union of shard lists is the global Top-k.  The
// export kernel recomputes each selected row's key with the rescore kernel's
// exact instruction sequence (same MMA fragments, same epilogue), so the keys
// it exchanges are bit-identical to those the local selection ranked.
#include <cuda_bf16.h>

#include <utility>

#include "csa2_internal.cuh"
#include "kernels.h"
#include "select.cuh"

namespace csa2 {

// ----------------------------------------------------------- shard sizes
__global__ void cp_local_rows_kernel(const int32_t* n_rows, int32_t batch, int64_t lo,
                                     int32_t shard_rows, int32_t* local_rows, uint32_t* status) {
  pdl_launch_dependents();
  pdl_wait();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    const int n = n_rows[b];
    if (n < 0) set_status(status, ST_DEVICE_CHECK);
    const int64_t v = (int64_t)n - lo;
    local_rows[b] = v < 0 ? 0 : (v > shard_rows ? shard_rows : (int32_t)v);
  }
}

// [world][B][nb] -> [B][world * nb]: sequence b's block maxima in global block order.
__global__ void cp_bm_regroup_kernel(const float* __restrict__ src, int32_t world, int32_t batch,
                                     int32_t nb, float* __restrict__ dst) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t per_seq = (int64_t)world * nb, total = per_seq * batch;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / per_seq, rem = i - b * per_seq;
    const int64_t g = rem / nb, j = rem - g * nb;
    dst[i] = src[(g * batch + b) * nb + j];
  }
}

// ------------------------------------------------------------ range filter
// For each list u and sequence: out = [x - lo for x in list[:count] if lo <= x
// < hi], in list order (ascending stays ascending), -1 padded to out_stride.
// copy, when given, receives the list and its count verbatim.  One CTA per
// (sequence, list): every layer's filter is one launch.
constexpr int CPF_NT = 256;

__global__ void __launch_bounds__(CPF_NT) cp_filter_kernel(const CpFilterParams p) {
  __shared__ uint32_t wsum[32];
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x, u = blockIdx.y, t = threadIdx.x;
  const int32_t* list = p.list[u];
  int32_t* copy = p.copy[u];
  int n = p.count[u][b];
  if (n < 0 || n > p.stride) {
    if (t == 0) set_status(p.status, ST_DEVICE_CHECK);
    n = n < 0 ? 0 : p.stride;
  }
  const int32_t* src = list + (int64_t)b * p.stride;
  const int per = (p.stride + CPF_NT - 1) / CPF_NT;  // <= 8: stride <= CSA2_MAX_POOL
  const int i0 = t * per;
  uint32_t mine = 0u;
  for (int j = 0; j < per; j++) {
    const int i = i0 + j;
    if (i < n) {
      const int x = src[i];
      mine += (x >= p.lo && x < p.hi) ? 1u : 0u;
    }
  }
  uint32_t total;
  uint32_t at = block_excl_scan<CPF_NT>(mine, wsum, total);
  int32_t* dst = p.out[u] + (int64_t)b * p.out_stride;
  for (int j = 0; j < per; j++) {
    const int i = i0 + j;
    if (i < n) {
      const int x = src[i];
      if (x >= p.lo && x < p.hi && (int)at < p.out_stride) dst[at++] = x - p.lo;
    }
  }
  const int m = (int)total < p.out_stride ? (int)total : p.out_stride;
  for (int i = m + t; i < p.out_stride; i += CPF_NT) dst[i] = -1;
  if (t == 0) p.out_count[u][b] = m;
  if (copy) {
    for (int i = t; i < p.stride; i += CPF_NT) copy[(int64_t)b * p.stride + i] = src[i];
    if (t == 0) p.copy_count[u][b] = n;
  }
}

// -------------------------------------------------------------- key export
__device__ __forceinline__ int64_t cp_row(const CpExportParams& p, int b, int pos) {
  if (p.page_table) {
    const int page = pos >> 6;
    const int64_t pid =
        page < p.max_pages ? (int64_t)p.page_table[(int64_t)b * p.max_pages + page] : -1;
    const int64_t row = pid * 64 + (pos & 63);
    return (pid < 0 || row >= p.pool_rows) ? -1 : row;
  }
  const int64_t row = (int64_t)b * p.seq_stride + pos;
  return row < p.pool_rows ? row : -1;
}

__device__ __forceinline__ void cp_mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One warp scores 16 selected rows per MMA (rows grp and grp + 8), with the
// fragment layout, channel permutation and epilogue of the rescore kernel:
// s = sum over heads of w_h * relu(q_h . k), heads (2c, 2c+1) per lane, then
// two butterfly adds.  Writes (key, global position), or (0, -1) past count.
constexpr int CPX_NT = 256;
constexpr int CPX_ROWS = CPX_NT / 32 * 16;  // rows per CTA

__global__ void __launch_bounds__(CPX_NT) cp_export_kernel(const CpExportParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y, j = blockIdx.z, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = lane & 3, grp = lane >> 2;
  const int32_t* idx = p.idx[j];
  int n = p.idx_count[j][b];
  if (n < 0 || n > p.top_k) {
    if (t == 0 && blockIdx.x == 0) set_status(p.status, ST_DEVICE_CHECK);
    n = n < 0 ? 0 : p.top_k;
  }
  int C = p.n_rows[b];
  C = C < 0 ? 0 : (C > p.max_rows ? p.max_rows : C);
  uint32_t bq[8];
  {
    const uint4* qp =
        reinterpret_cast<const uint4*>(p.q_idx[j] + ((int64_t)b * CSA2_HI + grp) * CSA2_DI + 16 * c);
    const uint4 q0 = __ldg(qp), q1 = __ldg(qp + 1);
    bq[0] = q0.x; bq[1] = q0.y; bq[2] = q0.z; bq[3] = q0.w;
    bq[4] = q1.x; bq[5] = q1.y; bq[6] = q1.z; bq[7] = q1.w;
  }
  const float w0 = __ldg(p.w[j] + b * CSA2_HI + 2 * c),
              w1 = __ldg(p.w[j] + b * CSA2_HI + 2 * c + 1);
  const int g0 = blockIdx.x * CPX_ROWS + warp * 16;  // first row of this warp's group
  uint32_t av[2][8];
  bool valid[2];
  int pos[2];
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const int e = g0 + grp + 8 * h;
    pos[h] = e < n ? idx[(int64_t)b * p.top_k + e] : -1;
    valid[h] = pos[h] >= 0 && pos[h] < C;
    if (e < n && !valid[h]) set_status(p.status, ST_DEVICE_CHECK);
    int64_t row = -1;
    if (valid[h]) {
      row = cp_row(p, b, pos[h]);
      if (row < 0) {
        set_status(p.status, ST_DEVICE_CHECK);
        valid[h] = false;
      }
    }
    if (row >= 0) {
      const uint4* kp = reinterpret_cast<const uint4*>(p.idx_k + row * CSA2_DI + 16 * c);
      const uint4 k0 = __ldg(kp), k1 = __ldg(kp + 1);
      av[h][0] = k0.x; av[h][1] = k0.y; av[h][2] = k0.z; av[h][3] = k0.w;
      av[h][4] = k1.x; av[h][5] = k1.y; av[h][6] = k1.z; av[h][7] = k1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; i++) av[h][i] = 0u;
    }
  }
  float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    const uint32_t a[4] = {av[0][2 * ks], av[1][2 * ks], av[0][2 * ks + 1], av[1][2 * ks + 1]};
    cp_mma_bf16_16816(d, a, bq[2 * ks], bq[2 * ks + 1]);
  }
  float s0 = fmaf(w1, fmaxf(d[1], 0.f), w0 * fmaxf(d[0], 0.f));
  float s1 = fmaf(w1, fmaxf(d[3], 0.f), w0 * fmaxf(d[2], 0.f));
  s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
  s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
  s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
  s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
  if (c == 0) {
    const float s[2] = {s0, s1};
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int e = g0 + grp + 8 * h;
      if (e < p.top_k) {
        uint2 v = make_uint2(0u, 0xFFFFFFFFu);
        if (valid[h]) v = make_uint2(float_key(s[h]), (uint32_t)(pos[h] + p.pos_base));
        p.send[j][(int64_t)b * p.top_k + e] = v;
      }
    }
  }
}

// ------------------------------------------------------------- Top-k merge
constexpr int CPM_NT = 1024;
constexpr int CPM_KPT = 8;
struct CpMergeSmem {
  SelectSmem<CPM_NT, CPM_KPT> sel;
  int32_t gpos[CPM_NT * CPM_KPT];
};

// One CTA per (sequence, job): element e = g * top_k + i is entry i of rank g's list;
// rank-major order with ascending positions inside each rank is ascending
// global position, so the selection's element-order tie rule is the
// lower-position rule and its element-order output is ascending.
__global__ void __launch_bounds__(CPM_NT) cp_merge_select_kernel(const CpMergeParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  CpMergeSmem& sm = *reinterpret_cast<CpMergeSmem*>(smem_raw);
  pdl_launch_dependents();
  cluster_select_prologue(sm.sel, /*cluster_wide=*/false);
  pdl_wait();
  const int b = blockIdx.x, jl = blockIdx.y, t = threadIdx.x;
  const int job = p.job0 + jl;
  const int n = p.world * p.top_k;  // <= CPM_NT * CPM_KPT, checked by the host
  uint32_t key[CPM_KPT];
#pragma unroll
  for (int j = 0; j < CPM_KPT; j++) {
    const int e = t * CPM_KPT + j;
    key[j] = 0u;
    sm.gpos[e] = -1;
    if (e < n) {
      const int g = e / p.top_k, i = e - g * p.top_k;
      const uint2 v = p.gathered[(((int64_t)g * p.n_jobs + job) * p.batch + b) * p.top_k + i];
      if (v.x != 0u) {
        key[j] = v.x;
        sm.gpos[e] = (int32_t)v.y;
      }
    }
  }
  __syncthreads();
  const int32_t* gpos = sm.gpos;
  cluster_select_topk<CPM_NT, CPM_KPT>(sm.sel, key, [gpos](int e) { return gpos[e]; }, p.top_k,
                                       p.idx[jl] + (int64_t)b * p.top_k, p.idx_count[jl] + b,
                                       /*cluster_wide=*/false, nullptr, /*top_window=*/true,
                                       /*gather_finish=*/true);
}

// ------------------------------------------------------- attention merge
// Log-sum-exp merge of nparts partials of one (layer, sequence, head):
// part r of slot s has O at part_o + r * o_pstride + s * o_sstride (16 x 512
// floats, unnormalised, relative to its max) and (max, sum) at part_ml + ...
// (maxima in log2 units).  FINAL writes O / sum as bf16; otherwise the merged
// (O, max, sum) in the same form.
template <bool FINAL>
__global__ void __launch_bounds__(128) cp_attn_merge_kernel(const CpAttnMergeParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y, li = blockIdx.z;
  const int t = threadIdx.x, np = p.nparts;
  const int64_t slot = (int64_t)li * p.batch + b;
  __shared__ float f[CP_MAX_PARTS];
  __shared__ float mx_s, den_s;
  float4 v[CP_MAX_PARTS];
#pragma unroll
  for (int r = 0; r < CP_MAX_PARTS; r++)
    v[r] = r < np ? *reinterpret_cast<const float4*>(p.part_o + r * p.o_pstride +
                                                     slot * p.o_sstride + h * CSA2_D + 4 * t)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  if (t < 32) {
    float m = -INFINITY, l = 0.f;
    if (t < np) {
      const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + t * p.ml_pstride +
                                                         slot * p.ml_sstride + h * 2);
      m = ml.x;
      l = ml.y;
    }
    float mx = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float fw = (mx == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - mx);
    float den = fw * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (t < np) f[t] = fw;
    if (t == 0) {
      mx_s = mx;
      den_s = den;
    }
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int r = 0; r < CP_MAX_PARTS; r++) {
    if (r >= np) break;
    acc.x = fmaf(f[r], v[r].x, acc.x);
    acc.y = fmaf(f[r], v[r].y, acc.y);
    acc.z = fmaf(f[r], v[r].z, acc.z);
    acc.w = fmaf(f[r], v[r].w, acc.w);
  }
  const int64_t o_off = (slot * CSA2_H + h) * CSA2_D + 4 * t;
  if constexpr (FINAL) {
    const float inv = den_s > 0.f ? 1.0f / den_s : 0.f;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p.out + o_off) = pk;
  } else {
    *reinterpret_cast<float4*>(p.out_o + o_off) = acc;
    if (t == 0)
      *reinterpret_cast<float2*>(p.out_ml + (slot * CSA2_H + h) * 2) = make_float2(mx_s, den_s);
  }
}

// --------------------------------------------------------------- launchers
// Every kernel here starts with griddepcontrol.launch_dependents + .wait and is
// launched with programmatic stream serialisation, like the rest of the
// library, so a chain of them overlaps each launch with its predecessor's tail.
template <typename... P, typename... A>
static cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, A&&... args) {
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

cudaError_t launch_cp_local_rows(const int32_t* n_rows, int batch, int64_t lo, int shard_rows,
                                 int32_t* local_rows, uint32_t* status, cudaStream_t st) {
  trace_mark("cp_local_rows", st);
  return launch_pdl(cp_local_rows_kernel, dim3((batch + 255) / 256), dim3(256), 0, st, n_rows,
                    (int32_t)batch, lo, (int32_t)shard_rows, local_rows, status);
}

cudaError_t launch_cp_bm_regroup(const float* src, int world, int batch, int nb, float* dst,
                                 cudaStream_t st) {
  const int64_t total = (int64_t)world * batch * nb;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
  if (blocks < 1) blocks = 1;
  trace_mark("cp_bm_regroup", st);
  return launch_pdl(cp_bm_regroup_kernel, dim3((unsigned)blocks), dim3(256), 0, st, src,
                    (int32_t)world, (int32_t)batch, (int32_t)nb, dst);
}

cudaError_t launch_cp_filter(const CpFilterParams& p, int batch, cudaStream_t st) {
  trace_mark("cp_filter", st);
  return launch_pdl(cp_filter_kernel, dim3(batch, p.n_lists), dim3(CPF_NT), 0, st, p);
}

cudaError_t launch_cp_export(const CpExportParams& p, int batch, cudaStream_t st) {
  trace_mark("cp_export", st);
  return launch_pdl(cp_export_kernel,
                    dim3((p.top_k + CPX_ROWS - 1) / CPX_ROWS, batch, p.n_jobs), dim3(CPX_NT), 0,
                    st, p);
}

cudaError_t launch_cp_merge_select(const CpMergeParams& p, cudaStream_t st) {
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([](int&) {
    return cudaFuncSetAttribute(cp_merge_select_kernel,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(CpMergeSmem));
  });
  if (ea != cudaSuccess) return ea;
  trace_mark("cp_merge_select", st);
  return launch_pdl(cp_merge_select_kernel, dim3(p.batch, p.n_sel), dim3(CPM_NT),
                    sizeof(CpMergeSmem), st, p);
}

cudaError_t launch_cp_attn_merge(const CpAttnMergeParams& p, int n_layers, bool final_out,
                                 cudaStream_t st) {
  const dim3 grid(CSA2_H, p.batch, n_layers);
  trace_mark(final_out ? "cp_attn_combine" : "cp_attn_local_merge", st);
  if (final_out) return launch_pdl(cp_attn_merge_kernel<true>, grid, dim3(128), 0, st, p);
  return launch_pdl(cp_attn_merge_kernel<false>, grid, dim3(128), 0, st, p);
}

int cp_merge_capacity() { return CPM_NT * CPM_KPT; }

}  // namespace csa2
