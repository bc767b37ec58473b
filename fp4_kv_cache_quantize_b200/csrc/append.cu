// append.cu -- the cache-append step that precedes a decode step: for every
// sequence, the new main-KV entry goes into the FP4 global cache together
// with its indexer-K projection, and every layer's new sliding-window entry
// goes into that layer's FP8 window ring.
//
//  * The indexer K is projected from the main-KV entry (yomxxx.com CSA2
//    paper notes, section 二, last paragraph: the indexer key is derived from
//    the main KV entry instead of a separate compression path; tucaod.com
//    walk-through, CSA2 section: the Full mode projects the indexer K from
//    its own global KV).  The entry is projected as produced (bf16, before its
//    FP4 storage rounding) by a 512 x 64 bf16 matrix, fp32 accumulation,
//    bf16 round-to-nearest-even output.
//  * Main KV: E2M1 + one E4M3 scale per 16 channels (fp4_codec.cuh).
//  * Window KV stays FP8 (yomxxx.com notes, section 三; each layer keeps its
//    own window: release note, section "Compressed Sparse Attention 2
//    (CSA2)"): E4M3, round to nearest even, saturating to +-448, no scale,
//    written to slot swa_pos % 128 of a 128-row ring.
//
// cache_append_kernel: grid (B, 1 + ceil(L / 4)), 256 threads.  Part 0 of a
// sequence packs the entry (64 threads, one 16-byte chunk each) and projects
// it (256 threads: 8 outputs x 16 channels each, partial sums reduced through
// shared memory in a fixed order); parts 1.. convert four layers' window
// entries each (64 threads per layer).  Every CTA reads the sequence's
// counters on entry; append_commit_kernel, launched after it with
// programmatic serialisation, advances them once all writes are done.
#include <cuda_bf16.h>

#include "csa2_internal.cuh"
#include "fp4_codec.cuh"
#include "kernels.h"

namespace csa2 {

constexpr int AP_NT = 256;
constexpr int AP_LAYERS_PER_CTA = AP_NT / 64;

// Pool row of the new entry at position pos, or -1 (not dereferenced) when
// the position is negative, beyond the sequence's capacity, or unmapped.
__device__ __forceinline__ int64_t append_row(const AppendParams& p, int b, int pos) {
  if (pos < 0) return -1;
  int64_t row;
  if (p.page_table) {
    const int page = pos >> 6;
    if (page >= p.max_pages) return -1;
    const int64_t pid = p.page_table[(int64_t)b * p.max_pages + page];
    row = pid * 64 + (pos & 63);
    if (pid < 0) return -1;
  } else {
    if (pos >= p.seq_stride) return -1;
    row = (int64_t)b * p.seq_stride + pos;
  }
  return row < p.pool_rows ? row : -1;
}

__global__ void __launch_bounds__(AP_NT) cache_append_kernel(const AppendParams p) {
  __shared__ float xs[CSA2_D];
  __shared__ float part[32][CSA2_DI + 1];
  const int b = blockIdx.x, t = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();  // counters and rows of the previous append (or other writers)

  if (blockIdx.y == 0) {
    const int pos = p.n_rows[b];
    const int64_t row = append_row(p, b, pos);
    if (row < 0) {
      if (t == 0) set_status(p.status, ST_DEVICE_CHECK);
      return;
    }
    if (t < CSA2_D / 8) {  // 64 threads, one 16-byte chunk of 8 channels each
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x + (int64_t)b * CSA2_D) + t);
      float f[8];
      unpack_bf16x8(v, f);
      float amax = amax8(f);
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // lanes 2j, 2j+1: one group
      uint8_t sb;
      const uint32_t packed = fp4_encode8(f, amax, &sb);
      reinterpret_cast<uint32_t*>(p.codes + row * (CSA2_D / 2))[t] = packed;
      if ((t & 1) == 0) p.scales[row * (CSA2_D / 16) + (t >> 1)] = sb;
#pragma unroll
      for (int k = 0; k < 8; k++) xs[8 * t + k] = f[k];
    }
    __syncthreads();
    // Projection: thread t owns outputs [8 jg, 8 jg + 8) over channels
    // [16 cs, 16 cs + 16); W rows are 128 B, so each load is 16 B aligned.
    const int jg = t & 7, cs = t >> 3;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4* wp = reinterpret_cast<const uint4*>(p.w_idx) + (int64_t)(16 * cs) * 8 + jg;
    uint4 wv[16];
#pragma unroll
    for (int c = 0; c < 16; c++) wv[c] = __ldg(wp + c * 8);
#pragma unroll
    for (int c = 0; c < 16; c++) {
      float wf[8];
      unpack_bf16x8(wv[c], wf);
      const float xc = xs[16 * cs + c];
#pragma unroll
      for (int k = 0; k < 8; k++) acc[k] = fmaf(xc, wf[k], acc[k]);
    }
#pragma unroll
    for (int k = 0; k < 8; k++) part[cs][8 * jg + k] = acc[k];
    __syncthreads();
    if (t < CSA2_DI) {
      float sum = 0.f;
#pragma unroll 8
      for (int i = 0; i < 32; i++) sum += part[i][t];
      p.idx_k[row * CSA2_DI + t] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    return;
  }

  // Window entries of up to four layers: 64 threads per layer, 8 channels each.
  const int l = (blockIdx.y - 1) * AP_LAYERS_PER_CTA + (t >> 6);
  if (l >= p.n_layers) return;
  const int spos = p.swa_pos[b];
  if (spos < 0) {
    if ((t & 63) == 0) set_status(p.status, ST_DEVICE_CHECK);
    return;
  }
  const int slot = spos % CSA2_W, ch = t & 63;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x_swa + ((int64_t)l * p.batch + b) * CSA2_D) + ch);
  float f[8];
  unpack_bf16x8(v, f);
  uint32_t w2[4];
#pragma unroll
  for (int k = 0; k < 4; k++)
    w2[k] = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(f[2 * k], f[2 * k + 1]), __NV_SATFINITE,
                                               __NV_E4M3);
  uint8_t* dst = p.swa + (((int64_t)l * p.batch + b) * CSA2_W + slot) * CSA2_D + 8 * ch;
  *reinterpret_cast<uint2*>(dst) = make_uint2((w2[0] & 0xFFFFu) | (w2[1] << 16),
                                              (w2[2] & 0xFFFFu) | (w2[3] << 16));
}

// Advances the counters once every write of the step has landed.
__global__ void __launch_bounds__(AP_NT) append_commit_kernel(const AppendParams p) {
  pdl_launch_dependents();
  pdl_wait();
  for (int b = threadIdx.x; b < p.batch; b += AP_NT) {
    const int pos = p.n_rows[b];
    if (append_row(p, b, pos) >= 0) p.n_rows[b] = pos + 1;
    if (p.n_layers > 0) {
      const int spos = p.swa_pos[b];
      if (spos >= 0) {
        p.swa_pos[b] = spos + 1;
        p.swa_len[b] = spos + 1 < CSA2_W ? spos + 1 : CSA2_W;
      }
    }
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t st) {
  if (p.batch <= 0) return cudaSuccess;
  const int parts = 1 + (p.n_layers + AP_LAYERS_PER_CTA - 1) / AP_LAYERS_PER_CTA;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.batch, parts);
  cfg.blockDim = dim3(AP_NT);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  trace_mark("append", st);
  cudaError_t e = cudaLaunchKernelEx(&cfg, cache_append_kernel, p);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(1);
  trace_mark("append_commit", st);
  return cudaLaunchKernelEx(&cfg, append_commit_kernel, p);
}

}  // namespace csa2
