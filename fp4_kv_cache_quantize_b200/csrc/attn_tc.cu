// attn_tc.cu -- sparse + sliding-window decode attention on the tensor cores.
//
// For one (layer, sequence): keys = values = [the Top-k main-KV rows, FP4
// dequantised exactly ; the layer's 128-row E4M3 window], one softmax over
// both branches, 16 query heads sharing every row (tucaod.com walk-through,
// core-attention figure: selection, Top-K and concatenation of main KV and
// SWA; release note, section "Causal Encoder-Decoder": 128-token SWA at every
// layer; section "FP4 KV": FP8 window KV).
//
// One thread-block cluster of five CTAs per (layer, sequence): CTA c < 4
// takes keys [128 c, 128 c + 128) of the sparse branch, CTA 4 the window.
// With 16 heads a per-CTA tile is too narrow for the tensor core's 128-row
// MMA in its natural orientation, so both products run transposed, keys and
// channels on the MMA's M axis and the heads on N (tcgen05.mma, M = 128,
// N = 16, fp32 accumulators in tensor memory):
//   S^T[key][head]  = K[key][:] . Q'[head][:]       (K-major A and B)
//   O^T[chan][head] = V^T[chan][key] . P^T[head][key] (A read MN-major from
//                                                     the same K = V tile)
// Every operand is fp16: E2M1 x E4M3 products and E4M3 window values are
// exact in fp16, and each query head is scaled by a power of two (undone on
// its logits) so that any bf16 query is represented to fp16 precision
// without overflow.  Rows are gathered with cp.async (16 bytes per copy)
// into shared memory and dequantised there into the 128-byte-swizzled tile
// the MMA reads.  The softmax runs on the S^T accumulator (one thread per
// key); P^T in fp16 is the second MMA's B operand.  The five partial results
// (normalised O in fp16, max and sum per head) are pushed through
// distributed shared memory to the CTA owning each 128-channel block with
// asynchronous stores counted on the owner's mbarrier (no cluster barrier
// at the end: an owner waits only for its own 5 x 4,224 bytes), and the
// owners merge them with log-sum-exp weights and write the bf16 output: no
// partials go through global memory.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "csa2_internal.cuh"
#include "kernels.h"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int TA_NT = 512;
constexpr int TA_TPR = TA_NT / 128;  // threads per key row (4): a quarter of the row each
constexpr int TA_KEYS = 128;                        // keys per CTA: the MMA's M
constexpr int TA_SPARSE = CSA2_MAX_TOPK / TA_KEYS;  // CTAs of the sparse branch
constexpr int TA_CTAS = TA_SPARSE + 1;              // and the window's
static_assert(TA_CTAS == ATTN_TC_CTAS_PER_UNIT, "cluster size the launcher plans with");
static_assert(CSA2_W == TA_KEYS, "one CTA holds the whole window");
constexpr int TA_KB = TA_KEYS * 128;                // one 64-channel block of the tile
constexpr uint32_t TA_IDESC_QK = idesc_f16_f32(128, 16, false);
constexpr uint32_t TA_IDESC_PV = idesc_f16_f32(128, 16, true);
constexpr uint32_t TA_TMEM_COLS = 128;  // S^T in columns [0, 16), O^T in [64, 128)
constexpr uint32_t TA_O_COL = 64;

struct TaSmem {
  // K = V in fp16: channel block kb at kb * TA_KB, 128 rows (keys) of 128 B,
  // 16-byte chunks swizzled by row % 8.  Before the rows are dequantised it
  // holds the raw bf16 queries.
  alignas(1024) uint8_t tile[8 * TA_KB];
  alignas(1024) uint8_t q[8 * 2048];       // Q': channel block kb, 16 rows (heads) of 128 B
  alignas(1024) uint8_t p[2 * 2048];       // P^T: key block kb, 16 rows (heads) of 128 B
  alignas(16) float sS[CSA2_H * TA_KEYS];  // logits [head][key], log2 units
  // the normalised partials this CTA receives as the owner of a channel
  // block: [source CTA][channel][head] fp16
  alignas(16) uint8_t recv[TA_CTAS * 128 * CSA2_H * 2];
  int64_t row[TA_KEYS];
  float scl1[CSA2_H], scl2[CSA2_H];        // logit = acc * scl1 * scl2 (log2 units)
  float m[CSA2_H], lsum[CSA2_H], linv[CSA2_H];
  alignas(16) float2 ml[TA_CTAS][CSA2_H];  // (max, sum) per source CTA, at the owners
  alignas(16) float wts[TA_CTAS][CSA2_H];
  uint64_t mbar;
  uint64_t rbar;  // an owner's partials have arrived (TA_RECV_BYTES)
  uint32_t tmem_base;
};
// bytes each owner receives: per source CTA, 128 channels x 16 heads of fp16
// O and 16 (max, sum) pairs
constexpr uint32_t TA_RECV_BYTES = TA_CTAS * (128 * CSA2_H * 2 + CSA2_H * 8);
constexpr size_t TA_SMEM = sizeof(TaSmem) + 1024;

__device__ __forceinline__ int64_t ta_kv_row(const AttnParams& p, int b, int pos) {
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

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }


// Byte offset of 16-byte chunk cc (0..7) of row r in a 128-byte-swizzled block.
__device__ __forceinline__ uint32_t sw_off(int r, int cc) {
  return (uint32_t)(r * 128 + ((cc ^ (r & 7)) << 4));
}

// The code below runs once per CTA: every instruction is fetched cold, so
// loops are kept rolled (a rolled loop body is fetched once, an unrolled one
// costs its full length in instruction fetch).
__global__ void __launch_bounds__(TA_NT, 1) attn_tc_kernel(const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  TaSmem& s = *reinterpret_cast<TaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
  cg::cluster_group cluster = cg::this_cluster();
  const int c = (int)cluster.block_rank();
  const bool window = c == TA_SPARSE;
  const int b = blockIdx.y, li = blockIdx.z;
  const AttnLayer L = p.layer[li];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  pdl_launch_dependents();

  if (t == 0) {
    mbar_init(&s.mbar, 1);
    mbar_init(&s.rbar, 1);
    fence_mbar_init();
  }
  // every CTA's receive barrier is initialised before any partial is sent:
  // the cluster barrier that orders this completes long before the sends
  cluster_arrive_release();
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, TA_TMEM_COLS);
    tmem_relinquish();
  }
  // The queries are inputs (no kernel of this library writes them): their
  // copy into shared memory starts before the wait for the indices.
  {
    const uint8_t* qg = reinterpret_cast<const uint8_t*>(L.q + (int64_t)b * CSA2_H * CSA2_D);
#pragma unroll 1
    for (int i = t; i < CSA2_H * CSA2_D * 2 / 16; i += TA_NT) cp_async16(s.tile + 16 * i, qg + 16 * i);
    cp_async_commit();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  pdl_wait();  // the indices come from the previous kernel

  // ---- this CTA's keys.  b runs over sequences x queries: query tq of
  // sequence bp sees the sequence's entries minus the drafts after it, and
  // the window rows that end at its own entry.  Threads r, r + 128, r + 256
  // and r + 384 all resolve key r's row (from the same index) and copy a
  // quarter of it each, so no thread waits for another before its copies
  // start.
  const int bp = b / p.nq, tq = b - bp * p.nq, later = p.nq - 1 - tq;
  const int r = t & (TA_KEYS - 1), qq = t >> 7;
  static_assert(TA_TPR == 4, "four threads per key row");
  const int32_t* idx = L.idx + (int64_t)b * p.idx_stride;
  const int kt = c * TA_KEYS + r;
  // this thread's index, read before the counts arrive (within the index
  // array's stride either way): the three loads are in flight together
  const int pos_t = !window && kt < p.idx_stride ? __ldg(idx + kt) : -1;
  int C = p.n_rows[bp];
  if (C < 0 || C > p.max_rows) {
    if (t == 0) set_status(p.status, ST_DEVICE_CHECK);
    C = C < 0 ? 0 : p.max_rows;
  }
  C = C - later < 0 ? 0 : C - later;
  int nk;          // candidate keys of this CTA: keys j < nk
  int64_t row = -1;  // key r's row of the cache (or of the window), -1: none
  // this thread's quarter of row r, loaded straight into registers (no
  // shared-memory staging): the dequantisation below consumes it
  uint4 rv[8];
  uint2 sv = make_uint2(0u, 0u);
#pragma unroll
  for (int i = 0; i < 8; i++) rv[i] = make_uint4(0u, 0u, 0u, 0u);
  if (!window) {
    int n_idx = L.idx_count[b];
    if (n_idx < 0 || n_idx > p.idx_stride) {
      if (t == 0) set_status(p.status, ST_DEVICE_CHECK);
      n_idx = n_idx < 0 ? 0 : p.idx_stride;
    }
    nk = min(max(n_idx - c * TA_KEYS, 0), TA_KEYS);
    if (L.idx_copy && qq == 0) {  // Reuse layer: publish the indices it used
      if (kt < p.idx_stride) L.idx_copy[(int64_t)b * p.idx_stride + kt] = pos_t;
      if (c == 0 && t == 0) L.idx_copy_count[b] = L.idx_count[b];
    }
    if (r < nk) {
      if (pos_t >= 0 && pos_t < C) row = ta_kv_row(p, bp, pos_t);
      if (row < 0 && qq == 0) set_status(p.status, ST_DEVICE_CHECK);
    }
    if (row >= 0) {  // channels [128 qq, 128 qq + 128): 64 code bytes, 8 scales
      const uint4* cg_ = reinterpret_cast<const uint4*>(p.codes + row * (CSA2_D / 2) + 64 * qq);
#pragma unroll
      for (int i = 0; i < 4; i++) rv[i] = __ldg(cg_ + i);
      sv = __ldg(reinterpret_cast<const uint2*>(p.scales + row * (CSA2_D / 16) + 8 * qq));
    }
  } else {
    int n_win = p.swa_len[bp];
    if (n_win < 0 || n_win > p.swa_rows) {
      if (t == 0) set_status(p.status, ST_DEVICE_CHECK);
      n_win = n_win < 0 ? 0 : p.swa_rows;
    }
    const int win_end = n_win - later < 0 ? 0 : n_win - later;
    const int win_lo = win_end > CSA2_W ? win_end - CSA2_W : 0;
    nk = win_end - win_lo;
    if (r < nk) {  // channels [128 qq, 128 qq + 128): 128 E4M3 values
      row = r;
      const uint4* wr = reinterpret_cast<const uint4*>(
          L.swa + ((int64_t)bp * p.swa_rows + win_lo + r) * CSA2_D + 128 * qq);
#pragma unroll
      for (int i = 0; i < 8; i++) rv[i] = __ldg(wr + i);
    }
  }
  if (qq == 0) s.row[r] = row;  // read after the barriers below
  // the queries' copies have landed; the rows may still be in flight (in
  // registers) while the queries are converted
  cp_async_wait_all();
  __syncthreads();

  // ---- Q' = Q * 2^e_h in fp16, max |Q'_h| in [2^14, 2^15): warp h converts
  // head h, 16 channels per lane
  {
    const int h = warp, g = lane;
    const uint4* src = reinterpret_cast<const uint4*>(s.tile + h * (CSA2_D * 2) + g * 32);
    uint4 v[2];
    uint32_t mx = 0u;
#pragma unroll
    for (int k = 0; k < 2; k++) {
      v[k] = src[k];
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int j = 0; j < 4; j++) mx = max(mx, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    const int e = q_pow2_exponent(mx);
    const int e1 = e / 2, e2 = e - e1;  // each within a float's exponent range
    const float f = pow2i(e1), f2 = pow2i(e2);
    if (g == 0) {
      s.scl1[h] = pow2i(-e1);
      s.scl2[h] = p.scale_log2 * pow2i(-e2);
    }
#pragma unroll
    for (int k = 0; k < 2; k++) {  // channels 16 g + 8 k .. + 8: block g / 4, chunk 2 (g & 3) + k
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      uint32_t o4[4];
#pragma unroll
      for (int j = 0; j < 4; j++)
        o4[j] = h2u(__floats2half2_rn(__uint_as_float(w[j] << 16) * f * f2,
                                      __uint_as_float(w[j] & 0xFFFF0000u) * f * f2));
      *reinterpret_cast<uint4*>(s.q + (g >> 2) * 2048 + sw_off(h, 2 * (g & 3) + k)) =
          make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
  __syncthreads();  // the raw queries in the tile are consumed

  // ---- dequantise into the fp16 tile: four threads per row, 128 channels
  // (channel blocks 2 qq and 2 qq + 1) each
  if (nk > 0) {
    uint8_t* trow = s.tile + r * 128;
    const int sw = r & 7;
    if (row < 0) {
#pragma unroll 1
      for (int j = 0; j < 16; j++)
        *reinterpret_cast<uint4*>(trow + (2 * qq + (j >> 3)) * TA_KB + (((j & 7) ^ sw) << 4)) =
            make_uint4(0, 0, 0, 0);
    } else if (!window) {
#pragma unroll
      for (int i = 0; i < 4; i++) {  // 16 code bytes: channels 128 qq + 32 i + [0, 32)
        const uint4 cv = rv[i];
        const uint32_t words[4] = {cv.x, cv.y, cv.z, cv.w};
        const uint32_t sb = ((i < 2 ? sv.x : sv.y) >> (16 * (i & 1))) & 0xFFFFu;  // groups 2i, 2i+1
        const __half s0 = __half(__nv_cvt_fp8_to_halfraw((uint8_t)(sb & 0xFF), __NV_E4M3));
        const __half s1 = __half(__nv_cvt_fp8_to_halfraw((uint8_t)(sb >> 8), __NV_E4M3));
        uint8_t* dst = trow + (2 * qq + (i >> 1)) * TA_KB;
#pragma unroll
        for (int q4 = 0; q4 < 4; q4++) {  // 8 channels per 16-byte store
          const uint32_t word = words[q4];
          const __half2 scv = q4 < 2 ? __half2(s0, s0) : __half2(s1, s1);
          uint32_t hv[4];
#pragma unroll
          for (int k = 0; k < 4; k++)
            hv[k] = h2u(__hmul2(__half2(__nv_cvt_fp4x2_to_halfraw2(
                                    (__nv_fp4x2_storage_t)((word >> (8 * k)) & 0xFF), __NV_E2M1)),
                                scv));
          *reinterpret_cast<uint4*>(dst + (((4 * (i & 1) + q4) ^ sw) << 4)) =
              make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; j++) {  // 16 E4M3 bytes: channels 128 qq + 16 j + [0, 16)
        const uint4 v = rv[j];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        uint32_t hv[8];
#pragma unroll
        for (int k = 0; k < 4; k++) {
          hv[2 * k] = h2u(__half2(__nv_cvt_fp8x2_to_halfraw2(
              (__nv_fp8x2_storage_t)(wv[k] & 0xFFFF), __NV_E4M3)));
          hv[2 * k + 1] = h2u(__half2(__nv_cvt_fp8x2_to_halfraw2(
              (__nv_fp8x2_storage_t)(wv[k] >> 16), __NV_E4M3)));
        }
        uint8_t* dst = trow + (2 * qq + (j >> 2)) * TA_KB;
        const int cc = 2 * (j & 3);
        *reinterpret_cast<uint4*>(dst + ((cc ^ sw) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(dst + (((cc + 1) ^ sw) << 4)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();

  // ---- S^T = K . Q'^T (one thread issues 32 MMAs of K = 16)
  if (nk > 0 && t == 0) {
    tc_fence_after();
    // descriptors advance by adding (byte offset >> 4) to the start-address
    // field (every operand lies below 256 KB, so the field never carries)
    const uint64_t da = sdesc_k128(smem_u32(s.tile)), db = sdesc_k128(smem_u32(s.q));
#pragma unroll 1
    for (int i = 0; i < 32; i++) {  // K = 512 in 32 steps: block kb = i / 4, 32-byte step i % 4
      const uint32_t kb = (uint32_t)i >> 2, sub = (uint32_t)i & 3;
      umma_bf16(tmem + 16 * sub, da + ((kb * TA_KB + 32 * sub) >> 4), db + ((kb * 2048 + 32 * sub) >> 4),
                TA_IDESC_QK, kb != 0);
    }
    umma_commit(&s.mbar);
  }
  float* sS = s.sS;
  bool ok = true;
  if (nk > 0 && warp < 4) {
    ok = __all_sync(0xffffffffu, mbar_wait(&s.mbar, 0, nullptr));
    if (!ok && lane == 0) set_status(p.status, ST_TIMEOUT);
    tc_fence_after();
    uint32_t r[4][16];
#pragma unroll
    for (int a = 0; a < 4; a++) tmem_ld_x16(tmem + ((uint32_t)(32 * warp) << 16) + 16 * a, r[a]);
    tmem_ld_wait();
    const int key = 32 * warp + lane;
    const bool valid = ok && key < nk && s.row[key] >= 0;
#pragma unroll
    for (int h = 0; h < 16; h++) {
      const float acc = (__uint_as_float(r[0][h]) + __uint_as_float(r[1][h])) +
                        (__uint_as_float(r[2][h]) + __uint_as_float(r[3][h]));
      sS[h * TA_KEYS + key] = valid ? acc * s.scl1[h] * s.scl2[h] : -INFINITY;
    }
  }
  __syncthreads();
  // ---- softmax: warp h for head h, 4 keys per lane; P^T in fp16, the sum
  // of the fp16 probabilities the MMA reads
  if (nk > 0) {
    const int h = warp, g = lane;
    const float4 x = *reinterpret_cast<const float4*>(sS + h * TA_KEYS + 4 * g);
    const float m = warp_max_f32(fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
    __half2 ph0, ph1;
    if (m == -INFINITY) {
      ph0 = ph1 = __floats2half2_rn(0.0f, 0.0f);
    } else {
      ph0 = __floats2half2_rn(exp2f(x.x - m), exp2f(x.y - m));
      ph1 = __floats2half2_rn(exp2f(x.z - m), exp2f(x.w - m));
    }
    const float2 p0 = __half22float2(ph0), p1 = __half22float2(ph1);
    float l = (p0.x + p0.y) + (p1.x + p1.y);
    // keys 4g .. 4g + 3: key block g / 16, 16-byte chunk (g / 2) % 8, half g % 2
    *reinterpret_cast<uint2*>(s.p + (g >> 4) * 2048 + sw_off(h, (g >> 1) & 7) + 8 * (g & 1)) =
        make_uint2(h2u(ph0), h2u(ph1));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (g == 0) {
      s.m[h] = m;
      s.lsum[h] = l;
      s.linv[h] = l > 0.0f ? 1.0f / l : 0.0f;
    }
    fence_proxy_async_smem();
  } else if (t < CSA2_H) {
    s.m[t] = -INFINITY;
    s.lsum[t] = 0.0f;
  }
  tc_fence_before();
  __syncthreads();

  // ---- O^T = V^T . P^T: four channel blocks of 128, K = 128 keys in 8 steps
  if (nk > 0 && t == 0) {
    tc_fence_after();
    const uint64_t da = sdesc_mn128(smem_u32(s.tile), TA_KB, 1024), db = sdesc_k128(smem_u32(s.p));
#pragma unroll 1
    for (int i = 0; i < 32; i++) {  // 16 keys ks = i / 4, channel block cb = i % 4
      const uint32_t cb = (uint32_t)i & 3, ks = (uint32_t)i >> 2;
      umma_bf16(tmem + TA_O_COL + 16 * cb, da + ((cb * 2 * TA_KB + ks * 2048) >> 4),
                db + (((ks >> 2) * 2048 + (ks & 3) * 32) >> 4), TA_IDESC_PV, ks > 0);
    }
    umma_commit(&s.mbar);
  }

  // ---- normalised partial O^T -> the owners of the channel blocks: warp w
  // reads TMEM lanes 32 (w % 4).., channel block w / 4
  bool live = nk > 0 && ok;
  if (nk > 0) {
    const bool done = __all_sync(0xffffffffu, ok && mbar_wait(&s.mbar, 1, nullptr));
    if (!done && ok && lane == 0) set_status(p.status, ST_TIMEOUT);
    live = __syncthreads_and(done);
  }
  cluster_wait_acquire();  // (the arrival above) every owner's barrier is ready
  if (c < TA_SPARSE && t == 0) mbar_arrive_expect_tx(&s.rbar, TA_RECV_BYTES);
  {
    // every CTA sends all of its bytes (zeros, with weight 0, when it has
    // no keys), so each owner's count is fixed
    const int chl = 32 * (warp & 3) + lane;
    if (live) tc_fence_after();
    {
      const int cb = warp >> 2;
      uint32_t hv[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (live) {
        uint32_t o[16];
        tmem_ld_x16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + TA_O_COL + 16 * cb, o);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 8; k++)
          hv[k] = h2u(__floats2half2_rn(__uint_as_float(o[2 * k]) * s.linv[2 * k],
                                        __uint_as_float(o[2 * k + 1]) * s.linv[2 * k + 1]));
      }
      const uint32_t dst = mapa_rank(s.recv + ((c * 128 + chl) * CSA2_H) * 2, cb);
      const uint32_t bar = mapa_rank(&s.rbar, cb);
      st_async_v4(dst, make_uint4(hv[0], hv[1], hv[2], hv[3]), bar);
      st_async_v4(dst + 16, make_uint4(hv[4], hv[5], hv[6], hv[7]), bar);
    }
  }
  if (t < CSA2_H / 2 * TA_SPARSE) {  // (max, sum) of heads 2j, 2j + 1 to owner o2
    const int j = t & 7, o2 = t >> 3;
    float4 v = make_float4(-INFINITY, 0.0f, -INFINITY, 0.0f);
    if (live) v = make_float4(s.m[2 * j], s.lsum[2 * j], s.m[2 * j + 1], s.lsum[2 * j + 1]);
    st_async_v4(mapa_rank(&s.ml[c][2 * j], o2),
                make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                           __float_as_uint(v.w)),
                mapa_rank(&s.rbar, o2));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TA_TMEM_COLS);
  }

  // ---- owners: log-sum-exp merge of the five partials of 128 channels
  if (c < TA_SPARSE) {
    // every source's partial has landed here (bounded wait)
    if (!mbar_wait_cluster(&s.rbar, 0) && t == 0) set_status(p.status, ST_TIMEOUT);
    if (t < CSA2_H) {
      float M = -INFINITY;
#pragma unroll
      for (int src = 0; src < TA_CTAS; src++) M = fmaxf(M, s.ml[src][t].x);
      float Lsum = 0.0f, wv[TA_CTAS];
#pragma unroll
      for (int src = 0; src < TA_CTAS; src++) {
        const float2 ml = s.ml[src][t];
        wv[src] = ml.x == -INFINITY ? 0.0f : ml.y * exp2f(ml.x - M);
        Lsum += wv[src];
      }
      const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
#pragma unroll
      for (int src = 0; src < TA_CTAS; src++) s.wts[src][t] = wv[src] * inv;
    }
    __syncthreads();
    // four threads per channel, four heads each
    const int ch = t & 127, hh = 4 * (t >> 7);
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
    for (int src = 0; src < TA_CTAS; src++) {
      const float4 w4 = *reinterpret_cast<const float4*>(&s.wts[src][hh]);
      if (w4.x == 0.0f && w4.y == 0.0f && w4.z == 0.0f && w4.w == 0.0f)
        continue;  // nothing from this source for these heads
      const uint2 v = *reinterpret_cast<const uint2*>(s.recv +
                                                      ((src * 128 + ch) * CSA2_H + hh) * 2);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
      acc[0] = fmaf(w4.x, f0.x, acc[0]);
      acc[1] = fmaf(w4.y, f0.y, acc[1]);
      acc[2] = fmaf(w4.z, f1.x, acc[2]);
      acc[3] = fmaf(w4.w, f1.y, acc[3]);
    }
    uint16_t* out = L.out + ((int64_t)b * CSA2_H + hh) * CSA2_D + c * 128 + ch;
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const __nv_bfloat16 v = __float2bfloat16_rn(acc[k]);
      out[k * CSA2_D] = *reinterpret_cast<const uint16_t*>(&v);
    }
  }
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t st) {
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([](int&) {
    return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)TA_SMEM);
  });
  if (ea != cudaSuccess) return ea;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = TA_CTAS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(TA_CTAS, p.batch, p.n_layers);
  cfg.blockDim = dim3(TA_NT);
  cfg.dynamicSmemBytes = TA_SMEM;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  trace_mark("attn", st);
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, p);
}

}  // namespace csa2
