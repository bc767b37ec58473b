// attn.cu -- sparse + sliding-window decode attention over the FP4 cache.
//
// For one (layer, sequence): keys = values = [the Top-k main-KV rows, FP4
// dequantised exactly ; the layer's 128-row E4M3 window], one softmax over
// both branches, 16 query heads sharing every row (tucaod.com walk-through,
// core-attention figure: selection, Top-K and concatenation of main KV and
// SWA; release note, section "Causal Encoder-Decoder": 128-token SWA at every
// layer; section "FP4 KV": FP8 window KV).
//
// The 640 keys are cut into 10 chunks of 64 (8 sparse, 2 window).  A CTA of
// 4 warps takes a contiguous range of chunks (split-KV), gathers each chunk's
// rows from HBM with 16-byte loads, dequantises them to fp16 in a 128B-XOR-
// swizzled shared tile (E2M1 x E4M3 and E4M3 are exact in fp16), computes
// S = Q K^T and O += P V with m16n8k16 tensor-core tiles (M = the 16 heads:
// a per-step tile far too small for tcgen05's 64/128-row MMA), keeps the
// online-softmax state in fp32.  With one split the CTA normalises and writes
// the output; otherwise each split writes its unnormalised O, max and sum
// (coalesced, to the workspace, where they stay in L2) and attn_merge_kernel,
// one CTA per (layer, sequence, head), combines them with log-sum-exp
// weights.  Each thread derives its gather addresses from the indices
// directly, and the query load overlaps the first gather.  With several
// queries per sequence, blockIdx.y runs over sequences x queries: each query
// sees the entries and the window rows up to its own position.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "csa2_internal.cuh"
#include "kernels.h"

namespace csa2 {

constexpr int AT_NT = 128;
constexpr int AT_CH = 64;  // keys per chunk
constexpr int AT_SPARSE_CHUNKS = CSA2_MAX_TOPK / AT_CH;
constexpr int AT_CHUNKS = AT_SPARSE_CHUNKS + CSA2_W / AT_CH;



struct AttnSmem {
  __half q[CSA2_H * CSA2_D];   // swizzled rows of 1024 B
  __half kv[AT_CH * CSA2_D];   // swizzled rows of 1024 B
  __half p[CSA2_H * AT_CH];    // swizzled rows of 128 B
  float s[CSA2_H][AT_CH + 4];
  float m[CSA2_H], l[CSA2_H], alpha[CSA2_H];
  uint32_t qmax[CSA2_H][2];  // per head, the two warps' largest |q| (bf16 bits)
  int64_t row[AT_CH];
};

__device__ __forceinline__ uint32_t sw1024(int row, int chunk) {  // byte offset
  return (uint32_t)(row * 1024 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Pool row of position pos of sequence b, or -1 (never dereferenced).
__device__ __forceinline__ int64_t kv_row(const AttnParams& p, int b, int pos) {
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

__global__ void __launch_bounds__(AT_NT, 2) attn_decode_kernel(const AttnParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  AttnSmem& s = *reinterpret_cast<AttnSmem*>(smem_raw);
  pdl_launch_dependents();
  pdl_wait();  // the indices come from the previous kernel
  const int split = blockIdx.x, b = blockIdx.y, li = blockIdx.z;
  const AttnLayer L = p.layer[li];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const uint32_t q_base = smem_u32(s.q), kv_base = smem_u32(s.kv), p_base = smem_u32(s.p);

  // b runs over sequences x queries: query tq of sequence bp sees the
  // sequence's entries minus the drafts after it, and the window rows that
  // end at its own entry.
  const int bp = b / p.nq, tq = b - bp * p.nq, later = p.nq - 1 - tq;
  int C = p.n_rows[bp];
  if (C < 0 || C > p.max_rows) {
    set_status(p.status, ST_DEVICE_CHECK);
    C = C < 0 ? 0 : p.max_rows;
  }
  C = C - later < 0 ? 0 : C - later;
  int n_idx = L.idx_count[b];
  if (n_idx < 0 || n_idx > p.idx_stride) {
    set_status(p.status, ST_DEVICE_CHECK);
    n_idx = n_idx < 0 ? 0 : p.idx_stride;
  }
  if (n_idx > CSA2_MAX_TOPK) n_idx = CSA2_MAX_TOPK;
  int n_win = p.swa_len[bp];
  if (n_win < 0 || n_win > p.swa_rows) {
    set_status(p.status, ST_DEVICE_CHECK);
    n_win = n_win < 0 ? 0 : p.swa_rows;
  }
  const int win_end = n_win - later < 0 ? 0 : n_win - later;
  const int win_lo = win_end > CSA2_W ? win_end - CSA2_W : 0;
  const int n_swa = win_end - win_lo;
  const int32_t* idx = L.idx + (int64_t)b * p.idx_stride;

  if (split == 0 && L.idx_copy) {  // Reuse layer: publish the indices it used
    for (int i = t; i < p.idx_stride; i += AT_NT) L.idx_copy[(int64_t)b * p.idx_stride + i] = idx[i];
    if (t == 0) L.idx_copy_count[b] = L.idx_count[b];
  }

  // Q (bf16) is loaded now and converted to fp16, each head scaled by a power
  // of two (q_pow2_exponent) that is undone on its logits, into swizzled rows
  // once the first chunk's gathers are in flight.  Chunk i = t + u AT_NT
  // belongs to head i / 64: warps 2h' and 2h' + 1 hold head h' + 2u.
  constexpr int QV = (CSA2_H * CSA2_D / 8) / AT_NT;
  static_assert(AT_NT == 128 && QV * 2 == CSA2_H, "two warps per head and chunk set");
  uint4 qv[QV];
  {
    const uint4* qg = reinterpret_cast<const uint4*>(L.q + (int64_t)b * CSA2_H * CSA2_D);
#pragma unroll
    for (int u = 0; u < QV; u++) qv[u] = __ldg(qg + t + u * AT_NT);
#pragma unroll
    for (int u = 0; u < QV; u++) {
      const uint32_t w[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
      uint32_t mx = 0u;
#pragma unroll
      for (int k = 0; k < 4; k++) mx = max(mx, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (lane == 0) s.qmax[(t >> 6) + 2 * u][warp & 1] = mx;  // read after a barrier
    }
  }
  bool q_ready = false;
  float ls1[2], ls2[2];  // logit factors of heads g and g + 8
  auto store_q = [&]() {
#pragma unroll
    for (int u = 0; u < QV; u++) {
      const int i = t + u * AT_NT;  // 16-byte chunk of 8 channels
      const int row = i >> 6, ch = i & 63;
      const int e = q_pow2_exponent(max(s.qmax[row][0], s.qmax[row][1]));
      const float f1 = pow2i(e / 2), f2 = pow2i(e - e / 2);
      const uint32_t w[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
      uint32_t o4[4];
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
        o4[k] = h2_bits(__floats2half2_rn(lo * f1 * f2, hi * f1 * f2));
      }
      *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(s.q) + sw1024(row, ch)) =
          make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
#pragma unroll
    for (int j = 0; j < 2; j++) {
      const int h = g + 8 * j;
      const int e = q_pow2_exponent(max(s.qmax[h][0], s.qmax[h][1]));
      ls1[j] = pow2i(-(e / 2));
      ls2[j] = p.scale_log2 * pow2i(-(e - e / 2));
    }
    q_ready = true;
  };
  if (t < CSA2_H) {
    s.m[t] = -INFINITY;
    s.l[t] = 0.0f;
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;

  const int c_lo = split * AT_CHUNKS / p.nsplit, c_hi = (split + 1) * AT_CHUNKS / p.nsplit;
  for (int chunk = c_lo; chunk < c_hi; chunk++) {
    const bool sparse = chunk < AT_SPARSE_CHUNKS;
    const int k0 = sparse ? chunk * AT_CH : (chunk - AT_SPARSE_CHUNKS) * AT_CH;
    const int nk = sparse ? n_idx : n_swa;
    if (k0 >= nk) continue;  // uniform across the CTA
    __syncthreads();         // previous chunk fully consumed
    if (t < AT_CH) {  // validity of each key, for the logits mask
      int64_t row = -1;
      const int pos = sparse && k0 + t < p.idx_stride ? __ldg(idx + k0 + t) : -1;
      if (k0 + t < nk) {
        if (sparse) {
          if (pos >= 0 && pos < C) row = kv_row(p, bp, pos);
          if (row < 0) set_status(p.status, ST_DEVICE_CHECK);
        } else {
          row = k0 + t;
        }
      }
      s.row[t] = row;
    }
    if (sparse) {
      // 64 rows x 16 chunks of 16 code bytes (32 channels, 2 scale groups);
      // each thread resolves its own rows from the indices.
      uint4 cv[8];
      uint32_t sv[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int i = t + u * AT_NT, r = i >> 4, cc = i & 15;
        // the index is read without waiting for the count (in bounds of the
        // index array either way), so both loads are in flight together
        const int pos = k0 + r < p.idx_stride ? __ldg(idx + k0 + r) : -1;
        int64_t row = -1;
        if (k0 + r < nk && pos >= 0 && pos < C) row = kv_row(p, bp, pos);
        if (row >= 0) {
          cv[u] = __ldg(reinterpret_cast<const uint4*>(p.codes + row * (CSA2_D / 2)) + cc);
          sv[u] = __ldg(reinterpret_cast<const uint16_t*>(p.scales + row * (CSA2_D / 16)) + cc);
        } else {
          cv[u] = make_uint4(0, 0, 0, 0);
          sv[u] = 0;
        }
      }
      if (!q_ready) store_q();
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int i = t + u * AT_NT, r = i >> 4, cc = i & 15;
        const __half s0 = __half(__nv_cvt_fp8_to_halfraw((uint8_t)(sv[u] & 0xFF), __NV_E4M3));
        const __half s1 = __half(__nv_cvt_fp8_to_halfraw((uint8_t)(sv[u] >> 8), __NV_E4M3));
#pragma unroll
        for (int q4i = 0; q4i < 4; q4i++) {  // 4 bytes of codes = 8 channels
          // rotate by cc so that one store instruction spreads over all banks
          const int q4 = (q4i + cc) & 3;
          const uint32_t word = q4 == 0 ? cv[u].x : q4 == 1 ? cv[u].y : q4 == 2 ? cv[u].z : cv[u].w;
          const __half2 sc = q4 < 2 ? __half2(s0, s0) : __half2(s1, s1);
          uint32_t hv[4];
#pragma unroll
          for (int k = 0; k < 4; k++) {
            const __half2 v = __half2(__nv_cvt_fp4x2_to_halfraw2(
                (__nv_fp4x2_storage_t)((word >> (8 * k)) & 0xFF), __NV_E2M1));
            hv[k] = h2_bits(__hmul2(v, sc));
          }
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(s.kv) + sw1024(r, cc * 4 + q4)) =
              make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
      }
    } else {
      // 64 window rows x 32 chunks of 16 E4M3 bytes.
      const uint8_t* swa = L.swa + ((int64_t)bp * p.swa_rows + win_lo) * CSA2_D;
      uint4 cv[16];
#pragma unroll
      for (int u = 0; u < 16; u++) {
        const int i = t + u * AT_NT, r = i >> 5, cc = i & 31;
        const int64_t row = k0 + r < nk ? (int64_t)(k0 + r) : -1;
        cv[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(swa + row * CSA2_D) + cc)
                         : make_uint4(0, 0, 0, 0);
      }
      if (!q_ready) store_q();
#pragma unroll
      for (int u = 0; u < 16; u++) {
        const int i = t + u * AT_NT, r = i >> 5, cc = i & 31;
        const uint32_t wv[4] = {cv[u].x, cv[u].y, cv[u].z, cv[u].w};
        uint32_t hv[8];
#pragma unroll
        for (int k = 0; k < 4; k++) {
          hv[2 * k] = h2_bits(__half2(__nv_cvt_fp8x2_to_halfraw2(
              (__nv_fp8x2_storage_t)(wv[k] & 0xFFFF), __NV_E4M3)));
          hv[2 * k + 1] = h2_bits(__half2(__nv_cvt_fp8x2_to_halfraw2(
              (__nv_fp8x2_storage_t)(wv[k] >> 16), __NV_E4M3)));
        }
        uint8_t* base = reinterpret_cast<uint8_t*>(s.kv);
        const uint4 lo = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        const uint4 hi = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        const int odd = cc & 1;  // alternate the order across lanes (bank spread)
        *reinterpret_cast<uint4*>(base + sw1024(r, 2 * cc + odd)) = odd ? hi : lo;
        *reinterpret_cast<uint4*>(base + sw1024(r, 2 * cc + 1 - odd)) = odd ? lo : hi;
      }
    }
    __syncthreads();

    // S = Q K^T for this warp's 16 keys.
    {
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int qrow = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int krow = warp * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll 8
      for (int ks = 0; ks < CSA2_D / 16; ks++) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(q_base + sw1024(qrow, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
        ldsm_x4(kv_base + sw1024(krow, 2 * ks + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_f16_16816(acc[0], a0, a1, a2, a3, b0, b1);
        mma_f16_16816(acc[1], a0, a1, a2, a3, b2, b3);
      }
#pragma unroll
      for (int nt = 0; nt < 2; nt++) {
        const int key = warp * 16 + nt * 8 + 2 * tig;
        const bool v0 = s.row[key] >= 0, v1 = s.row[key + 1] >= 0;
        s.s[g][key] = v0 ? acc[nt][0] * ls1[0] * ls2[0] : -INFINITY;
        s.s[g][key + 1] = v1 ? acc[nt][1] * ls1[0] * ls2[0] : -INFINITY;
        s.s[g + 8][key] = v0 ? acc[nt][2] * ls1[1] * ls2[1] : -INFINITY;
        s.s[g + 8][key + 1] = v1 ? acc[nt][3] * ls1[1] * ls2[1] : -INFINITY;
      }
    }
    __syncthreads();

    // Online softmax: 8 threads per head row, 8 keys each.
    {
      const int h = t >> 3, seg = t & 7;
      float x[8], cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        x[i] = s.s[h][seg * 8 + i];
        cm = fmaxf(cm, x[i]);
      }
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 4));
      const float m_old = s.m[h];
      const float m_new = fmaxf(m_old, cm);
      float alpha = 1.0f, rs = 0.0f;
      uint32_t pv[4];
      if (m_new == -INFINITY) {
        pv[0] = pv[1] = pv[2] = pv[3] = 0u;
      } else {
        alpha = exp2f(m_old - m_new);
        float e[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
          e[i] = exp2f(x[i] - m_new);
          rs += e[i];
        }
#pragma unroll
        for (int k = 0; k < 4; k++) pv[k] = h2_bits(__floats2half2_rn(e[2 * k], e[2 * k + 1]));
      }
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(s.p) + sw128(h, seg)) =
          make_uint4(pv[0], pv[1], pv[2], pv[3]);
      __syncwarp();
      if (seg == 0) {
        s.m[h] = m_new;
        s.l[h] = s.l[h] * alpha + rs;
        s.alpha[h] = alpha;
      }
    }
    __syncthreads();

    // O = O * alpha + P V over this warp's 128 channels.
    {
      const float al0 = s.alpha[g], al1 = s.alpha[g + 8];
#pragma unroll
      for (int i = 0; i < 16; i++) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      const int prow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < AT_CH / 16; ks++) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(p_base + sw128(prow, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
        const int vrow = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int np = 0; np < 8; np++) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(kv_base + sw1024(vrow, warp * 16 + np * 2 + (lane >> 4)), b0, b1, b2, b3);
          mma_f16_16816(o[2 * np], a0, a1, a2, a3, b0, b1);
          mma_f16_16816(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }
  __syncthreads();

  uint16_t* out = L.out + (int64_t)b * CSA2_H * CSA2_D;
  if (p.nsplit == 1) {
    const float l0 = s.l[g], l1 = s.l[g + 8];
    const float inv0 = l0 > 0.f ? 1.0f / l0 : 0.f, inv1 = l1 > 0.f ? 1.0f / l1 : 0.f;
#pragma unroll
    for (int nt = 0; nt < 16; nt++) {
      const int ch = warp * 128 + nt * 8 + 2 * tig;
      const __nv_bfloat162 r0 = __floats2bfloat162_rn(o[nt][0] * inv0, o[nt][1] * inv0);
      const __nv_bfloat162 r1 = __floats2bfloat162_rn(o[nt][2] * inv1, o[nt][3] * inv1);
      *reinterpret_cast<__nv_bfloat162*>(out + g * CSA2_D + ch) = r0;
      *reinterpret_cast<__nv_bfloat162*>(out + (g + 8) * CSA2_D + ch) = r1;
    }
    return;
  }
  // Split partial: unnormalised O through the idle key/value tile (rows padded
  // to 520 floats against bank conflicts) to coalesced 16-byte stores.
  constexpr int OS = 520;
  float* ob = reinterpret_cast<float*>(s.kv);
#pragma unroll
  for (int nt = 0; nt < 16; nt++) {
    const int ch = warp * 128 + nt * 8 + 2 * tig;
    *reinterpret_cast<float2*>(ob + g * OS + ch) = make_float2(o[nt][0], o[nt][1]);
    *reinterpret_cast<float2*>(ob + (g + 8) * OS + ch) = make_float2(o[nt][2], o[nt][3]);
  }
  __syncthreads();
  const int64_t slot = ((int64_t)li * p.batch + b) * p.nsplit + split;
  float4* dst = reinterpret_cast<float4*>(p.part_o + slot * (CSA2_H * CSA2_D));
  for (int i = t; i < CSA2_H * CSA2_D / 4; i += AT_NT) {
    const int row = i >> 7, c4 = i & 127;
    dst[i] = *reinterpret_cast<const float4*>(ob + row * OS + 4 * c4);
  }
  if (t < CSA2_H)
    *reinterpret_cast<float2*>(p.part_ml + (slot * CSA2_H + t) * 2) = make_float2(s.m[t], s.l[t]);
}

// Log-sum-exp merge of the split partials of one (layer, sequence, head).
__global__ void __launch_bounds__(128) attn_merge_kernel(const AttnParams p) {
  pdl_wait();  // the partials come from attn_decode_kernel
  const int h = blockIdx.x, b = blockIdx.y, li = blockIdx.z;
  const int t = threadIdx.x, ns = p.nsplit;
  const int64_t slot0 = ((int64_t)li * p.batch + b) * ns;
  __shared__ float f[16];
  __shared__ float invl;
  // every split's slice is requested before any is used (one L2 round trip,
  // overlapping the max/sum reduction below)
  float4 v[AT_CHUNKS];
#pragma unroll
  for (int r = 0; r < AT_CHUNKS; r++)
    v[r] = r < ns ? *reinterpret_cast<const float4*>(p.part_o + (slot0 + r) * (CSA2_H * CSA2_D) +
                                                     h * CSA2_D + 4 * t)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  if (t < 32) {
    float m = -INFINITY, l = 0.f;
    if (t < ns) {
      const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + ((slot0 + t) * CSA2_H + h) * 2);
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
    if (t < ns) f[t] = fw;
    if (t == 0) invl = den > 0.f ? 1.0f / den : 0.f;
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int r = 0; r < AT_CHUNKS; r++) {
    if (r >= ns) break;
    acc.x = fmaf(f[r], v[r].x, acc.x);
    acc.y = fmaf(f[r], v[r].y, acc.y);
    acc.z = fmaf(f[r], v[r].z, acc.z);
    acc.w = fmaf(f[r], v[r].w, acc.w);
  }
  uint16_t* out = p.layer[li].out + ((int64_t)b * CSA2_H + h) * CSA2_D + 4 * t;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * invl, acc.y * invl);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * invl, acc.w * invl);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out) = pk;
}

int attn_nsplit(int pairs, int num_sms) {
  const int opts[4] = {1, 2, 5, 10};
  const int64_t slots = 2LL * num_sms;  // CTAs resident at once: two per SM
  if ((int64_t)pairs < slots) {         // fill the GPU once
    for (int i = 0; i < 4; i++)
      if ((int64_t)pairs * opts[i] >= slots) return opts[i];
    return 10;
  }
  // More units than resident CTAs: the whole-unit CTAs run in waves and the
  // last, partial wave costs a full CTA time.  Split when it shortens the
  // waves by a clear margin (a CTA's time is its share of the keys plus a
  // fixed ~6%; a split adds the merge, ~10% of a whole-unit CTA).
  auto cost = [&](int ns) {
    const int64_t waves = ((int64_t)pairs * ns + slots - 1) / slots;
    return (double)waves * (1.0 / ns + 0.06) + (ns > 1 ? 0.1 : 0.0);
  };
  int best = 1;
  for (int i = 1; i < 4; i++)
    if (cost(opts[i]) < 0.9 * cost(best)) best = opts[i];
  return best;
}

cudaError_t launch_attn(const AttnParams& p, cudaStream_t st, bool merge) {
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([](int&) {
    return cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(AttnSmem));
  });
  if (ea != cudaSuccess) return ea;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nsplit, p.batch, p.n_layers);
  cfg.blockDim = dim3(AT_NT);
  cfg.dynamicSmemBytes = sizeof(AttnSmem);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  trace_mark("attn", st);
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_decode_kernel, p);
  if (e != cudaSuccess || p.nsplit == 1 || !merge) return e;
  cudaLaunchConfig_t mc = {};
  mc.gridDim = dim3(CSA2_H, p.batch, p.n_layers);
  mc.blockDim = dim3(128);
  mc.stream = st;
  mc.attrs = at;
  mc.numAttrs = 1;
  trace_mark("attn_merge", st);
  return cudaLaunchKernelEx(&mc, attn_merge_kernel, p);
}

size_t attn_partial_bytes(int batch, int n_layers, int nsplit) {
  if (nsplit <= 1) return 0;
  const size_t slots = (size_t)batch * n_layers * nsplit;
  return slots * CSA2_H * CSA2_D * sizeof(float) + slots * CSA2_H * 2 * sizeof(float);
}

}  // namespace csa2
