// select.cuh -- exact cluster-wide Top-K by radix select over 32-bit keys.
//
// Selection rule (the reading this library takes of "Top-512" / "top 2,048
// blocks", which the pages leave unspecified for ties): the k largest keys,
// ties broken towards the lower element index, returned in ascending element
// order.  Elements are spread over the CTAs of one thread-block cluster;
// histograms are merged through distributed shared memory, so one cluster
// selects from up to 16 x NT x KPT elements without a second kernel.
#pragma once

#include <cooperative_groups.h>

#include "csa2_internal.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

template <int NT>
struct SelectSmem {
  uint32_t hist[256];
  uint32_t acc[4][256];  // cluster-wide histograms; only rank 0's copy is used
  uint32_t wsum[32];
  uint32_t bcast[4];
  uint32_t tot[4];       // this CTA's counts: [0] candidates, [1] > T, [2] == T
};

// Exclusive block-wide prefix sum of v over threads in index order.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t& total) {
  static_assert(NT % 32 == 0 && NT <= 1024, "block size");
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < NT / 32 ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) wsum[lane] = w;
  }
  __syncthreads();
  total = wsum[NT / 32 - 1];
  const uint32_t before = wid ? wsum[wid - 1] : 0u;
  __syncthreads();
  return before + x - v;
}

// Thread t of cluster rank r owns elements e = (r * NT + t) * KPT + j,
// key[j] (0 = not a candidate) and id[j] (written to out when selected).
// Every thread of every CTA of the cluster must call this with the same
// k_req.  Writes out[0..k) (k = min(k_req, candidates)), out[k..k_req) = -1,
// and *out_count = k.
template <int NT, int KPT>
__device__ void cluster_select_topk(SelectSmem<NT>& sm, const uint32_t (&key)[KPT],
                                    const int32_t (&id)[KPT], int k_req, int32_t* out,
                                    int32_t* out_count) {
  static_assert(NT >= 256, "one thread per histogram bin");
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank(), ncta = cluster.num_blocks();
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;

  for (int i = t; i < 4 * 256; i += NT) (&sm.acc[0][0])[i] = 0u;
  uint32_t nv = 0;
#pragma unroll
  for (int j = 0; j < KPT; j++) nv += key[j] != 0u;
  uint32_t cta_valid;
  block_excl_scan<NT>(nv, sm.wsum, cta_valid);
  if (t == 0) sm.tot[0] = cta_valid;
  cluster.sync();
  if (t == 0) {
    uint32_t n = 0;
    for (unsigned r = 0; r < ncta; r++) n += *cluster.map_shared_rank(&sm.tot[0], r);
    sm.bcast[2] = n;
  }
  __syncthreads();
  const uint32_t n_valid = sm.bcast[2];
  const uint32_t k = (uint32_t)k_req < n_valid ? (uint32_t)k_req : n_valid;

  uint32_t prefix = 0, mask = 0, krem = k;
  if (k > 0) {
    for (int pass = 0; pass < 4; pass++) {
      const int shift = 24 - 8 * pass;
      for (int i = t; i < 256; i += NT) sm.hist[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < KPT; j++) {
        const uint32_t kk = key[j];
        const uint32_t bin = (kk != 0u && (kk & mask) == prefix) ? (kk >> shift) & 255u : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], __popc(peers));
      }
      __syncthreads();
      if (t < 256 && sm.hist[t] != 0u)
        atomicAdd(cluster.map_shared_rank(&sm.acc[pass][t], 0), sm.hist[t]);
      cluster.sync();
      if (wid == 0) {
        const uint32_t* acc0 = cluster.map_shared_rank(&sm.acc[pass][0], 0);
        uint32_t c[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
          c[i] = acc0[8 * lane + i];
          s += c[i];
        }
        uint32_t v = s;  // suffix sum over lanes >= this one
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, v, o);
          if (lane + o < 32) v += y;
        }
        const unsigned ball = __ballot_sync(0xffffffffu, v >= krem);
        const int L = 31 - __clz(ball);
        uint32_t above = __shfl_sync(0xffffffffu, v, (L + 1) & 31);
        if (L == 31) above = 0;
        if (lane == L) {
          uint32_t run = above;
          int d = 8 * L;
          for (int i = 7; i >= 0; i--) {
            if (run + c[i] >= krem) {
              d = 8 * L + i;
              break;
            }
            run += c[i];
          }
          sm.bcast[0] = (uint32_t)d;
          sm.bcast[1] = krem - run;
        }
      }
      __syncthreads();
      prefix |= sm.bcast[0] << shift;
      mask |= 0xFFu << shift;
      krem = sm.bcast[1];
    }
  }
  const uint32_t T = prefix;

  // Compaction in element order: every key > T, then the first krem keys == T.
  uint32_t gt = 0, eq = 0;
  if (k > 0) {
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      gt += key[j] > T;
      eq += key[j] == T;
    }
  }
  uint32_t eq_tot, gt_tot;
  const uint32_t eq_excl = block_excl_scan<NT>(eq, sm.wsum, eq_tot);
  block_excl_scan<NT>(gt, sm.wsum, gt_tot);
  if (t == 0) {
    sm.tot[1] = gt_tot;
    sm.tot[2] = eq_tot;
  }
  cluster.sync();
  if (t == 0) {
    uint32_t eq_before = 0, sel_before = 0;
    for (unsigned r = 0; r < rank; r++) {
      const uint32_t g = *cluster.map_shared_rank(&sm.tot[1], r);
      const uint32_t e = *cluster.map_shared_rank(&sm.tot[2], r);
      const uint32_t take = krem > eq_before ? min(krem - eq_before, e) : 0u;
      sel_before += g + take;
      eq_before += e;
    }
    sm.bcast[2] = eq_before;
    sm.bcast[3] = sel_before;
  }
  __syncthreads();
  const uint32_t my_eq_rank = sm.bcast[2] + eq_excl;
  const uint32_t take_eq = krem > my_eq_rank ? min(krem - my_eq_rank, eq) : 0u;
  uint32_t sel_tot;
  const uint32_t sel_excl = block_excl_scan<NT>(gt + take_eq, sm.wsum, sel_tot);
  if (k > 0) {
    uint32_t pos = sm.bcast[3] + sel_excl, taken = 0;
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const bool pick = key[j] > T || (key[j] == T && taken < take_eq);
      if (key[j] == T && pick) taken++;
      if (pick) out[pos++] = id[j];
    }
  }
  if (rank == 0) {
    for (int i = (int)k + t; i < k_req; i += NT) out[i] = -1;
    if (t == 0 && out_count) *out_count = (int32_t)k;
  }
  cluster.sync();  // no CTA leaves while others may still read its shared memory
}

}  // namespace csa2
