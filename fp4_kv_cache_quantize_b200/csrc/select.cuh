// select.cuh -- exact cluster-wide Top-K over 32-bit order-preserving keys.
//
// Selection rule (this library's reading of "Top-512" / "top 2,048 blocks",
// which the pages leave open for ties): the k largest keys, ties broken
// towards the lower element index, returned in ascending element order.
//
// Radix select, four 8-bit passes from the most significant digit, over the
// keys of a thread-block cluster (thread t of rank r owns elements
// (r*NT + t)*KPT + j, j < KPT; a cluster of one CTA is the common case).
// Per pass:
//   * counting: every lane owns a row of 256 counters (rows padded to 257
//     words), so no two lanes of one shared atomic meet on an address or a
//     bank whatever the keys; warps with no key in play skip the atomic;
//   * thread b < 256 sums bin b over the 32 rows (conflict-free) and clears;
//   * across the cluster, bins are pulled after a cluster barrier in the
//     first pass and pushed (remote reductions) before it in later passes;
//   * the digit: a suffix scan over the 256 bins held one per thread; the one
//     thread where the suffix count crosses the number still wanted writes
//     the digit.
// Then one packed prefix scan places every selected element in element order.
#pragma once

#include <cooperative_groups.h>

#include "csa2_internal.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

template <int NT, int KPT>
struct SelectSmem {
  uint32_t cnt[32][257];   // lane-private counters, padded rows
  uint32_t hist[256];      // this CTA's pass-0 histogram (read by the other ranks)
  uint32_t acc[4][256];    // cluster-wide histograms of passes 1..3
  uint32_t wsum[32];
  uint32_t digit[4];
  uint32_t info[16];       // per cluster rank: (keys > T) << 16 | (keys == T)
};
static_assert(sizeof(SelectSmem<256, 4>) % 16 == 0, "keeps what follows 16-byte aligned");

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
  __syncthreads();  // wsum is free again
  if (lane == 31) wsum[wid] = x;
  __syncthreads();
  uint32_t w = lane < NT / 32 ? wsum[lane] : 0u;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
    if (lane >= o) w += y;
  }
  total = __shfl_sync(0xffffffffu, w, NT / 32 - 1);
  const uint32_t before = wid ? __shfl_sync(0xffffffffu, w, (wid - 1) & 31) : 0u;
  return before + x - v;
}

// Every thread of every CTA of the cluster calls this with the same k_req.
// key[j] is element (rank*NT + t)*KPT + j's key (0 = not a candidate).
// id_of(e) maps a cluster-wide element index to the id written to out.
// Writes out[0..k) (k = min(k_req, candidates)) in ascending element order,
// out[k..k_req) = -1 and *out_count = k (rank 0 writes the last two).
// With cluster_wide = false the calling CTA selects on its own (rank 0 of a
// one-CTA selection) even inside a larger cluster.
template <int NT, int KPT, class IdOf>
__device__ void cluster_select_topk(SelectSmem<NT, KPT>& sm, const uint32_t (&key)[KPT],
                                    IdOf id_of, int k_req, int32_t* out, int32_t* out_count,
                                    bool cluster_wide = true) {
  static_assert(NT >= 256 && NT % 32 == 0, "one thread per histogram bin");
  static_assert(KPT <= 64 && NT * KPT < 65536, "16-bit packed counts");
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster_wide ? cluster.block_rank() : 0u;
  const unsigned ncta = cluster_wide ? cluster.num_blocks() : 1u;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;

  for (int i = t; i < 32 * 257; i += NT) (&sm.cnt[0][0])[i] = 0u;
  if (ncta > 1)
    for (int i = t; i < 4 * 256; i += NT) (&sm.acc[0][0])[i] = 0u;
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u, krem = 0u, k = 0u;
  for (int pass = 0; pass < 4; pass++) {
    const int shift = 24 - 8 * pass;
    uint32_t* row = sm.cnt[lane];
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const uint32_t kk = key[j];
      const bool hit = kk != 0u && (kk & mask) == prefix;
      if (__any_sync(0xffffffffu, hit) && hit) atomicAdd(&row[(kk >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t c = 0u;
    if (t < 256) {
#pragma unroll 8
      for (int l = 0; l < 32; l++) {
        c += sm.cnt[l][t];
        sm.cnt[l][t] = 0u;
      }
    }
    if (ncta > 1) {
      if (pass == 0) {
        if (t < 256) sm.hist[t] = c;
        cluster.sync();  // every rank's pass-0 histogram is complete
        if (t < 256) {
          c = 0u;
          for (unsigned r = 0; r < ncta; r++) c += *cluster.map_shared_rank(&sm.hist[t], r);
        }
      } else {
        if (t < 256 && c != 0u)
          for (unsigned r = 0; r < ncta; r++)
            atomicAdd(cluster.map_shared_rank(&sm.acc[pass][t], r), c);
        cluster.sync();
        if (t < 256) c = sm.acc[pass][t];
      }
    }
    // suffix counts S(b) = sum over bins >= b, with bin b held by thread b
    uint32_t v = c;
    if (t < 256) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, v, o);
        if (lane + o < 32) v += y;
      }
      if (lane == 0) sm.wsum[wid] = v;
    }
    __syncthreads();
    uint32_t above = 0u, all = 0u;
#pragma unroll
    for (int w = 0; w < 8; w++) {
      const uint32_t x = sm.wsum[w];
      all += x;
      if (w > wid) above += x;
    }
    if (pass == 0) {
      k = (uint32_t)k_req < all ? (uint32_t)k_req : all;  // cluster-uniform
      krem = k;
      if (k == 0u) break;
    }
    if (t < 256) {
      const uint32_t S = v + above;
      if (S >= krem && S - c < krem) {
        sm.digit[0] = (uint32_t)t;
        sm.digit[1] = krem - (S - c);
      }
    }
    __syncthreads();
    prefix |= sm.digit[0] << shift;
    mask |= 0xFFu << shift;
    krem = sm.digit[1];
  }
  const uint32_t T = prefix;

  // every key > T, then the first krem keys == T in element order
  uint32_t gt = 0u, eq = 0u;
  if (k > 0u) {
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      gt += key[j] > T;
      eq += key[j] == T;
    }
  }
  uint32_t tot;
  const uint32_t excl = block_excl_scan<NT>((gt << 16) | eq, sm.wsum, tot);
  uint32_t gt_before = 0u, eq_before = 0u;  // over the cluster ranks below this one
  if (ncta > 1) {
    if (t < (int)ncta) *cluster.map_shared_rank(&sm.info[rank], t) = tot;
    cluster.sync();  // the last cluster barrier: no remote access after it
    for (unsigned r = 0; r < rank; r++) {
      gt_before += sm.info[r] >> 16;
      eq_before += sm.info[r] & 0xFFFFu;
    }
  }
  if (k > 0u) {
    const uint32_t eq_rank = eq_before + (excl & 0xFFFFu);  // keys == T before this thread
    const uint32_t take_eq = krem > eq_rank ? min(krem - eq_rank, eq) : 0u;
    uint32_t pos = gt_before + (excl >> 16) + min(krem, eq_rank), taken = 0u;
    const int e0 = ((int)rank * NT + t) * KPT;
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const bool pick = key[j] > T || (key[j] == T && taken < take_eq);
      if (key[j] == T && pick) taken++;
      if (pick) out[pos++] = id_of(e0 + j);
    }
  }
  if (rank == 0) {
    for (int i = (int)k + t; i < k_req; i += NT) out[i] = -1;
    if (t == 0 && out_count) *out_count = (int32_t)k;
  }
}

}  // namespace csa2
