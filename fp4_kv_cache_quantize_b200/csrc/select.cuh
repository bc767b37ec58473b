// select.cuh -- exact Top-K over 32-bit order-preserving keys held in the
// registers of the threads of one CTA or of a thread-block cluster.
//
// Selection rule (this library's reading of "Top-512" / "top 2,048 blocks",
// which the pages leave open for ties): the k largest keys, ties broken
// towards the lower element index, returned in ascending element order.
//
// The k-th largest key is found by narrowing a bracket [lo, hi] of key
// values round by round, with counting only (no shared-memory atomics: on
// this GPU a CTA of shared atomics over a few thousand keys costs several
// microseconds, which is what a histogram-per-pass radix select spends):
//   * round 0: the candidates' maximum, minimum and number, one warp
//     reduction (redux.sync) per quantity, then across warps and ranks;
//   * each further round cuts [lo, hi] into SEL_NB equal bins of key values
//     (a power-of-two width, so the bin is a subtraction and a shift); every
//     lane counts its keys inside the bracket into 4-bit fields of packed
//     64-bit counters, a warp adds its lanes' counts with one redux.sync per
//     pair of bins, CTA and cluster totals follow; the bin holding the k-th
//     key becomes the new bracket.  A round ends the search when the bin's
//     keys are exactly the ones still wanted, or when the bracket holds a
//     single key value (then the lowest element indices among the keys equal
//     to it are taken).
// Cluster exchanges push each CTA's few counters into every rank's shared
// memory before a cluster barrier (remote stores never wait), so every read
// after a barrier is local.  One packed prefix scan then places every
// selected element in element order.
#pragma once

#include <cooperative_groups.h>

#include "csa2_internal.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int SEL_DB0 = 4;             // key bits the first counting round resolves (at best)
constexpr int SEL_DB = 6;              // ... and every later round
constexpr int SEL_NB = 1 << SEL_DB;    // bins of a round, at most
constexpr int SEL_MAX_RANKS = 16;

template <int NT, int KPT>
struct SelectSmem {
  static constexpr int NW = NT / 32;
  uint32_t wcnt[NW][SEL_NB / 2];                 // per-warp counts, bins (2i, 2i+1) as 16-bit halves
  uint32_t xbuf[2][SEL_MAX_RANKS][SEL_NB / 2];   // per-rank CTA counts, by round parity
  uint32_t wred[NW][4];                          // round 0: per-warp max, min, count
  uint32_t cinfo[SEL_MAX_RANKS][4];              // round 0: per-rank max, min, count
  uint32_t verdict[4];                           // the round's chosen bin, keys above it, keys in it
  uint32_t wsum[32];
  uint32_t info[SEL_MAX_RANKS];                  // placement: per rank (keys > T) << 16 | (keys == T)
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

// One counting round: this CTA's counts of the keys in [lo, lo + span] per
// bin (key - lo) >> s, bins 0..2^DB-1, pushed as pairs of 16-bit halves into
// xbuf[par][rank][*] of every rank (the caller's barrier completes them).
template <int NT, int KPT, int DB>
__device__ __forceinline__ void count_bins(SelectSmem<NT, KPT>& sm, const uint32_t (&key)[KPT],
                                           uint32_t lo, uint32_t span, int s, int par,
                                           unsigned rank, unsigned ncta,
                                           cg::cluster_group& cluster) {
  constexpr int NB = 1 << DB, NP = NB / 16, NW = NT / 32;
  static_assert(NB >= 16 && NB <= SEL_NB, "bins per round");
  constexpr uint32_t FULL = 0xffffffffu;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  uint64_t c[NP];
#pragma unroll
  for (int q = 0; q < NP; q++) c[q] = 0ull;
  bool any = false;
#pragma unroll
  for (int j = 0; j < KPT; j++) {
    const uint32_t d = key[j] - lo;  // keys below lo (and 0) wrap past span
    if (d <= span) {
      const uint32_t b = d >> s;
      const uint64_t inc = 1ull << ((b & 15u) * 4u);
      if constexpr (NP == 1) {
        c[0] += inc;
      } else {
#pragma unroll
        for (int q = 0; q < NP; q++) c[q] += (b >> 4) == (uint32_t)q ? inc : 0ull;
      }
      any = true;
    }
  }
  if (__any_sync(FULL, any)) {
    // nibbles -> 16-bit halves: word w holds bins 2w (low) and 2w+1 (high)
#pragma unroll
    for (int h = 0; h < 2 * NP; h++) {
      const uint32_t x = (uint32_t)(c[h >> 1] >> (32 * (h & 1)));
      const uint32_t ev = x & 0x0F0F0F0Fu, od = (x >> 4) & 0x0F0F0F0Fu;
      const uint32_t i01 = __byte_perm(ev, od, 0x5140), i23 = __byte_perm(ev, od, 0x7362);
      const uint32_t w4[4] = {__byte_perm(i01, 0u, 0x4140), __byte_perm(i01, 0u, 0x4342),
                              __byte_perm(i23, 0u, 0x4140), __byte_perm(i23, 0u, 0x4342)};
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const uint32_t v = __reduce_add_sync(FULL, w4[u]);
        if (lane == 0) sm.wcnt[wid][4 * h + u] = v;
      }
    }
  } else if (lane < NB / 2) {
    sm.wcnt[wid][lane] = 0u;
  }
  __syncthreads();
  if (t < SEL_NB / 2) {  // this CTA's counts of bins (2t, 2t+1), pushed to every rank
    uint32_t v = 0u;
    if (t < NB / 2) {
#pragma unroll 8
      for (int w = 0; w < NW; w++) v += sm.wcnt[w][t];
    }
    if (ncta > 1) {
      for (unsigned r = 0; r < ncta; r++) *cluster.map_shared_rank(&sm.xbuf[par][rank][t], r) = v;
    } else {
      sm.xbuf[par][0][t] = v;
    }
  }
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
  static_assert(NT >= 64 && NT % 32 == 0, "at least two warps");
  static_assert(KPT <= 15, "4-bit per-lane counters");
  static_assert(NT * KPT < 65536, "16-bit packed counts");
  constexpr int NW = NT / 32;
  constexpr uint32_t FULL = 0xffffffffu;
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster_wide ? cluster.block_rank() : 0u;
  const unsigned ncta = cluster_wide ? cluster.num_blocks() : 1u;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;

  // ---- round 0: maximum, minimum and number of candidates
  {
    uint32_t mx = 0u, mn = FULL, cnt = 0u;
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const uint32_t kk = key[j];
      if (kk != 0u) {
        mx = max(mx, kk);
        mn = min(mn, kk);
        cnt++;
      }
    }
    mx = __reduce_max_sync(FULL, mx);
    mn = __reduce_min_sync(FULL, mn);
    cnt = __reduce_add_sync(FULL, cnt);
    if (lane == 0) {
      sm.wred[wid][0] = mx;
      sm.wred[wid][1] = mn;
      sm.wred[wid][2] = cnt;
    }
    __syncthreads();
    if (wid == 0) {
      uint32_t a = 0u, b = FULL, c = 0u;
      if (lane < NW) {
        a = sm.wred[lane][0];
        b = sm.wred[lane][1];
        c = sm.wred[lane][2];
      }
      a = __reduce_max_sync(FULL, a);
      b = __reduce_min_sync(FULL, b);
      c = __reduce_add_sync(FULL, c);
      if (lane < (int)ncta) {  // push this CTA's figures to every rank
        uint32_t* dst = ncta > 1 ? cluster.map_shared_rank(&sm.cinfo[rank][0], lane)
                                 : &sm.cinfo[0][0];
        dst[0] = a;
        dst[1] = b;
        dst[2] = c;
      }
    }
    if (ncta > 1) cluster.sync();
    else __syncthreads();
  }
  uint32_t gmx = 0u, gmn = FULL, gcnt = 0u;
  for (unsigned r = 0; r < ncta; r++) {
    gmx = max(gmx, sm.cinfo[r][0]);
    gmn = min(gmn, sm.cinfo[r][1]);
    gcnt += sm.cinfo[r][2];
  }
  const uint32_t k = (uint32_t)(k_req > 0 ? k_req : 0) < gcnt ? (uint32_t)(k_req > 0 ? k_req : 0)
                                                              : gcnt;

  // The selection: every key > Tx, then the first keq keys == Tx in element
  // order (keq = 0 when every key >= Tx + 1 is taken).
  uint32_t Tx = FULL, keq = 0u;
  if (k > 0u && k == gcnt) {
    Tx = gmn - 1u;  // every candidate (gmn >= 1)
  } else if (k > 0u) {
    uint32_t lo = gmn, hi = gmx, krem = k;
    // each round leaves at most 2^(span bits - SEL_DB0 or SEL_DB) key values:
    // the bracket is a single value after at most 8 rounds
    for (int round = 0;; round++) {
      if (lo == hi || round == 12) {  // one key value left: ties by element order
        Tx = lo;
        keq = krem;
        break;
      }
      const uint32_t span = hi - lo;
      const int nbits = 32 - __clz(span);
      int shift;
      const int par = round & 1;
      // the first round sees every key: fewer bins keep it cheap; later
      // rounds see few keys and resolve more bits each
      if (round == 0) {
        const int s = nbits > SEL_DB0 ? nbits - SEL_DB0 : 0;
        shift = s;
        count_bins<NT, KPT, SEL_DB0>(sm, key, lo, span, s, par, rank, ncta, cluster);
      } else {
        const int s = nbits > SEL_DB ? nbits - SEL_DB : 0;
        shift = s;
        count_bins<NT, KPT, SEL_DB>(sm, key, lo, span, s, par, rank, ncta, cluster);
      }
      if (ncta > 1) cluster.sync();
      else __syncthreads();
      // ---- warp 0: totals of bins (2 lane, 2 lane + 1), the bin of the k-th key
      if (wid == 0) {
        uint32_t c0 = 0u, c1 = 0u;
        for (unsigned r = 0; r < ncta; r++) {
          const uint32_t v = sm.xbuf[par][r][lane];
          c0 += v & 0xFFFFu;
          c1 += v >> 16;
        }
        // keys in bins above 2 lane + 1: suffix sum over the higher lanes
        uint32_t pair = c0 + c1, suf = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(FULL, suf, o);
          if (lane + o < 32) suf += y;
        }
        const uint32_t above_hi = suf - pair;  // bins > 2 lane + 1
        if (above_hi < krem && above_hi + pair >= krem) {
          const bool in_hi = above_hi + c1 >= krem;
          sm.verdict[0] = in_hi ? 2u * lane + 1u : 2u * lane;
          sm.verdict[1] = in_hi ? above_hi : above_hi + c1;
          sm.verdict[2] = in_hi ? c1 : c0;
        }
      }
      __syncthreads();
      const uint32_t jb = sm.verdict[0], above = sm.verdict[1], inbin = sm.verdict[2];
      krem -= above;
      const uint32_t nlo = lo + (jb << shift);
      const uint64_t nhi = (uint64_t)nlo + ((1ull << shift) - 1ull);
      if (inbin == krem) {  // the whole bin: every key >= nlo
        Tx = nlo - 1u;
        keq = 0u;
        break;
      }
      lo = nlo;
      hi = nhi < (uint64_t)hi ? (uint32_t)nhi : hi;
    }
  }

  // ---- placement: every key > Tx, then the first keq keys == Tx
  uint32_t gt = 0u, eq = 0u;
#pragma unroll
  for (int j = 0; j < KPT; j++) {
    gt += key[j] > Tx;
    eq += key[j] == Tx;
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
    const uint32_t eq_rank = eq_before + (excl & 0xFFFFu);  // keys == Tx before this thread
    const uint32_t take_eq = keq > eq_rank ? min(keq - eq_rank, eq) : 0u;
    uint32_t pos = gt_before + (excl >> 16) + min(keq, eq_rank), taken = 0u;
    const int e0 = ((int)rank * NT + t) * KPT;
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const bool pick = key[j] > Tx || (key[j] == Tx && taken < take_eq);
      if (key[j] == Tx && pick) taken++;
      if (pick) out[pos++] = id_of(e0 + j);
    }
  }
  if (rank == 0) {
    for (int i = (int)k + t; i < k_req; i += NT) out[i] = -1;
    if (t == 0 && out_count) *out_count = (int32_t)k;
  }
}

}  // namespace csa2
