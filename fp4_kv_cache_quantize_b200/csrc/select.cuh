// select.cuh -- exact Top-K over 32-bit order-preserving keys held in the
// registers of the threads of one CTA or of a thread-block cluster.
//
// Selection rule (this library's reading of "Top-512" / "top 2,048 blocks",
// which the pages leave open for ties): the k largest keys, ties broken
// towards the lower element index, returned in ascending element order.
//
// The k-th largest key is found by narrowing a bracket [lo, hi] of key
// values round by round:
//   * round 0: the candidates' maximum, minimum and number (warp reductions,
//     then across warps and cluster ranks);
//   * each counting round cuts [lo, hi] into equal bins of key values (a
//     power-of-two width: the bin is a subtraction and a shift) and counts
//     the bracket's keys per bin; the bin holding the k-th largest key
//     becomes the new bracket.  The first round sees every key: it uses 16
//     bins, each lane counts into 4-bit fields of one 64-bit register, and a
//     warp adds its lanes' counters with six shuffles (a reduce-scatter that
//     leaves one bin's warp total per lane pair) before one shared-memory
//     atomic per bin.  Later rounds see few keys: 64 bins, one shared atomic
//     per key in the bracket.
//     With top_window, when the keys span more than SEL_TOP_SPAN, the first
//     round's 16 bins cover only the SEL_TOP_SPAN key values below the
//     maximum (two octaves of the float values the keys encode: the k
//     largest scores lie there unless the maximum is an outlier far above
//     them); if fewer than k keys fall there, every one of them is above the
//     k-th, and the next round counts the rest of the range the same way.
//   * a round ends the search when the bin's keys are exactly the ones still
//     wanted, or when the bin is a single key value (the lowest element
//     indices among the keys equal to it are taken), or (with gather_finish)
//     when the bin holds at most SEL_GATHER keys: then every rank sends its
//     keys in the bin (with their element indices) to every rank, and each
//     rank ranks the same gathered set locally, so no further counting round
//     is needed.
// The code runs once per CTA and every instruction of it is fetched cold
// (instruction fetch, not arithmetic, bounds this kernel's latency), so all
// rounds run the same rolled loop body.
// Cluster exchanges push each CTA's counts into every rank's shared memory
// with asynchronous stores (st.async) that count their bytes on the
// receiver's mbarrier: a rank waits only until every rank's counts have
// landed in its own shared memory, never on a cluster barrier, and every
// rank can work out every rank's share of the result from local reads.
// Round parities alternate two receive buffers and two mbarriers; a rank can
// send round r + 2's counts only after it has received round r + 1's from
// every rank, which each sent after reading its round r buffer, so a buffer
// is never overwritten while it is read.  The placement needs no further
// exchange: each rank knows how many selected elements precede it and how
// many of its keys equal to the threshold it takes, and places its own with
// one block prefix scan.
#pragma once

#include <cooperative_groups.h>

#include "csa2_internal.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int SEL_NB = 64;             // bins of a light round
constexpr int SEL_MAX_RANKS = 16;
constexpr uint32_t SEL_TOP_SPAN = 1u << 24;  // key values the first round looks at below the max
constexpr int SEL_GATHER = 64;               // largest bin that is gathered instead of counted
constexpr uint32_t SEL_NONE = 0xFFFFFFFFu;   // find_bin: the k-th key is below the counted range

template <int NT, int KPT>
struct SelectSmem {
  static constexpr int NW = NT / 32;
  alignas(16) uint32_t hist[2][SEL_NB];          // this CTA's counts, by round parity
  alignas(16) uint32_t xbuf[2][SEL_MAX_RANKS][SEL_NB];  // every rank's counts, by round parity
  uint32_t wred[NW][4];                          // round 0: per-warp max, min, count
  alignas(16) uint32_t cinfo[SEL_MAX_RANKS][4];  // round 0: per-rank max, min, count
  uint32_t above[SEL_MAX_RANKS];                 // per rank: keys above the bracket
  uint32_t last[SEL_MAX_RANKS];                  // per rank: keys in the bracket
  uint32_t verdict[4];
  uint32_t fin[4];                               // this rank's rule: T, keys == T taken, first output slot
  uint32_t wsum[32];
  alignas(8) uint2 gbuf[SEL_GATHER];             // gathered (key, element) pairs of the final bin
  uint32_t grank[SEL_GATHER];                    // their ranks (key descending, element ascending)
  uint32_t gt_in[SEL_MAX_RANKS], keq[SEL_MAX_RANKS];  // per rank: gathered keys > T, taken keys == T
  uint32_t gcnt, gT;
  uint64_t xbar[2];  // every rank's counts of the round have arrived (by parity)
  uint64_t cbar;     // every rank's round-0 figures have arrived
  uint64_t gbar;     // the gathered bin has arrived
};
static_assert(sizeof(SelectSmem<256, 4>) % 16 == 0, "keeps what follows 16-byte aligned");

// Every thread of every CTA calls this before the selection, before any
// other use of sm, with the same cluster_wide as the selection; it starts a
// cluster barrier that the selection completes, so a kernel issues it early
// (before waiting for its inputs) and other work hides the barrier.  No
// other cluster barrier may come between the two.
template <int NT, int KPT>
__device__ __forceinline__ void cluster_select_prologue(SelectSmem<NT, KPT>& sm,
                                                        bool cluster_wide = true) {
  const int t = threadIdx.x;
  for (int i = t; i < 2 * SEL_NB; i += NT) sm.hist[i / SEL_NB][i % SEL_NB] = 0u;
  if (t < SEL_MAX_RANKS) {
    sm.gt_in[t] = 0u;
    sm.keq[t] = 0u;
  }
  if (t == 0) {
    sm.gcnt = 0u;
    mbar_init(&sm.xbar[0], 1);
    mbar_init(&sm.xbar[1], 1);
    mbar_init(&sm.cbar, 1);
    mbar_init(&sm.gbar, 1);
    fence_mbar_init();
  }
  if (cluster_wide && cg::this_cluster().num_blocks() > 1) cluster_arrive_release();
}

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

// First counting round: 16 bins of width 2^s over [lo, lo + span], every
// lane's keys counted into nibbles, warp totals by a shuffle reduce-scatter,
// one shared atomic per bin and warp into hist.
template <int N>
__device__ __forceinline__ void count16(uint32_t* hist, const uint32_t (&key)[N], uint32_t lo,
                                        uint32_t span, int s) {
  static_assert(N <= 15, "4-bit per-lane counters");
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  uint64_t c = 0ull;
#pragma unroll
  for (int j = 0; j < N; j++) {
    const uint32_t d = key[j] - lo;  // keys below lo (and 0) wrap past span
    if (d <= span) c += 1ull << (((d >> s) & 15u) * 4u);
  }
  // nibbles -> bytes: w_i holds bins 4i..4i+3 (at most 15 each)
  const uint32_t x0 = (uint32_t)c, x1 = (uint32_t)(c >> 32);
  const uint32_t e0 = x0 & 0x0F0F0F0Fu, o0 = (x0 >> 4) & 0x0F0F0F0Fu;
  const uint32_t e1 = x1 & 0x0F0F0F0Fu, o1 = (x1 >> 4) & 0x0F0F0F0Fu;
  const uint32_t w0 = __byte_perm(e0, o0, 0x5140), w1 = __byte_perm(e0, o0, 0x7362);
  const uint32_t w2 = __byte_perm(e1, o1, 0x5140), w3 = __byte_perm(e1, o1, 0x7362);
  // lanes with bit 4 clear keep bins 0-7 (w0, w1), the others bins 8-15
  const bool b4 = lane & 16;
  uint32_t k0 = b4 ? w2 : w0, k1 = b4 ? w3 : w1;
  k0 += __shfl_xor_sync(FULL, b4 ? w0 : w2, 16);
  k1 += __shfl_xor_sync(FULL, b4 ? w1 : w3, 16);
  // bit 3: one word of 4 bins (bytes; at most 4 x 15 = 60)
  const bool b3 = lane & 8;
  uint32_t k = b3 ? k1 : k0;
  k += __shfl_xor_sync(FULL, b3 ? k0 : k1, 8);
  // bit 2: two bins as 16-bit halves
  const bool b2 = lane & 4;
  const uint32_t lo2 = __byte_perm(k, 0u, 0x4140), hi2 = __byte_perm(k, 0u, 0x4342);
  uint32_t h = b2 ? hi2 : lo2;
  h += __shfl_xor_sync(FULL, b2 ? lo2 : hi2, 4);
  // bit 1: one bin
  const bool b1 = lane & 2;
  uint32_t v = b1 ? (h >> 16) : (h & 0xFFFFu);
  v += __shfl_xor_sync(FULL, b1 ? (h & 0xFFFFu) : (h >> 16), 2);
  // bit 0: lanes 2i and 2i+1 hold bin i; the pair's sum is the warp total
  v += __shfl_xor_sync(FULL, v, 1);
  if ((lane & 1) == 0 && v != 0u) atomicAdd(&hist[lane >> 1], v);
}

// Later rounds: 64 bins, one shared atomic per key in the bracket.
template <int N>
__device__ __forceinline__ void count64(uint32_t* hist, const uint32_t (&key)[N], uint32_t lo,
                                        uint32_t span, int s) {
#pragma unroll
  for (int j = 0; j < N; j++) {
    const uint32_t d = key[j] - lo;
    if (d <= span) atomicAdd(&hist[d >> s], 1u);
  }
}

// Warp 0: the bin of the krem-th largest key from per-rank counts
// xs[r][b] (r < nr); writes (bin, keys above it, keys in it) to verdict, or
// (SEL_NONE, keys in the range, 0) when the range holds fewer than krem.
template <class Smem>
__device__ __forceinline__ void find_bin(Smem& sm, const uint32_t (*xs)[SEL_NB], unsigned nr,
                                         uint32_t krem) {
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
  for (unsigned r = 0; r < SEL_MAX_RANKS; r++) {  // all loads in flight at once
    if (r < nr) {
      c0 += xs[r][2 * lane];
      c1 += xs[r][2 * lane + 1];
    }
  }
  const uint32_t pair = c0 + c1;
  uint32_t suf = pair;  // keys in bins >= 2 lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(FULL, suf, o);
    if (lane + o < 32) suf += y;
  }
  const uint32_t above_hi = suf - pair;  // bins > 2 lane + 1
  if (lane == 0) {  // (no bin holds it: fewer than krem keys in the range)
    sm.verdict[0] = SEL_NONE;
    sm.verdict[1] = suf;
    sm.verdict[2] = 0u;
  }
  __syncwarp();
  if (above_hi < krem && above_hi + pair >= krem) {
    const bool in_hi = above_hi + c1 >= krem;
    sm.verdict[0] = in_hi ? 2u * lane + 1u : 2u * lane;
    sm.verdict[1] = in_hi ? above_hi : above_hi + c1;
    sm.verdict[2] = in_hi ? c1 : c0;
  }
}

__device__ __forceinline__ int round_shift(uint32_t span, int bits) {
  const int nbits = 32 - __clz(span);
  return nbits > bits ? nbits - bits : 0;
}

// Every thread of every CTA of the cluster calls this with the same k_req,
// after cluster_select_prologue.
// key[j] is element (rank*NT + t)*KPT + j's key (0 = not a candidate).
// id_of(e) maps a cluster-wide element index to the id written to out.
// Writes out[0..k) (k = min(k_req, candidates)) in ascending element order,
// out[k..k_req) = -1 and *out_count = k (rank 0 writes the last two).
// With cluster_wide = false the calling CTA selects on its own (rank 0 of a
// one-CTA selection) even inside a larger cluster.  top_window and
// gather_finish choose the first round's range and the last step (header
// comment); they change the work, not the result.  A wait for another
// rank's counts that gives up (after kWaitCycles) sets ST_TIMEOUT in
// *status (when given) and the result is not defined.
// cluster_select_emit: the same selection, handing each selected element to
// emit(output slot, id) instead of writing an array; returns k.
template <int NT, int KPT, class IdOf, class Emit>
__device__ uint32_t cluster_select_emit(SelectSmem<NT, KPT>& sm, const uint32_t (&key)[KPT],
                                        IdOf id_of, int k_req, Emit emit,
                                        bool cluster_wide = true, uint32_t* status = nullptr,
                                        bool top_window = false, bool gather_finish = false) {
  static_assert(NT >= 64 && NT % 32 == 0, "at least 64 threads");
  static_assert(KPT <= 15, "4-bit per-lane counters");
  static_assert(NT * KPT < 65536, "16-bit packed counts");
  constexpr int NW = NT / 32;
  constexpr uint32_t FULL = 0xffffffffu;
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster_wide ? cluster.block_rank() : 0u;
  const unsigned ncta = cluster_wide ? cluster.num_blocks() : 1u;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  bool failed = false;  // a wait gave up: later waits are skipped
  auto wait_counts = [&](uint64_t* bar, uint32_t parity) {
    if (!failed && !mbar_wait_cluster(bar, parity)) {
      failed = true;
      if (status) set_status(status, ST_TIMEOUT);
    }
  };
  // every rank's barriers are initialised (the prologue's arrival)
  if (ncta > 1) cluster_wait_acquire();

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
      if (ncta > 1) {  // push this CTA's figures to every rank
        if (lane == 0) mbar_arrive_expect_tx(&sm.cbar, 16u * ncta);
        __syncwarp();
        if (lane < (int)ncta)
          st_async_v4(mapa_rank(&sm.cinfo[rank][0], lane), make_uint4(a, b, c, 0u),
                      mapa_rank(&sm.cbar, lane));
      } else if (lane == 0) {
        *reinterpret_cast<uint4*>(sm.cinfo[0]) = make_uint4(a, b, c, 0u);
      }
    }
    if (ncta > 1) wait_counts(&sm.cbar, 0u);
    else __syncthreads();
  }
  uint32_t gmx = 0u, gmn = FULL, gcnt = 0u, cnt_below = 0u;
#pragma unroll
  for (unsigned r = 0; r < SEL_MAX_RANKS; r++) {
    if (r < ncta) {
      const uint4 ci = *reinterpret_cast<const uint4*>(sm.cinfo[r]);
      gmx = max(gmx, ci.x);
      gmn = min(gmn, ci.y);
      gcnt += ci.z;
      if (r < rank) cnt_below += ci.z;
    }
  }
  const uint32_t kr = (uint32_t)(k_req > 0 ? k_req : 0);
  const uint32_t k = kr < gcnt ? kr : gcnt;

  // The result on every rank r: every key > Tx, then the first keq_r keys
  // == Tx of the rank in element order, placed from output slot off_r.
  if (k == 0u || k == gcnt) {
    if (t == 0) {
      sm.fin[0] = k ? gmn - 1u : FULL;  // every candidate, or none
      sm.fin[1] = 0u;
      sm.fin[2] = k ? cnt_below : 0u;
    }
    __syncthreads();
  } else {
    uint32_t lo = gmn, hi = gmx, krem = k;
    if (t < SEL_MAX_RANKS) sm.above[t] = 0u;
    int mode = 0;  // 1: the whole bin; 2: one key value; 3: the bin is gathered
    uint32_t nlo = lo, nhi = hi, inbin = 0u;
    bool wide = true;  // this round sees every key: 16 bins in nibble counters
#pragma unroll 1  // one copy of the body: its instructions are fetched once
    for (int round = 0; round < 14; round++) {
      const int par = round & 1;
      // the counted range [clo, hi]; the first round looks only below the max
      const bool top = top_window && round == 0 && hi - lo >= SEL_TOP_SPAN;
      const uint32_t clo = top ? hi - (SEL_TOP_SPAN - 1u) : lo;
      const uint32_t span = hi - clo;  // > 0 here
      int s;
      if (wide) {
        s = round_shift(span, 4);
        count16<KPT>(sm.hist[par], key, clo, span, s);
      } else {
        s = round_shift(span, 6);
        count64<KPT>(sm.hist[par], key, clo, span, s);
      }
      __syncthreads();
      // the other parity's counts were pushed last round, before that
      // round's find: clear them for the next round
      if (t < SEL_NB) sm.hist[par ^ 1][t] = 0u;
      if (ncta > 1) {  // push this CTA's counts to every rank, 16 bytes per thread
        if (t == 0) mbar_arrive_expect_tx(&sm.xbar[par], (uint32_t)(SEL_NB * 4) * ncta);
        for (int i = t; i < (SEL_NB / 4) * (int)ncta; i += NT) {
          const int g = i % (SEL_NB / 4), r = i / (SEL_NB / 4);
          st_async_v4(mapa_rank(&sm.xbuf[par][rank][4 * g], r),
                      *reinterpret_cast<const uint4*>(&sm.hist[par][4 * g]),
                      mapa_rank(&sm.xbar[par], r));
        }
        wait_counts(&sm.xbar[par], (uint32_t)(round >> 1) & 1u);
      } else {
        if (t < SEL_NB) sm.xbuf[par][0][t] = sm.hist[par][t];
        __syncthreads();
      }
      if (wid == 0) find_bin(sm, sm.xbuf[par], ncta, krem);
      __syncthreads();
      const uint32_t jb = sm.verdict[0], above = sm.verdict[1];
      inbin = sm.verdict[2];
      // warp r: rank r's keys above the bin (every counted key when the
      // k-th lies below the range) and in it
      const int jbi = jb == SEL_NONE ? -1 : (int)jb;
      for (int r = wid; r < (int)ncta; r += NW) {
        const uint32_t* xr = sm.xbuf[par][r];
        uint32_t a = (2 * lane > jbi ? xr[2 * lane] : 0u) + (2 * lane + 1 > jbi ? xr[2 * lane + 1] : 0u);
        a = __reduce_add_sync(FULL, a);
        if (lane == 0) {
          sm.above[r] += a;
          if (jbi >= 0) sm.last[r] = xr[jbi];
        }
      }
      krem -= above;
      if (jb == SEL_NONE) {  // (first round only) the rest of the range, counted wide
        hi = clo - 1u;
        continue;
      }
      wide = false;
      nlo = clo + (jb << s);
      const uint64_t h64 = (uint64_t)nlo + ((1ull << s) - 1ull);
      nhi = h64 < (uint64_t)hi ? (uint32_t)h64 : hi;
      if (inbin == krem) { mode = 1; break; }
      if (nlo == nhi || round == 13) { mode = 2; break; }  // 32 bits take at most 7 rounds
      if (gather_finish && inbin <= (uint32_t)SEL_GATHER) { mode = 3; break; }
      lo = nlo;
      hi = nhi;
    }
    __syncthreads();  // above / last complete
    if (mode == 3) {
      // ---- gather the bin: rank r's keys in [nlo, nhi] go to slots from
      // sum_{r' < r} last[r'] on every rank; then every rank ranks them
      uint32_t off = 0u;
      for (unsigned r = 0; r < rank; r++) off += sm.last[r];
      if (ncta > 1 && t == 0) mbar_arrive_expect_tx(&sm.gbar, inbin * 8u);
      const int e0 = ((int)rank * NT + t) * KPT;
#pragma unroll
      for (int j = 0; j < KPT; j++) {
        if (key[j] >= nlo && key[j] <= nhi) {
          const uint32_t slot = off + atomicAdd(&sm.gcnt, 1u);
          // (always below inbin <= SEL_GATHER; a bound only in case a failed
          // wait left the counts inconsistent)
          if (slot >= (uint32_t)SEL_GATHER) continue;
          if (ncta > 1) {
            for (unsigned r = 0; r < ncta; r++)
              st_async_v2(mapa_rank(&sm.gbuf[slot], r), key[j], (uint32_t)(e0 + j),
                          mapa_rank(&sm.gbar, r));
          } else {
            sm.gbuf[slot] = make_uint2(key[j], (uint32_t)(e0 + j));
          }
        }
      }
      if (ncta > 1) wait_counts(&sm.gbar, 0u);
      else __syncthreads();
      // rank of candidate i: candidates before it (key descending, element
      // ascending); warp w takes candidates w, w + NW, ...
      for (int i = wid; i < (int)inbin; i += NW) {
        const uint2 ci = sm.gbuf[i];
        uint32_t c = 0u;
        for (int j = lane; j < (int)inbin; j += 32) {
          const uint2 cj = sm.gbuf[j];
          c += cj.x > ci.x || (cj.x == ci.x && cj.y < ci.y);
        }
        c = __reduce_add_sync(FULL, c);
        if (lane == 0) {
          sm.grank[i] = c;
          if (c == krem - 1u) sm.gT = ci.x;  // the k-th largest key
        }
      }
      __syncthreads();
      const uint32_t T = sm.gT;
      if (t < (int)inbin) {
        const uint2 ci = sm.gbuf[t];
        const uint32_t src = ci.y / (uint32_t)(NT * KPT);
        if (ci.x > T) atomicAdd(&sm.gt_in[src], 1u);
        else if (ci.x == T && sm.grank[t] < krem) atomicAdd(&sm.keq[src], 1u);
      }
      __syncthreads();
      if (t == 0) {
        uint32_t o = 0u;
        for (unsigned r = 0; r < rank; r++) o += sm.above[r] + sm.gt_in[r] + sm.keq[r];
        sm.fin[0] = T;
        sm.fin[1] = sm.keq[rank];
        sm.fin[2] = o;
      }
      __syncthreads();
    } else {
      if (wid == 0) {
        // lane r = rank r.  mode 1: every key of the bin (>= nlo); mode 2:
        // the first krem keys == nlo in element order (ranks in order)
        const bool in = lane < (int)ncta;
        const uint32_t e = in ? sm.last[lane] : 0u, ab = in ? sm.above[lane] : 0u;
        uint32_t eqi = e;  // inclusive prefix over ranks of the keys in the bin
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(FULL, eqi, o);
          if (lane >= o) eqi += y;
        }
        const uint32_t eqb = eqi - e;
        const uint32_t kq = mode == 1 ? 0u : (krem > eqb ? min(krem - eqb, e) : 0u);
        const uint32_t sel = ab + (mode == 1 ? e : kq);
        uint32_t seli = sel;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(FULL, seli, o);
          if (lane >= o) seli += y;
        }
        if (lane == (int)rank) {
          sm.fin[0] = mode == 1 ? nlo - 1u : nlo;
          sm.fin[1] = kq;
          sm.fin[2] = seli - sel;
        }
      }
      __syncthreads();
    }
  }

  // ---- placement: every key > Tx, then the first keq keys == Tx of this rank
  const uint32_t Tx = sm.fin[0], keq = sm.fin[1], out_off = sm.fin[2];
  uint32_t gt = 0u, eq = 0u;
#pragma unroll
  for (int j = 0; j < KPT; j++) {
    gt += key[j] > Tx;
    eq += key[j] == Tx && key[j] != 0u;
  }
  uint32_t tot;
  const uint32_t excl = block_excl_scan<NT>((gt << 16) | eq, sm.wsum, tot);
  if (k > 0u) {
    const uint32_t eq_rank = excl & 0xFFFFu;  // keys == Tx of this rank before this thread
    const uint32_t take_eq = keq > eq_rank ? min(keq - eq_rank, eq) : 0u;
    uint32_t pos = out_off + (excl >> 16) + min(keq, eq_rank), taken = 0u;
    const int e0 = ((int)rank * NT + t) * KPT;
#pragma unroll
    for (int j = 0; j < KPT; j++) {
      const bool tie = key[j] == Tx && key[j] != 0u;
      const bool pick = key[j] > Tx || (tie && taken < take_eq);
      if (tie && pick) taken++;
      if (pick) emit((int)pos++, id_of(e0 + j));
    }
  }
  return k;
}

template <int NT, int KPT, class IdOf>
__device__ void cluster_select_topk(SelectSmem<NT, KPT>& sm, const uint32_t (&key)[KPT],
                                    IdOf id_of, int k_req, int32_t* out, int32_t* out_count,
                                    bool cluster_wide = true, uint32_t* status = nullptr,
                                    bool top_window = false, bool gather_finish = false) {
  const uint32_t k = cluster_select_emit(
      sm, key, id_of, k_req, [out](int pos, int id) { out[pos] = id; }, cluster_wide, status,
      top_window, gather_finish);
  const unsigned rank = cluster_wide ? cg::this_cluster().block_rank() : 0u;
  if (rank == 0) {
    for (int i = (int)k + (int)threadIdx.x; i < k_req; i += NT) out[i] = -1;
    if (threadIdx.x == 0 && out_count) *out_count = (int32_t)k;
  }
}

}  // namespace csa2
