// score.cu -- the CSA2 indexer kernels.
//
//  * score_scan_kernel: the Full-mode scan [release note, section
//    "Compressed Sparse Attention 2 (CSA2)": the Full layer scores every
//    causally visible position; yomxxx.com CSA2 notes, section 二, HSI
//    paragraph: it keeps the top 2,048 blocks of 8 positions by block max].
//    It streams the bf16 indexer K (128 B per position) from HBM with TMA
//    into a 3-stage shared-memory ring (128B-swizzled tiles of 128 positions),
//    four CTAs per SM (four independent producer/MMA/epilogue pipelines keep
//    more requests in flight than one deep ring per CTA does),
//    one thread issues tcgen05.mma (M = 128 positions, N = 8 indexer heads
//    per query padded to 16/32/64, K = 64) into a ring of TMEM accumulators,
//    and four (eight for N = 64) epilogue warps read the dot products back
//    (tcgen05.ld), apply s = sum_h w_h * relu(q_h . k) per query, and write
//    only the block maxima of 8-position blocks.  Scores never touch HBM.
//    With several queries per sequence (draft verification, chunked
//    prefill) one launch scores up to 8 of them per indexer-K row.
//  * rescore_select_kernel: scores the positions of a set of candidate blocks
//    (the HSI pool for Reindex layers, the Full layer's top blocks for its own
//    Top-512) with mma.sync tensor-core tiles over gathered rows, then
//    selects the exact Top-k in the same cluster with the radix select of
//    select.cuh.  Several (layer, sequence) jobs run in one launch.
//  * block_select_kernel: the HSI pool, the top blocks by block maximum, with
//    the same radix select over a cluster of up to 16 CTAs per sequence.
#include <cuda_bf16.h>

#include "csa2_internal.cuh"
#include "kernels.h"
#include "select.cuh"

namespace csa2 {

// ------------------------------------------------------------- the scan
constexpr int SC_BOX = 64;                 // rows per TMA box
constexpr int SC_STAGES = 3;
constexpr int SC_CTAS_PER_SM = 4;          // up to four independent pipelines per SM
constexpr int SC_A_BYTES = SC_TILE * 128;  // 16 KB of indexer K per stage

// One instantiation per MMA width N: the 8 indexer heads of every query of a
// sequence (nq queries, 8 nq <= N), padded to 16, 32 or 64; ACC accumulators
// of N fp32 columns in TMEM.
template <int N, int ACC>
struct ScanCfg {
  // N = 64: 8 epilogue warps, two per TMEM lane quarter, each with half the
  // queries (the per-row work of 8 queries would otherwise limit the pipeline)
  static constexpr int EPI_WARPS = N > 32 ? 8 : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int B_BYTES = N * 128;  // indexer queries per stage
  static constexpr uint32_t IDESC = idesc_bf16_f32(SC_TILE, N);
  static constexpr uint32_t TMEM_COLS = N * ACC;
  static_assert(TMEM_COLS >= 32 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation size");
  static_assert(TMEM_COLS * SC_CTAS_PER_SM <= 512, "TMEM columns of one SM");
  struct Smem {
    uint8_t a[SC_STAGES][SC_A_BYTES];
    uint8_t b[SC_STAGES][B_BYTES];
    uint64_t full[SC_STAGES], empty[SC_STAGES];
    uint64_t tfull[ACC], tempty[ACC], tinfo[ACC], done;
    int32_t tile[SC_STAGES];  // the tile each stage holds (-1: no more tiles)
    int32_t acc_tile[ACC];    // the tile each accumulator holds (-1: no more tiles)
    uint32_t tmem_base;
    int abort;
    // N = 64 (two batches of TMEM loads per tile): each epilogue warp's copy
    // of the launch's query weights, loaded once per sequence
    float wq[N > 32 ? 8 * CSA2_SCAN_QUERIES * CSA2_HI : 2];
  };
  static constexpr size_t SMEM = sizeof(Smem) + 1024;
};

__device__ __forceinline__ int visible_rows(const int32_t* n_rows, int b, int max_rows,
                                            uint32_t* status) {
  int c = n_rows[b];
  if (c < 0 || c > max_rows) {
    set_status(status, ST_DEVICE_CHECK);
    c = c < 0 ? 0 : max_rows;
  }
  return c;
}

// Entries visible to query v % nq of sequence v / nq: the sequence's count
// minus the drafts after that query (never negative).
__device__ __forceinline__ int visible_query(const int32_t* n_rows, int v, int nq, int max_rows,
                                             uint32_t* status) {
  const int b = v / nq, t = v - b * nq;
  const int c = visible_rows(n_rows, b, max_rows, status) - (nq - 1 - t);
  return c < 0 ? 0 : c;
}

// First pool row of the 64-row box holding position pos0 (a multiple of 64),
// or pool_rows (out of range: TMA fills zeros) when the row map is invalid.
__device__ __forceinline__ int32_t box_row(const ScanParams& p, int b, int pos0) {
  int64_t row;
  if (p.page_table) {
    const int page = pos0 / SC_BOX;
    const int64_t pid = page < p.max_pages ? (int64_t)p.page_table[(int64_t)b * p.max_pages + page]
                                           : -1;
    row = pid * SC_BOX;
    if (pid < 0 || row + SC_BOX > p.pool_rows) {
      set_status(p.status, ST_DEVICE_CHECK);
      row = p.pool_rows;
    }
  } else {
    row = (int64_t)b * p.seq_stride + pos0;
  }
  return (int32_t)row;
}

// ONE: the single-query specialisation (weights held in registers, one TMEM
// load per tile).
template <int N, int ACC, bool ONE>
__global__ void __launch_bounds__(ScanCfg<N, ACC>::THREADS, N <= 16 ? SC_CTAS_PER_SM : (N <= 32 ? 3 : 2))
    score_scan_kernel(const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_q, const ScanParams p) {
  using Cfg = ScanCfg<N, ACC>;
  using ScanSmem = typename Cfg::Smem;
  extern __shared__ uint8_t smem_raw[];
  ScanSmem& s = *reinterpret_cast<ScanSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int64_t total = (int64_t)p.batch * p.tiles_per_seq;
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < SC_STAGES; i++) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < ACC; i++) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], Cfg::EPI_WARPS * 32);
      mbar_init(&s.tinfo[i], 1);
    }
    mbar_init(&s.done, 1);
    s.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_q);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, Cfg::TMEM_COLS);  // ACC accumulators of N fp32 columns
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort = &s.abort;
  // The prologue above overlaps the previous kernel (e.g. the cache append
  // that wrote the newest rows); nothing it wrote is read before this.
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------- TMA producer
      int stage = 0, cur_b = -1, C = 0;
      uint32_t phase = 0, issued = 0, issued_phase = 0;
      const uint64_t stream_once = l2_policy_evict_first();  // indexer K is read once per step
      // Tiles are handed out by a counter in the workspace header, one at a
      // time, so that CTAs that run faster take more of them (a fixed
      // interleave leaves a tail of slow CTAs); the next tile is requested
      // while the current one is issued.  Every CTA stops at its first
      // request past the last tile, so a launch makes exactly total +
      // gridDim requests: the one that receives the last number is the last
      // request of the launch, and it returns the counter to zero for the
      // next launch (no end-of-kernel counter that every CTA would contend
      // for).
      const uint64_t last_req = (uint64_t)total + gridDim.x - 1u;
      auto request = [&]() {
        const uint32_t v = atomicAdd(p.sched, 1u);
        if ((uint64_t)v == last_req) *p.sched = 0u;
        return v;
      };
      uint32_t next = request();
      while (true) {
        const int64_t g = next;
        if (g >= total) break;
        next = request();
        const int b = (int)(g / p.tiles_per_seq), t = (int)(g % p.tiles_per_seq);
        if (b != cur_b) {
          C = visible_rows(p.n_rows, b, p.max_rows, p.status);
          cur_b = b;
        }
        if (t * SC_TILE >= C - p.tail) continue;
        if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort)) {
          s.abort = 1;
          set_status(p.status, ST_TIMEOUT);
          break;
        }
        s.tile[stage] = (int32_t)g;
        const int pos0 = t * SC_TILE;
        const int32_t y0 = box_row(p, b, pos0);
        const int32_t y1 = pos0 + SC_BOX < C - p.tail ? box_row(p, b, pos0 + SC_BOX) : y0;
        mbar_arrive_expect_tx(&s.full[stage], SC_A_BYTES + Cfg::B_BYTES);
        tma_load_2d_hint(s.a[stage], &map_k, &s.full[stage], 0, y0, stream_once);
        tma_load_2d_hint(s.a[stage] + SC_BOX * 128, &map_k, &s.full[stage], 0, y1, stream_once);
        tma_load_2d(s.b[stage], &map_q, &s.full[stage], 0, (b * p.nq + p.q_first) * CSA2_HI);
        issued |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == SC_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // end of the tiles: a stage that carries no data, only the marker
      if (!*abort) {
        if (mbar_wait(&s.empty[stage], phase ^ 1u, abort)) {
          // this stage's earlier copy has been consumed, so it has landed
          issued &= ~(1u << stage);
          s.tile[stage] = -1;
          mbar_arrive(&s.full[stage]);
        } else {
          s.abort = 1;
          set_status(p.status, ST_TIMEOUT);
        }
      }
      // Drain: every issued copy lands before the CTA may exit.
      for (int i = 0; i < SC_STAGES; i++)
        if ((issued >> i) & 1u)
          if (!mbar_wait(&s.full[i], (issued_phase >> i) & 1u, nullptr))
            set_status(p.status, ST_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------- MMA issuer
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      while (true) {
        if (!mbar_wait(&s.full[stage], phase, abort) ||
            !mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort)) {
          s.abort = 1;
          set_status(p.status, ST_TIMEOUT);
          break;
        }
        const int32_t tile = s.tile[stage];
        s.acc_tile[acc] = tile;
        mbar_arrive(&s.tinfo[acc]);  // the epilogue learns the tile (or the end)
        if (tile < 0) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(s.a[stage]), b_addr = smem_u32(s.b[stage]);
        const uint32_t d = tmem + (uint32_t)(acc * N);
#pragma unroll
        for (int k = 0; k < 4; k++)  // K = 64 as four K = 16 steps inside the swizzle atom
          umma_bf16(d, sdesc_k128(a_addr + 32 * k), sdesc_k128(b_addr + 32 * k), Cfg::IDESC,
                    k > 0);
        umma_commit(&s.empty[stage]);
        umma_commit(&s.tfull[acc]);
        if (++stage == SC_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (++acc == ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      umma_commit(&s.done);  // completes once every MMA issued above has
      if (!mbar_wait(&s.done, 0, nullptr)) set_status(p.status, ST_TIMEOUT);
    }
  } else {  // ------------------------------------------ epilogue, 4 warps
    // Thread = one TMEM lane = one position of the tile.  Query tq's score
    // is the weighted ReLU sum over accumulator columns [8 tq, 8 tq + 8).
    constexpr int QPB = ONE ? 1 : (N / 8 < 4 ? N / 8 : 4);  // queries per batch of TMEM loads
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const int nq = ONE ? 1 : p.nq_pass;  // queries of this launch
    const int nq_all = p.nq, q_first = p.q_first;
    int acc = 0;
    uint32_t acc_phase = 0;
    int cur_b = -1, C = 0, w_b = -1, w_t0 = -1;
    float wr[QPB][CSA2_HI];
    while (true) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s.tinfo[acc], acc_phase, abort))) {
        s.abort = 1;
        set_status(p.status, ST_TIMEOUT);
        break;
      }
      const int64_t g = s.acc_tile[acc];
      if (g < 0) break;
      const int b = (int)(g / p.tiles_per_seq), t = (int)(g % p.tiles_per_seq);
      if (b != cur_b) {
        C = visible_rows(p.n_rows, b, p.max_rows, nullptr);  // the last query's view
        cur_b = b;
        if constexpr (N > 32) {
          float* wq = s.wq + (warp - 2) * (CSA2_SCAN_QUERIES * CSA2_HI);
          __syncwarp();
          for (int i = lane; i < nq * CSA2_HI; i += 32)
            wq[i] = __ldg(p.w + ((int64_t)b * nq_all + q_first) * CSA2_HI + i);
          __syncwarp();
        }
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&s.tfull[acc], acc_phase, abort));
      if (!ok) {
        s.abort = 1;
        set_status(p.status, ST_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * N);
      const int pos = t * SC_TILE + row;
      // this warp's queries: all of them, or its half when 8 warps share a tile
      const int qlo = Cfg::EPI_WARPS == 8 ? 4 * ((warp - 2) >> 2) : 0;
      const int qhi = Cfg::EPI_WARPS == 8 ? min(nq, qlo + 4) : nq;
      bool arrived = false;
      for (int t0 = qlo; t0 < qhi; t0 += QPB) {
        uint32_t r[QPB][8];
#pragma unroll
        for (int qq = 0; qq < QPB; qq++)
          if (t0 + qq < qhi) tmem_ld_x8(tbase + (uint32_t)(8 * (t0 + qq)), r[qq]);
        tmem_ld_wait();
        if (t0 + QPB >= qhi) {  // every load of this warp from the accumulator has completed
          tc_fence_before();
          mbar_arrive(&s.tempty[acc]);
          if constexpr (Cfg::EPI_WARPS == 8) arrived = true;
        }
        if (N <= 32 && (b != w_b || t0 != w_t0)) {  // one batch: weights stay in registers
#pragma unroll
          for (int qq = 0; qq < QPB; qq++)
#pragma unroll
            for (int h = 0; h < CSA2_HI; h++)
              wr[qq][h] = t0 + qq < nq
                              ? __ldg(p.w + ((int64_t)b * nq_all + q_first + t0 + qq) * CSA2_HI + h)
                              : 0.0f;
          w_b = b;
          w_t0 = t0;
        }
        // the QPB queries are independent chains: no early exit, so that
        // they interleave; a query past the launch's last stores nothing
#pragma unroll
        for (int qq = 0; qq < QPB; qq++) {
          const int tq = t0 + qq;
          const bool live = tq < qhi;             // warp-uniform
          const int gq = q_first + tq;            // query index within the sequence
          const int Cq = C - (nq_all - 1 - gq);  // entries that query sees
          float sc = 0.0f;
#pragma unroll
          for (int h = 0; h < CSA2_HI; h++) {
            float wh;
            if constexpr (N > 32)
              wh = s.wq[(warp - 2) * (CSA2_SCAN_QUERIES * CSA2_HI) + tq * CSA2_HI + h];
            else
              wh = wr[qq][h];
            sc = fmaf(wh, fmaxf(__uint_as_float(r[qq][h]), 0.0f), sc);
          }
          if (pos >= Cq) sc = -INFINITY;
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 1));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 2));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 4));
          if (live && (lane & 7) == 0 && pos < Cq)
            p.bm[((int64_t)b * nq_all + gq) * p.bm_stride + pos / CSA2_BLK] = sc;
        }
      }
      if constexpr (Cfg::EPI_WARPS == 8) {
        if (!arrived) {  // a warp with no query of this launch still releases the tile
          tc_fence_before();
          mbar_arrive(&s.tempty[acc]);
        }
      }
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------- rescore + Top-k select
constexpr int RS_GB = 4;      // groups of 16 candidates whose loads a warp keeps in flight
constexpr int RS_EPC = 1024;  // candidates per CTA (threads x candidates per thread)

// Two shapes of the same CTA: 512 threads x 2 candidates when the launch's
// clusters fit on the GPU at once (shorter scoring and counting chains),
// 256 x 4 otherwise (twice the CTAs per SM for many (layer, sequence) jobs).
template <int NT>
struct RescoreSmem {
  SelectSmem<NT, RS_EPC / NT> sel;
  alignas(16) uint32_t keys[RS_EPC];
  int32_t blocks[RS_EPC / CSA2_BLK];
};

__device__ __forceinline__ int64_t pos_row(const RescoreParams& p, int b, int pos) {
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

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Scores this CTA's RS_EPC candidates (positions of blocks[0..RS_EPC/8),
// -1 = none) against one job's indexer query into keys[] (0 = not a
// candidate).  16 candidates per MMA: rows grp and grp + 8 of a group; a warp
// issues the row loads of RS_GB groups before their MMAs, so that several
// gathered rows are in flight per lane.
template <int NT>
__device__ __forceinline__ void score_candidates(const RescoreParams& p, const int32_t* blocks,
                                                 uint32_t* keys, int bp, int C,
                                                 const uint32_t (&bq)[8], float w0, float w1) {
  constexpr int NW = NT / 32;
  constexpr int GPW = RS_EPC / 16 / NW;  // groups per warp
  constexpr int GB = GPW < RS_GB ? GPW : RS_GB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane & 3, grp = lane >> 2;
  for (int gb = 0; gb < GPW; gb += GB) {
    uint32_t av[GB][2][8];
    bool valid[GB][2];
#pragma unroll
    for (int u = 0; u < GB; u++) {
      const int g = warp + NW * (gb + u);
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int e = g * 16 + grp + 8 * h;  // candidate index within this CTA
        const int blk = blocks[e / CSA2_BLK];
        const int pos = blk * CSA2_BLK + (e % CSA2_BLK);
        int64_t row = -1;
        valid[u][h] = blk >= 0 && pos < C;
        if (valid[u][h]) {
          row = pos_row(p, bp, pos);
          if (row < 0) {
            set_status(p.status, ST_DEVICE_CHECK);
            valid[u][h] = false;
          }
        }
        if (row >= 0) {
          const uint4* kp = reinterpret_cast<const uint4*>(p.idx_k + row * CSA2_DI + 16 * c);
          const uint4 k0 = __ldg(kp), k1 = __ldg(kp + 1);
          av[u][h][0] = k0.x; av[u][h][1] = k0.y; av[u][h][2] = k0.z; av[u][h][3] = k0.w;
          av[u][h][4] = k1.x; av[u][h][5] = k1.y; av[u][h][6] = k1.z; av[u][h][7] = k1.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; i++) av[u][h][i] = 0u;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < GB; u++) {
      const int g = warp + NW * (gb + u);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 4; ks++) {
        const uint32_t a[4] = {av[u][0][2 * ks], av[u][1][2 * ks], av[u][0][2 * ks + 1],
                               av[u][1][2 * ks + 1]};
        mma_bf16_16816(d, a, bq[2 * ks], bq[2 * ks + 1]);
      }
      float s0 = fmaf(w1, fmaxf(d[1], 0.f), w0 * fmaxf(d[0], 0.f));
      float s1 = fmaf(w1, fmaxf(d[3], 0.f), w0 * fmaxf(d[2], 0.f));
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (c == 0) {
        keys[g * 16 + grp] = valid[u][0] ? float_key(s0) : 0u;
        keys[g * 16 + grp + 8] = valid[u][1] ? float_key(s1) : 0u;
      }
    }
  }
}

// B fragments of one job's indexer query: head n = lane / 4 (8 heads = MMA
// N), this thread's 16 contiguous channels [16c, 16c + 16) of the 64,
// c = lane % 4.  The K axis is permuted identically for A and B so that each
// thread loads 32 contiguous bytes of a row; a dot product does not depend on
// K order.  The query and weights are inputs: read before the wait.
__device__ __forceinline__ void job_query(const RescoreJob& job, int b, uint32_t (&bq)[8],
                                          float& w0, float& w1) {
  const int lane = threadIdx.x & 31, c = lane & 3, grp = lane >> 2;
  const uint4* qp =
      reinterpret_cast<const uint4*>(job.q_idx + ((int64_t)b * CSA2_HI + grp) * CSA2_DI + 16 * c);
  const uint4 q0 = __ldg(qp), q1 = __ldg(qp + 1);
  bq[0] = q0.x; bq[1] = q0.y; bq[2] = q0.z; bq[3] = q0.w;
  bq[4] = q1.x; bq[5] = q1.y; bq[6] = q1.z; bq[7] = q1.w;
  w0 = __ldg(job.w + b * CSA2_HI + 2 * c);
  w1 = __ldg(job.w + b * CSA2_HI + 2 * c + 1);
}

template <int RS_NT>
__global__ void __launch_bounds__(RS_NT) rescore_select_kernel(const RescoreParams p) {
  constexpr int EPC = RS_EPC;  // candidates per CTA
  constexpr int RS_KPT = RS_EPC / RS_NT;
  using RescoreSmem = csa2::RescoreSmem<RS_NT>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RescoreSmem& s = *reinterpret_cast<RescoreSmem*>(smem_raw);
  pdl_launch_dependents();
  cluster_select_prologue(s.sel);
  const int b = blockIdx.y;
  const RescoreJob job = p.job[blockIdx.z];
  uint32_t bq[8];
  float w0, w1;
  job_query(job, b, bq, w0, w1);
  pdl_wait();  // the candidate blocks come from the previous kernel
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int t = threadIdx.x;
  const int e0 = rank * EPC;  // first candidate of this CTA
  // the candidate blocks are read without waiting for their count (within
  // the list's stride), so both loads are in flight together
  int cblk = -1;
  if (t < EPC / CSA2_BLK && e0 / CSA2_BLK + t < p.cand_stride)
    cblk = p.cand[(int64_t)b * p.cand_stride + e0 / CSA2_BLK + t];
  const int C = visible_query(p.n_rows, b, p.nq, p.max_rows, p.status);
  const int bp = b / p.nq;  // the sequence whose rows the candidates index
  int ncb = p.cand_count[b];
  if (ncb < 0 || ncb > p.cand_stride) {
    set_status(p.status, ST_DEVICE_CHECK);
    ncb = ncb < 0 ? 0 : p.cand_stride;
  }
  static_assert(EPC / CSA2_BLK <= RS_NT, "one candidate block per thread");
  if (t < EPC / CSA2_BLK) s.blocks[t] = e0 / CSA2_BLK + t < ncb ? cblk : -1;
  __syncthreads();
  score_candidates<RS_NT>(p, s.blocks, s.keys, bp, C, bq, w0, w1);
  __syncthreads();

  uint32_t key[RS_KPT];
#pragma unroll
  for (int j = 0; j < RS_KPT; j++) key[j] = s.keys[t * RS_KPT + j];
  const int32_t* blocks = s.blocks;
  auto id_of = [blocks, e0](int e) {  // candidate index -> position
    const int el = e - e0;
    return blocks[el / CSA2_BLK] * CSA2_BLK + (el % CSA2_BLK);
  };
  __syncthreads();
  cluster_select_topk<RS_NT, RS_KPT>(s.sel, key, id_of, p.top_k,
                                     job.idx + (int64_t)b * job.idx_stride, job.idx_count + b,
                                     true, p.status, /*top_window=*/true, /*gather_finish=*/true);
}

// --------------------------------------------- block Top-k (pool) select
constexpr int BS_NT = 1024;
constexpr int BS_KPT = 8;   // 131,072 block maxima (1M positions) over a 16-CTA cluster

__global__ void __launch_bounds__(BS_NT) block_select_kernel(
    const float* __restrict__ bm, int32_t bm_stride, const int32_t* __restrict__ n_rows,
    int32_t max_rows, int32_t nq, int32_t k_req, int32_t* sel, int32_t sel_stride,
    int32_t* sel_count, uint32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelectSmem<BS_NT, BS_KPT>& sm = *reinterpret_cast<SelectSmem<BS_NT, BS_KPT>*>(smem_raw);
  pdl_launch_dependents();
  cluster_select_prologue(sm);
  pdl_wait();  // the block maxima come from the scan
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = blockIdx.y;
  const int e0 = (rank * BS_NT + threadIdx.x) * BS_KPT;
  // the block maxima are read without waiting for the count (within the
  // row's stride, a multiple of 16), so both loads are in flight together
  const float* src = bm + (int64_t)b * bm_stride + e0;
  float4 v[BS_KPT / 4];
#pragma unroll
  for (int j = 0; j < BS_KPT / 4; j++)
    v[j] = e0 + 4 * j < bm_stride ? *reinterpret_cast<const float4*>(src + 4 * j)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  const int C = visible_query(n_rows, b, nq, max_rows, status);
  const int nblk = (C + CSA2_BLK - 1) / CSA2_BLK;
  uint32_t key[BS_KPT];
#pragma unroll
  for (int j = 0; j < BS_KPT / 4; j++) {
    const float f[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int u = 0; u < 4; u++) key[4 * j + u] = (e0 + 4 * j + u < nblk) ? float_key(f[u]) : 0u;
  }
  cluster_select_topk<BS_NT, BS_KPT>(sm, key, [](int e) { return e; }, k_req,
                                     sel + (int64_t)b * sel_stride, sel_count + b, true, status);
}

// ------------------------------------------------------------ launchers
template <int N, int ACC, bool ONE>
static cudaError_t launch_scan_n(const CUtensorMap& map_k, const CUtensorMap& map_q,
                                 const ScanParams& p, int num_sms, cudaStream_t st) {
  using Cfg = ScanCfg<N, ACC>;
  auto kern = score_scan_kernel<N, ACC, ONE>;
  static PerDeviceOnce setup;  // resident CTAs per SM for this instantiation
  int per_sm = 0;
  cudaError_t es = setup.run([&](int& v) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg::SMEM);
    if (e != cudaSuccess) return e;
    // Resident CTAs per SM from the shared memory, registers and TMEM each
    // one takes (the runtime's occupancy calculator reports 1 for kernels
    // that allocate tensor memory, so the limits are applied here).
    int dev = 0, smem_sm = 0, reserved = 0, regs_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    const int warp_regs = (fa.numRegs * 32 + 255) / 256 * 256;
    int n = smem_sm / ((int)Cfg::SMEM + reserved);
    const int by_regs = regs_sm / (warp_regs * (Cfg::THREADS / 32));
    const int by_tmem = 512 / (int)Cfg::TMEM_COLS;
    n = n < by_regs ? n : by_regs;
    n = n < by_tmem ? n : by_tmem;
    if (n < 1) return cudaErrorInvalidConfiguration;
    v = n < SC_CTAS_PER_SM ? n : SC_CTAS_PER_SM;
    return cudaSuccess;
  }, &per_sm);
  if (es != cudaSuccess) return es;
  const int64_t total = (int64_t)p.batch * p.tiles_per_seq;
  const int64_t slots = (int64_t)per_sm * num_sms;
  const int grid = (int)(total < slots ? total : slots);
  if (grid <= 0) return cudaSuccess;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map_k, map_q, p);
}

// Query box rows the scan loads per stage for nq_pass queries of a sequence.
int scan_query_rows(int nq_pass) { return nq_pass <= 2 ? 16 : (nq_pass <= 4 ? 32 : 64); }

cudaError_t launch_scan(const CUtensorMap& map_k, const CUtensorMap& map_q, const ScanParams& p,
                        int num_sms, cudaStream_t st) {
  if (p.nq_pass < 1 || p.nq_pass > CSA2_SCAN_QUERIES || p.q_first < 0 ||
      p.q_first + p.nq_pass > p.nq || p.tail != p.nq - (p.q_first + p.nq_pass))
    return cudaErrorInvalidValue;
  if (p.nq_pass == 1) return launch_scan_n<16, 4, true>(map_k, map_q, p, num_sms, st);
  if (p.nq_pass <= 2) return launch_scan_n<16, 4, false>(map_k, map_q, p, num_sms, st);
  if (p.nq_pass <= 4) return launch_scan_n<32, 4, false>(map_k, map_q, p, num_sms, st);
  return launch_scan_n<64, 2, false>(map_k, map_q, p, num_sms, st);
}

// Candidates per sequence: n_cand_blocks * 8, RS_EPC per CTA of a cluster of
// up to 16 CTAs that scores and selects them together.
template <int NT>
static cudaError_t launch_rescore_nt(const RescoreParams& p, int n_jobs, int batch, int cs,
                                     cudaStream_t st) {
  const size_t smem = sizeof(RescoreSmem<NT>);
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([smem](int&) {
    cudaError_t e = cudaFuncSetAttribute(rescore_select_kernel<NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(rescore_select_kernel<NT>,
                                cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, batch, n_jobs);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, rescore_select_kernel<NT>, p);
}

cudaError_t launch_rescore(const RescoreParams& p, int n_jobs, int batch, int n_cand_blocks,
                           cudaStream_t st) {
  const int ncand = n_cand_blocks * CSA2_BLK;
  int cs = 1;
  while (cs * RS_EPC < ncand) cs <<= 1;
  if (cs > 16) return cudaErrorInvalidValue;
  const int64_t ctas = (int64_t)cs * batch * n_jobs;
  if (ctas <= num_sms()) return launch_rescore_nt<512>(p, n_jobs, batch, cs, st);
  return launch_rescore_nt<256>(p, n_jobs, batch, cs, st);
}

cudaError_t launch_block_select(const float* bm, int bm_stride, const int32_t* n_rows,
                                int max_rows, int batch, int nq, int k_req, int32_t* sel,
                                int sel_stride, int32_t* sel_count, uint32_t* status,
                                cudaStream_t st) {
  const int nblk_max = (max_rows + CSA2_BLK - 1) / CSA2_BLK;
  int cs = (nblk_max + BS_NT * BS_KPT - 1) / (BS_NT * BS_KPT);
  if (cs < 1) cs = 1;
  int c2 = 1;
  while (c2 < cs) c2 <<= 1;
  if (c2 > 16) return cudaErrorInvalidValue;
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([](int&) {
    cudaError_t e = cudaFuncSetAttribute(block_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(SelectSmem<BS_NT, BS_KPT>));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(block_select_kernel,
                                cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c2, batch, 1);
  cfg.blockDim = dim3(BS_NT);
  cfg.dynamicSmemBytes = sizeof(SelectSmem<BS_NT, BS_KPT>);
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = c2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, block_select_kernel, bm, (int32_t)bm_stride, n_rows,
                            (int32_t)max_rows, (int32_t)nq, (int32_t)k_req, sel,
                            (int32_t)sel_stride, sel_count, status);
}

}  // namespace csa2
