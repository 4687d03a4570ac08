// Prefill scorer on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// followed by an exact per-query top-512.
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): in prefill a GPU kernel computes
// the index scores and a fast top-k keeps the best 512 blocks of every query;
// query t sees the complete blocks b < floor((t+1)/4).  Score (stated reading):
// s = sum_h w_h * max(0, q~_h . k^_b); ties keep the lower block index.
//
// Design (B200).  For a causal chunk of queries of one sequence the scores are
// a dense product Q~ K^T with K = 128: 1024 FLOP per (query, block) pair.
// D[b][(t,h)] = k^_b . q~_{t,h} is computed with tcgen05.mma (cta_group::1,
// kind::f16, bf16 in / fp32 out): M = 128 compressed keys (A, streamed by TMA
// from the paged cache through a ring of stages), N = 256 = 64 queries x 4
// heads (B, the rotated queries of one work tile, resident in shared memory),
// accumulators double-buffered in TMEM (2 x 256 of the 512 columns).  Keys on
// the M side put the 4 heads of one (block, query) pair in 4 adjacent TMEM
// columns of one lane, so one thread combines them without shuffles.
//
// Warp roles (one CTA per SM, persistent): warp 0 issues TMA, warp 1 owns TMEM
// and issues the MMAs (one elected thread), the other warps are the epilogue:
// each reads its 32-lane TMEM quadrant (32 blocks) for a group of queries,
// combines the heads and writes the score of every visible (query, block) pair
// as an order-preserving 32-bit key, 32 consecutive blocks of one query per
// warp store (one 128-byte line).  Writing every score costs the same HBM
// bytes as a filtered candidate list (key + block id) of the usual size, and
// keeps the epilogue to a few instructions per score so that it hides under
// the MMAs.  Work tiles are ordered longest first (causal imbalance) and dealt
// to CTAs in a snake.
//
// Selection (k_prefill_select): one warp per query row, longest rows first:
// a lower bound from a sample of the row's keys, one pass collecting the keys
// at or above it, the exact cut among those (score desc, block asc), and the
// kept blocks written in ascending order.  Rows that do not fit that path
// (longer than 8192 blocks, heavy ties, a bound that keeps too few or too
// many) go to k_prefill_select_overflow: an exact CTA-wide selection.
#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int PF_QT = 64;              // queries per work tile
constexpr int PF_N = PF_QT * HI;       // 256 MMA columns
constexpr int PF_M = 128;              // compressed keys per M-tile
#ifndef QSA_PF_STAGES
#define QSA_PF_STAGES 3
#endif
#ifndef QSA_PF_EPI_WARPS
#define QSA_PF_EPI_WARPS 16
#endif
constexpr int PF_STAGES = QSA_PF_STAGES;       // A ring depth
constexpr int PF_EPI_WARPS = QSA_PF_EPI_WARPS;  // 8 or 16
constexpr int PF_THREADS = (2 + PF_EPI_WARPS) * 32;
constexpr int PF_QPW = PF_QT * 4 / PF_EPI_WARPS;  // queries per epilogue warp (32 or 16)
constexpr int PF_A_BYTES = PF_M * D * 2;  // 32 KiB
constexpr int PF_B_BYTES = PF_N * D * 2;  // 64 KiB
constexpr uint32_t PF_TMEM_COLS = 512;
static_assert(PF_EPI_WARPS % 4 == 0 && PF_QPW % 8 == 0, "epilogue warps cover the four TMEM quadrants evenly");

struct __align__(1024) PfSmem {
  uint8_t a[PF_STAGES][2][PF_A_BYTES / 2];  // [stage][K half][128 rows x 128 B], 128B-swizzled
  uint8_t b[2][PF_B_BYTES / 2];              // [K half][256 rows x 128 B]
  float4 w[2][PF_QT];                        // halved head weights of the work tile's queries (by tile parity)
  uint64_t full_a[PF_STAGES], empty_a[PF_STAGES], full_b, empty_b, tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;  // set by the first role whose wait gives up: every role then stops issuing work
};

// Wait of one role: bounded, and it stops as soon as any role of the CTA has given up, so that one
// barrier that never completes ends the whole CTA instead of costing a full limit per later wait.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, int* err, uint64_t limit_ns,
                                        volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!*abort) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      set_error(err, QSA_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
  return false;
}

// Phases armed (or committed) on stage s of a ring after `n` uses in round-robin order.
__device__ __forceinline__ int ring_uses(int n, int s, int stages) { return n / stages + (s < n % stages ? 1 : 0); }

// ---- tcgen05 / TMEM wrappers ----
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; completes at the next tc_wait_ld.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Ties the registers of a tc_ld32 to a point after tc_wait_ld, so no use of
// them is scheduled before the wait.
__device__ __forceinline__ void tc_after_wait(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// K-major operand in 128-byte-swizzled rows of 128 B (8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t pf_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PF_N >> 3) << 17) | ((uint32_t)(PF_M >> 4) << 24);
}

// ---- work schedule: tiles longest first, dealt in a snake ----
struct PfSched {
  int ntiles, grid, pos0, T;
  __device__ int tile_at(int k) const {  // k-th tile in descending cost order
    return ntiles - 1 - k;
  }
  // j-th tile of CTA c, or -1
  __device__ int nth(int c, int j) const {
    const int k = j * grid + ((j & 1) ? (grid - 1 - c) : c);
    return k < ntiles ? tile_at(k) : -1;
  }
  __device__ int nbv_of(int t) const { return (pos0 + t + 1) >> 2; }
  __device__ int mtiles(int qt) const {  // M-tiles of a work tile (0: every query keeps all its blocks)
    const int tl = min(T, (qt + 1) * PF_QT) - 1;
    const int nb = nbv_of(tl);
    return nb <= TOPK ? 0 : ceil_div(nb, PF_M);
  }
};

__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill_score(PrefillParams p, const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap) {
  extern __shared__ uint8_t smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>(smem_aligned<1024>(smem_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  PfSched sch{ceil_div(p.T, PF_QT), (int)gridDim.x, p.pos0, p.T};
  const uint64_t lim = p.wait_ns ? p.wait_ns : WAIT_LIMIT_NS;
  volatile int* abort = &S.abort;

  if (tid == 0) {
    S.abort = 0;
    for (int s = 0; s < PF_STAGES; ++s) {
      mbar_init(&S.full_a[s], 1);
      mbar_init(&S.empty_a[s], 1);
    }
    mbar_init(&S.full_b, 1);
    mbar_init(&S.empty_b, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.tfull[i], 1);
      mbar_init(&S.tempty[i], PF_EPI_WARPS);
    }
    fence_mbar_init();
  }
  if (warp == 1) {  // TMEM: the whole warp allocates all 512 columns (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(PF_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // =============================== TMA producer ===============================
    // The whole warp walks the schedule: lane i fetches the physical page of
    // logical page 32g + i for the group g of four M-tiles (32 pages) ahead of
    // use, so no page-table load sits on the path of a copy; lane 0 waits for
    // the stage and expects its bytes, then 16 lanes issue one copy each.
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
    }
    const int32_t* pt = p.c.page_table + (int64_t)p.req * p.c.max_pages;
    const int oob_row = (int)(p.c.num_pages * PAGE_BLOCKS);  // a row past the cache: TMA fills zeros
    constexpr int GROUP = 32 / (PF_M / PAGE_BLOCKS);         // M-tiles per page group (4)
    auto page_row = [&](int lp, int nbv_hi) {                // lane's page -> first cache row
      int row = oob_row;
      if (lp < p.c.max_pages) {
        const int phys = __ldg(pt + lp);
        if (phys >= 0 && phys < p.c.num_pages) row = phys * PAGE_BLOCKS;
        else if (lp * PAGE_BLOCKS < nbv_hi) set_error(p.err, QSA_DEVERR_PAGE);
      }
      return row;
    };
    int a_it = 0, wt = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      const int qt = sch.nth(blockIdx.x, j);
      if (qt < 0) break;
      const int nm = sch.mtiles(qt);
      if (nm == 0) continue;
      const int nbv_hi = sch.nbv_of(min(p.T, (qt + 1) * PF_QT) - 1);
      int go = 1;
      if (lane == 0) {
        go = wt == 0 || pf_wait(&S.empty_b, (wt - 1) & 1, p.err, lim, abort);
        if (go) {
          mbar_arrive_expect_tx(&S.full_b, PF_B_BYTES);
          tma_load_2d(S.b[0], &qmap, 0, qt * PF_N, &S.full_b);
          tma_load_2d(S.b[1], &qmap, 64, qt * PF_N, &S.full_b);
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      ++wt;
      int rows_cur = page_row(lane, nbv_hi), rows_nxt = oob_row;
      for (int mt = 0; mt < nm; ++mt, ++a_it) {
        const int g = mt / GROUP, r = mt % GROUP;
        if (r == 0 && (g + 1) * GROUP < nm) rows_nxt = page_row((g + 1) * 32 + lane, nbv_hi);
        const int s = a_it % PF_STAGES;
        if (lane == 0) {
          go = a_it < PF_STAGES || pf_wait(&S.empty_a[s], ((a_it / PF_STAGES) - 1) & 1, p.err, lim, abort);
          if (go) mbar_arrive_expect_tx(&S.full_a[s], PF_A_BYTES);
        }
        // the stage is free (and its bytes expected) before any lane copies into it
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        // 16 lanes issue the M-tile's 16 copies at once: lane 2*pg + half copies the 64-dim half
        // `half` of page pg (16 keys)
        constexpr int PAGES = PF_M / PAGE_BLOCKS;  // 8 pages per M-tile
        const int pg = (lane >> 1) & (PAGES - 1), half = lane & 1;
        const int row = __shfl_sync(0xffffffffu, rows_cur, r * PAGES + pg);
        if (lane < 2 * PAGES)
          tma_load_2d(S.a[s][half] + pg * PAGE_BLOCKS * 128, &kmap, half * 64, row, &S.full_a[s]);
        if (r == GROUP - 1) rows_cur = rows_nxt;
      }
    }
    // drain: every copy issued above has landed before the CTA may exit (in the normal case these
    // phases completed long ago and the waits return at once)
    if (lane == 0) {
      if (wt > 0) mbar_wait(&S.full_b, (wt - 1) & 1, p.err, lim);
      for (int s = 0; s < PF_STAGES; ++s) {
        const int uses = ring_uses(a_it, s, PF_STAGES);
        if (uses > 0) mbar_wait(&S.full_a[s], (uses - 1) & 1, p.err, lim);
      }
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      const uint32_t idesc = pf_idesc();
      int a_it = 0, m_it = 0, wt = 0, b_commits = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int qt = sch.nth(blockIdx.x, j);
        if (qt < 0) break;
        const int nm = sch.mtiles(qt);
        if (nm == 0) continue;
        if (!pf_wait(&S.full_b, wt & 1, p.err, lim, abort)) break;
        ++wt;
        for (int mt = 0; mt < nm; ++mt, ++a_it, ++m_it) {
          const int s = a_it % PF_STAGES;
          const int buf = m_it & 1;
          if (!pf_wait(&S.full_a[s], (a_it / PF_STAGES) & 1, p.err, lim, abort) ||
              (m_it >= 2 && !pf_wait(&S.tempty[buf], ((m_it >> 1) - 1) & 1, p.err, lim, abort))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(buf * PF_N);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)((kk & 3) * 32);
            const uint64_t ad = smem_desc_sw128(smem_u32(S.a[s][kk >> 2]) + off);
            const uint64_t bd = smem_desc_sw128(smem_u32(S.b[kk >> 2]) + off);
            tc_mma(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(&S.empty_a[s]);
          tc_commit(&S.tfull[buf]);
        }
        tc_commit(&S.empty_b);
        ++b_commits;
      }
      // tail: every commit issued above has arrived (its MMAs are done) before the CTA may exit
      if (b_commits > 0) mbar_wait(&S.empty_b, (b_commits - 1) & 1, p.err, lim);
      for (int s = 0; s < PF_STAGES; ++s) {
        const int uses = ring_uses(a_it, s, PF_STAGES);
        if (uses > 0) mbar_wait(&S.empty_a[s], (uses - 1) & 1, p.err, lim);
      }
    }
  } else {
    // =============================== epilogue ===============================
    const int e = warp - 2;           // 0 .. PF_EPI_WARPS-1
    const int quad = warp & 3;        // TMEM lanes 32*quad .. +31 = blocks of the M-tile
    const int qg = e >> 2;            // query group: queries qg*PF_QPW .. +PF_QPW-1 of the tile
    const int etid = tid - 64;        // 0 .. 32*PF_EPI_WARPS-1
    const int nmax = p.cap / PF_M;    // M-tile slots per work tile in the score array
    int m_it = 0, wt = 0;
    for (int j = 0;; ++j) {
      const int qt = sch.nth(blockIdx.x, j);
      if (qt < 0) break;
      const int nm = sch.mtiles(qt);
      if (nm == 0) continue;
      const int par = wt & 1;
      ++wt;
      // this tile's head weights, halved (see below); the other parity's copy
      // may still be read by warps finishing the previous tile, so a barrier
      // is needed only after writing
      if (etid < PF_QT) {
        const int t = qt * PF_QT + etid;
        float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < p.T) w4 = __ldg(reinterpret_cast<const float4*>(p.w) + t);
        S.w[par][etid] = make_float4(0.5f * w4.x, 0.5f * w4.y, 0.5f * w4.z, 0.5f * w4.w);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(PF_EPI_WARPS * 32) : "memory");
      const float4* wq = &S.w[par][qg * PF_QPW];
      // score-key tile (qt, mt): [64 queries][128 blocks]; this thread writes column quad*32+lane
      uint32_t* col = p.keys + (int64_t)qt * nmax * (PF_QT * PF_M) + qg * PF_QPW * PF_M + quad * 32 + lane;

      for (int mt = 0; mt < nm; ++mt, ++m_it) {
        const int buf = m_it & 1;
        // after a timeout anywhere in the CTA the loops still run to their end (no work, no waits), so
        // that every epilogue warp meets the same named barriers
        if (!pf_wait(&S.tfull[buf], (m_it >> 1) & 1, p.err, lim, abort)) continue;
        tc_fence_after();
        uint32_t r[PF_QPW / 8][32];
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * PF_N + qg * PF_QPW * 4);
#pragma unroll
        for (int g = 0; g < PF_QPW / 8; ++g) tc_ld32(taddr + 32u * g, r[g]);
        tc_wait_ld();
#pragma unroll
        for (int g = 0; g < PF_QPW / 8; ++g) tc_after_wait(r[g]);
        // the accumulators are in registers: hand the TMEM buffer back at once
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.tempty[buf]);

        // w * max(x, 0) == (w/2) * (x + |x|) exactly (doubling and halving are
        // exact), which keeps the ReLU on the FMA pipe.  Every column of the
        // tile is written: the blocks past a query's visible range are never
        // read back.
        uint32_t* out = col + (int64_t)mt * (PF_QT * PF_M);
#pragma unroll
        for (int jl = 0; jl < PF_QPW; ++jl) {
          const float4 w4 = wq[jl];
          const uint32_t* rr = &r[jl >> 3][4 * (jl & 7)];
          const float x0 = __uint_as_float(rr[0]), x1 = __uint_as_float(rr[1]);
          const float x2 = __uint_as_float(rr[2]), x3 = __uint_as_float(rr[3]);
          float sc = fmaf(w4.x, x0 + fabsf(x0), 0.f);
          sc = fmaf(w4.y, x1 + fabsf(x1), sc);
          sc = fmaf(w4.z, x2 + fabsf(x2), sc);
          sc = fmaf(w4.w, x3 + fabsf(x3), sc) + 0.f;  // + 0: an underflowed -0 becomes +0
          const uint32_t u = __float_as_uint(sc);
          out[jl * PF_M] = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);  // order-preserving key
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(PF_TMEM_COLS));
  }
}

// ----------------------------------------------------------------------------
// Selection: one warp per query row, longest rows first.  Row t's keys are the
// 128-key chunks (t & 63) of its work tile's M-tiles, 32 KiB apart; a chunk is
// one 16-byte load per lane (lane l: blocks 4l .. 4l+3).
//
// (1) A bound L below the cut: rows of at most PW_ALL_N blocks take L = 0.
//     Longer rows sample every 8th chunk; L is the smallest sample key in
//     the bin (256 bins linear in the score) that holds the sample's R-th
//     largest key, R set for about 1.5 x 512 row keys at or above L.
// (2) One streaming pass appends every key >= L (with its block) to
//     lane-private lists; a lane keeps its blocks in ascending order.
// (3) The exact cut (key T, block I of the 512th element in (key desc, block
//     asc) order) is found on the lists: a histogram of the list's scores
//     (256 linear bins) gives the bin holding the cut, and that bin's few keys are
//     ranked among themselves.
// (4) The kept list entries set their bits in a block bitmap, which is
//     written out in ascending order.
// A row that does not fit (a lane list overflows, fewer than 512 keys reach
// L, heavily tied keys, or a row longer than PW_FAST_N) goes to the overflow
// list, which k_prefill_select_overflow resolves with a CTA-wide exact
// selection.
// ----------------------------------------------------------------------------
#ifndef QSA_PW_WARPS
#define QSA_PW_WARPS 4
#endif
#ifndef QSA_PW_UNROLL
#define QSA_PW_UNROLL 8
#endif
constexpr int PW_WARPS = QSA_PW_WARPS;    // rows in flight per CTA
constexpr int PW_UNROLL = QSA_PW_UNROLL;  // chunks loaded back to back
constexpr int PW_LIST = 48;               // list entries per lane
constexpr int PW_FAST_N = 8192;           // longer rows take the CTA-wide path
constexpr int PW_ALL_N = PW_LIST * 32;    // rows this short keep every key as a candidate
constexpr int PW_SAMPLE = 8;              // sample chunks at most (every 8th of <= 64)
constexpr int PW_BINS = 256;
constexpr int PW_L3 = 64;

struct __align__(16) PwWarp {
  uint32_t lkey[(PW_LIST + 1) * 32];  // [slot][lane]; slot PW_LIST is a spare for writes past a full list
  uint16_t lidx[(PW_LIST + 1) * 32];
  uint32_t hist[PW_BINS];
  uint32_t bitmap[PW_FAST_N / 32];
  uint32_t k3[PW_L3];
  int i3[PW_L3];
};

// Bin D of hist[0..256) counted from the top: count(> D) < k <= count(>= D);
// `above` = count(> D).  Returns false when the histogram holds fewer than k.
__device__ __forceinline__ bool pw_top_bin(const uint32_t* hist, int k, int& D, int& above) {
  const int lane = threadIdx.x & 31;
  const int lo = PW_BINS - 8 * (lane + 1);
  const uint4 h0 = *reinterpret_cast<const uint4*>(hist + lo);
  const uint4 h1 = *reinterpret_cast<const uint4*>(hist + lo + 4);
  const int local = (int)(h0.x + h0.y + h0.z + h0.w + h1.x + h1.y + h1.z + h1.w);
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, x - local < k && x >= k);
  if (!hit) return false;
  const int L = __ffs(hit) - 1;
  int c = __shfl_sync(0xffffffffu, x - local, L);
  const int topL = PW_BINS - 1 - 8 * L;
  int d = topL - 7;
  for (int i = 0; i < 8; ++i) {
    const int h = (int)hist[topL - i];
    if (c + h >= k) {
      d = topL - i;
      break;
    }
    c += h;
  }
  D = d;
  above = c;
  return true;
}

// Bins linear in the score between the scores of keys kmin and kmax.
// Monotone in the key: decoding, subtraction, scaling by a positive factor
// and truncation all preserve order.
struct PwBins {
  float smin, scale;
  __device__ int operator()(uint32_t k) const { return min(PW_BINS - 1, (int)((key_score(k) - smin) * scale)); }
};

__device__ __forceinline__ PwBins pw_bins(uint32_t kmin, uint32_t kmax) {
  PwBins b;
  b.smin = key_score(kmin);
  const float span = key_score(kmax) - b.smin;
  b.scale = span > 0.f && span < 3.0e38f ? (float)PW_BINS / (span * 1.0001f) : 0.f;
  return b;
}

__device__ __forceinline__ void pw_zero(uint32_t* a, int words) {  // words: a multiple of 4
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < words / 4; i += 32) reinterpret_cast<uint4*>(a)[i] = make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(PW_WARPS * 32) k_prefill_select(PrefillParams p) {
  extern __shared__ uint8_t pw_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  PwWarp& W = reinterpret_cast<PwWarp*>(pw_raw)[warp];
  const int nmax = p.cap / PF_M;
  const uint32_t lt = (1u << lane) - 1u;
  const int gw = blockIdx.x * PW_WARPS + warp, nw = gridDim.x * PW_WARPS;
  for (int k = gw; k < p.T; k += nw) {
    const int t = p.T - 1 - k;
    const int n = (p.pos0 + t + 1) >> 2;
    int32_t* sel = p.sel + (int64_t)t * TOPK;
    __syncwarp();  // the previous row's shared data is no longer read
    if (n <= TOPK) {
      for (int i = lane; i < n; i += 32) sel[i] = i;
      if (lane == 0) p.sel_n[t] = n;
      continue;
    }
    bool overflow = n > PW_FAST_N;
    if (!overflow) {
      const uint32_t* row = p.keys + ((int64_t)(t >> 6) * nmax * PF_QT + (t & 63)) * PF_M + 4 * lane;
      auto chunk = [&](int c) { return __ldcg(reinterpret_cast<const uint4*>(row + (int64_t)c * (PF_QT * PF_M))); };
      const int nch = ceil_div(n, PF_M);
      // ---- (1) the bound L ----
      uint32_t L = 0u;
      if (n > PW_ALL_N) {
        const int ns_ch = max(2, nch / 8);
        uint32_t sk[PW_SAMPLE][4];
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
        for (int i = 0; i < PW_SAMPLE; ++i) {
          const int c = (i * nch) / ns_ch;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (i < ns_ch) v = chunk(c);
          const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool valid = i < ns_ch && c * PF_M + 4 * lane + e < n;
            sk[i][e] = kk[e];
            if (valid) {
              mn = min(mn, kk[e]);
              mx = max(mx, kk[e]);
            }
          }
        }
        mn = __reduce_min_sync(0xffffffffu, mn);
        mx = __reduce_max_sync(0xffffffffu, mx);
        const PwBins bin = pw_bins(mn, mx);
        pw_zero(W.hist, PW_BINS);
        __syncwarp();
        int ns = 0;
#pragma unroll
        for (int i = 0; i < PW_SAMPLE; ++i) {
          const int c = (i * nch) / ns_ch;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (i < ns_ch && c * PF_M + 4 * lane + e < n) {
              atomicAdd(&W.hist[bin(sk[i][e])], 1u);
              ++ns;
            }
          }
        }
        ns = __reduce_add_sync(0xffffffffu, ns);
        __syncwarp();
        const int R = min(ns, (3 * TOPK / 2 * ns) / n + 8);
        int Ds = 0, as = 0;
        if (pw_top_bin(W.hist, R, Ds, as)) {
          uint32_t lm = 0xFFFFFFFFu;
#pragma unroll
          for (int i = 0; i < PW_SAMPLE; ++i) {
            const int c = (i * nch) / ns_ch;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (i < ns_ch && c * PF_M + 4 * lane + e < n && bin(sk[i][e]) >= Ds) lm = min(lm, sk[i][e]);
          }
          L = __reduce_min_sync(0xffffffffu, lm);
        }
      }
      // ---- (2) candidates: every key >= L ----
      int lc = 0;
      const int nfull = n / PF_M;
      for (int c0 = 0; c0 < nch; c0 += PW_UNROLL) {
        uint4 v[PW_UNROLL];
#pragma unroll
        for (int u = 0; u < PW_UNROLL; ++u)
          if (c0 + u < nch) v[u] = chunk(c0 + u);
#pragma unroll
        for (int u = 0; u < PW_UNROLL; ++u) {
          const int c = c0 + u;
          if (c >= nch) break;
          const int b0 = c * PF_M + 4 * lane;
          const uint32_t kk[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          // branch-free: every key is written to the lane's next slot, which advances only for a
          // key >= L; past a full list the writes go to a spare slot (the row then overflows)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int slot = min(lc, PW_LIST) * 32 + lane;
            W.lkey[slot] = kk[e];
            W.lidx[slot] = (uint16_t)(b0 + e);
            lc += (kk[e] >= L && (c < nfull || b0 + e < n)) ? 1 : 0;
          }
        }
      }
      const int ln = __reduce_add_sync(0xffffffffu, (unsigned)lc);
      overflow = __any_sync(0xffffffffu, lc > PW_LIST) || ln < TOPK;
      if (!overflow) {
        __syncwarp();
        // ---- (3) the cut ----
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
        for (int j = 0; j < lc; ++j) {
          const uint32_t kk = W.lkey[j * 32 + lane];
          mn = min(mn, kk);
          mx = max(mx, kk);
        }
        mn = __reduce_min_sync(0xffffffffu, mn);
        mx = __reduce_max_sync(0xffffffffu, mx);
        const PwBins bin = pw_bins(mn, mx);
        pw_zero(W.hist, PW_BINS);
        __syncwarp();
        for (int j = 0; j < lc; ++j) atomicAdd(&W.hist[bin(W.lkey[j * 32 + lane])], 1u);
        __syncwarp();
        int D = 0, above = 0;
        bool ok = pw_top_bin(W.hist, TOPK, D, above);
        const int need = TOPK - above;
        int n3 = 0;
        const int lmax = __reduce_max_sync(0xffffffffu, (unsigned)lc);
        for (int j = 0; j < lmax; ++j) {
          const bool have = j < lc;
          const uint32_t kk = have ? W.lkey[j * 32 + lane] : 0u;
          const bool in = have && bin(kk) == D;
          const uint32_t mm = __ballot_sync(0xffffffffu, in);
          const int slot = n3 + __popc(mm & lt);
          if (in && slot < PW_L3) {
            W.k3[slot] = kk;
            W.i3[slot] = W.lidx[j * 32 + lane];
          }
          n3 += __popc(mm);
        }
        __syncwarp();
        overflow = !ok || n3 > PW_L3 || need < 1 || need > n3;
        if (!overflow) {
          uint32_t T = 0u;
          int I = -1;
          for (int j0 = 0; j0 < n3; j0 += 32) {
            const int j = j0 + lane;
            bool hit = false;
            uint32_t kj = 0u;
            int ij = 0;
            if (j < n3) {
              kj = W.k3[j];
              ij = W.i3[j];
              int rank = 0;
              for (int q = 0; q < n3; ++q) {
                const uint32_t kq = W.k3[q];
                rank += (kq > kj) || (kq == kj && W.i3[q] < ij);
              }
              hit = rank == need - 1;
            }
            const uint32_t hm = __ballot_sync(0xffffffffu, hit);
            if (hm) {
              const int src = __ffs(hm) - 1;
              T = __shfl_sync(0xffffffffu, kj, src);
              I = __shfl_sync(0xffffffffu, ij, src);
            }
          }
          // ---- (4) bitmap of the kept blocks, written out in order ----
          const int words = ceil_div(n, 128) * 4;
          pw_zero(W.bitmap, words);
          __syncwarp();
          for (int j = 0; j < lc; ++j) {
            const uint32_t kk = W.lkey[j * 32 + lane];
            const int b = W.lidx[j * 32 + lane];
            if (kk > T || (kk == T && b <= I)) atomicOr(&W.bitmap[b >> 5], 1u << (b & 31));
          }
          __syncwarp();
          int out = 0;
          for (int w0 = 0; w0 < words; w0 += 32) {
            const int wi = w0 + lane;
            uint32_t bits = wi < words ? W.bitmap[wi] : 0u;
            const int cn = __popc(bits);
            int x = cn;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(0xffffffffu, x, o);
              if (lane >= o) x += y;
            }
            int o = out + x - cn;
            while (bits) {
              const int bit = __ffs(bits) - 1;
              bits &= bits - 1u;
              if (o < TOPK) sel[o] = wi * 32 + bit;
              ++o;
            }
            out += __shfl_sync(0xffffffffu, x, 31);
          }
          if (lane == 0) {
            if (out != TOPK) set_error(p.err, QSA_DEVERR_SELECTION);
            p.sel_n[t] = min(out, TOPK);
          }
        }
      }
    }
    if (overflow && lane == 0) {
      const int slot = atomicAdd(p.ovf_n, 1);
      p.ovf_list[slot] = t;
    }
  }
}

// Overflow rows: exact CTA-wide selection over the row's keys in L2.
__global__ void __launch_bounds__(256) k_prefill_select_overflow(PrefillParams p) {
  __shared__ FastTopScratch fs;
  using All = Group<256, 0>;
  const int nmax = p.cap / PF_M;
  const int nov = *p.ovf_n;
  for (int o = blockIdx.x; o < nov; o += gridDim.x) {
    const int t = p.ovf_list[o];
    const int n = (p.pos0 + t + 1) >> 2;
    const uint32_t* row = p.keys + ((int64_t)(t >> 6) * nmax * PF_QT + (t & 63)) * PF_M;
    int32_t* sel = p.sel + (int64_t)t * TOPK;
    auto key_at = [&](int i) { return __ldcg(row + (int64_t)(i >> 7) * (PF_QT * PF_M) + (i & (PF_M - 1))); };
    fast_topk<All>(key_at, n, TOPK, [&](int i, int out) { sel[out] = i; }, &fs);
    if (threadIdx.x == 0) p.sel_n[t] = TOPK;
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// Rotation of the chunk's index queries (bf16, [T*4][128] rows for TMA).
// ----------------------------------------------------------------------------
// One warp per query: lane i owns the rotation pairs (i, i+64) and (i+32, i+96)
// of all four heads; the angles pos * inv_freq_i are taken once per query in
// FP64 and each rotated value is rounded once to bf16.
constexpr int PR_WARPS = 8;

__global__ void __launch_bounds__(PR_WARPS * 32) k_prefill_rotate(PrefillParams p, const __nv_bfloat16* __restrict__ idx_q,
                                                                 RopeFreqs fr) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * PR_WARPS + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const double pos = (double)(p.pos0 + t);
  double sn[2], cs[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) sincos(pos * fr.f[lane + 32 * e], &sn[e], &cs[e]);
  const uint16_t* qin = reinterpret_cast<const uint16_t*>(idx_q + (int64_t)t * HI * D);
  uint16_t* qo = reinterpret_cast<uint16_t*>(p.qrot + (int64_t)t * HI * D);
#pragma unroll
  for (int h = 0; h < HI; ++h) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = h * D + lane + 32 * e;
      const double x0 = (double)bf16_bits_to_f32(__ldg(qin + i));
      const double x1 = (double)bf16_bits_to_f32(__ldg(qin + i + D / 2));
      qo[i] = f64_to_bf16_bits(x0 * cs[e] - x1 * sn[e]);
      qo[i + D / 2] = f64_to_bf16_bits(x0 * sn[e] + x1 * cs[e]);
    }
  }
}

// ---- host side ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor [rows][128], boxes of 64 columns x box_rows rows, 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill(const PrefillParams& p, const __nv_bfloat16* idx_q, const RopeFreqs& fr, int num_sms,
                           cudaStream_t st, const cudaEvent_t* ev, int n_ev) {
  auto mark = [&](int i) {
    if (ev && i < 2 * n_ev) cudaEventRecord(ev[i], st);
  };
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(PfSmem) + 1024;
  const size_t pw_smem = sizeof(PwWarp) * PW_WARPS;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_prefill_score, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_prefill_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pw_smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (p.cap % PF_M != 0) return cudaErrorInvalidValue;  // whole M-tile slots per work tile
  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, p.c.cidx, (uint64_t)p.c.num_pages * PAGE_BLOCKS, PAGE_BLOCKS)) return cudaErrorInvalidValue;
  if (!make_map(&qmap, p.qrot, (uint64_t)p.T * HI, PF_N)) return cudaErrorInvalidValue;
  mark(0);
  k_prefill_rotate<<<ceil_div(p.T, PR_WARPS), PR_WARPS * 32, 0, st>>>(p, idx_q, fr);
  mark(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(p.T, PF_QT);
  mark(2);
  k_prefill_score<<<std::min(num_sms, tiles), PF_THREADS, smem, st>>>(p, kmap, qmap);
  mark(3);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  mark(4);
  if ((e = cudaMemsetAsync(p.ovf_n, 0, sizeof(int), st)) != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_prefill_select, PW_WARPS * 32, pw_smem)) !=
      cudaSuccess)
    return e;
  k_prefill_select<<<std::min(ceil_div(p.T, PW_WARPS), std::max(1, per_sm) * num_sms), PW_WARPS * 32, pw_smem, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_prefill_select_overflow<<<std::min(p.T, 2 * num_sms), 256, 0, st>>>(p);
  mark(5);
  return cudaGetLastError();
}

}  // namespace qsa
