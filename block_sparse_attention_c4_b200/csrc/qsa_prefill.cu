// Prefill scoring of a causal chunk on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), with the exact per-query top-512 taken from a
// filtered candidate list instead of from every score.
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
// columns of one lane, so one thread combines them without shuffles.  Warp
// roles (one CTA per SM, persistent): warp 0 issues TMA, warp 1 owns TMEM and
// issues the MMAs, 16 epilogue warps read the accumulators.  Work tiles are
// ordered longest first (causal imbalance) and dealt to CTAs in a snake.
//
// Short contexts: a work tile whose queries see at most PF_DENSE_MAX (8192)
// blocks writes every score key (4 bytes per pair, 128 coalesced bytes per
// warp and query) and k_prefill_select reads them all: there a threshold would
// pass a quarter or more of each query's blocks, and emitting candidates costs
// the epilogue more instructions than the keys cost bytes.
//
// Longer contexts: scores never go to memory as a whole.  Per work tile the
// M-tiles run in two phases:
//   (1) sample: every 8th M-tile of the tile's visible range (a stratified
//       sample, 1/8 of the blocks) fills, per query, a log-scale histogram of
//       its score keys in shared memory (1/16 octave per bin, the range fixed
//       per query by an upper bound of its scores from the rotation kernel).
//       From it each query gets a threshold tau expected to pass about
//       2 x 512 of its blocks;
//   (2) main: every M-tile (the sampled ones again); a score key >= tau is
//       written as a candidate (key << 32 | ~block, so a larger word ranks
//       first under (score desc, block asc)) to the query's list for the TMEM
//       quadrant of the block; each epilogue warp owns its lists' counters.
// Exactness does not rest on the sample: if a query's candidates number at
// least 512, its top-512 is among them (every block below tau has 512 blocks
// at or above it, ties at tau included), and k_prefill_select takes the exact
// cut among the candidates.  A query whose lists hold fewer than 512 or
// overflowed (an unlucky sample, heavily tied scores) is re-scored in full by
// k_prefill_rescore (mma.sync over its pages, exact radix top-k).  Queries
// with at most PF_EMIT_ALL blocks skip the sample and emit every block.
#include <cmath>
#include <mutex>
#include <type_traits>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int PF_QT = 64;              // queries per work tile
static_assert(PF_QT == 64, "pf_tile_nbv_hi counts 64 queries per work tile");
constexpr int PF_N = PF_QT * HI;       // 256 MMA columns
constexpr int PF_M = 128;              // compressed keys per M-tile
constexpr int PF_STAGES = 3;           // A ring depth
// Epilogue warps: 16 (576 threads; two of the SM's four register-file quarters hold five warps, so
// at most 96 registers per thread) for calls with candidate tiles, 8 (320 threads, up to 168
// registers) when every work tile writes dense keys: there the wider warps carry 32 queries each
// without spilling and the 32K chunk scores faster, while candidate emission needs the 16.
constexpr int PF_EPI_WARPS_CAND = 16;
constexpr int PF_EPI_WARPS_DENSE = 8;
template <int EW>
constexpr int pf_threads() { return (2 + EW) * 32; }
constexpr int PF_A_BYTES = PF_M * D * 2;  // 32 KiB
constexpr int PF_B_BYTES = PF_N * D * 2;  // 64 KiB
constexpr uint32_t PF_TMEM_COLS = 512;
constexpr int PF_PAGES = PF_M / PAGE_BLOCKS;  // 8 pages per M-tile
constexpr int PF_SAMPLE = 8;              // one M-tile in PF_SAMPLE is scored first, as the sample
constexpr float PF_SAMPLE_KEEP = 0.5f;    // tau passes about 512 / PF_SAMPLE_KEEP blocks
constexpr int PF_BINS = 128;              // histogram bins per query: 8 octaves below the bound
constexpr int PF_BIN_SHIFT = 19;          // key >> 19 = sign, exponent, 4 mantissa bits (1/16 octave)
constexpr int PF_HIST_STRIDE = PF_BINS + 1;  // padded rows: conflict-free per-query scans

struct __align__(1024) PfSmem {
  uint8_t a[PF_STAGES][2][PF_A_BYTES / 2];  // [stage][K half][128 rows x 128 B], 128B-swizzled
  uint8_t b[2][PF_B_BYTES / 2];              // [K half][256 rows x 128 B]
  float4 w[PF_QT];                           // halved head weights, query pairs interleaved by head
  uint32_t hist[PF_QT * PF_HIST_STRIDE];     // sample histograms of the work tile's queries
  alignas(16) float tau[PF_QT];              // emission thresholds (scores; -inf: every block)
  int32_t base[PF_QT];                       // histogram bases (bin 0 = key >> 19 at or below base)
  uint64_t full_a[PF_STAGES], empty_a[PF_STAGES], full_b, empty_b, tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;  // set by the first role whose wait gives up: every role then stops issuing work
};

// Two lanes of fma.rn.f32x2: each is fmaf(a, b, c) of its lane (round to nearest, subnormals kept).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n.reg .b64 ra, rb, rc, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %5};\nmov.b64 rc, {%6, %7};\n"
      "fma.rn.f32x2 rd, ra, rb, rc;\nmov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Histogram bin of a score key for a query whose bins start at `base` (monotone in the key).
__device__ __forceinline__ int pf_bin(uint32_t key, int base) {
  return min(PF_BINS - 1, max(0, (int)(key >> PF_BIN_SHIFT) - base));
}

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


// ---- work schedule: tiles longest first, dealt in a snake; per tile the sample M-tiles first ----
// A work tile: 64 consecutive queries of one segment.  Local query index t (0 .. T-1 within the
// segment), global row q_off + t of the call's arrays.
struct PfTile {
  int req, pos0, T, q_off, qt;
  __device__ int nbv_of(int t) const { return (pos0 + t + 1) >> 2; }
  __device__ int nbv_hi() const { return pf_tile_nbv_hi(pos0, T, qt); }
  // every score key of the tile is written (no sample, no threshold)
  __device__ bool dense() const { return nbv_hi() <= PF_DENSE_MAX; }
  // M-tiles of the main phase (0: every query keeps all its blocks, nothing to score)
  __device__ int mtiles() const {
    const int nb = nbv_hi();
    return nb <= TOPK ? 0 : ceil_div(nb, PF_M);
  }
  // M-tiles of the sample phase (0: every query of the tile emits all its blocks)
  __device__ int stiles() const {
    const int nb = nbv_hi();
    return nb <= PF_EMIT_ALL || nb <= PF_DENSE_MAX ? 0 : ceil_div(ceil_div(nb, PF_M), PF_SAMPLE);
  }
};

// M-tile of step k of a tile with ns sample steps
__device__ __forceinline__ int pf_mt_of(int k, int ns) { return k < ns ? k * PF_SAMPLE : k - ns; }

// The k-th tile in schedule order: segments in their listed order, each segment's tiles from its last
// (longest context) down.
__device__ __forceinline__ PfTile pf_tile(const PrefillParams& p, int k) {
  int lo = 0, hi = p.nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seg[mid].tile_off <= k) lo = mid;
    else hi = mid - 1;
  }
  const PfSeg& s = p.seg[lo];
  return PfTile{s.req, s.pos0, s.T, s.q_off, ceil_div(s.T, PF_QT) - 1 - (k - s.tile_off)};
}

// j-th tile of CTA c, dealt in a snake over the schedule, or false
__device__ __forceinline__ bool pf_nth(const PrefillParams& p, int c, int j, PfTile& tile) {
  const int grid = (int)gridDim.x;
  const int k = j * grid + ((j & 1) ? (grid - 1 - c) : c);
  if (k >= p.ntiles) return false;
  tile = pf_tile(p, k);
  return true;
}

// Segment holding global row g (rows of one warp or CTA share it: uniform lookups).
__device__ __forceinline__ const PfSeg& pf_seg_of_row(const PrefillParams& p, int g) {
  int s = 0;
  while (s + 1 < p.nseg && (unsigned)(g - p.seg[s].q_off) >= (unsigned)p.seg[s].T) ++s;
  return p.seg[s];
}

// Emission threshold of one query from its sample histogram: the lower edge of the highest bin at
// which the sample holds R keys, R = (512 / PF_SAMPLE_KEEP) x (sampled blocks / visible blocks), so
// that about 512 / PF_SAMPLE_KEEP of the query's blocks pass.  0 (emit every
// visible block) for queries with few blocks, no histogram range, or too small a sample.
__device__ __forceinline__ uint32_t pf_threshold(const uint32_t* hist_row, int base, int nbv, int ns) {
  if (nbv <= PF_EMIT_ALL || base == PF_NO_BASE) return 0u;
  int ns_q = 0;
  for (int i = 0; i < ns; ++i) ns_q += min(PF_M, max(0, nbv - i * PF_SAMPLE * PF_M));
  const int R = max(1, (int)((float)TOPK / PF_SAMPLE_KEEP * (float)ns_q / (float)nbv));
  int acc = 0;
  for (int b = PF_BINS - 1; b > 0; --b) {
    acc += (int)hist_row[b];
    if (acc >= R) return base + b > 0 ? (uint32_t)(base + b) << PF_BIN_SHIFT : 0u;
  }
  return 0u;
}

// One CTA per SM: a TMA producer warp, an MMA warp and EW epilogue warps.
template <int EW>
__global__ void __launch_bounds__(pf_threads<EW>(), 1)
    k_prefill_score(PrefillParams p, const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap) {
  constexpr int PF_EPI_WARPS = EW;
  constexpr int PF_QPW = PF_QT * 4 / EW;  // queries per epilogue warp
  // the 8-warp form runs only calls whose tiles all write dense keys: no sample, no candidate code
  constexpr bool DENSE_ONLY = EW == PF_EPI_WARPS_DENSE;
  static_assert(EW % 4 == 0 && PF_QPW % 8 == 0, "epilogue warps cover the four TMEM quadrants evenly");
  static_assert(PF_QPW <= 32, "one lane per query of an epilogue warp holds its list counter");
  extern __shared__ uint8_t smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>(smem_aligned<1024>(smem_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    // Lane i < 8 looks up the physical page of page i of the next step's M-tile one step ahead, so
    // no page-table load sits on the path of a copy; lane 0 waits for the stage and expects its
    // bytes, then 16 lanes issue one copy each (a 64-dim half of one page of 16 keys).
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
    }
    const int oob_row = (int)(p.c.num_pages * PAGE_BLOCKS);  // a row past the cache: TMA fills zeros
    const int32_t* pt = p.c.page_table;
    auto page_row = [&](int lp, int nbv_hi) {                // logical page of the tile's request -> first cache row
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
    PfTile tl;
    for (int j = 0; ok && pf_nth(p, blockIdx.x, j, tl); ++j) {
      const int nm = tl.mtiles();
      if (nm == 0) continue;
      const int ns = tl.stiles(), nk = ns + nm;
      const int nbv_hi = tl.nbv_hi();
      pt = p.c.page_table + (int64_t)tl.req * p.c.max_pages;
      int go = 1;
      if (lane == 0) {
        go = wt == 0 || pf_wait(&S.empty_b, (wt - 1) & 1, p.err, lim, abort);
        if (go) {  // the tile's 64 queries x 4 heads of rotated index queries (rows past the call's end: zeros)
          const int qrow = (tl.q_off + tl.qt * PF_QT) * HI;
          mbar_arrive_expect_tx(&S.full_b, PF_B_BYTES);
          tma_load_2d(S.b[0], &qmap, 0, qrow, &S.full_b);
          tma_load_2d(S.b[1], &qmap, 64, qrow, &S.full_b);
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      ++wt;
      int rows_cur = lane < PF_PAGES ? page_row(pf_mt_of(0, ns) * PF_PAGES + lane, nbv_hi) : oob_row;
      for (int k = 0; k < nk; ++k, ++a_it) {
        const int rows_nxt =
            (k + 1 < nk && lane < PF_PAGES) ? page_row(pf_mt_of(k + 1, ns) * PF_PAGES + lane, nbv_hi) : oob_row;
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
        const int pg = (lane >> 1) & (PF_PAGES - 1), half = lane & 1;
        const int row = __shfl_sync(0xffffffffu, rows_cur, pg);
        if (lane < 2 * PF_PAGES)
          tma_load_2d(S.a[s][half] + pg * PAGE_BLOCKS * 128, &kmap, half * 64, row, &S.full_a[s]);
        rows_cur = rows_nxt;
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
      PfTile tl;
      for (int j = 0; ok && pf_nth(p, blockIdx.x, j, tl); ++j) {
        const int nm = tl.mtiles();
        if (nm == 0) continue;
        const int nk = tl.stiles() + nm;
        if (!pf_wait(&S.full_b, wt & 1, p.err, lim, abort)) break;
        ++wt;
        for (int k = 0; k < nk; ++k, ++a_it, ++m_it) {
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
    // Thread = one block of the M-tile (TMEM lane 32*quad + lane), registers = the 4 heads of the
    // warp's 16 queries.  Lane jl < 16 of a warp keeps the candidate count of query jl's list for
    // the warp's quadrant, so a list is never shared between warps.
    const int e = warp - 2;           // 0 .. PF_EPI_WARPS-1
    const int quad = warp & 3;        // TMEM lanes 32*quad .. +31 = blocks of the M-tile
    const int qg = e >> 2;            // query group: queries qg*PF_QPW .. +PF_QPW-1 of the tile
    const int etid = tid - 64;        // 0 .. 32*PF_EPI_WARPS-1
    const uint32_t lt = (1u << lane) - 1u;
    auto to_key = [](float sc) {  // order-preserving score key
      const uint32_t u = __float_as_uint(sc);
      return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    };
    int m_it = 0;
    PfTile tl;
    for (int j = 0; pf_nth(p, blockIdx.x, j, tl); ++j) {
      const int nm = tl.mtiles();
      if (nm == 0) continue;
      const int ns = tl.stiles(), nk = ns + nm;
      // every epilogue warp is done with the previous tile's shared state before it is replaced
      asm volatile("bar.sync 1, %0;" ::"n"(PF_EPI_WARPS * 32) : "memory");
      if (etid < PF_QT) {
        const int t = tl.qt * PF_QT + etid;
        float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
        int bs = PF_NO_BASE;
        if (t < tl.T) {
          w4 = __ldg(reinterpret_cast<const float4*>(p.w) + tl.q_off + t);
          bs = __ldg(p.qbase + tl.q_off + t);
        }
        {  // query pairs interleaved: S.w[2i] = (x, x', y, y'), S.w[2i+1] = (z, z', w, w') of queries 2i, 2i+1
          float* wf = reinterpret_cast<float*>(S.w) + (etid >> 1) * 8 + (etid & 1);
          wf[0] = 0.5f * w4.x;
          wf[2] = 0.5f * w4.y;
          wf[4] = 0.5f * w4.z;
          wf[6] = 0.5f * w4.w;
        }

        S.base[etid] = bs;
        S.tau[etid] = -INFINITY;
      }
      if (ns > 0)
        for (int i = etid; i < PF_QT * PF_HIST_STRIDE; i += PF_EPI_WARPS * 32) S.hist[i] = 0u;
      asm volatile("bar.sync 1, %0;" ::"n"(PF_EPI_WARPS * 32) : "memory");
      const int q0 = qg * PF_QPW;          // first query of this warp's group, in the tile
      const int t0 = tl.qt * PF_QT + q0;   // ... in the segment
      int cntq[PF_QPW];                    // every lane: candidates of query q0 + j in this quadrant's list
#pragma unroll
      for (int j2 = 0; j2 < PF_QPW; ++j2) cntq[j2] = 0;
      // this quadrant's list of the warp's first query; query q0 + jl's list is PF_ROW_WORDS further on
      unsigned long long* list0 = p.cand + (int64_t)(tl.q_off + t0) * PF_ROW_WORDS + quad * PF_QCAP;
      // dense tile: the score keys of the warp's first query's row; query q0 + jl's are 2 * PF_ROW_WORDS on
      uint32_t* dkeys0 = reinterpret_cast<uint32_t*>(p.cand + (int64_t)(tl.q_off + t0) * PF_ROW_WORDS);
      const bool dense = DENSE_ONLY || tl.dense();

      for (int k = 0; k < nk; ++k, ++m_it) {
        const int mt = pf_mt_of(k, ns);
        const int buf = m_it & 1;
        // after a timeout anywhere in the CTA the loop still runs to its end (no work, no waits), so
        // that every epilogue warp meets the same named barriers
        if (pf_wait(&S.tfull[buf], (m_it >> 1) & 1, p.err, lim, abort)) {
          tc_fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * PF_N + q0 * 4);
          const int b = mt * PF_M + quad * 32 + lane;  // this thread's block
          const uint32_t nb_word = ~(uint32_t)b;       // low word of its candidates: lower block ranks first
          // which of the warp's 16 queries see this thread's block (all of them except in a tile's last
          // M-tiles), as a mask computed once per M-tile
          uint32_t vmask = PF_QPW == 32 ? 0xFFFFFFFFu : (1u << PF_QPW) - 1u;
          if (!((mt + 1) * PF_M <= tl.nbv_of(t0) && t0 + PF_QPW <= tl.T)) {
            vmask = 0u;
#pragma unroll
            for (int jl = 0; jl < PF_QPW; ++jl)
              vmask |= (t0 + jl < tl.T && b < tl.nbv_of(t0 + jl)) ? (1u << jl) : 0u;
          }
          // the warp's queries' 4 heads in loads of 8 queries (32 columns each); the TMEM buffer goes back
          // to the MMA warp once the last is in registers
#pragma unroll
          for (int half = 0; half < PF_QPW / 8; ++half) {
            uint32_t r[32];
            tc_ld32(taddr + 32u * half, r);
            tc_wait_ld();
            tc_after_wait(r);
            if (half == PF_QPW / 8 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&S.tempty[buf]);
            }
            // the 8 scores first (independent chains); w * max(x, 0) == (w/2) * (x + |x|) exactly (doubling
            // and halving are exact), which keeps the ReLU on the FMA pipe; + 0 turns an underflowed -0 into +0
            float sc[8];
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2) {  // two queries per packed FMA, heads in order from +0
              const float4 wa = S.w[q0 + half * 8 + jj], wb = S.w[q0 + half * 8 + jj + 1];
              float y[2][4];
#pragma unroll
              for (int o = 0; o < 2; ++o)
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const float x = __uint_as_float(r[4 * (jj + o) + h]);
                  y[o][h] = x + fabsf(x);
                }
              float2 acc = fma2(make_float2(wa.x, wa.y), make_float2(y[0][0], y[1][0]), make_float2(0.f, 0.f));
              acc = fma2(make_float2(wa.z, wa.w), make_float2(y[0][1], y[1][1]), acc);
              acc = fma2(make_float2(wb.x, wb.y), make_float2(y[0][2], y[1][2]), acc);
              acc = fma2(make_float2(wb.z, wb.w), make_float2(y[0][3], y[1][3]), acc);
              sc[jj] = acc.x + 0.f;
              sc[jj + 1] = acc.y + 0.f;
            }
            const uint32_t vis8 = (vmask >> (8 * half)) & 0xFFu;
            if (dense) {  // every visible key, coalesced: the warp's 32 blocks of one query are 128 bytes
              if (vis8 == 0xFFu) {  // no per-query test in the M-tiles every query sees
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) dkeys0[(int64_t)(half * 8 + jj) * (2 * PF_ROW_WORDS) + b] = to_key(sc[jj]);
              } else
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                if ((vis8 >> jj) & 1u) dkeys0[(int64_t)(half * 8 + jj) * (2 * PF_ROW_WORDS) + b] = to_key(sc[jj]);
            } else if constexpr (!DENSE_ONLY) {
              if (k < ns) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                  if ((vis8 >> jj) & 1u)
                    atomicAdd(&S.hist[(q0 + half * 8 + jj) * PF_HIST_STRIDE + pf_bin(to_key(sc[jj]), S.base[q0 + half * 8 + jj])], 1u);
              } else {
              uint32_t em = 0u;  // queries this thread's block is a candidate of
              const float4 ta = *reinterpret_cast<const float4*>(&S.tau[q0 + half * 8]);
              const float4 tb = *reinterpret_cast<const float4*>(&S.tau[q0 + half * 8 + 4]);
              const float tq[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) em |= (sc[jj] >= tq[jj] ? 1u : 0u) << jj;
              em &= vis8;
              const uint32_t qm = __reduce_or_sync(0xffffffffu, em);  // queries with a candidate in this warp
              if (qm) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  if ((qm >> jj) & 1u) {  // warp-uniform
                    const int jl = half * 8 + jj;
                    const bool e = (em >> jj) & 1u;
                    const unsigned m = __ballot_sync(0xffffffffu, e);
                    const int slot = cntq[jl] + __popc(m & lt);
                    if (e && slot < PF_QCAP)
                      list0[(int64_t)jl * PF_ROW_WORDS + slot] = ((unsigned long long)to_key(sc[jj]) << 32) | nb_word;
                    cntq[jl] += __popc(m);
                  }
                }
              }
              }
            }
          }
        }
        if (!DENSE_ONLY && k == ns - 1) {  // the sample is complete: each query's threshold
          asm volatile("bar.sync 1, %0;" ::"n"(PF_EPI_WARPS * 32) : "memory");
          if (etid < PF_QT) {
            const int t = tl.qt * PF_QT + etid;
            const uint32_t tk =
                t < tl.T ? pf_threshold(S.hist + etid * PF_HIST_STRIDE, S.base[etid], tl.nbv_of(t), ns) : 0u;
            S.tau[etid] = tk == 0u ? -INFINITY : key_score(tk);
          }
          asm volatile("bar.sync 1, %0;" ::"n"(PF_EPI_WARPS * 32) : "memory");
        }
      }
      if constexpr (!DENSE_ONLY) {  // dense rows' lists are never read
        int mine = 0;
#pragma unroll
        for (int j2 = 0; j2 < PF_QPW; ++j2) mine = lane == j2 ? cntq[j2] : mine;
        if (lane < PF_QPW && t0 + lane < tl.T) p.cand_n[(int64_t)(tl.q_off + t0 + lane) * 4 + quad] = mine;
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
// Selection: one warp per query row, longest rows first, from the row's
// candidates (long contexts) or from all its score keys (dense tiles).
// (1) a histogram of the keys' log-scale bins (the scorer's bins of the
//     query; 4 times finer for a dense row) gives the bin D holding the
//     512th key;
// (2) one pass marks the blocks of every key above bin D in a block bitmap
//     (a dense row: one ballot per 32 blocks) and gathers bin D's keys; when
//     bin D holds more than the warp can gather, a second pass splits it by
//     the next 8 key bits first;
// (3) when many were gathered, they are split by the next 8 key bits in
//     shared memory: the sub-bins above the cut are marked, the cut sub-bin's
//     kept; what remains is ranked by whole word (key, then lower block
//     first; words are distinct), the best `need` marked;
// (4) the bitmap is written out in ascending block order.
// Rows with fewer than 512 candidates, an overflowed list, more ties in bin D
// than the warp holds (after the split; bin 0, which also holds the keys below
// the histogram's range, is never split) or no score bound go to the
// re-scoring list.
// ----------------------------------------------------------------------------
constexpr int PS_MAX_WARPS = 8;
// A single-segment call whose tiles all wrote dense keys selects first the rows whose keys the scorer
// wrote last (its last work tiles are the shortest rows), about this many bytes of them, while they are
// still in L2 (126 MB): 64 MiB measured best (402 us against 415 for the plain order, 411 for 32 MiB,
// 407 for 96 MiB at L = 32768).
constexpr double PS_L2_FIRST_BYTES = 64.0 * 1048576.0;
constexpr int PS_TIE_CAP = 256;
constexpr int PS_SUB_BINS = 256;   // second level: the 8 key bits below a first-level bin
constexpr int PS_TIE_RANK = 48;    // more gathered ties than this are split by sub-bin before ranking
constexpr int PS_U = 8;            // candidate rows: 8-byte loads in flight per lane
constexpr int PS_DENSE_U = 6;      // dense rows: 16-byte loads in flight per lane (4: +8 us, 8: +18 us at L = 32768)
constexpr int PS_DSPLIT_LOG = 2;                 // dense rows: 4 bins per candidate bin, i.e. 512 bins
constexpr int PS_DSPLIT = 1 << PS_DSPLIT_LOG;     // of 1/64 octave (key >> 17) over the same 8 octaves
constexpr int PS_DBINS = PF_BINS * PS_DSPLIT;
constexpr int PS_HIST_WORDS = PS_DBINS > PS_SUB_BINS ? PS_DBINS : PS_SUB_BINS;
static_assert(PF_BIN_SHIFT - PS_DSPLIT_LOG >= 8, "a dense bin keeps 8 key bits below it for the tie split");

__host__ __device__ constexpr int ps_warp_bytes(int bm_words) {
  return PS_HIST_WORDS * 4 + PS_TIE_CAP * 8 + ((bm_words + 3) / 4) * 16;
}

// Bin D of hist[0 .. NB) counted from the top: count(> D) < k <= count(>= D); `above` = count(> D).
// The caller guarantees count(all) >= k.  One warp; lane l owns the NB/32 bins below the top NB/32*l.
template <int NB>
__device__ __forceinline__ void ps_top_bin(const uint32_t* hist, int k, int& D, int& above) {
  constexpr int PER = NB / 32;
  const int lane = threadIdx.x & 31;
  const int top = NB - 1 - PER * lane;
  int local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) local += (int)hist[top - i];
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, x - local < k && x >= k);
  const int L = __ffs(hit) - 1;
  int c = __shfl_sync(0xffffffffu, x - local, L);
  const int topL = NB - 1 - PER * L;
  int d = topL - (PER - 1);
  for (int i = 0; i < PER; ++i) {
    const int h = (int)hist[topL - i];
    if (c + h >= k) {
      d = topL - i;
      break;
    }
    c += h;
  }
  D = d;
  above = c;
}

// The two row forms.  A candidate row: 4 lists (one per TMEM quadrant) of words key << 32 | ~block,
// binned like the scorer's sample (1/16 octave).  A dense row: the score key of every block, binned
// 4 times finer (a bin then holds a few dozen keys of a few thousand), the block being the key's index.
template <bool DENSE>
struct PsForm {
  static constexpr int BINS = DENSE ? PS_DBINS : PF_BINS;
  static constexpr int SHIFT = DENSE ? PF_BIN_SHIFT - PS_DSPLIT_LOG : PF_BIN_SHIFT;
  static constexpr int SUB_SHIFT = SHIFT - 8;  // the 8 key bits below a bin's
  int base;  // bin 0 = key >> SHIFT at or below base
  __device__ int bin_of_key(uint32_t key) const { return __vimin_s32_relu((int)(key >> SHIFT) - base, BINS - 1); }
  __device__ int bin(unsigned long long e) const { return bin_of_key((uint32_t)(e >> 32)); }
  __device__ static int sub(unsigned long long e) {
    return (int)((uint32_t)(e >> 32) >> SUB_SHIFT) & (PS_SUB_BINS - 1);
  }
};

// The end of a row's selection, one warp: the blocks above the cut bin are marked in the bitmap, the
// cut bin's nt entries (words key << 32 | ~block) are in tie[], `need` of them to take.  Many ties are
// first split by their next 8 key bits in shared memory (when the cut bin is not clamped), the rest
// ranked pairwise; then the bitmap is written out in ascending block order.  False: the row must be
// re-scored in full (more ties than the warp holds).
template <class Sub>
__device__ bool ps_finish(int nt, int need, bool splittable, Sub sub, int words, uint32_t* hist,
                          unsigned long long* tie, uint32_t* bitmap, int32_t* sel, int* err, int* sel_n) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  if (nt > PS_TIE_CAP || need > nt) return false;
  if (nt > PS_TIE_RANK && splittable) {
    // sub-bins above the cut sub-bin D2 are kept; D2's ties are packed to the front (each chunk of 32 is
    // read into registers before the ballot, and written only at or below its own indices); the pairwise
    // ranking costs nt^2 / 32 steps per lane, so it only sees D2's
    for (int i = lane; i < PS_SUB_BINS; i += 32) hist[i] = 0u;
    __syncwarp();
    for (int j = lane; j < nt; j += 32) atomicAdd(&hist[sub(tie[j])], 1u);
    __syncwarp();
    int D2, above2;
    ps_top_bin<PS_SUB_BINS>(hist, need, D2, above2);
    need -= above2;
    int nt2 = 0;
    for (int j0 = 0; j0 < nt; j0 += 32) {
      const int j = j0 + lane;
      unsigned long long e = 0ull;
      int sb = -1;
      if (j < nt) {
        e = tie[j];
        sb = sub(e);
      }
      if (sb > D2) {
        const uint32_t blk = ~(uint32_t)e;
        atomicOr(&bitmap[blk >> 5], 1u << (blk & 31));
      }
      const unsigned m = __ballot_sync(0xffffffffu, sb == D2);
      if (sb == D2) tie[nt2 + __popc(m & lt)] = e;
      nt2 += __popc(m);
    }
    __syncwarp();
    nt = nt2;
  }
  // ---- the best `need` of the cut bin's ties, by whole word (words are distinct) ----
  for (int j = lane; j < nt; j += 32) {
    const unsigned long long ej = tie[j];
    int rank = 0;
    for (int m = 0; m < nt; ++m) rank += tie[m] > ej;
    if (rank < need) {
      const uint32_t blk = ~(uint32_t)ej;
      atomicOr(&bitmap[blk >> 5], 1u << (blk & 31));
    }
  }
  __syncwarp();
  // ---- ascending output ----
  int out = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int wi = w0 + lane;
    uint32_t bits = wi < words ? bitmap[wi] : 0u;
    const int cn = __popc(bits);
    int xx = cn;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, xx, o);
      if (lane >= o) xx += y;
    }
    int o = out + xx - cn;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (o < TOPK) sel[o] = wi * 32 + bit;
      ++o;
    }
    out += __shfl_sync(0xffffffffu, xx, 31);
  }
  if (lane == 0) {
    if (out != TOPK) set_error(err, QSA_DEVERR_SELECTION);
    *sel_n = min(out, TOPK);
  }
  return true;
}

// Exact top-512 of a candidate row (n > 512 visible blocks) by one warp.  for_each(f) calls
// f(word, valid) for every candidate, all lanes together, PS_U loads in flight per lane.  False: the
// row must be re-scored in full.
template <class ForEach>
__device__ bool ps_candidate_row(ForEach for_each, int n, int qbase, uint32_t* hist, unsigned long long* tie,
                                 uint32_t* bitmap, int32_t* sel, int* err, int* sel_n) {
  using F = PsForm<false>;
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  if (qbase == PF_NO_BASE) return false;  // no score bound: every key would fall in one clamped bin
  const F f{qbase};
  // ---- (1) histogram ----
  for (int i = lane; i < F::BINS; i += 32) hist[i] = 0u;
  __syncwarp();
  for_each([&](unsigned long long e, bool valid) {
    if (valid) atomicAdd(&hist[f.bin(e)], 1u);
  });
  __syncwarp();
  int D, above;
  ps_top_bin<F::BINS>(hist, TOPK, D, above);
  int need = TOPK - above;  // taken from bin D, >= 1
  // ---- (2) bitmap of the blocks above bin D; bin D gathered ----
  const int words = (n + 31) >> 5;
  for (int i = lane; i < words; i += 32) bitmap[i] = 0u;
  __syncwarp();
  auto sweep = [&](auto in_above, auto in_tie) {  // one pass: bits for in_above, in_tie gathered
    int cnt_t = 0;
    for_each([&](unsigned long long e, bool valid) {
      const bool up = valid && in_above(e);
      const bool tie_e = valid && in_tie(e);
      if (up) {
        const uint32_t blk = ~(uint32_t)e;
        atomicOr(&bitmap[blk >> 5], 1u << (blk & 31));
      }
      const unsigned tm = __ballot_sync(0xffffffffu, tie_e);
      if (tie_e) {
        const int slot = cnt_t + __popc(tm & lt);
        if (slot < PS_TIE_CAP) tie[slot] = e;
      }
      cnt_t += __popc(tm);
    });
    return cnt_t;
  };
  int nt = sweep([&](unsigned long long e) { return f.bin(e) > D; }, [&](unsigned long long e) { return f.bin(e) == D; });
  __syncwarp();
  // the sub-bits order the keys of one bin only when it is not clamped: bin 0 also holds every key below
  // the range, so it is never split
  const bool splittable = D > 0;
  if (nt > PS_TIE_CAP && splittable) {
    // a crowded cut bin: split it by the next 8 key bits and keep only the cut sub-bin's ties
    for (int i = lane; i < PS_SUB_BINS; i += 32) hist[i] = 0u;
    __syncwarp();
    for_each([&](unsigned long long e, bool valid) {
      if (valid && f.bin(e) == D) atomicAdd(&hist[F::sub(e)], 1u);
    });
    __syncwarp();
    int D2, above2;
    ps_top_bin<PS_SUB_BINS>(hist, need, D2, above2);
    need -= above2;
    nt = sweep([&](unsigned long long e) { return f.bin(e) == D && F::sub(e) > D2; },
               [&](unsigned long long e) { return f.bin(e) == D && F::sub(e) == D2; });
    __syncwarp();
  }
  return ps_finish(nt, need, splittable, F::sub, words, hist, tie, bitmap, sel, err, sel_n);
}

// Exact top-512 of a dense row (n > 512 visible blocks, the score key of block b at keys[b]) by one
// warp, in two passes over the keys read 4 per 16-byte load: (1) the histogram; (2) the cut as key
// thresholds (the bins are monotone in the key): the bitmap words of the blocks above the cut bin are
// built from lane masks (a 128-key chunk is 8 lanes per 32-block word), the cut bin's keys gathered.
// A step whose U x 128 keys all lie below n skips the per-key bound test.  False: the row must be
// re-scored in full (no score bound, or more keys in the cut bin than the warp holds).
__device__ bool ps_dense_row(const uint32_t* keys, int n, int qbase, uint32_t* hist, unsigned long long* tie,
                             uint32_t* bitmap, int32_t* sel, int* err, int* sel_n) {
  using F = PsForm<true>;
  constexpr int U = PS_DENSE_U;  // 16-byte loads in flight per lane
  const int lane = threadIdx.x & 31;
  if (qbase == PF_NO_BASE) return false;
  const F f{qbase * PS_DSPLIT};
  const uint4* k4 = reinterpret_cast<const uint4*>(keys);  // the row area is 16-byte aligned and holds
  const int n4 = (n + 3) >> 2;                              // at least 4 * n4 keys
  auto load = [&](int c0, uint4 (&r)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * 32 + lane;
      r[u] = c < n4 ? __ldcg(k4 + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // ---- (1) histogram ----
  for (int i = lane; i < F::BINS; i += 32) hist[i] = 0u;
  __syncwarp();
  for (int c0 = 0; c0 < n4; c0 += 32 * U) {
    uint4 r[U];
    load(c0, r);
    if (4 * (c0 + 32 * U) <= n) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t kk[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) atomicAdd(&hist[f.bin_of_key(kk[j])], 1u);
      }
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = 4 * (c0 + u * 32 + lane);
        const uint32_t kk[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (v + j < n) atomicAdd(&hist[f.bin_of_key(kk[j])], 1u);
      }
    }
  }
  __syncwarp();
  int D, above;
  ps_top_bin<F::BINS>(hist, TOPK, D, above);
  const int need = TOPK - above;  // taken from bin D, >= 1
  // bin D as keys klo .. khm1; above it: keys > khm1 (none when D is the top bin, which holds every key
  // above the range); bin 0 also holds every key below the range
  const bool top = D == F::BINS - 1;
  const uint32_t klo = D == 0 ? 0u : (uint32_t)(f.base + D) << F::SHIFT;
  const uint32_t khm1 = top ? 0xFFFFFFFFu : ((uint32_t)(f.base + D + 1) << F::SHIFT) - 1u;
  const uint32_t span = khm1 - klo;  // key in bin D  <=>  key - klo <= span (unsigned)
  // ---- (2) bitmap words of the blocks above bin D; bin D gathered (slots from a shared counter: the
  // order of the gathered keys does not matter, the finishing step ranks them by whole word) ----
  const int words = (n + 31) >> 5;
  unsigned* tie_count = hist;  // the histogram is no longer read
  __syncwarp();
  if (lane == 0) *tie_count = 0u;
  __syncwarp();
  auto step = [&](const uint4 (&r)[U], int c0, auto full) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int cb = c0 + u * 32;  // this step's first 4-key group: blocks 4 cb .. 4 cb + 127
      const int v = 4 * (cb + lane);
      const uint32_t kk[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
      uint32_t m4 = 0u, t4 = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m4 |= (kk[j] > khm1 ? 1u : 0u) << j;
        t4 |= (kk[j] - klo <= span ? 1u : 0u) << j;
      }
      if constexpr (!decltype(full)::value) {
        const int rem = n - v;  // keys of this lane's group below n
        const uint32_t vm = rem >= 4 ? 0xFu : rem <= 0 ? 0u : (1u << rem) - 1u;
        m4 &= vm;
        t4 &= vm;
      }
      if (t4 != 0u) {
        int slot = (int)atomicAdd(tie_count, (unsigned)__popc(t4));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((t4 >> j) & 1u) {
            if (slot < PS_TIE_CAP) tie[slot] = ((unsigned long long)kk[j] << 32) | (uint32_t)~(uint32_t)(v + j);
            ++slot;
          }
      }
      // lanes 8 w .. 8 w + 7 hold the 32 blocks of word cb / 8 + w
      uint32_t wd = m4 << (4 * (lane & 7));
      wd |= __shfl_xor_sync(0xffffffffu, wd, 1);
      wd |= __shfl_xor_sync(0xffffffffu, wd, 2);
      wd |= __shfl_xor_sync(0xffffffffu, wd, 4);
      const int wi = cb / 8 + (lane >> 3);
      if ((lane & 7) == 0 && wi < words) bitmap[wi] = wd;
    }
  };
  for (int c0 = 0; c0 < n4; c0 += 32 * U) {
    uint4 r[U];
    load(c0, r);
    if (4 * (c0 + 32 * U) <= n)
      step(r, c0, std::true_type{});
    else
      step(r, c0, std::false_type{});
  }
  __syncwarp();
  const int nt = (int)*tie_count;
  __syncwarp();  // every lane has read the count before the finishing step reuses the histogram
  return ps_finish(nt, need, D > 0 && !top, F::sub, words, hist, tie, bitmap, sel, err, sel_n);
}

__global__ void __launch_bounds__(PS_MAX_WARPS * 32) k_prefill_select(PrefillParams p, int bm_words) {
  extern __shared__ __align__(16) uint8_t ps_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* mine = ps_raw + warp * ps_warp_bytes(bm_words);
  uint32_t* hist = reinterpret_cast<uint32_t*>(mine);
  unsigned long long* tie = reinterpret_cast<unsigned long long*>(mine + PS_HIST_WORDS * 4);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(mine + PS_HIST_WORDS * 4 + PS_TIE_CAP * 8);
  const int wpb = blockDim.x >> 5;
  const int gw = blockIdx.x * wpb + warp, nw = gridDim.x * wpb;
  for (int k = gw; k < p.T; k += nw) {
    // k-th row in schedule order: segments in listed order, each from its last (longest) row down
    int si = 0;
    while (si + 1 < p.nseg && p.seg[si + 1].row_off <= k) ++si;
    const PfSeg& sg = p.seg[si];
    int t = sg.q_off + (sg.T - 1 - (k - sg.row_off));  // global row
    if (p.sel_pivot > 0) {
      // one segment: rows sel_r0 .. sel_pivot-1 first (the scorer's last work tiles, their keys still in
      // L2), then the rest longest first, the rows of at most 512 blocks last
      const int na = p.sel_pivot - p.sel_r0, nb = p.T - p.sel_pivot;
      t = k < na ? p.sel_r0 + k : k < na + nb ? p.T - 1 - (k - na) : p.sel_r0 - 1 - (k - na - nb);
    }
    const int n = (sg.pos0 + (t - sg.q_off) + 1) >> 2;
    int32_t* sel = p.sel + (int64_t)t * TOPK;
    __syncwarp();  // the previous row's shared data is no longer read
    if (n <= TOPK) {
      for (int i = lane; i < n; i += 32) sel[i] = i;
      if (lane == 0) p.sel_n[t] = n;
      continue;
    }
    const unsigned long long* row = p.cand + (int64_t)t * PF_ROW_WORDS;
    const int qbase = p.qbase[t];
    bool done;
    if (pf_tile_nbv_hi(sg.pos0, sg.T, (t - sg.q_off) / PF_QT) <= PF_DENSE_MAX) {
      // a dense tile's row: the score key of every block, in block order
      done = ps_dense_row(reinterpret_cast<const uint32_t*>(row), n, qbase, hist, tie, bitmap, sel, p.err,
                          p.sel_n + t);
    } else {
      // a candidate row: its four lists, re-scored in full when they overflowed or hold fewer than 512
      const int cl = lane < 4 ? p.cand_n[(int64_t)t * 4 + lane] : 0;
      const int total = (int)__reduce_add_sync(0xffffffffu, (unsigned)cl);
      done = false;
      if (__reduce_max_sync(0xffffffffu, (unsigned)cl) <= (unsigned)PF_QCAP && total >= TOPK) {
        auto for_each = [&](auto fn) {
          for (int q = 0; q < 4; ++q) {
            const int cn = __shfl_sync(0xffffffffu, cl, q);
            const unsigned long long* list = row + q * PF_QCAP;
            for (int i0 = 0; i0 < cn; i0 += 32 * PS_U) {
              unsigned long long e[PS_U];
#pragma unroll
              for (int u = 0; u < PS_U; ++u) {
                const int i = i0 + u * 32 + lane;
                e[u] = i < cn ? __ldcg(list + i) : 0ull;
              }
#pragma unroll
              for (int u = 0; u < PS_U; ++u) fn(e[u], i0 + u * 32 + lane < cn);
            }
          }
        };
        done = ps_candidate_row(for_each, n, qbase, hist, tie, bitmap, sel, p.err, p.sel_n + t);
      }
    }
    if (!done && lane == 0) p.fb_list[atomicAdd(p.fb_n, 1)] = t;
  }
}

// ----------------------------------------------------------------------------
// Exact re-scoring of the rows the candidates could not settle: one CTA per
// row, its warps stream the row's pages (16 compressed keys each) through
// mma.sync into order-preserving score keys in global scratch, then an exact
// CTA-wide top-512 (radix refinement for heavy ties) emits the kept blocks in
// ascending order.
// ----------------------------------------------------------------------------
constexpr int PB_WARPS = 8;

__global__ void __launch_bounds__(PB_WARPS * 32) k_prefill_rescore(PrefillParams p) {
  __shared__ FastTopScratch fs;
  using All = Group<PB_WARPS * 32, 0>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, cq = lane & 3;
  const int nfb = *p.fb_n;
  uint32_t* keys = p.fb_keys + (int64_t)blockIdx.x * p.fb_cap;
  const uint4* cidx = reinterpret_cast<const uint4*>(p.c.cidx);
  for (int o = blockIdx.x; o < nfb; o += gridDim.x) {
    const int t = p.fb_list[o];  // global row
    const PfSeg& sg = pf_seg_of_row(p, t);
    const int n = (sg.pos0 + (t - sg.q_off) + 1) >> 2;
    const int32_t* pt = p.c.page_table + (int64_t)sg.req * p.c.max_pages;
    // B fragments of the rotated query (permuted like the page loads) and the lane's head weights
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.qrot + (int64_t)t * HI * D);
    uint32_t bq[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int d0 = 8 * (cq + 4 * (j >> 1)) + 4 * (j & 1);
      bq[j][0] = g8 < HI ? __ldg(q32 + ((g8 * D + d0) >> 1)) : 0u;
      bq[j][1] = g8 < HI ? __ldg(q32 + ((g8 * D + d0 + 2) >> 1)) : 0u;
    }
    const float wa = cq < 2 ? __ldg(p.w + (int64_t)t * HI + 2 * cq) : 0.f;
    const float wb = cq < 2 ? __ldg(p.w + (int64_t)t * HI + 2 * cq + 1) : 0.f;
    const int np = ceil_div(n, PAGE_BLOCKS);
    for (int lp = warp; lp < np; lp += PB_WARPS) {
      int phys = lp < p.c.max_pages ? __ldg(pt + lp) : -1;
      if (phys >= p.c.num_pages) phys = -1;  // flagged by the scorer already
      PageRegs pr;
      if (phys >= 0) load_page(pr, cidx + (int64_t)phys * (PAGE_BLOCKS * D / 8), g8, cq);
      float lo = 0.f, hi = 0.f;
      if (phys >= 0) score_page(pr, bq, wa, wb, lo, hi);
      if (cq < 2) {
        const int local = lp * PAGE_BLOCKS + g8 + 8 * cq;
        if (local < n) keys[local] = score_key(cq ? hi : lo);
      }
    }
    __syncthreads();
    int32_t* sel = p.sel + (int64_t)t * TOPK;
    fast_topk<All>([&](int i) { return keys[i]; }, n, TOPK, [&](int i, int out) { sel[out] = i; }, &fs);
    if (tid == 0) p.sel_n[t] = TOPK;
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// Rotation of the chunk's index queries (bf16, [T*4][128] rows for TMA), and
// each query's histogram base: an upper bound of its scores,
//   s <= sum_h max(w_h, 0) * |q~_h| * |k^|,  |k^| <= 1 + 2^-8 (a bf16 unit vector),
// taken with 2% of slack, sets the top bin; the 127 bins below it cover
// eight octaves at 1/16 octave each.
// ----------------------------------------------------------------------------
// One warp per query: lane i owns the rotation pairs (2i, 2i+64) and (2i+1, 2i+65) of all four heads,
// read and written as 32-bit words of two bf16 dims; the angles pos * inv_freq_j are taken once per
// query in FP64.
//
// Each rotated value is rounded once to bf16 (nearest even) from its exact value x0 c - x1 s (or
// x0 s + x1 c) with the FP64 terms c, s.  FP32 first: with cf, sf the FP32 roundings of c and s (|c|,
// |s| <= 1) and two more FP32 roundings, the FP32 result y lies within 2^-23 (|x0| + |x1| + |y|) +
// 2^-149 of the exact value (each rounding at most 2^-24 relative, or 2^-150 below the normal range).
// Rounding to bf16 is monotone, so when y minus and plus twice that bound round to the same bf16
// value, y rounds to the exact value's; otherwise (a value that close to a rounding boundary, about
// one in 10^4) that component is redone in FP64.
__device__ __forceinline__ uint32_t rope_pair_bf16(float x0, float x1, float cf, float sf, double c, double s) {
  const float y0 = fmaf(x0, cf, -(x1 * sf));
  const float y1 = fmaf(x0, sf, x1 * cf);
  const float m = fmaf(fabsf(x0) + fabsf(x1), 0x1p-22f, 0x1p-126f);
  const float e0 = fmaf(fabsf(y0), 0x1p-22f, m), e1 = fmaf(fabsf(y1), 0x1p-22f, m);
  const uint32_t b0 = pack_bf16x2(y0 - e0, y0 + e0), b1 = pack_bf16x2(y1 - e1, y1 + e1);
  uint32_t r = pack_bf16x2(y0, y1);  // low half: the first component
  if ((b0 >> 16) != (b0 & 0xFFFFu))
    r = (r & 0xFFFF0000u) | f64_to_bf16_bits((double)x0 * c - (double)x1 * s);
  if ((b1 >> 16) != (b1 & 0xFFFFu))
    r = (r & 0x0000FFFFu) | ((uint32_t)f64_to_bf16_bits((double)x0 * s + (double)x1 * c) << 16);
  return r;
}

constexpr int PR_WARPS = 8;

__global__ void __launch_bounds__(PR_WARPS * 32) k_prefill_rotate(PrefillParams p, const __nv_bfloat16* __restrict__ idx_q,
                                                                 RopeFreqs fr) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * PR_WARPS + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.fb_n = 0;  // the re-scoring list of this call starts empty
  if (t >= p.T) return;
  const PfSeg& sg = pf_seg_of_row(p, t);
  const double pos = (double)(sg.pos0 + (t - sg.q_off));
  const uint32_t* qin = reinterpret_cast<const uint32_t*>(idx_q + (int64_t)t * HI * D) + lane;
  uint32_t x[HI][2];  // [head][dims 2i, 2i+1 | dims 2i+64, 2i+65]
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    x[h][0] = __ldg(qin + h * (D / 2));
    x[h][1] = __ldg(qin + h * (D / 2) + D / 4);
  }
  double sn[2], cs[2];
  float sf[2], cf[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    sincos(pos * fr.f[2 * lane + j], &sn[j], &cs[j]);
    sf[j] = (float)sn[j];
    cf[j] = (float)cs[j];
  }
  uint32_t* qo = reinterpret_cast<uint32_t*>(p.qrot + (int64_t)t * HI * D) + lane;
  float nrm2[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    uint32_t rp[2];  // pair j: low half dim 2i+j rotated, high half dim 2i+64+j rotated
#pragma unroll
    for (int j = 0; j < 2; ++j)
      rp[j] = rope_pair_bf16(__uint_as_float(x[h][0] << (16 - 16 * j) & 0xFFFF0000u),
                             __uint_as_float(x[h][1] << (16 - 16 * j) & 0xFFFF0000u), cf[j], sf[j], cs[j], sn[j]);
    const uint32_t lo = __byte_perm(rp[0], rp[1], 0x5410), hi = __byte_perm(rp[0], rp[1], 0x7632);
    qo[h * (D / 2)] = lo;
    qo[h * (D / 2) + D / 4] = hi;
    const float a0 = __uint_as_float(lo << 16), a1 = __uint_as_float(lo & 0xFFFF0000u);
    const float b0 = __uint_as_float(hi << 16), b1 = __uint_as_float(hi & 0xFFFF0000u);
    nrm2[h] = fmaf(a0, a0, fmaf(b0, b0, fmaf(a1, a1, b1 * b1)));
  }
#pragma unroll
  for (int h = 0; h < HI; ++h)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nrm2[h] += __shfl_xor_sync(0xffffffffu, nrm2[h], o);
  if (lane == 0) {
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(p.w) + t);
    const float bound = 1.02f * (fmaxf(w4.x, 0.f) * sqrtf(nrm2[0]) + fmaxf(w4.y, 0.f) * sqrtf(nrm2[1]) +
                                 fmaxf(w4.z, 0.f) * sqrtf(nrm2[2]) + fmaxf(w4.w, 0.f) * sqrtf(nrm2[3]));
    p.qbase[t] = bound > 0.f && bound < 3.0e38f ? (int)(score_key(bound) >> PF_BIN_SHIFT) - (PF_BINS - 1)
                                                : PF_NO_BASE;
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


// Warps per CTA of the selection: 8, fewer when each warp's block bitmap is large.
static int select_warps(int bm_words) { return std::max(1, std::min(8, (200 * 1024) / ps_warp_bytes(bm_words))); }

cudaError_t launch_prefill(PrefillParams p, const __nv_bfloat16* idx_q, const RopeFreqs& fr, int num_sms,
                           cudaStream_t st, const cudaEvent_t* ev, int n_ev) {
  auto mark = [&](int i) {
    if (ev && i < 2 * n_ev) cudaEventRecord(ev[i], st);
  };
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(PfSmem) + 1024;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_prefill_score<PF_EPI_WARPS_CAND>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_prefill_score<PF_EPI_WARPS_DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_prefill_select, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (p.fb_cap % 32 != 0 || p.fb_ctas < 1 || p.nseg < 1 || p.nseg > PF_MAX_SEGS) return cudaErrorInvalidValue;
  for (int i = 0; i < p.nseg; ++i)
    if (p.fb_cap < ((p.seg[i].pos0 + p.seg[i].T) >> 2)) return cudaErrorInvalidValue;
  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, p.c.cidx, (uint64_t)p.c.num_pages * PAGE_BLOCKS, PAGE_BLOCKS)) return cudaErrorInvalidValue;
  if (!make_map(&qmap, p.qrot, (uint64_t)p.T * HI, PF_N)) return cudaErrorInvalidValue;
  mark(0);
  k_prefill_rotate<<<ceil_div(p.T, PR_WARPS), PR_WARPS * 32, 0, st>>>(p, idx_q, fr);
  mark(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int tiles = p.ntiles;
  mark(2);
  bool all_dense = true;  // every work tile of the call writes dense keys
  for (int i = 0; i < p.nseg; ++i)
    all_dense = all_dense && pf_tile_nbv_hi(p.seg[i].pos0, p.seg[i].T, (p.seg[i].T - 1) / PF_QT) <= PF_DENSE_MAX;
  if (all_dense)
    k_prefill_score<PF_EPI_WARPS_DENSE>
        <<<std::min(num_sms, tiles), pf_threads<PF_EPI_WARPS_DENSE>(), smem, st>>>(p, kmap, qmap);
  else
    k_prefill_score<PF_EPI_WARPS_CAND><<<std::min(num_sms, tiles), pf_threads<PF_EPI_WARPS_CAND>(), smem, st>>>(p, kmap, qmap);
  mark(3);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  mark(4);
  if (all_dense && p.nseg == 1) {
    // the selection starts with the rows whose keys the scorer wrote last: about PS_L2_FIRST_BYTES of
    // them, from the first row of more than 512 blocks up (rows r0 .. P-1 hold about
    // ((pos0 + P)^2 - (pos0 + r0)^2) / 2 bytes of keys)
    const int pos0 = p.seg[0].pos0;
    const int r0 = std::min(p.T, std::max(0, 4 * TOPK - pos0));
    const double a = (double)(pos0 + r0);
    const int P = (int)std::min<double>(p.T, std::sqrt(2.0 * PS_L2_FIRST_BYTES + a * a) - pos0);
    p.sel_r0 = r0;
    p.sel_pivot = P > r0 ? P : 0;
  }
  const int bm_words = p.fb_cap / 32;
  const int warps = select_warps(bm_words);
  const size_t ps_smem = (size_t)warps * ps_warp_bytes(bm_words);
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_prefill_select, warps * 32, ps_smem)) !=
      cudaSuccess)
    return e;
  k_prefill_select<<<std::min(ceil_div(p.T, warps), std::max(1, per_sm) * num_sms), warps * 32, ps_smem, st>>>(
      p, bm_words);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_prefill_rescore<<<p.fb_ctas, PB_WARPS * 32, 0, st>>>(p);
  mark(5);
  return cudaGetLastError();
}

}  // namespace qsa
