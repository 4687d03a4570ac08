// Prefill scorer on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// with a fused per-query candidate filter and an exact top-512 finalize.
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
// from the paged cache through a 3-deep ring), N = 256 = 64 queries x 4 heads
// (B, the rotated queries of one work tile, resident in shared memory),
// accumulators double-buffered in TMEM (2 x 256 of the 512 columns).  Keys on
// the M side put the 4 heads of one (block, query) pair in 4 adjacent TMEM
// columns of one lane, so one thread combines them without shuffles.
//
// Warp roles (one CTA per SM, persistent): warp 0 issues TMA, warp 1 owns TMEM
// and issues the MMAs (one elected thread), warps 2..9 are the epilogue: each
// reads its 32-lane TMEM quadrant (32 blocks) for 32 of the 64 queries.
//
// Top-512 without keeping scores: each query has a rising admission threshold.
// Admitted candidates are counted in a 128-bin log-scale histogram of the
// query's scaled scores (scale from the query alone); the threshold bin D is
// raised while at least 512 counted candidates lie above it, so every element
// of the final top-512 is admitted when it is scored (a bin >= D element can
// only be beaten by >= 512 elements of higher bins).  Candidates are appended
// in block order (per-tile ballots, prefix over the four quadrant warps), so a
// query's list is sorted; the finalize kernel (one warp per query) keeps the
// bins above D, ranks the few elements of bin D to find the exact cut, and
// compacts in order.  Work tiles are ordered longest first (causal imbalance)
// and dealt to CTAs in a snake.
#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int PF_QT = 64;              // queries per work tile
constexpr int PF_N = PF_QT * HI;       // 256 MMA columns
constexpr int PF_M = 128;              // compressed keys per M-tile
constexpr int PF_STAGES = 3;           // A ring depth
constexpr int PF_EPI_WARPS = 8;
constexpr int PF_THREADS = (2 + PF_EPI_WARPS) * 32;
constexpr int PF_BINS = 128;
constexpr int PF_A_BYTES = PF_M * D * 2;  // 32 KiB
constexpr int PF_B_BYTES = PF_N * D * 2;  // 64 KiB
constexpr uint32_t PF_TMEM_COLS = 512;

struct __align__(16) PfQuery {
  float4 w;     // head weights
  float theta;  // admit s > theta
  float scale;  // score -> histogram scale
  int nbv;      // visible complete blocks
  int D;        // threshold bin
};

struct __align__(1024) PfSmem {
  uint8_t a[PF_STAGES][2][PF_A_BYTES / 2];  // [stage][K half][128 rows x 128 B], 128B-swizzled
  uint8_t b[2][PF_B_BYTES / 2];              // [K half][256 rows x 128 B]
  int hist[PF_QT][PF_BINS];
  PfQuery q[PF_QT];
  int count[2][PF_QT];
  int acnt[PF_QT];
  int new_ge[PF_QT];
  uint32_t masks[2][4][32];  // [half][quadrant][query of the half]
  uint64_t full_a[PF_STAGES], empty_a[PF_STAGES], full_b, empty_b, tfull[2], tempty[2];
  uint32_t tmem_base;
};

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

__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

// Histogram bin of a score: 16 bins per octave of s * scale over [2^-3, 2^5),
// everything lower (and every s <= 0) in bin 0.  Monotone in s.
__device__ __forceinline__ int pf_bin(float s, float scale) {
  if (!(s > 0.f)) return 0;
  const int b = (int)(__float_as_uint(s * scale) >> 19) - (int)(0x3E000000u >> 19) + 1;
  return min(max(b, 0), PF_BINS - 1);
}

// Admission threshold for bin D (a hair below the bin's lower edge in score
// units, so no score of bin >= D is ever rejected by rounding).
__device__ __forceinline__ float pf_theta(int D, float scale) {
  if (D <= 0) return -INFINITY;
  const float edge = __uint_as_float((uint32_t)(D - 1 + (int)(0x3E000000u >> 19)) << 19);
  return edge / scale * (1.0f - 1.0f / 1048576.0f);
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
  PfSmem& S = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  PfSched sch{ceil_div(p.T, PF_QT), (int)gridDim.x, p.pos0, p.T};

  if (tid == 0) {
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
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
      const int32_t* pt = p.c.page_table + (int64_t)p.req * p.c.max_pages;
      const int oob_row = (int)(p.c.num_pages * PAGE_BLOCKS);  // a row past the cache: TMA fills zeros
      int a_it = 0, wt = 0;
      for (int j = 0;; ++j) {
        const int qt = sch.nth(blockIdx.x, j);
        if (qt < 0) break;
        const int nm = sch.mtiles(qt);
        if (nm == 0) continue;
        if (wt > 0) mbar_wait(&S.empty_b, (wt - 1) & 1, p.err);
        mbar_arrive_expect_tx(&S.full_b, PF_B_BYTES);
        tma_load_2d(S.b[0], &qmap, 0, qt * PF_N, &S.full_b);
        tma_load_2d(S.b[1], &qmap, 64, qt * PF_N, &S.full_b);
        ++wt;
        for (int mt = 0; mt < nm; ++mt, ++a_it) {
          const int s = a_it % PF_STAGES;
          if (a_it >= PF_STAGES) mbar_wait(&S.empty_a[s], ((a_it / PF_STAGES) - 1) & 1, p.err);
          mbar_arrive_expect_tx(&S.full_a[s], PF_A_BYTES);
          for (int pg = 0; pg < PF_M / PAGE_BLOCKS; ++pg) {
            const int lp = (mt * PF_M) / PAGE_BLOCKS + pg;  // logical page of the request
            int row = oob_row;
            if (lp < p.c.max_pages) {
              const int phys = __ldg(pt + lp);
              if (phys >= 0 && phys < p.c.num_pages) row = phys * PAGE_BLOCKS;
              else if (lp * PAGE_BLOCKS < sch.nbv_of(min(p.T, (qt + 1) * PF_QT) - 1)) set_error(p.err, QSA_DEVERR_PAGE);
            }
            tma_load_2d(S.a[s][0] + pg * PAGE_BLOCKS * 128, &kmap, 0, row, &S.full_a[s]);
            tma_load_2d(S.a[s][1] + pg * PAGE_BLOCKS * 128, &kmap, 64, row, &S.full_a[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      const uint32_t idesc = pf_idesc();
      int a_it = 0, m_it = 0, wt = 0;
      for (int j = 0;; ++j) {
        const int qt = sch.nth(blockIdx.x, j);
        if (qt < 0) break;
        const int nm = sch.mtiles(qt);
        if (nm == 0) continue;
        mbar_wait(&S.full_b, wt & 1, p.err);
        ++wt;
        for (int mt = 0; mt < nm; ++mt, ++a_it, ++m_it) {
          const int s = a_it % PF_STAGES;
          const int buf = m_it & 1;
          mbar_wait(&S.full_a[s], (a_it / PF_STAGES) & 1, p.err);
          if (m_it >= 2) mbar_wait(&S.tempty[buf], ((m_it >> 1) - 1) & 1, p.err);
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
      }
      // tail: every commit issued above must have arrived before the CTA may exit
      if (wt > 0) mbar_wait(&S.empty_b, (wt - 1) & 1, p.err);
      for (int s = 0; s < PF_STAGES; ++s) {
        const int uses = a_it / PF_STAGES + (s < a_it % PF_STAGES ? 1 : 0);
        if (uses > 0) mbar_wait(&S.empty_a[s], (uses - 1) & 1, p.err);
      }
    }
  } else {
    // =============================== epilogue ===============================
    const int e = warp - 2;           // 0..7
    const int quad = warp & 3;        // TMEM lanes 32*quad .. +31 = blocks of the M-tile
    const int half = e >> 2;          // queries 32*half .. +31
    const bool leader = quad == 0;    // the warp that updates the half's per-query state
    const int bar_half = 2 + half;    // named barrier of the 4 warps of this half
    const int etid = tid - 64;        // 0..255
    int m_it = 0;
    for (int j = 0;; ++j) {
      const int qt = sch.nth(blockIdx.x, j);
      if (qt < 0) break;
      const int nm = sch.mtiles(qt);
      if (nm == 0) continue;
      // ---- per-tile query state ----
      for (int i = etid; i < PF_QT * PF_BINS; i += 256) (&S.hist[0][0])[i] = 0;
      if (etid < PF_QT) {
        const int t = qt * PF_QT + etid;
        PfQuery qi;
        if (t < p.T) {
          qi.w = __ldg(reinterpret_cast<const float4*>(p.w) + t);
          qi.scale = __ldg(p.scale + t);
          qi.nbv = sch.nbv_of(t);
        } else {
          qi.w = make_float4(0.f, 0.f, 0.f, 0.f);
          qi.scale = 1.f;
          qi.nbv = 0;
        }
        qi.D = 0;
        qi.theta = -INFINITY;
        S.q[etid] = qi;
        S.count[0][etid] = 0;
        S.acnt[etid] = 0;
        S.new_ge[etid] = 0;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");

      for (int mt = 0; mt < nm; ++mt, ++m_it) {
        const int buf = m_it & 1;
        mbar_wait(&S.tfull[buf], (m_it >> 1) & 1, p.err);
        tc_fence_after();
        const int b = mt * PF_M + quad * 32 + lane;  // this thread's block
        float sc[32];
        uint32_t my_masks = 0;  // lane i: this quadrant's admission mask of query 32*half + i
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
          uint32_t r[2][32];
          const uint32_t col = (uint32_t)(buf * PF_N + half * 128 + g2 * 64);
          const uint32_t lanes = (uint32_t)(quad * 32) << 16;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
              "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
              : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]),
                "=r"(r[0][6]), "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]),
                "=r"(r[0][12]), "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]), "=r"(r[0][16]), "=r"(r[0][17]),
                "=r"(r[0][18]), "=r"(r[0][19]), "=r"(r[0][20]), "=r"(r[0][21]), "=r"(r[0][22]), "=r"(r[0][23]),
                "=r"(r[0][24]), "=r"(r[0][25]), "=r"(r[0][26]), "=r"(r[0][27]), "=r"(r[0][28]), "=r"(r[0][29]),
                "=r"(r[0][30]), "=r"(r[0][31])
              : "r"(tmem + lanes + col));
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
              "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
              : "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]),
                "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]), "=r"(r[1][10]), "=r"(r[1][11]),
                "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15]), "=r"(r[1][16]), "=r"(r[1][17]),
                "=r"(r[1][18]), "=r"(r[1][19]), "=r"(r[1][20]), "=r"(r[1][21]), "=r"(r[1][22]), "=r"(r[1][23]),
                "=r"(r[1][24]), "=r"(r[1][25]), "=r"(r[1][26]), "=r"(r[1][27]), "=r"(r[1][28]), "=r"(r[1][29]),
                "=r"(r[1][30]), "=r"(r[1][31])
              : "r"(tmem + lanes + col + 32u));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int qq = 0; qq < 16; ++qq) {
            const int jl = g2 * 16 + qq;  // query of the half
            const PfQuery* qp = &S.q[half * 32 + jl];
            const float4 w4 = qp->w;
            const float4 tz = *reinterpret_cast<const float4*>(&qp->theta);  // theta, scale, nbv, D
            const uint32_t* rr = &r[qq >> 3][4 * (qq & 7)];
            float s = w4.x * fmaxf(__uint_as_float(rr[0]), 0.f);
            s = fmaf(w4.y, fmaxf(__uint_as_float(rr[1]), 0.f), s);
            s = fmaf(w4.z, fmaxf(__uint_as_float(rr[2]), 0.f), s);
            s = fmaf(w4.w, fmaxf(__uint_as_float(rr[3]), 0.f), s);
            sc[jl] = s;
            const bool admit = s > tz.x && b < __float_as_int(tz.z);
            const uint32_t m = __ballot_sync(0xffffffffu, admit);
            if (lane == jl) my_masks = m;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.tempty[buf]);
        S.masks[half][quad][lane] = my_masks;
        asm volatile("bar.sync %0, 128;" ::"r"(bar_half) : "memory");

        // ---- ordered append: quadrant q's blocks follow quadrants < q ----
        // lane i prepares query 32*half + i: its masks, this warp's base offset, scale and D
        const int cur = mt & 1;
        const int jq_l = half * 32 + lane;
        uint32_t total_l, base_l;
        {
          const uint32_t m0 = S.masks[half][0][lane], m1 = S.masks[half][1][lane];
          const uint32_t m2 = S.masks[half][2][lane], m3 = S.masks[half][3][lane];
          const uint32_t p0 = __popc(m0), p1 = __popc(m1), p2 = __popc(m2), p3 = __popc(m3);
          total_l = p0 + p1 + p2 + p3;
          base_l = (uint32_t)S.count[cur][jq_l] + (quad > 0 ? p0 : 0u) + (quad > 1 ? p1 : 0u) + (quad > 2 ? p2 : 0u);
        }
        const float scale_l = S.q[jq_l].scale;
        const int D_l = S.q[jq_l].D;
        const uint32_t any = __ballot_sync(0xffffffffu, my_masks != 0);
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (!(any & (1u << i))) continue;
          const uint32_t mq = __shfl_sync(0xffffffffu, my_masks, i);
          const int base = (int)__shfl_sync(0xffffffffu, base_l, i);
          const float scale = __shfl_sync(0xffffffffu, scale_l, i);
          const int Dq = __shfl_sync(0xffffffffu, D_l, i);
          const bool mine = (mq >> lane) & 1u;
          const int jq = half * 32 + i;
          const int t = qt * PF_QT + jq;
          const int pos = base + __popc(mq & lt);
          const float s = sc[i];
          int bin = -1;
          if (mine) {
            if (t < p.T && pos < p.cap) {
              p.cand_key[(int64_t)t * p.cap + pos] = score_key(s);
              p.cand_id[(int64_t)t * p.cap + pos] = b;
            } else {  // cannot happen: each visible block is admitted once per query
              set_error(p.err, QSA_DEVERR_SELECTION);
            }
            bin = pf_bin(s, scale);
            if (bin < Dq) bin = -1;  // admitted on an older threshold: not counted
          }
          const uint32_t counted = __ballot_sync(0xffffffffu, bin >= 0);
          if (counted) {
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (bin >= 0 && (peers & lt) == 0) atomicAdd(&S.hist[jq][bin], __popc(peers));
            if (lane == 0) atomicAdd(&S.new_ge[jq], __popc(counted));
          }
        }
        asm volatile("bar.sync %0, 128;" ::"r"(bar_half) : "memory");
        if (leader) {  // lane i: query 32*half + i
          const int jq = jq_l;
          S.count[cur ^ 1][jq] = S.count[cur][jq] + (int)total_l;
          int a = S.acnt[jq] + S.new_ge[jq];
          S.new_ge[jq] = 0;
          int Dq = D_l;
          while (Dq < PF_BINS - 1 && a - S.hist[jq][Dq] >= TOPK) {
            a -= S.hist[jq][Dq];
            ++Dq;
          }
          S.acnt[jq] = a;
          if (Dq != D_l) {
            S.q[jq].D = Dq;
            S.q[jq].theta = pf_theta(Dq, scale_l);
          }
        }
      }
      // ---- the tile's per-query results ----
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (etid < PF_QT) {
        const int t = qt * PF_QT + etid;
        if (t < p.T) {
          p.cand_n[t] = S.count[nm & 1][etid];
          p.thr_bin[t] = S.q[etid].D;
        }
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
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
// Finalize: one warp per query.  Keeps the candidates of bins above D, ranks
// the (few) candidates of bin D to place the exact cut (score key, list
// position; the list is in block order, so position order is block order),
// and compacts in order.  A bin D holding more than PF_FIN_CAP candidates is
// handed to the CTA-wide radix path (overflow list).
// ----------------------------------------------------------------------------
constexpr int PF_FIN_WARPS = 8;
constexpr int PF_FIN_CAP = 256;

__global__ void __launch_bounds__(PF_FIN_WARPS * 32) k_prefill_finalize(PrefillParams p) {
  __shared__ uint32_t eq_key[PF_FIN_WARPS][PF_FIN_CAP];
  __shared__ int eq_pos[PF_FIN_WARPS][PF_FIN_CAP];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * PF_FIN_WARPS + warp;
  if (t >= p.T) return;
  const int nbv = (p.pos0 + t + 1) >> 2;
  int32_t* sel = p.sel + (int64_t)t * TOPK;
  if (nbv <= TOPK) {
    for (int i = lane; i < nbv; i += 32) sel[i] = i;
    if (lane == 0) p.sel_n[t] = nbv;
    return;
  }
  const int n = min(p.cand_n[t], p.cap);
  const int Dq = p.thr_bin[t];
  const float scale = __ldg(p.scale + t);
  const uint32_t* keys = p.cand_key + (int64_t)t * p.cap;
  const int32_t* ids = p.cand_id + (int64_t)t * p.cap;
  int gt = 0, neq = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    int bin = -1;
    uint32_t k = 0;
    if (i < n) {
      k = __ldcg(keys + i);
      bin = pf_bin(key_score(k), scale);
    }
    gt += __popc(__ballot_sync(0xffffffffu, bin > Dq));
    const uint32_t me = __ballot_sync(0xffffffffu, bin == Dq);
    const int slot = neq + __popc(me & ((1u << lane) - 1u));
    if (bin == Dq && slot < PF_FIN_CAP) {
      eq_key[warp][slot] = k;
      eq_pos[warp][slot] = i;
    }
    neq += __popc(me);
  }
  const int need = TOPK - gt;
  if (need < 1 || need > neq || neq > PF_FIN_CAP) {  // degenerate ties (or a broken invariant): CTA path
    if (lane == 0) {
      if (need < 1 || need > neq) set_error(p.err, QSA_DEVERR_SELECTION);
      const int slot = atomicAdd(p.ovf_n, 1);
      p.ovf_list[slot] = t;
    }
    return;
  }
  __syncwarp();
  uint32_t T = 0;
  int I = 0;
  for (int j = lane; j < neq; j += 32) {
    const uint32_t kj = eq_key[warp][j];
    const int ij = eq_pos[warp][j];
    int rank = 0;
    for (int m = 0; m < neq; ++m) {
      const uint32_t km = eq_key[warp][m];
      rank += (km > kj) || (km == kj && eq_pos[warp][m] < ij);
    }
    if (rank == need - 1) {
      T = kj;
      I = ij;
    }
  }
  // broadcast the cut from the lane that found it
  const uint32_t who = __ballot_sync(0xffffffffu, (T != 0u) || (I != 0));
  const int src = who ? __ffs(who) - 1 : 0;
  T = __shfl_sync(0xffffffffu, T, src);
  I = __shfl_sync(0xffffffffu, I, src);
  int out = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    bool keep = false;
    if (i < n) {
      const uint32_t k = __ldcg(keys + i);
      keep = k > T || (k == T && i <= I);
    }
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    const int o = out + __popc(m & ((1u << lane) - 1u));
    if (keep && o < TOPK) sel[o] = __ldcg(ids + i);
    out += __popc(m);
  }
  if (lane == 0) {
    if (out != TOPK) set_error(p.err, QSA_DEVERR_SELECTION);
    p.sel_n[t] = min(out, TOPK);
  }
}

// Overflow queries: exact CTA-wide radix selection over the query's candidate list.
__global__ void __launch_bounds__(256) k_prefill_overflow(PrefillParams p) {
  __shared__ SelectScratch sc;
  using All = Group<256, 0>;
  const int nov = *p.ovf_n;
  for (int o = blockIdx.x; o < nov; o += gridDim.x) {
    const int t = p.ovf_list[o];
    const int n = min(p.cand_n[t], p.cap);
    if (n <= 0) {
      if (threadIdx.x == 0) p.sel_n[t] = 0;
      continue;
    }
    const uint32_t* keys = p.cand_key + (int64_t)t * p.cap;
    const int32_t* ids = p.cand_id + (int64_t)t * p.cap;
    int32_t* sel = p.sel + (int64_t)t * TOPK;
    auto key_at = [&](int i) { return __ldcg(keys + i); };
    const SelectResult r = radix_select<All>(key_at, n, min(n, TOPK), &sc);
    select_compact<All>(key_at, n, r, [&](int i, int out) { sel[out] = __ldcg(ids + i); }, &sc);
    if (threadIdx.x == 0) p.sel_n[t] = min(n, TOPK);
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// Rotation of the chunk's index queries (bf16, [T*4][128] rows for TMA) and
// the per-query histogram scale 16 / sum_h max(w_h, 0) * ||q~_h||.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_prefill_rotate(PrefillParams p, const __nv_bfloat16* __restrict__ idx_q,
                                                        RopeFreqs fr) {
  const int t = blockIdx.x;
  const int tid = threadIdx.x, h = tid >> 5, lane = tid & 31;
  __shared__ double cs_s[D / 2], sn_s[D / 2];
  __shared__ float nrm[HI];
  const int pos = p.pos0 + t;
  if (tid < D / 2) sincos((double)pos * fr.f[tid], &sn_s[tid], &cs_s[tid]);
  __syncthreads();
  const uint16_t* qin = reinterpret_cast<const uint16_t*>(idx_q + ((int64_t)t * HI + h) * D);
  uint16_t* qo = reinterpret_cast<uint16_t*>(p.qrot + ((int64_t)t * HI + h) * D);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int i = lane + 32 * e;
    const double x0 = (double)bf16_bits_to_f32(qin[i]);
    const double x1 = (double)bf16_bits_to_f32(qin[i + D / 2]);
    const uint16_t y0 = f64_to_bf16_bits(x0 * cs_s[i] - x1 * sn_s[i]);
    const uint16_t y1 = f64_to_bf16_bits(x0 * sn_s[i] + x1 * cs_s[i]);
    qo[i] = y0;
    qo[i + D / 2] = y1;
    const float f0 = bf16_bits_to_f32(y0), f1 = bf16_bits_to_f32(y1);
    ss += f0 * f0 + f1 * f1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) nrm[h] = sqrtf(ss);
  __syncthreads();
  if (tid == 0) {
    float hi = 0.f;
    for (int k = 0; k < HI; ++k) hi += fmaxf(__ldg(p.w + (int64_t)t * HI + k), 0.f) * nrm[k];
    hi *= 1.01f;  // the bf16-rounded compressed keys have norm <= 1.01
    p.scale[t] = hi > 1e-30f ? 16.f / hi : 1.f;
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
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_prefill_score, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, p.c.cidx, (uint64_t)p.c.num_pages * PAGE_BLOCKS, PAGE_BLOCKS)) return cudaErrorInvalidValue;
  if (!make_map(&qmap, p.qrot, (uint64_t)p.T * HI, PF_N)) return cudaErrorInvalidValue;
  mark(0);
  k_prefill_rotate<<<p.T, 128, 0, st>>>(p, idx_q, fr);
  mark(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(p.T, PF_QT);
  mark(2);
  k_prefill_score<<<std::min(num_sms, tiles), PF_THREADS, smem, st>>>(p, kmap, qmap);
  mark(3);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.ovf_n, 0, sizeof(int), st)) != cudaSuccess) return e;
  mark(4);
  k_prefill_finalize<<<ceil_div(p.T, PF_FIN_WARPS), PF_FIN_WARPS * 32, 0, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_prefill_overflow<<<std::min(p.T, 4 * num_sms), 256, 0, st>>>(p);
  mark(5);
  return cudaGetLastError();
}

}  // namespace qsa
